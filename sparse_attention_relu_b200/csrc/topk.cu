// Per-query top-k selection: a radix select on order-preserving keys.
//
// "Sparse Attention Architecture Evolution in LLMs" (Top-K Selection): each
// query keeps k positions (k = 2048); "GLM sparse attention" (threshold
// figure): the cut-off is the k-th best score.  Ties go to the lower
// position; -0 == +0; NaN ranks as -inf.
//
// One CTA of 512 threads owns a row, and several CTAs share an SM (about
// 25 KB of shared memory each) so that one row's reads overlap another's
// arithmetic.  Scores become 32-bit keys whose unsigned order is the float
// order, and the row is read twice (the second time from L2):
//   pass 1  a 2048-bin histogram fixes the bin b1 that holds the k-th best
//           score.  A bin is the sign and 32 steps per binade of the
//           magnitude over 2^-16 .. 2^16 (saturating outside): monotone, so a
//           higher bin means a strictly larger score, and indexer scores,
//           which crowd a few binades, spread over hundreds of bins instead
//           of the few dozen that the top bits of the fp32 key would give
//           (the histogram atomics would serialise on them);
//   pass 2  b1 is an interval [lo, hi] of floats: every score above hi is
//           written out at once (in any order), the members of b1 --
//           typically a hundred or so -- go to a candidate buffer in shared
//           memory with their fp32 keys.
// The candidates are then split once more: a histogram of their keys over
// 2048 buckets spanning the candidates' key range finds the bucket at the
// cut, the buckets above it go out, and only that bucket's members (one or
// two, typically) are ranked (key, then position: ties go to the lower
// position) for the last of the k - |above b1| slots.  A bin b1 with more members than the buffer holds is resolved by radix
// passes over the row instead (11 + 11 + 10 bits of the fp32 key), with
// ties at the cut filled from the lowest positions by an ordered pass over
// the row (ballot + warp prefix + a scan of warp totals).
#include "kernels.cuh"
#include "select.cuh"

namespace dsa {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
using sel::kBins;
using sel::kCand;
using sel::rank_key;
using sel::score_bin;
using sel::bin_bounds;
using sel::warp_append;
using B512 = sel::Blk<kThreads, 0, 0>;  // the whole CTA, __syncthreads()
using Smem = sel::Smem<kWarps>;
__device__ __forceinline__ void find_bin(Smem& sm, int nbins, uint32_t need) {
  sel::find_bin<B512>(sm, nbins, need);
}
__device__ __forceinline__ void rank_candidates(Smem& sm, uint32_t* ckey, int32_t* cpos, int m,
                                                uint32_t need, int32_t* dst) {
  sel::rank_candidates<B512>(sm, ckey, cpos, m, need, dst);
}
constexpr int kBatch = 4;    // float4 loads each thread keeps in flight per step
constexpr int kBatchRow = 2;  // the same at three CTAs per SM (42 registers)

// The members of bin b1 (more than the candidate buffer holds) resolved from
// the row itself: three radix levels over their fp32 keys find the k-th key
// tau; members above tau are written after the `above1` scores above b1
// (sm.n_out counts the written slots), and ties at tau fill the rest from
// the lowest positions by an ordered pass over the row.  All threads call it.
__device__ void resolve_by_row(Smem& sm, const float* row, int n, int k, uint32_t b1,
                               uint32_t above1, int32_t* out) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  auto member_key = [&](int i, uint32_t& u) -> bool {
    const float x = __ldg(row + i);
    u = rank_key(x);
    return score_bin(x) == b1;
  };
  uint32_t prefix = 0, c_gt = above1;
  const int shift[3] = {21, 10, 0};
  const uint32_t width[3] = {11, 11, 10};
#pragma unroll
  for (int lvl = 0; lvl < 3; ++lvl) {
    for (int i = tid; i < kBins; i += kThreads) sm.hist[i] = 0;
    __syncthreads();
    const int hi = shift[lvl] + (int)width[lvl];  // bits above this level must match prefix
    for (int i = tid; i < n; i += kThreads) {
      uint32_t u;
      if (member_key(i, u) && (hi >= 32 || (u >> hi) == prefix))
        atomicAdd(&sm.hist[(u >> shift[lvl]) & ((1u << width[lvl]) - 1u)], 1u);
    }
    __syncthreads();
    find_bin(sm, 1 << width[lvl], (uint32_t)k - c_gt);
    prefix = (prefix << width[lvl]) | sm.sel_bin;
    c_gt += sm.sel_above;
    __syncthreads();
  }
  const uint32_t tau = prefix;                  // the k-th best key
  const uint32_t need_eq = (uint32_t)k - c_gt;  // >= 1 keys equal to tau to take
  const uint32_t n_eq = sm.hist[tau & 0x3ffu];
  __syncthreads();
  // b1's members above tau in any order; those equal to tau all go when
  // exactly need_eq of them exist, else the need_eq lowest positions.
  const bool all_eq = n_eq == need_eq;
  for (int base = 0; base < n; base += kThreads) {
    const int i = base + tid;
    uint32_t u = 0;
    const bool take = i < n && member_key(i, u) && (u > tau || (all_eq && u == tau));
    uint32_t slot;
    if (warp_append(take, &sm.n_out, slot) && take) out[slot] = i;
  }
  if (all_eq) return;
  __syncthreads();
  uint32_t eq_base = 0;
  for (int base = 0; base < n && eq_base < need_eq; base += kThreads) {  // uniform
    const int i = base + tid;
    const bool eq = i < n && rank_key(__ldg(row + i)) == tau;
    const uint32_t emask = __ballot_sync(0xffffffffu, eq);
    if (lane == 0) sm.warp_tot[warp] = (uint32_t)__popc(emask);
    __syncthreads();
    uint32_t before = 0, total = 0;
    for (int w2 = 0; w2 < kWarps; ++w2) {
      const uint32_t c = sm.warp_tot[w2];
      if (w2 < warp) before += c;
      total += c;
    }
    const uint32_t rank = eq_base + before + __popc(emask & ((1u << lane) - 1u));
    if (eq && rank < need_eq) out[c_gt + rank] = i;
    eq_base += total;
    __syncthreads();
  }
}

__global__ void __launch_bounds__(kThreads, 3) topk_kernel(Rows R, int32_t row0, const float* scores,
                                                           int64_t ld, int k, int32_t* idx) {
  __shared__ uint32_t ckey[kCand];
  __shared__ int32_t cpos[kCand];
  __shared__ Smem sm;
  const int tid = threadIdx.x, lane = tid & 31;
  const int32_t r = row0 + blockIdx.x;
  const RowInfo ri = row_info(R, r);
  const int n = ri.t + 1;
  int32_t* out = idx + (int64_t)blockIdx.x * k;
  if (n <= k) {
    for (int i = tid; i < k; i += kThreads) out[i] = i < n ? i : -1;
    return;
  }
  const float* row = scores + (int64_t)blockIdx.x * ld;
  // The row as a scalar head up to the first 16-byte boundary, n4 float4
  // vectors from a0, and a scalar tail from t0 (row strides need not be
  // multiples of four floats).
  const int a0 =
      min(n, (int)((4u - (uint32_t)((reinterpret_cast<uintptr_t>(row) >> 2) & 3u)) & 3u));
  const int n4 = (n - a0) >> 2, t0 = a0 + 4 * n4;
  const int n_head = a0, n_edge = n_head + (n - t0);  // <= 6 scalar scores
  const float4* row4 = reinterpret_cast<const float4*>(row + a0);

  // ------------------------------------------------------------ pass 1
  for (int i = tid; i < kBins; i += kThreads) sm.hist[i] = 0;
  if (tid == 0) {
    sm.n_out = 0;
    sm.n_cand = 0;
  }
  __syncthreads();
  if (tid < n_edge) {
    const int i = tid < n_head ? tid : t0 + (tid - n_head);
    atomicAdd(&sm.hist[score_bin(__ldg(row + i))], 1u);
  }
  for (int base = tid; base < n4; base += kBatchRow * kThreads) {
    float4 xv[kBatchRow];
#pragma unroll
    for (int u = 0; u < kBatchRow; ++u) {
      const int v = base + u * kThreads;
      if (v < n4) xv[u] = __ldg(row4 + v);
    }
#pragma unroll
    for (int u = 0; u < kBatchRow; ++u) {
      const int v = base + u * kThreads;
      const float xs[4] = {xv[u].x, xv[u].y, xv[u].z, xv[u].w};
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (v < n4) atomicAdd(&sm.hist[score_bin(xs[e])], 1u);
    }
  }
  __syncthreads();
  find_bin(sm, kBins, (uint32_t)k);
  const uint32_t b1 = sm.sel_bin;
  const uint32_t above1 = sm.sel_above;  // scores in bins above b1
  const uint32_t in_b1 = sm.hist[b1];
  const uint32_t need = (uint32_t)k - above1;  // 1 <= need <= in_b1
  __syncthreads();

  // ------------------------------------------------------------ pass 2
  // Everything above b1 is selected; the members of b1 become candidates
  // (when they all fit the buffer).  b1 is the float interval [lo, hi]; the
  // -inf bin 0 holds NaN too, which no float comparison admits, so bins are
  // compared there.
  const bool collect = in_b1 <= (uint32_t)kCand;
  float lo, hi;
  bin_bounds(b1, lo, hi);
  auto classify = [&](float x, bool valid, bool& gt, bool& eq) {
    if (b1 != 0) {
      gt = valid && x > hi;
      eq = valid && !gt && x >= lo;
    } else {
      const uint32_t b = valid ? score_bin(x) : 0u;
      gt = valid && b > b1;
      eq = valid && b == b1;
    }
    eq = eq && collect;
  };
  if (tid < 32) {  // the scalar head and tail in warp 0
    const bool mine = tid < n_edge;
    const int i = tid < n_head ? tid : t0 + (tid - n_head);
    const float x = mine ? __ldg(row + i) : 0.f;
    bool gt, eq;
    classify(x, mine, gt, eq);
    uint32_t slot;
    if (warp_append(gt, &sm.n_out, slot) && gt) out[slot] = i;
    if (warp_append(eq, &sm.n_cand, slot) && eq) {
      ckey[slot] = rank_key(x);
      cpos[slot] = i;
    }
  }
  // four scores per vector: above b1 -> written out (one atomic per warp and
  // vector), members of b1 -> candidates (rare: per-score appends)
  const uint32_t lt = (1u << lane) - 1u;
  for (int base = 0; base < n4; base += kBatchRow * kThreads) {  // uniform trip count
    float4 xv[kBatchRow];
#pragma unroll
    for (int u = 0; u < kBatchRow; ++u) {
      const int v = base + u * kThreads + tid;
      xv[u] = v < n4 ? __ldg(row4 + v) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < kBatchRow; ++u) {
      const int v = base + u * kThreads + tid;
      const float xs[4] = {xv[u].x, xv[u].y, xv[u].z, xv[u].w};
      bool gt[4], eq[4];
      bool any_eq = false;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        classify(xs[e], v < n4, gt[e], eq[e]);
        any_eq |= eq[e];
      }
      uint32_t g[4], tot = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        g[e] = __ballot_sync(0xffffffffu, gt[e]);
        tot += __popc(g[e]);
      }
      if (tot) {
        uint32_t slot = 0;
        if (lane == 0) slot = atomicAdd(&sm.n_out, tot);
        slot = __shfl_sync(0xffffffffu, slot, 0);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if (gt[e]) out[slot + __popc(g[e] & lt)] = a0 + 4 * v + e;
          slot += __popc(g[e]);
        }
      }
      if (__any_sync(0xffffffffu, any_eq)) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          uint32_t slot;
          if (warp_append(eq[e], &sm.n_cand, slot) && eq[e]) {
            ckey[slot] = rank_key(xs[e]);
            cpos[slot] = a0 + 4 * v + e;
          }
        }
      }
    }
  }
  __syncthreads();

  if (collect) {
    rank_candidates(sm, ckey, cpos, (int)in_b1, need, out + above1);
    return;
  }

  resolve_by_row(sm, row, n, k, b1, above1, out);
}

// ---------------------------------------------------------------- split rows
// Few long rows (decode) leave most SMs idle with one CTA per row, so each
// row is split over a cluster of P CTAs.  Each histograms its slice;
// the slices' histograms are summed into the leader's (CTA 0) through
// distributed shared memory (a reduction per non-empty bin), and the leader
// fixes b1.  Each CTA then filters its slice into local buffers -- scores
// above b1, and b1's members -- reserves space with one remote atomic on the
// leader's counters, writes its scores above b1 to the output and its
// candidates into the leader's buffer.  The leader ranks the candidates (or
// resolves an overflowing b1 from the row) exactly as the one-CTA kernel.

__device__ __forceinline__ uint32_t cl_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cl_map(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
               : "=r"(r)
               : "r"((uint32_t)__cvta_generic_to_shared(p)), "r"(rank));
  return r;
}
__device__ __forceinline__ void cl_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}
__device__ __forceinline__ void cl_red_add(uint32_t addr, uint32_t v) {
  asm volatile("red.shared::cluster.add.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t cl_atom_add(uint32_t addr, uint32_t v) {
  uint32_t old;
  asm volatile("atom.shared::cluster.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(addr), "r"(v) : "memory");
  return old;
}
__device__ __forceinline__ uint32_t cl_ld(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ void cl_st(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

template <int P>
__global__ void __cluster_dims__(P, 1, 1) __launch_bounds__(kThreads, 2)
    topk_split_kernel(Rows R, int32_t row0, const float* scores, int64_t ld, int k,
                      int32_t* idx) {
  extern __shared__ uint32_t dyn[];
  uint32_t* ckey = dyn;                                      // [kCand] this slice's candidates
  int32_t* cpos = reinterpret_cast<int32_t*>(dyn + kCand);   // [kCand]
  uint32_t* mkey = dyn + 2 * kCand;                          // [kCand] leader: the row's candidates
  int32_t* mpos = reinterpret_cast<int32_t*>(dyn + 3 * kCand);  // [kCand]
  __shared__ int32_t gpos[kCand];                            // this slice's scores above b1
  __shared__ Smem sm;
  __shared__ uint32_t info[4];  // leader: b1, above1, |b1|; every CTA: its two reservations
  __shared__ uint32_t local_gt, local_cand;
  const int tid = threadIdx.x, lane = tid & 31;
  const uint32_t crank = cl_rank();
  const int32_t rloc = blockIdx.x / P;
  const RowInfo ri = row_info(R, row0 + rloc);
  const int n = ri.t + 1;
  int32_t* out = idx + (int64_t)rloc * k;
  if (n <= k) {  // the same for every CTA of the cluster
    if (crank == 0)
      for (int i = tid; i < k; i += kThreads) out[i] = i < n ? i : -1;
    return;
  }
  const float* row = scores + (int64_t)rloc * ld;
  const int chunk = ((n + P - 1) / P + 3) & ~3;
  const int p0 = min(n, (int)crank * chunk), p1 = min(n, p0 + chunk);
  // The slice as a scalar head up to the first 16-byte boundary, m4 float4
  // vectors from a0, and a scalar tail from t0 (row strides need not be
  // multiples of four floats).
  const int a0 = min(
      p1, p0 + (int)((4u - (uint32_t)((reinterpret_cast<uintptr_t>(row + p0) >> 2) & 3u)) & 3u));
  const int m4 = (p1 - a0) >> 2, t0 = a0 + 4 * m4;
  const int n_head = a0 - p0, n_edge = n_head + (p1 - t0);  // <= 6 scalar scores
  const float4* s4 = reinterpret_cast<const float4*>(row + a0);

  // ------------------------------------------------------------ slice histogram
  for (int i = tid; i < kBins; i += kThreads) sm.hist[i] = 0;
  if (tid == 0) {
    sm.n_out = 0;  // leader: output slots reserved so far
    sm.n_cand = 0;  // leader: candidate slots reserved so far
    local_gt = 0;
    local_cand = 0;
  }
  __syncthreads();
  if (tid < n_edge) {
    const int i = tid < n_head ? p0 + tid : t0 + (tid - n_head);
    atomicAdd(&sm.hist[score_bin(__ldg(row + i))], 1u);
  }
  for (int base = tid; base < m4; base += kBatch * kThreads) {
    float4 xv[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int v = base + u * kThreads;
      if (v < m4) xv[u] = __ldg(s4 + v);
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int v = base + u * kThreads;
      const float xs[4] = {xv[u].x, xv[u].y, xv[u].z, xv[u].w};
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (v < m4) atomicAdd(&sm.hist[score_bin(xs[e])], 1u);
    }
  }
  __syncthreads();
  cl_sync();  // every slice histogram complete
  if (crank != 0)
    for (int b = tid; b < kBins; b += kThreads) {
      const uint32_t c = sm.hist[b];
      if (c) cl_red_add(cl_map(&sm.hist[b], 0), c);
    }
  cl_sync();  // the leader holds the row's histogram
  if (crank == 0) {
    find_bin(sm, kBins, (uint32_t)k);
    if (tid == 0) {
      info[0] = sm.sel_bin;
      info[1] = sm.sel_above;
      info[2] = sm.hist[sm.sel_bin];
    }
  }
  cl_sync();
  if (tid < 3) info[tid] = cl_ld(cl_map(&info[tid], 0));
  __syncthreads();
  const uint32_t b1 = info[0], above1 = info[1], in_b1 = info[2];
  const bool collect = in_b1 <= (uint32_t)kCand;
  __syncthreads();  // info[0..2] read before the reservations reuse it

  // ------------------------------------------------------------ filter the slice
  float lo, hi;
  bin_bounds(b1, lo, hi);
  // score i of the slice is above b1 / a member of b1 (the -inf bin 0 holds
  // NaN too, which no float comparison admits: compare bins there)
  auto classify = [&](float x, bool valid, bool& gt, bool& eq) {
    if (b1 != 0) {
      gt = valid && x > hi;
      eq = valid && !gt && x >= lo;
    } else {
      const uint32_t b = valid ? score_bin(x) : 0u;
      gt = valid && b > b1;
      eq = valid && b == b1;
    }
    eq = eq && collect;
  };
  // the scalar head and tail (at most six scores) in warp 0
  if (tid < 32) {
    const bool mine = tid < n_edge;
    const int i = tid < n_head ? p0 + tid : t0 + (tid - n_head);
    const float x = mine ? __ldg(row + i) : 0.f;
    bool gt, eq;
    classify(x, mine, gt, eq);
    uint32_t slot;
    if (warp_append(gt, &local_gt, slot) && gt) gpos[slot] = i;
    if (warp_append(eq, &local_cand, slot) && eq) {
      ckey[slot] = rank_key(x);
      cpos[slot] = i;
    }
  }
  for (int base = 0; base < m4; base += kBatch * kThreads) {  // uniform trip count
    float4 xv[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int v = base + u * kThreads + tid;
      xv[u] = v < m4 ? __ldg(s4 + v) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    // classify the batch into two bit masks, then reserve the slots of the
    // whole warp's batch with one atomic per list (lane 0), the lanes
    // taking consecutive ranges by a prefix sum of their counts
    uint32_t gtm = 0, eqm = 0;
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int v = base + u * kThreads + tid;
      const float xs[4] = {xv[u].x, xv[u].y, xv[u].z, xv[u].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        bool gt, eq;
        classify(xs[e], v < m4, gt, eq);
        gtm |= (gt ? 1u : 0u) << (4 * u + e);
        eqm |= (eq ? 1u : 0u) << (4 * u + e);
      }
    }
    const uint32_t own = (uint32_t)__popc(gtm) | ((uint32_t)__popc(eqm) << 16);
    uint32_t incl = own;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const uint32_t tot = __shfl_sync(0xffffffffu, incl, 31);
    if (!tot) continue;  // warp-uniform
    uint32_t wb = 0;
    if (lane == 0) {
      const uint32_t bg = (tot & 0xffffu) ? atomicAdd(&local_gt, tot & 0xffffu) : 0u;
      const uint32_t be = (tot >> 16) ? atomicAdd(&local_cand, tot >> 16) : 0u;
      wb = bg | (be << 16);  // both below kCand
    }
    wb = __shfl_sync(0xffffffffu, wb, 0) + (incl - own);
    uint32_t sg = wb & 0xffffu, se = wb >> 16;
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int v = base + u * kThreads + tid;
      const float xs[4] = {xv[u].x, xv[u].y, xv[u].z, xv[u].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = a0 + 4 * v + e;
        if ((gtm >> (4 * u + e)) & 1u) gpos[sg++] = i;  // < above1 < k <= kCand
        if ((eqm >> (4 * u + e)) & 1u) {
          ckey[se] = rank_key(xs[e]);
          cpos[se++] = i;
        }
      }
    }
  }
  __syncthreads();
  const uint32_t ngt = local_gt, ncand = local_cand;
  if (tid == 0) {
    info[0] = cl_atom_add(cl_map(&sm.n_out, 0), ngt);
    info[1] = ncand ? cl_atom_add(cl_map(&sm.n_cand, 0), ncand) : 0u;
  }
  __syncthreads();
  const uint32_t base_gt = info[0], base_c = info[1];
  for (uint32_t j = tid; j < ngt; j += kThreads) out[base_gt + j] = gpos[j];
  for (uint32_t j = tid; j < ncand; j += kThreads) {
    cl_st(cl_map(&mkey[base_c + j], 0), ckey[j]);
    cl_st(cl_map(&mpos[base_c + j], 0), (uint32_t)cpos[j]);
  }
  cl_sync();  // every score above b1 written, every candidate with the leader

  if (crank == 0) {
    if (collect)
      rank_candidates(sm, mkey, mpos, (int)in_b1, (uint32_t)k - above1, out + above1);
    else
      resolve_by_row(sm, row, n, k, b1, above1, out);  // sm.n_out == above1 here
  }
}

// The rows' k best from the candidate lists of the fused decode indexer
// (indexer_decode_kernel with SEL): one CTA per row.  A row's list is in
// segments: the segment that starts at key tile j holds segcnt[j] entries at
// cand[j * 128 ...].  The row's histogram, built by the indexer over all its
// scores, fixes the bin b1 of the k-th best; the segments hold every score of
// b1 and above, from which the k best are written as select_list does.  Rows
// with n <= k candidates take 0 .. n-1.
constexpr int kMaxSeg = 1024;  // segments a row can have (one per key tile at most)
__global__ void __launch_bounds__(kThreads, 1)
    select_rows_kernel(Rows R, int32_t row0, const uint64_t* __restrict__ cand, int64_t cap,
                       const uint32_t* __restrict__ segcnt, const uint32_t* __restrict__ rhist,
                       int k, int32_t* __restrict__ idx) {
  __shared__ uint32_t ckey[kCand];
  __shared__ int32_t cpos[kCand];
  __shared__ Smem sm;
  __shared__ uint32_t seg_first[kMaxSeg];  // entry offset of the segment's list in the row
  __shared__ uint32_t seg_pre[kMaxSeg + 1];  // candidates before the segment
  __shared__ int nseg;
  const int tid = threadIdx.x, lane = tid & 31;
  const int32_t r = blockIdx.x;
  const RowInfo ri = row_info(R, row0 + r);
  const int n = ri.t + 1;
  int32_t* out = idx + (int64_t)r * k;
  if (n <= k) {
    for (int i = tid; i < k; i += kThreads) out[i] = i < n ? i : -1;
    return;
  }
  // the row's segments, in tile order (a warp-wide scan of the tile counts)
  const int ntile = (int)((n + 127) / 128);
  const uint32_t* sc = segcnt + (int64_t)r * (cap / 128);
  if (tid < 32) {
    uint32_t total = 0;
    int ns = 0;
    for (int j0 = 0; j0 < ntile && j0 < kMaxSeg; j0 += 32) {
      const int j = j0 + lane;
      const uint32_t c = j < ntile ? __ldcg(sc + j) : 0u;
      const uint32_t nz = __ballot_sync(0xffffffffu, c != 0);
      uint32_t incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (c) {
        const int slot = ns + __popc(nz & ((1u << lane) - 1u));
        seg_first[slot] = (uint32_t)j * 128u;
        seg_pre[slot] = total + incl - c;
      }
      total += __shfl_sync(0xffffffffu, incl, 31);
      ns += __popc(nz);
    }
    if (lane == 0) {
      seg_pre[ns] = total;
      nseg = ns;
    }
  }
  const uint32_t* h = rhist + (int64_t)r * kBins;
  for (int i = tid; i < kBins; i += kThreads) sm.hist[i] = __ldcg(h + i);
  __syncthreads();
  const int ns = nseg;
  const uint32_t m = seg_pre[ns];
  const unsigned long long* row = reinterpret_cast<const unsigned long long*>(cand + (int64_t)r * cap);
  // entry i of the row's list: its segment by binary search over the prefix counts
  auto get = [&](uint32_t i) -> uint64_t {
    int lo = 0, hi = ns - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (seg_pre[mid] <= i) lo = mid; else hi = mid - 1;
    }
    return __ldcg(row + seg_first[lo] + (i - seg_pre[lo]));
  };
  sel::select_list<B512>(sm, get, m, k, out, ckey, cpos, true);
}

}  // namespace

dsa_status_t launch_select_rows(const Rows& R, int32_t row0, int32_t nrows, const uint64_t* cand,
                                int64_t cap, const uint32_t* segcnt, const uint32_t* rhist, int k,
                                int32_t* idx, cudaStream_t st) {
  if (nrows <= 0) return DSA_OK;
  if (cap / 128 > kMaxSeg || cap % 128) return DSA_ERR_UNSUPPORTED;
  select_rows_kernel<<<nrows, kThreads, 0, st>>>(R, row0, cand, cap, segcnt, rhist, k, idx);
  return launch_status();
}

dsa_status_t launch_topk(const Rows& R, int32_t row0, int32_t nrows, const float* scores,
                         int64_t ld, int k, int32_t* idx, cudaStream_t st) {
  if (nrows <= 0) return DSA_OK;
  // Few long rows: one cluster of 4 or 8 CTAs per row (8 while all the
  // clusters fit one wave at two CTAs per SM); otherwise one CTA per row,
  // several per SM.
  if (k <= kCand && nrows * 4 <= 4 * num_sms() && R.max_len >= 8 * k) {
    const size_t smem = 4 * kCand * sizeof(uint32_t);  // + static: above the 48 KB default
    const bool eight = nrows * 8 <= 2 * num_sms() && R.max_len >= 16 * k;
    auto kfn = eight ? topk_split_kernel<8> : topk_split_kernel<4>;
    if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return DSA_ERR_CUDA;
    kfn<<<nrows * (eight ? 8 : 4), kThreads, smem, st>>>(R, row0, scores, ld, k, idx);
    return launch_status();
  }
  topk_kernel<<<nrows, kThreads, 0, st>>>(R, row0, scores, ld, k, idx);
  return launch_status();
}

}  // namespace dsa
