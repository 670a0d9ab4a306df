// Per-query top-k selection: a radix select on order-preserving keys.
//
// "Sparse Attention Architecture Evolution in LLMs" (Top-K Selection): each
// query keeps k positions (k = 2048); "GLM sparse attention" (threshold
// figure): the cut-off is the k-th best score.  Ties go to the lower
// position; -0 == +0; NaN ranks as -inf.
//
// One CTA owns a row.  Scores become 32-bit keys whose unsigned order is
// the float order.  Three histogram passes (11 + 11 + 10 bits) pin down the
// exact key tau of the k-th best element and the number c_gt of elements
// strictly above it; a final pass writes every element above tau (any
// order) and the first k - c_gt elements equal to tau in position order,
// the latter through a block-wide ordered compaction (ballot + warp prefix
// + a scan of warp totals).  When the row fits, the first pass parks the
// keys in shared memory and the later passes never touch global memory.
#include "kernels.cuh"

namespace dsa {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 2048;
// Largest row cached in shared memory (keys): 48K entries = 192 KB.
constexpr int kCacheCap = 48 * 1024;

__device__ __forceinline__ uint32_t rank_key(float x) {
  uint32_t u = __float_as_uint(x);
  if ((u & 0x7fffffffu) > 0x7f800000u) u = 0xff800000u;  // NaN -> -inf
  if (u == 0x80000000u) u = 0u;                          // -0 -> +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct Smem {
  uint32_t hist[kBins];
  uint32_t warp_tot[kWarps];
  uint32_t sel_bin;
  uint32_t sel_above;
  uint32_t gt_pos;
};

// Given hist[0..nbins) and the number `need` of elements still to take,
// finds bin b with above(b) < need <= above(b) + hist[b], where above(b) is
// the count in bins > b.  Result in sm.sel_bin / sm.sel_above.
__device__ void find_bin(Smem& sm, int nbins, uint32_t need) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = nbins / kThreads;  // 4 or 2 contiguous bins per thread
  const int b0 = tid * per;
  uint32_t local = 0;
  for (int i = 0; i < per; ++i) local += sm.hist[b0 + i];
  // suffix sum over threads: elements in bins owned by higher threads
  uint32_t incl = local;  // inclusive suffix inside the warp (lanes >= lane)
  for (int off = 1; off < 32; off <<= 1) {
    uint32_t v = __shfl_down_sync(0xffffffffu, incl, off);
    if (lane + off < 32) incl += v;
  }
  if (lane == 0) sm.warp_tot[warp] = incl;
  __syncthreads();
  uint32_t above = incl - local;
  for (int w2 = warp + 1; w2 < kWarps; ++w2) above += sm.warp_tot[w2];
  for (int i = per - 1; i >= 0; --i) {
    uint32_t h = sm.hist[b0 + i];
    if (above < need && need <= above + h) {
      sm.sel_bin = (uint32_t)(b0 + i);
      sm.sel_above = above;
    }
    above += h;
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kThreads) topk_kernel(Rows R, int32_t row0, const float* scores,
                                                        int64_t ld, int k, int32_t* idx,
                                                        int cache_cap) {
  extern __shared__ uint32_t cache[];
  __shared__ Smem sm;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int32_t r = row0 + blockIdx.x;
  const RowInfo ri = row_info(R, r);
  const int n = ri.t + 1;
  int32_t* out = idx + (int64_t)blockIdx.x * k;
  if (n <= k) {
    for (int i = tid; i < k; i += kThreads) out[i] = i < n ? i : -1;
    return;
  }
  const float* row = scores + (int64_t)blockIdx.x * ld;
  const bool cached = n <= cache_cap;
  auto key_at = [&](int i) -> uint32_t { return cached ? cache[i] : rank_key(__ldg(row + i)); };

  // pass 1: top 11 bits
  for (int i = tid; i < kBins; i += kThreads) sm.hist[i] = 0;
  if (tid == 0) sm.gt_pos = 0;
  __syncthreads();
  for (int i = tid; i < n; i += kThreads) {
    uint32_t u = rank_key(__ldg(row + i));
    if (cached) cache[i] = u;
    atomicAdd(&sm.hist[u >> 21], 1u);
  }
  __syncthreads();
  find_bin(sm, kBins, (uint32_t)k);
  const uint32_t b1 = sm.sel_bin;
  uint32_t above = sm.sel_above;
  __syncthreads();

  // pass 2: middle 11 bits among keys whose top bits are b1
  for (int i = tid; i < kBins; i += kThreads) sm.hist[i] = 0;
  __syncthreads();
  for (int i = tid; i < n; i += kThreads) {
    uint32_t u = key_at(i);
    if ((u >> 21) == b1) atomicAdd(&sm.hist[(u >> 10) & 0x7ffu], 1u);
  }
  __syncthreads();
  find_bin(sm, kBins, (uint32_t)k - above);
  const uint32_t pre2 = (b1 << 11) | sm.sel_bin;
  above += sm.sel_above;
  __syncthreads();

  // pass 3: low 10 bits among keys whose top 22 bits are pre2
  for (int i = tid; i < kBins; i += kThreads) sm.hist[i] = 0;
  __syncthreads();
  for (int i = tid; i < n; i += kThreads) {
    uint32_t u = key_at(i);
    if ((u >> 10) == pre2) atomicAdd(&sm.hist[u & 0x3ffu], 1u);
  }
  __syncthreads();
  find_bin(sm, 1024, (uint32_t)k - above);
  const uint32_t tau = (pre2 << 10) | sm.sel_bin;
  const uint32_t c_gt = above + sm.sel_above;  // elements strictly above tau
  const uint32_t need_eq = (uint32_t)k - c_gt;  // >= 1
  __syncthreads();

  // pass 4: emit. Elements above tau in any order at [0, c_gt); the first
  // need_eq elements equal to tau, in position order, at [c_gt, k).
  uint32_t eq_base = 0;
  for (int base = 0; base < n; base += kThreads) {
    const int i = base + tid;
    const uint32_t u = i < n ? key_at(i) : 0u;
    const bool gt = i < n && u > tau;
    const bool eq = i < n && u == tau;
    const uint32_t gmask = __ballot_sync(0xffffffffu, gt);
    if (gmask) {
      uint32_t wbase = 0;
      if (lane == 0) wbase = atomicAdd(&sm.gt_pos, (uint32_t)__popc(gmask));
      wbase = __shfl_sync(0xffffffffu, wbase, 0);
      if (gt) out[wbase + __popc(gmask & ((1u << lane) - 1u))] = i;
    }
    if (eq_base < need_eq) {  // uniform across the block
      const uint32_t emask = __ballot_sync(0xffffffffu, eq);
      if (lane == 0) sm.warp_tot[warp] = (uint32_t)__popc(emask);
      __syncthreads();
      uint32_t before = 0, total = 0;
      for (int w2 = 0; w2 < kWarps; ++w2) {
        uint32_t c = sm.warp_tot[w2];
        if (w2 < warp) before += c;
        total += c;
      }
      const uint32_t rank = eq_base + before + __popc(emask & ((1u << lane) - 1u));
      if (eq && rank < need_eq) out[c_gt + rank] = i;
      eq_base += total;
      __syncthreads();
    }
  }
}

}  // namespace

dsa_status_t launch_topk(const Rows& R, int32_t row0, int32_t nrows, const float* scores,
                         int64_t ld, int k, int32_t* idx, cudaStream_t st) {
  if (nrows <= 0) return DSA_OK;
  // Rows up to cache_cap entries are parked in shared memory; longer rows
  // stream from global memory (L2) on every pass.
  const int cache_cap = R.max_len < kCacheCap ? R.max_len : kCacheCap;
  const size_t cache_bytes = (size_t)cache_cap * 4;
  if (cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)cache_bytes) != cudaSuccess)
    return DSA_ERR_CUDA;
  topk_kernel<<<nrows, kThreads, cache_bytes, st>>>(R, row0, scores, ld, k, idx, cache_cap);
  return launch_status();
}

}  // namespace dsa
