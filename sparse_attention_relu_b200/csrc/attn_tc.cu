// Sparse MLA attention on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// For query row r, head h and the selected positions S_r (k slots, -1 = empty):
//   z[h,s] = sm_scale * <q[r,h,0:576], C[s,0:576]>
//   o[r,h] = sum_s softmax_S(z[h,:])_s * C[s,0:512],   lse = log sum_s exp z
// ("GLM sparse attention", MLA passage: one cached latent row (512 latent +
// 64 rotary) per token, scored by the absorbed query of every head, so one
// gathered row serves all 128 heads; exact softmax over the survivors; the
// selected positions are scattered, so the gather must be efficient.)
//
// TMEM holds 128 lanes x 512 fp32 columns, exactly the size of the 128 x 512
// output accumulator, leaving no room for the score tile.  Each query row
// therefore runs on a 2-CTA cluster that splits both contractions without
// duplicating work:
//   CTA c computes the partial scores over its half of the 576-d contraction
//   (dims 288c .. 288c+287) and the output for its half of the 512 value
//   columns (256c .. 256c+255).
// The two partial score tiles are summed through distributed shared memory
// (IEEE addition commutes, so both CTAs hold bit-identical scores and make
// identical softmax decisions).
//
// Per CTA: the gathered tile holds the 5 swizzle atoms (64 columns each)
// 4c .. 4c+4 of 64 selected rows, fetched with 16-byte cp.async by 64
// producer threads, one row each, written straight into the 128-byte
// swizzled layout the MMA reads (an empty slot is zero-filled); 4 such
// stages are in flight.  Measured on B200: one thread issuing TMA
// tile::gather4 (4 rows per instruction) needs about 9.3K cycles per such
// tile, the spread cp.async gather a fraction of it.
//
// Both products take their A operand from TMEM (the .ts form), so shared
// memory holds only gathered rows and the exchange buffers:
//   columns   0..143  the CTA's 288 query dims of every head, bf16 pairs
//   columns 160..223  the 64-column partial score tile (fp32)
//   columns 224..255  P, the tile's probabilities as bf16 pairs
//   columns 256..511  the 256-column output accumulator
//
// Warp roles (352 threads per CTA):
//   warps 0-1  gather producer (indices -> shared memory, cp.async rows)
//   warp 2     TMEM allocator and MMA issuer (one thread, issues whichever of
//              QK(next tile) and PV(oldest tile with P ready) can go)
//   warps 3-10 softmax, two warpgroups: a thread owns one head (its TMEM lane)
//              and half of each tile's 64 rows.  Software-pipelined: tile
//              n+1's partial scores leave for the peer before tile n's
//              softmax runs (double-buffered exchange).  Online softmax in
//              the log2 domain with a lazy rescale (the reference max moves
//              only when a new score exceeds it by more than 2^8), P to TMEM
//              as bf16, final normalisation and store.
// Decode rows are split over several clusters; each writes a normalised
// partial output and its log-sum-exp, merged by attn_combine_kernel.
#include <cudaTypedefs.h>

#include "kernels.cuh"
#include "sm100.cuh"

namespace dsa {

using namespace sm100;

namespace {

constexpr int kH = 128, kDK = 576, kDV = 512;
constexpr int kNT = 64;         // selected rows per tile
constexpr int kProducers = 64;  // warps 0-1
constexpr int kSoftmax0 = 96;   // first softmax thread (warps 3-10)
constexpr int kSoftmaxThreads = 256;
constexpr int kThreads = kSoftmax0 + kSoftmaxThreads;  // 352
constexpr int kAtoms = 5;       // 64-column atoms held per CTA
constexpr int kCBytes = kAtoms * kNT * 128;   // 40960 per stage
constexpr int kStages = 4;
constexpr int kXBytes = kH * kNT * 4;         // 32768 per exchange buffer
constexpr int OFF_C = 0;
constexpr int OFF_X = OFF_C + kStages * kCBytes;         // [2] exchange buffers
constexpr int OFF_IDX = OFF_X + 2 * kXBytes;             // [stage][64] int32
constexpr int OFF_MASK = OFF_IDX + kStages * kNT * 4;    // [stage][2] uint32 validity bits
constexpr int OFF_HMAX = OFF_MASK + kStages * 2 * 4;     // [2 warpgroups][128] float
constexpr int OFF_BAR = OFF_HMAX + 2 * kH * 4;
constexpr int kNumBars = 20;
constexpr int OFF_MISC = OFF_BAR + kNumBars * 8;
// The dynamic window starts 1024-aligned (right after the driver's reserved
// kilobyte, with no static shared memory); the kernel checks it.
constexpr int kSmem = OFF_MISC + 16;
static_assert(kSmem <= 232448, "shared memory");
// TMEM columns
constexpr uint32_t TM_Q = 0;     // the CTA's 288 query dims of all heads, bf16 pairs (144 cols)
constexpr uint32_t TM_S = 160;   // 64-column score tile
constexpr uint32_t TM_P = 224;   // 32-column bf16 P tile (the PV A operand)
constexpr uint32_t TM_O = 256;   // 256-column output accumulator
constexpr uint32_t IDESC_QK = idesc(1, 128, kNT);
constexpr uint32_t IDESC_PV = idesc(1, 128, 256, false, true);
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescale = 8.0f;  // log2 headroom before the reference max moves

enum {
  B_QREADY = 0,  // the query is in TMEM (every softmax thread)
  B_CFULL = 1,   // [4] stage rows landed (producers)
  B_CEMPTY = 5,  // [4] PV of the stage retired
  B_SFULL = 9,   // QK retired
  B_SEMPTY = 10, // scores read (every softmax thread)
  B_PFULL = 11,  // P stored in TMEM (every softmax thread)
  B_PVDONE = 12, // PV retired
  B_XFULL = 13,  // [2] the peer's partial scores arrived
  B_XEMPTY = 15, // [2] the peer read our partial scores
  B_DRAIN = 17
};

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}
__device__ __forceinline__ uint32_t map_peer(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void st_cluster_v4(uint32_t addr, float a, float b, float c, float d) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b),
               "f"(c), "f"(d)
               : "memory");
}
__device__ __forceinline__ void arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
__device__ __forceinline__ bool try_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait with cluster-scope acquire (data written by the peer CTA).
__device__ __forceinline__ bool wait_cluster(uint32_t bar, uint32_t parity, unsigned* status) {
  if (try_cluster(bar, parity)) return true;
  const long long t0 = clock64();
  while (!try_cluster(bar, parity)) {
    if (clock64() - t0 > kSpinLimit) {
      atomicOr(status, kErrTimeout);
      return false;
    }
  }
  return true;
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n\t"
      "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
      "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]),
      "f"(v[8]), "f"(v[9]), "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]),
      "f"(v[15]), "f"(v[16]), "f"(v[17]), "f"(v[18]), "f"(v[19]), "f"(v[20]), "f"(v[21]),
      "f"(v[22]), "f"(v[23]), "f"(v[24]), "f"(v[25]), "f"(v[26]), "f"(v[27]), "f"(v[28]),
      "f"(v[29]), "f"(v[30]), "f"(v[31])
      : "memory");
}
// MMA with the A operand in TMEM (rows in lanes, 16-bit K pairs per column).
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b,
                                            uint32_t id, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(id), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&v)[8]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};\n\t"
      "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
      : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n\t"
      "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15])
      : "memory");
}

// Named barrier `id` over `n` threads, returning the AND of `v` (every
// participant must reach it, so failures are folded in rather than
// branched around).
template <int ID, int N>
__device__ __forceinline__ bool bar_and(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "n"(ID), "n"(N)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&p);
}

struct Split {
  int nsplit, tiles_per_split;
};

__host__ __device__ inline Split plan_split(int32_t nrows, int k) {
  const int tiles = (k + kNT - 1) / kNT;
  int want = nrows >= 148 ? 1 : (148 + nrows - 1) / nrows;
  if (want > tiles) want = tiles;
  if (want < 1) want = 1;
  Split s;
  s.tiles_per_split = (tiles + want - 1) / want;
  s.nsplit = (tiles + s.tiles_per_split - 1) / s.tiles_per_split;
  return s;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ kv, Rows R,
                   int32_t row0, const int32_t* __restrict__ idx, int k, float scale2, Split sp,
                   uint16_t* __restrict__ out, float* __restrict__ lse,
                   float* __restrict__ part_o, float* __restrict__ part_lse) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  const uint32_t sb = smem_u32(smem);
  if (sb & 1023u) {  // the swizzled operand layouts need 1024-byte alignment
    if (threadIdx.x == 0) raise_status(R, kErrLayout);
    return;  // uniform across the cluster: both CTAs share the layout
  }
  int32_t* sidx = reinterpret_cast<int32_t*>(smem + OFF_IDX);
  uint32_t* vmask = reinterpret_cast<uint32_t*>(smem + OFF_MASK);
  float* hmax = reinterpret_cast<float*>(smem + OFF_HMAX);
  auto bar = [&](int i) { return sb + OFF_BAR + 8u * i; };
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t crank = cluster_rank(), peer = crank ^ 1u;
  const int item = blockIdx.x >> 1;
  const int32_t rloc = item / sp.nsplit, split = item % sp.nsplit;
  const int32_t r = row0 + rloc;
  const RowInfo ri = row_info(R, r);
  const int slot_lo = split * sp.tiles_per_split * kNT;
  const int slot_hi = min(k, slot_lo + sp.tiles_per_split * kNT);
  const int ntiles = slot_hi > slot_lo ? (slot_hi - slot_lo + kNT - 1) / kNT : 0;

  if (tid == 0) {
    mbar_init(bar(B_QREADY), kSoftmaxThreads);
    for (int i = 0; i < kStages; ++i) {
      // per producer: a release-arrive after its index store and a cp.async arrive
      mbar_init(bar(B_CFULL + i), 2 * kProducers);
      mbar_init(bar(B_CEMPTY + i), 1);
    }
    mbar_init(bar(B_SFULL), 1);
    mbar_init(bar(B_SEMPTY), kSoftmaxThreads);
    mbar_init(bar(B_PFULL), kSoftmaxThreads);
    mbar_init(bar(B_PVDONE), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(B_XFULL + i), 1);  // one release-arrive from the peer per tile
      mbar_init(bar(B_XEMPTY + i), 1);
    }
    mbar_init(bar(B_DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(sb + OFF_MISC, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 2) {
    // ------------------------------------------------------------ gather producer
    const uint16_t* kvb = kv + ri.kbase * kDK + 256 * crank;  // atoms 4c .. 4c+4
    auto load_idx = [&](int n) -> int32_t {
      const int slot = slot_lo + n * kNT + tid;
      int32_t s = slot < slot_hi ? __ldg(idx + (int64_t)rloc * k + slot) : -1;
      if (s < -1 || s >= ri.len || ri.t < 0) {
        if (s != -1 && ri.t >= 0) raise_status(R, kErrBadIndex);
        s = -1;
      }
      return s;
    };
    // A warp instruction copies 4 rows x 128 contiguous bytes: lanes 8g..8g+7
    // take the 16-byte chunks of row 4j+g of this warp's 32 rows.
    const int sub = lane >> 3, ch = lane & 7;
    int32_t pre = ntiles > 0 ? load_idx(0) : -1;
    for (int n = 0; n < ntiles; ++n) {
      const int st = n % kStages;
      const bool ok = mbar_wait(bar(B_CEMPTY + st), ((n / kStages) & 1) ^ 1, R.status) &&
                      !*abort_flag;
      if (!bar_and<2, kProducers>(ok)) {
        *abort_flag = 1;
        break;
      }
      sidx[st * kNT + tid] = pre;
      const uint32_t bits = __ballot_sync(0xffffffffu, pre >= 0);
      if (lane == 0) vmask[st * 2 + warp] = bits;
      mbar_arrive(bar(B_CFULL + st));  // publishes indices and mask to the softmax threads
      asm volatile("bar.sync 2, 64;" ::: "memory");  // every producer sees the tile's indices
      pre = n + 1 < ntiles ? load_idx(n + 1) : -1;    // overlaps the copies below
      const uint32_t cb = sb + OFF_C + st * kCBytes;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int row = warp * 32 + 4 * j + sub;
        const int32_t s = sidx[st * kNT + row];
        const char* src = reinterpret_cast<const char*>(s >= 0 ? kvb + (int64_t)s * kDK : kv);
        const uint32_t nbytes = s >= 0 ? 16u : 0u;  // 0: zero-fill
        const uint32_t dst = cb + row * 128 + ((uint32_t)(ch ^ (row & 7)) << 4);
#pragma unroll
        for (int la = 0; la < kAtoms; ++la)
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst + la * kNT * 128),
                       "l"(src + (la * 64 + ch * 8) * 2), "r"(nbytes)
                       : "memory");
      }
      // arrives on the stage barrier once this thread's copies have landed
      asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar(B_CFULL + st))
                   : "memory");
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
  } else if (warp == 2) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(bar(B_QREADY), 0, R.status);
      // Issue whichever is ready: QK of the next tile (rows landed, score
      // tile free) or PV of the oldest tile whose P is in TMEM.  PV never
      // waits for a later tile's rows.
      int nq = 0, np = 0;
      long long t0 = clock64();
      while (ok && np < ntiles) {
        if (*abort_flag) {
          ok = false;
          break;
        }
        bool progressed = false;
        if (nq < ntiles) {
          const int st = nq % kStages;
          if (mbar_try(bar(B_CFULL + st), (nq / kStages) & 1) &&
              mbar_try(bar(B_SEMPTY), (nq & 1) ^ 1)) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // cp.async rows
            tc_fence_after();
            const uint32_t cb = sb + OFF_C + st * kCBytes;
#pragma unroll
            for (int kk = 0; kk < 18; ++kk) {
              const int e = 288 * (int)crank + 16 * kk;  // global contraction index
              const int la = e / 64 - 4 * (int)crank, off = (e % 64) * 2;
              mma_bf16_ts(tmem + TM_S, tmem + TM_Q + 8 * kk,
                          desc_sw128(cb + la * kNT * 128 + off, 1024), IDESC_QK, kk > 0 ? 1u : 0u);
            }
            mma_commit(bar(B_SFULL));
            ++nq;
            progressed = true;
          }
        }
        if (np < nq) {
          if (mbar_try(bar(B_PFULL), np & 1)) {
            tc_fence_after();
            const uint32_t cb = sb + OFF_C + (np % kStages) * kCBytes;  // stage of tile np
#pragma unroll
            for (int kk = 0; kk < kNT / 16; ++kk)
              mma_bf16_ts(tmem + TM_O, tmem + TM_P + kk * 8,
                          desc_sw128_mn(cb + kk * 2048, kNT * 128, 1024), IDESC_PV,
                          (np > 0 || kk > 0) ? 1u : 0u);
            mma_commit(bar(B_PVDONE));
            mma_commit(bar(B_CEMPTY + np % kStages));
            ++np;
            progressed = true;
          }
        }
        if (progressed) {
          t0 = clock64();
        } else if (clock64() - t0 > kSpinLimit) {
          atomicOr(R.status, kErrTimeout);
          ok = false;
        }
      }
      if (!ok) {
        *abort_flag = 1;
        mma_commit(bar(B_DRAIN));
        mbar_wait(bar(B_DRAIN), 0, R.status);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax
    // Two warpgroups; warpgroup wg handles rows 32wg .. 32wg+31 of every
    // tile for the head of its TMEM lane.  Software-pipelined: the partial
    // scores of tile n+1 go to the peer before tile n's softmax runs, so the
    // exchange overlaps the arithmetic (double-buffered exchange buffers).
    const int wg = (warp - 3) >> 2;
    const int quad = warp & 3;
    const int h = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    // The query: this CTA's 288 contraction dims of head h, as bf16 pairs in
    // TMEM columns TM_Q .. TM_Q+143 (warpgroup wg stores 72 of them).
    {
      const uint4* qsrc = reinterpret_cast<const uint4*>(
          q + ((int64_t)r * kH + h) * kDK + 288 * crank + 144 * wg);
#pragma unroll
      for (int part = 0; part < 3; ++part) {  // 3 x 48 dims = 3 x 24 columns
        uint32_t w24[24];
#pragma unroll
        for (int v = 0; v < 6; ++v) {
          const uint4 x = __ldg(qsrc + part * 6 + v);
          w24[4 * v] = x.x;
          w24[4 * v + 1] = x.y;
          w24[4 * v + 2] = x.z;
          w24[4 * v + 3] = x.w;
        }
        const uint32_t ta = tmem + lane_off + TM_Q + 72 * wg + 24 * part;
        uint32_t a8[8], b8[8], c8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          a8[e] = w24[e];
          b8[e] = w24[8 + e];
          c8[e] = w24[16 + e];
        }
        tmem_st8(ta, a8);
        tmem_st8(ta + 8, b8);
        tmem_st8(ta + 16, c8);
      }
      tc_fence_before();
      mbar_arrive(bar(B_QREADY));
    }
    const uint32_t xrow_peer0 = map_peer(sb + OFF_X + h * (kNT * 4), peer);
    const uint32_t xfull_peer0 = map_peer(bar(B_XFULL), peer);
    const uint32_t xempty_peer0 = map_peer(bar(B_XEMPTY), peer);
    float m2 = -INFINITY, l = 0.f;
    bool ok = true;
    float s_cur[32], s_nxt[32];
    // Loads tile m's partial scores into d and ships them to the peer.
    auto send = [&](int m, float (&d)[32]) -> bool {
      const int st = m % kStages, xb = m & 1;
      bool w_ok = __all_sync(0xffffffffu,
                             mbar_wait(bar(B_CFULL + st), (m / kStages) & 1, R.status) &&
                                 mbar_wait(bar(B_SFULL), m & 1, R.status) && !*abort_flag);
      if (w_ok) {
        tc_fence_after();
        tmem_ld32(tmem + lane_off + TM_S + 32 * wg, d);
        tc_fence_before();
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) d[j] = 0.f;
      }
      mbar_arrive(bar(B_SEMPTY));
      w_ok = w_ok && __all_sync(0xffffffffu, mbar_wait(bar(B_XEMPTY + xb), ((m >> 1) & 1) ^ 1,
                                                       R.status));
      if (w_ok) {
        const uint32_t xr = xrow_peer0 + xb * kXBytes;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const int cc = 8 * wg + c;
          st_cluster_v4(xr + ((cc ^ (h & 7)) * 16), d[4 * c], d[4 * c + 1], d[4 * c + 2],
                        d[4 * c + 3]);
        }
      }
      if (!bar_and<1, kSoftmaxThreads>(w_ok)) return false;  // all stores issued
      if (tid == kSoftmax0) arrive_remote(xfull_peer0 + 8u * xb);  // one cumulative release
      return true;
    };
    if (ntiles > 0) ok = send(0, s_cur);
    for (int n = 0; ok && n < ntiles; ++n) {
      const int st = n % kStages, xb = n & 1;
      if (n + 1 < ntiles && !send(n + 1, s_nxt)) {
        ok = false;
        break;
      }
      // the peer's half of tile n
      bool w_ok = __all_sync(0xffffffffu, wait_cluster(bar(B_XFULL + xb), (n >> 1) & 1, R.status));
      const uint32_t bits = vmask[st * 2 + wg];
      float hm = -INFINITY;
      {
        const float4* xr = reinterpret_cast<const float4*>(smem + OFF_X + xb * kXBytes +
                                                            h * (kNT * 4));
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const int cc = 8 * wg + c;
          const float4 v = w_ok ? xr[cc ^ (h & 7)] : make_float4(0.f, 0.f, 0.f, 0.f);
          const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j = 4 * c + e;
            s_cur[j] = ((bits >> j) & 1u) ? (s_cur[j] + vv[e]) * scale2 : -INFINITY;
            hm = fmaxf(hm, s_cur[j]);
          }
        }
      }
      hmax[wg * kH + h] = hm;
      if (!bar_and<1, kSoftmaxThreads>(w_ok)) {  // exchange buffer read, half maxima visible
        ok = false;
        break;
      }
      if (tid == kSoftmax0) arrive_remote(xempty_peer0 + 8u * xb);
      const float mt = fmaxf(hm, hmax[(wg ^ 1) * kH + h]);  // same value in both warpgroups
      // P of tile n-1 is consumed and O is final up to tile n-1 once PV(n-1) retired
      bool t_ok = n == 0 || __all_sync(0xffffffffu,
                                       mbar_wait(bar(B_PVDONE), (n - 1) & 1, R.status));
      if (mt > m2 + kRescale || (m2 == -INFINITY && mt != -INFINITY)) {
        const float m_new = fmaxf(mt, m2);
        const float alpha = ex2(m2 - m_new);  // 0 when m2 = -inf
        l *= alpha;
        if (n > 0 && t_ok) {  // rescale this warpgroup's 128 output columns
          tc_fence_after();
          for (int cc = 0; cc < 4; ++cc) {
            float v[32];
            const uint32_t ta = tmem + lane_off + TM_O + 128 * wg + cc * 32;
            tmem_ld32(ta, v);
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] *= alpha;
            tmem_st32(ta, v);
          }
        }
        m2 = m_new;
      }
      const float mref = m2 == -INFINITY ? 0.f : m2;  // all scores -inf: p = 0
      float lsum = 0.f;
      uint32_t pw[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float p0 = ex2(s_cur[2 * j] - mref);
        const float p1 = ex2(s_cur[2 * j + 1] - mref);
        pw[j] = pack_bf16(p0, p1);  // bf16 only as the MMA operand
        lsum += p0 + p1;            // the denominator keeps fp32 probabilities
      }
      if (t_ok) tmem_st16(tmem + lane_off + TM_P + 16 * wg, pw);
      l += lsum;
      if (!t_ok) *abort_flag = 1;  // seen by everyone at the next barrier reduction
      tc_fence_before();           // orders the P store (and a rescale) before the PV MMA
      mbar_arrive(bar(B_PFULL));
#pragma unroll
      for (int j = 0; j < 32; ++j) s_cur[j] = s_nxt[j];
    }
    if (!ok) *abort_flag = 1;
    // combine the two warpgroups' denominators (the first barrier retires the
    // last tile's reads of the half maxima)
    asm volatile("bar.sync 1, 256;" ::: "memory");
    hmax[wg * kH + h] = l;
    asm volatile("bar.sync 1, 256;" ::: "memory");
    l += hmax[(wg ^ 1) * kH + h];
    // final output: warpgroup wg writes columns 128wg .. 128wg+127 of this CTA's half
    bool have_o = ok && ntiles > 0;
    if (have_o) have_o = mbar_wait(bar(B_PVDONE), (ntiles - 1) & 1, R.status);
    have_o = __all_sync(0xffffffffu, have_o);
    tc_fence_after();
    const float inv = l > 0.f ? 1.f / l : 0.f;
    const float lse_v = l > 0.f ? (m2 + log2f(l)) * kLn2 : -INFINITY;
    const bool final_out = sp.nsplit == 1;
    for (int cc = 0; cc < 4; ++cc) {
      float v[32];
      const int c32 = 4 * wg + cc;  // 32-column block inside this CTA's 256 columns
      if (have_o) {
        tmem_ld32(tmem + lane_off + TM_O + c32 * 32, v);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = 0.f;
      }
      const int col = (int)crank * 256 + c32 * 32;
      if (final_out) {
        uint16_t* o = out + ((int64_t)r * kH + h) * kDV + col;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
          reinterpret_cast<uint4*>(o)[q4] =
              make_uint4(pack_bf16(v[8 * q4] * inv, v[8 * q4 + 1] * inv),
                         pack_bf16(v[8 * q4 + 2] * inv, v[8 * q4 + 3] * inv),
                         pack_bf16(v[8 * q4 + 4] * inv, v[8 * q4 + 5] * inv),
                         pack_bf16(v[8 * q4 + 6] * inv, v[8 * q4 + 7] * inv));
      } else {
        float* o = part_o + (((int64_t)rloc * sp.nsplit + split) * kH + h) * kDV + col;
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4)
          reinterpret_cast<float4*>(o)[q4] = make_float4(v[4 * q4] * inv, v[4 * q4 + 1] * inv,
                                                         v[4 * q4 + 2] * inv, v[4 * q4 + 3] * inv);
      }
    }
    if (crank == 0 && wg == 0) {
      if (final_out) {
        if (lse) lse[(int64_t)r * kH + h] = lse_v;
      } else {
        part_lse[((int64_t)rloc * sp.nsplit + split) * kH + h] = lse_v;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  cluster_sync();  // the peer may still write into our shared memory until here
}

// Merges split partials: out = sum_i exp(lse_i - lse) o_i, lse = log sum_i exp(lse_i).
__global__ void __launch_bounds__(128) attn_combine_kernel(int32_t row0, int nsplit,
                                                           const float* __restrict__ part_o,
                                                           const float* __restrict__ part_lse,
                                                           uint16_t* __restrict__ out,
                                                           float* __restrict__ lse) {
  const int32_t rloc = blockIdx.x, h = blockIdx.y;
  const int32_t r = row0 + rloc;
  const float* pl = part_lse + (int64_t)rloc * nsplit * kH + h;
  float mx = -INFINITY;
  for (int i = 0; i < nsplit; ++i) mx = fmaxf(mx, pl[(int64_t)i * kH]);
  float den = 0.f;
  for (int i = 0; i < nsplit; ++i) {
    const float li = pl[(int64_t)i * kH];
    if (li != -INFINITY) den += __expf(li - mx);
  }
  const int v = threadIdx.x * 4;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (den > 0.f) {
    for (int i = 0; i < nsplit; ++i) {
      const float li = pl[(int64_t)i * kH];
      if (li == -INFINITY) continue;
      const float wgt = __expf(li - mx) / den;
      const float4 o = *reinterpret_cast<const float4*>(
          part_o + (((int64_t)rloc * nsplit + i) * kH + h) * kDV + v);
      acc.x = fmaf(wgt, o.x, acc.x);
      acc.y = fmaf(wgt, o.y, acc.y);
      acc.z = fmaf(wgt, o.z, acc.z);
      acc.w = fmaf(wgt, o.w, acc.w);
    }
  }
  uint16_t* o = out + ((int64_t)r * kH + h) * kDV + v;
  *reinterpret_cast<uint2*>(o) = make_uint2(pack_bf16(acc.x, acc.y), pack_bf16(acc.z, acc.w));
  if (lse && threadIdx.x == 0) lse[(int64_t)r * kH + h] = den > 0.f ? mx + logf(den) : -INFINITY;
}

// Fixed scratch for callers that cannot allocate device memory (see
// launch_attn_tc_static): the split partials of one call, 64 MiB.
constexpr size_t kStaticScratchBytes = size_t(64) << 20;
static __device__ __align__(256) float g_attn_scratch[kStaticScratchBytes / sizeof(float)];

}  // namespace

bool attn_tc_supported(int H, int D_K, int D_V) { return H == kH && D_K == kDK && D_V == kDV; }

size_t attn_tc_workspace(int32_t nrows, int k, int H, int D_V) {
  if (nrows <= 0) return 0;
  const Split sp = plan_split(nrows, k);
  if (sp.nsplit == 1) return 0;
  return (size_t)nrows * sp.nsplit * kH * (kDV + 1) * sizeof(float) + 256;
}

dsa_status_t launch_attn_tc(const Rows& R, int32_t row0, int32_t nrows, const uint16_t* q,
                            const uint16_t* kv, const int32_t* idx, int k, float sm_scale,
                            uint16_t* out, float* lse, void* ws, size_t ws_bytes,
                            cudaStream_t st) {
  if (nrows <= 0) return DSA_OK;
  const Split sp = plan_split(nrows, k);
  float *part_o = nullptr, *part_lse = nullptr;
  if (sp.nsplit > 1) {
    if (!ws || ws_bytes < attn_tc_workspace(nrows, k, kH, kDV)) return DSA_ERR_WORKSPACE;
    part_o = reinterpret_cast<float*>(ws);
    part_lse = part_o + (size_t)nrows * sp.nsplit * kH * kDV;
  }
  if (cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) !=
      cudaSuccess)
    return DSA_ERR_CUDA;
  const dim3 grid(2 * nrows * sp.nsplit);
  attn_tc_kernel<<<grid, kThreads, kSmem, st>>>(q, kv, R, row0, idx, k, sm_scale * kLog2e, sp,
                                                out, lse, part_o, part_lse);
  if (cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;
  if (sp.nsplit > 1) {
    attn_combine_kernel<<<dim3(nrows, kH), 128, 0, st>>>(row0, sp.nsplit, part_o, part_lse, out,
                                                         lse);
    if (cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;
  }
  return DSA_OK;
}

size_t attn_tc_static_scratch_bytes() { return kStaticScratchBytes; }

// Same computation as launch_attn_tc, with the split partials placed in
// g_attn_scratch instead of a caller workspace.  The array's device address
// is looked up once per device, with that device current; host code may not
// use the symbol itself (it names a host-side shadow, not device memory).
dsa_status_t launch_attn_tc_static(const Rows& R, int32_t row0, int32_t nrows, const uint16_t* q,
                                   const uint16_t* kv, const int32_t* idx, int k, float sm_scale,
                                   uint16_t* out, float* lse, cudaStream_t st) {
  const size_t need = attn_tc_workspace(nrows, k, kH, kDV);
  if (need > kStaticScratchBytes) return DSA_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (need) {
    static void* addr[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return DSA_ERR_CUDA;
    if (!addr[dev]) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_attn_scratch) != cudaSuccess || !p) return DSA_ERR_CUDA;
      addr[dev] = p;
    }
    scratch = addr[dev];
  }
  return launch_attn_tc(R, row0, nrows, q, kv, idx, k, sm_scale, out, lse, scratch, need, st);
}

}  // namespace dsa
