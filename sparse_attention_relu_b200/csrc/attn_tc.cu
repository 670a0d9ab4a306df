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
// swizzled layout the MMA reads (an empty slot is zero-filled).  Measured on
// B200: one thread issuing TMA tile::gather4 (4 rows per instruction) needs
// about 9.3K cycles per such tile, the spread cp.async gather a fraction of it.
// TMEM: two 64-column score buffers and a 256-column output accumulator.
//
// Warp roles (352 threads per CTA):
//   warps 0-1  gather producer (indices -> shared memory, cp.async rows)
//   warp 2     TMEM allocator and MMA issuer (one thread)
//   warps 3-10 softmax, two warpgroups: a thread owns one head (its TMEM lane)
//              and half of each tile's 64 rows -- score exchange, online softmax
//              in the log2 domain with a lazy rescale (the reference max moves
//              only when a new score exceeds it by more than 2^8), P to shared
//              memory as bf16, final normalisation and store.
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
constexpr int kQBytes = kAtoms * kH * 128;    // 81920
constexpr int kCBytes = kAtoms * kNT * 128;   // 40960 per stage
constexpr int kStages = 2;
constexpr int kPBytes = kH * kNT * 2;         // 16384 per buffer
constexpr int kXBytes = kH * kNT * 4;         // 32768
constexpr int OFF_Q = 0;
constexpr int OFF_C = OFF_Q + kQBytes;
constexpr int OFF_P = OFF_C + kStages * kCBytes;
constexpr int OFF_X = OFF_P + 2 * kPBytes;
constexpr int OFF_IDX = OFF_X + kXBytes;                 // [stage][64] int32
constexpr int OFF_MASK = OFF_IDX + kStages * kNT * 4;    // [stage][2] uint32 validity bits
constexpr int OFF_HMAX = OFF_MASK + kStages * 2 * 4;     // [2 warpgroups][128] float
constexpr int OFF_BAR = OFF_HMAX + 2 * kH * 4;
constexpr int kNumBars = 16;
constexpr int OFF_MISC = OFF_BAR + kNumBars * 8;
constexpr int kSmem = OFF_MISC + 16 + 1024;
static_assert(kSmem <= 232448, "shared memory");
// TMEM columns
constexpr uint32_t TM_S = 0;     // two 64-column score buffers
constexpr uint32_t TM_O = 256;   // 256-column output accumulator
constexpr uint32_t IDESC_QK = idesc(1, 128, kNT);
constexpr uint32_t IDESC_PV = idesc(1, 128, 256, false, true);
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescale = 8.0f;  // log2 headroom before the reference max moves

enum {
  B_QFULL = 0, B_CFULL = 1, B_CEMPTY = 3, B_SFULL = 5, B_SEMPTY = 7, B_PFULL = 9,
  B_PVDONE = 11, B_XFULL = 13, B_XEMPTY = 14, B_DRAIN = 15
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
    attn_tc_kernel(const __grid_constant__ CUtensorMap qmap, const uint16_t* __restrict__ kv,
                   Rows R, int32_t row0, const int32_t* __restrict__ idx, int k, float scale2,
                   Split sp, uint16_t* __restrict__ out, float* __restrict__ lse,
                   float* __restrict__ part_o, float* __restrict__ part_lse) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
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
    mbar_init(bar(B_QFULL), 1);
    for (int i = 0; i < 2; ++i) {
      // per producer: a release-arrive after its index store and a cp.async arrive
      mbar_init(bar(B_CFULL + i), 2 * kProducers);
      mbar_init(bar(B_CEMPTY + i), 1);
      mbar_init(bar(B_SFULL + i), 1);
      mbar_init(bar(B_SEMPTY + i), kSoftmaxThreads);
      mbar_init(bar(B_PFULL + i), kSoftmaxThreads);
      mbar_init(bar(B_PVDONE + i), 1);
    }
    mbar_init(bar(B_XFULL), 1);  // one release-arrive from the peer per tile
    mbar_init(bar(B_XEMPTY), 1);
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
    if (tid == 0) {
      tma_prefetch(&qmap);
      mbar_expect_tx(bar(B_QFULL), kQBytes);
      for (int la = 0; la < kAtoms; ++la)
        tma_load_2d(sb + OFF_Q + la * kH * 128, &qmap, (int)(4 * crank + la) * 64, r * kH,
                    bar(B_QFULL));
    }
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
      const int st = n & 1;
      const bool ok = mbar_wait(bar(B_CEMPTY + st), ((n >> 1) & 1) ^ 1, R.status) && !*abort_flag;
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
    if (tid == 0) mbar_wait(bar(B_QFULL), 0, R.status);
  } else if (warp == 2) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(bar(B_QFULL), 0, R.status);
      const uint32_t qb = sb + OFF_Q;
      for (int n = 0; ok && n <= ntiles; ++n) {
        if (n < ntiles) {
          const int st = n & 1;
          if (!mbar_wait(bar(B_CFULL + st), (n >> 1) & 1, R.status) ||
              !mbar_wait(bar(B_SEMPTY + st), ((n >> 1) & 1) ^ 1, R.status) || *abort_flag) {
            ok = false;
            break;
          }
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // cp.async rows
          tc_fence_after();
          const uint32_t cb = sb + OFF_C + st * kCBytes;
#pragma unroll
          for (int kk = 0; kk < 18; ++kk) {
            const int e = 288 * (int)crank + 16 * kk;  // global contraction index
            const int la = e / 64 - 4 * (int)crank, off = (e % 64) * 2;
            mma_bf16(tmem + TM_S + st * kNT, desc_sw128(qb + la * kH * 128 + off, 1024),
                     desc_sw128(cb + la * kNT * 128 + off, 1024), IDESC_QK, kk > 0 ? 1u : 0u);
          }
          mma_commit(bar(B_SFULL + st));
        }
        if (n >= 1) {
          const int m = n - 1, pb = m & 1;
          if (!mbar_wait(bar(B_PFULL + pb), (m >> 1) & 1, R.status) || *abort_flag) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t cb = sb + OFF_C + pb * kCBytes;  // stage of tile m
          const uint32_t pbase = sb + OFF_P + pb * kPBytes;
#pragma unroll
          for (int kk = 0; kk < kNT / 16; ++kk)
            mma_bf16(tmem + TM_O, desc_sw128(pbase + kk * 32, 1024),
                     desc_sw128_mn(cb + kk * 2048, kNT * 128, 1024), IDESC_PV,
                     (m > 0 || kk > 0) ? 1u : 0u);
          mma_commit(bar(B_PVDONE + pb));
          mma_commit(bar(B_CEMPTY + pb));
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
    // Two warpgroups; warpgroup wg handles tokens 32wg .. 32wg+31 of every
    // tile for the head of its TMEM lane.
    const int wg = (warp - 3) >> 2;
    const int quad = warp & 3;
    const int h = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t xrow = sb + OFF_X + h * (kNT * 4);
    const uint32_t xrow_peer = map_peer(xrow, peer);
    const uint32_t xfull_peer = map_peer(bar(B_XFULL), peer);
    const uint32_t xempty_peer = map_peer(bar(B_XEMPTY), peer);
    float m2 = -INFINITY, l = 0.f;
    bool ok = true;
    for (int n = 0; n < ntiles; ++n) {
      const int st = n & 1;
      bool w_ok = __all_sync(0xffffffffu, mbar_wait(bar(B_CFULL + st), (n >> 1) & 1, R.status) &&
                                              mbar_wait(bar(B_SFULL + st), (n >> 1) & 1, R.status) &&
                                              !*abort_flag);
      float s[32];
      if (w_ok) {
        tc_fence_after();
        tmem_ld32(tmem + lane_off + TM_S + st * kNT + 32 * wg, s);
        tc_fence_before();
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) s[j] = 0.f;
      }
      mbar_arrive(bar(B_SEMPTY + st));
      // send this half of the partial scores to the peer CTA
      w_ok = w_ok && __all_sync(0xffffffffu, mbar_wait(bar(B_XEMPTY), (n & 1) ^ 1, R.status));
      if (w_ok) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const int cc = 8 * wg + c;
          st_cluster_v4(xrow_peer + ((cc ^ (h & 7)) * 16), s[4 * c], s[4 * c + 1], s[4 * c + 2],
                        s[4 * c + 3]);
        }
      }
      if (!bar_and<1, kSoftmaxThreads>(w_ok)) {  // all stores issued: one cumulative release
        ok = false;
        break;
      }
      if (tid == kSoftmax0) arrive_remote(xfull_peer);
      w_ok = __all_sync(0xffffffffu, wait_cluster(bar(B_XFULL), n & 1, R.status));
      const uint32_t bits = vmask[st * 2 + wg];
      float hm = -INFINITY;
      {
        const float4* xr = reinterpret_cast<const float4*>(smem + OFF_X + h * (kNT * 4));
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const int cc = 8 * wg + c;
          const float4 v = w_ok ? xr[cc ^ (h & 7)] : make_float4(0.f, 0.f, 0.f, 0.f);
          const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j = 4 * c + e;
            s[j] = ((bits >> j) & 1u) ? (s[j] + vv[e]) * scale2 : -INFINITY;
            hm = fmaxf(hm, s[j]);
          }
        }
      }
      hmax[wg * kH + h] = hm;
      if (!bar_and<1, kSoftmaxThreads>(w_ok)) {  // exchange buffer read, half maxima visible
        ok = false;
        break;
      }
      if (tid == kSoftmax0) arrive_remote(xempty_peer);
      const float mt = fmaxf(hm, hmax[(wg ^ 1) * kH + h]);  // same value in both warpgroups
      bool t_ok = true;
      if (mt > m2 + kRescale || (m2 == -INFINITY && mt != -INFINITY)) {
        const float m_new = fmaxf(mt, m2);
        const float alpha = ex2(m2 - m_new);  // 0 when m2 = -inf
        l *= alpha;
        if (n > 0) {  // rescale this warpgroup's 128 output columns (PV of tile n-1 first)
          const int m = n - 1;
          t_ok = __all_sync(0xffffffffu,
                            mbar_wait(bar(B_PVDONE + (m & 1)), (m >> 1) & 1, R.status));
          if (t_ok) {
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
        }
        m2 = m_new;
      }
      // P buffer n&1 is free once PV(n-2) completed
      if (n >= 2)
        t_ok = t_ok && __all_sync(0xffffffffu, mbar_wait(bar(B_PVDONE + (n & 1)),
                                                         ((n - 2) >> 1) & 1, R.status));
      uint8_t* prow = smem + OFF_P + (n & 1) * kPBytes + h * 128;
      const float mref = m2 == -INFINITY ? 0.f : m2;  // all scores -inf: p = 0
      float lsum = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t w4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float p0 = ex2(s[8 * c + 2 * e] - mref);
          const float p1 = ex2(s[8 * c + 2 * e + 1] - mref);
          w4[e] = pack_bf16(p0, p1);  // bf16 only as the MMA operand
          lsum += p0 + p1;            // the denominator keeps fp32 probabilities
        }
        const int cc = 4 * wg + c;
        if (t_ok)
          *reinterpret_cast<uint4*>(prow + ((cc ^ (h & 7)) * 16)) =
              make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
      l += lsum;
      if (!t_ok) *abort_flag = 1;  // seen by everyone at the next barrier reduction
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // P: generic -> async proxy
      tc_fence_before();  // orders a rescale's tcgen05.st before the next MMA
      mbar_arrive(bar(B_PFULL + (n & 1)));
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
    if (have_o) {
      const int m = ntiles - 1;
      have_o = mbar_wait(bar(B_PVDONE + (m & 1)), (m >> 1) & 1, R.status);
    }
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
  CUtensorMap qmap;
  if (!make_tmap_2d(&qmap, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kDK, (uint64_t)R.n_q * kH, 64,
                    kH))
    return DSA_ERR_CUDA;
  if (cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) !=
      cudaSuccess)
    return DSA_ERR_CUDA;
  const dim3 grid(2 * nrows * sp.nsplit);
  attn_tc_kernel<<<grid, kThreads, kSmem, st>>>(qmap, kv, R, row0, idx, k, sm_scale * kLog2e,
                                                sp, out, lse, part_o, part_lse);
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
