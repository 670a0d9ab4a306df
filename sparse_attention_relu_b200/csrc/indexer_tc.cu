// Lightning indexer on the 5th-generation tensor cores (tcgen05, sm_100a).
//
//   I[t, s] = sum_j w[t, j] * ReLU(<q_I[t, j, :], k_I[s, :]>),   s <= t
//
// ("GLM sparse attention", ReLU paragraph; "Sparse Attention Architecture
// Evolution in LLMs", Indexer section: a small scorer that scans every
// earlier position.)  H_I = 64 heads, D_I = 128, bf16 or fp8 e4m3 inputs.
//
// The contraction is a GEMM with the KEYS on M and (query, head) pairs on N:
//   D[key, (q, j)] = <k_I[key], q_I[q, j]>        M = 128 keys, N = G * 64
// so that one TMEM lane holds every head of one key for G queries, and the
// ReLU + weighted head sum is a private loop per thread in the epilogue,
// with no shuffles.  fp8 scales fold in for free: q_scale (positive) moves
// into w, k_scale multiplies the finished sum.
//
// Warp roles (prefill: 832 threads):
//   warp 0      TMA producer: the query block once, then a ring of key tiles
//   warp 1      TMEM allocator and MMA issuer (one thread)
//   warps 2-25  epilogue: TMEM -> registers, ReLU, weighted head sum, store.
//               Six sets of four warps (one warp per TMEM lane quadrant in
//               each) take the (accumulator, query) units in turn, so six
//               warps per SM sub-partition hide each other's latencies.  A
//               score costs per head one max (the ReLU) and half of a packed
//               two-lane fp32 FMA, into four independent accumulator pairs.
// Key tiles stream through an NK-stage shared-memory ring; accumulators
// rotate through NS TMEM slots so the MMA of the next job overlaps the
// epilogue of the previous one.
//
// Work: prefill -- a CTA owns NG*G consecutive queries of one sequence and
// every key tile up to the last query (blocks launched heaviest first);
// decode -- a persistent kernel of its own (indexer_decode_kernel, below).
#include <cudaTypedefs.h>

#include "kernels.cuh"
#include "select.cuh"
#include "sm100.cuh"

namespace dsa {

using namespace sm100;

namespace {

constexpr int kHI = 64, kDI = 128, kTileK = 128;  // heads, dims, keys per tile
constexpr int kThreads = 576;
constexpr int kEpiThreads = 512;  // warps 2-17
constexpr int kEpiSets = kEpiThreads / 128;
// Prefill: six sets of four epilogue warps (warps 2-25) share out the
// (accumulator, query) units in turn; the extra warps hide the latency of
// each unit's TMEM loads and weight reads behind the others' arithmetic.
constexpr int kEpiSetsP = 6;
constexpr int kEpiThreadsP = kEpiSetsP * 128;  // 768
constexpr int kThreadsP = 64 + kEpiThreadsP;   // 832

// Two fp32 FMAs in one instruction: {lo, hi} = {x0 * w0, x1 * w1} + acc.
__device__ __forceinline__ uint64_t fma2(float x0, float x1, float w0, float w1, uint64_t acc) {
  uint64_t d;
  asm("{\n\t.reg .b64 x, w;\n\t"
      "mov.b64 x, {%1, %2};\n\t"
      "mov.b64 w, {%3, %4};\n\t"
      "fma.rn.f32x2 %0, x, w, %5;\n\t}"
      : "=l"(d)
      : "f"(x0), "f"(x1), "f"(w0), "f"(w1), "l"(acc));
  return d;
}
__device__ __forceinline__ float lo32(uint64_t v) { return __uint_as_float((uint32_t)v); }
__device__ __forceinline__ float hi32(uint64_t v) { return __uint_as_float((uint32_t)(v >> 32)); }

// Weighted ReLU head sum of one key for one query: the 64 fp32 head scores
// at TMEM columns ta .. ta+63 of this warp's lanes, weights w[0..63] in
// shared memory.  Both 32-column loads are in flight before the one wait.
__device__ __forceinline__ float relu_wsum(uint32_t ta, const float4* __restrict__ wr) {
  uint32_t r[64];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%64];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%65];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
        "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]),
        "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]),
        "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]),
        "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
        "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]),
        "=r"(r[62]), "=r"(r[63])
      : "r"(ta), "r"(ta + 32)
      : "memory");
  uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
  for (int h4 = 0; h4 < 16; ++h4) {
    const float4 w4 = wr[h4];
    acc[(2 * h4) & 3] = fma2(fmaxf(__uint_as_float(r[4 * h4]), 0.f),
                             fmaxf(__uint_as_float(r[4 * h4 + 1]), 0.f), w4.x, w4.y,
                             acc[(2 * h4) & 3]);
    acc[(2 * h4 + 1) & 3] = fma2(fmaxf(__uint_as_float(r[4 * h4 + 2]), 0.f),
                                 fmaxf(__uint_as_float(r[4 * h4 + 3]), 0.f), w4.z, w4.w,
                                 acc[(2 * h4 + 1) & 3]);
  }
  return (lo32(acc[0]) + hi32(acc[0])) + (lo32(acc[1]) + hi32(acc[1])) +
         ((lo32(acc[2]) + hi32(acc[2])) + (lo32(acc[3]) + hi32(acc[3])));
}

// relu_wsum with one 32-column TMEM load at a time.
__device__ __forceinline__ float relu_wsum_halves(uint32_t ta, const float4* __restrict__ wr) {
  uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    float v[32];
    tmem_ld32(ta + 32 * half, v);
#pragma unroll
    for (int h4 = 0; h4 < 8; ++h4) {
      const float4 w4 = wr[8 * half + h4];
      acc[(2 * h4) & 3] = fma2(fmaxf(v[4 * h4], 0.f), fmaxf(v[4 * h4 + 1], 0.f), w4.x, w4.y,
                               acc[(2 * h4) & 3]);
      acc[(2 * h4 + 1) & 3] = fma2(fmaxf(v[4 * h4 + 2], 0.f), fmaxf(v[4 * h4 + 3], 0.f), w4.z,
                                   w4.w, acc[(2 * h4 + 1) & 3]);
    }
  }
  return (lo32(acc[0]) + hi32(acc[0])) + (lo32(acc[1]) + hi32(acc[1])) +
         ((lo32(acc[2]) + hi32(acc[2])) + (lo32(acc[3]) + hi32(acc[3])));
}

template <int DT, int G, int NG, int NK>
struct Cfg {
  static constexpr int ESZ = DT == DSA_BF16 ? 2 : 1;
  static constexpr int ROWB = kDI * ESZ;          // bytes per row
  static constexpr int KC = ROWB / 128;           // 128-byte column blocks per row
  static constexpr int N = G * kHI;               // MMA N
  static constexpr int QB = G * NG;               // queries per CTA
  static constexpr int QBYTES = NG * N * ROWB;
  static constexpr int KBYTES = kTileK * ROWB;
  static constexpr int NS = (512 / N) > 8 ? 8 : (512 / N);  // TMEM accumulator slots
  static constexpr int TCOLS = NS * N;
  static constexpr int UK = DT == DSA_BF16 ? 16 : 32;       // K per MMA instruction
  static constexpr int KSTEPS = kDI / UK;
  static constexpr uint32_t IDESC = idesc(DT == DSA_BF16 ? 1u : 0u, 128, N);
  // shared memory map (offsets from a 1024-aligned base)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + QBYTES;
  static constexpr int OFF_W = OFF_K + NK * KBYTES;
  static constexpr int OFF_BAR = OFF_W + QB * kHI * 4;
  static constexpr int NBAR = 2 * NK + 2 * NS + 2;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;  // + alignment slack
  static_assert(TCOLS == 512 || TCOLS == 256 || TCOLS == 128, "TMEM columns");
};

struct Work {
  int valid;          // CTA has work
  int64_t kbase;      // first key row of the sequence
  int32_t len;        // sequence length
  int32_t t0;         // local position of the first query of the block
  int32_t nq;         // queries in the block (<= QB)
  int32_t qrow0;      // global query row of query 0 of the block
  int32_t kt_begin, kt_end;  // key tiles
  int32_t qvalid_lo, qvalid_hi;  // valid query positions [lo, hi) (local)
};

// PREFILL and CHUNKED: a block owns QB consecutive query rows of sequence
// blockIdx.y.  In PREFILL a sequence's query rows are its cache rows
// (positions 0 ..); in CHUNKED they are q_offsets[b] .. q_offsets[b+1]-1 at
// the last C_b positions (the first at p0 = L_b - C_b).
template <int QB>
__device__ Work plan_prefill(const Rows& R, int32_t row0, int32_t nrows) {
  Work w{};
  const int b = blockIdx.y;
  const int32_t o0 = __ldg(R.offs + b), o1 = __ldg(R.offs + b + 1);
  int32_t q0 = o0, q1 = o1;
  if (R.mode == DSA_CHUNKED) {
    q0 = __ldg(R.qoffs + b);
    q1 = __ldg(R.qoffs + b + 1);
  }
  if (o0 < 0 || o1 < o0 || (int64_t)o1 > R.n_k || o1 - o0 > R.max_len || q0 < 0 || q1 < q0 ||
      q1 > R.n_q || q1 - q0 > o1 - o0) {
    if (threadIdx.x == 0 && blockIdx.x == 0) raise_status(R, kErrBadOffsets);
    return w;
  }
  const int32_t p0 = (o1 - o0) - (q1 - q0);  // position of the sequence's first query
  const int32_t lo = max(q0, row0), hi = min(q1, row0 + nrows);
  if (lo >= hi) return w;
  const int32_t i0 = (lo - q0) / QB, i1 = (hi - 1 - q0) / QB;
  if ((int32_t)blockIdx.x > i1 - i0) return w;
  const int32_t i = i1 - (int32_t)blockIdx.x;  // heaviest block first
  w.valid = 1;
  w.kbase = o0;
  w.len = o1 - o0;
  w.t0 = p0 + i * QB;
  w.qrow0 = q0 + i * QB;
  w.qvalid_lo = p0 + max(i * QB, lo - q0);
  w.qvalid_hi = p0 + min(i * QB + QB, hi - q0);
  w.nq = QB;
  w.kt_begin = 0;
  w.kt_end = (w.qvalid_hi - 1) / kTileK + 1;  // keys up to the last valid query
  return w;
}

template <int DT, int G, int NG, int NK>
__global__ void __launch_bounds__(kThreadsP, 1)
    indexer_tc_kernel(const __grid_constant__ CUtensorMap qmap,
                      const __grid_constant__ CUtensorMap kmap, Rows R, int32_t row0,
                      int32_t nrows, const float* __restrict__ w, const float* __restrict__ q_scale,
                      const float* __restrict__ k_scale, float* __restrict__ scores, int64_t ld,
                      int fill) {
  using C = Cfg<DT, G, NG, NK>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  float* wq = reinterpret_cast<float*>(smem + C::OFF_W);
  const uint32_t bar0 = sbase + C::OFF_BAR;
  auto k_full = [&](int i) { return bar0 + 8u * i; };
  auto k_empty = [&](int i) { return bar0 + 8u * (NK + i); };
  auto s_full = [&](int i) { return bar0 + 8u * (2 * NK + i); };
  auto s_empty = [&](int i) { return bar0 + 8u * (2 * NK + C::NS + i); };
  const uint32_t q_full = bar0 + 8u * (2 * NK + 2 * C::NS);
  const uint32_t drain = q_full + 8u;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const Work wk = plan_prefill<C::QB>(R, row0, nrows);
  if (!wk.valid) return;

  if (tid == 0) {
    for (int i = 0; i < NK; ++i) {
      mbar_init(k_full(i), 1);
      mbar_init(k_empty(i), 1);
    }
    for (int i = 0; i < C::NS; ++i) {
      mbar_init(s_full(i), 1);
      mbar_init(s_empty(i), 4 * G);  // the four lane-quadrant warps of each of the G queries
    }
    mbar_init(q_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(sbase + C::OFF_MISC, C::TCOLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_tiles = wk.kt_end - wk.kt_begin;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch(&qmap);
      tma_prefetch(&kmap);
      mbar_expect_tx(q_full, C::QBYTES);
      for (int g = 0; g < NG; ++g)
        for (int kc = 0; kc < C::KC; ++kc)
          tma_load_2d(sbase + C::OFF_Q + (g * C::KC + kc) * C::N * 128, &qmap, kc * (128 / C::ESZ),
                      (wk.qrow0 + g * G) * kHI, q_full);
      int issued = 0;
      for (int j = 0; j < n_tiles; ++j) {
        const int st = j % NK;
        if (!mbar_wait(k_empty(st), ((j / NK) & 1) ^ 1, R.status) || *abort_flag) {
          *abort_flag = 1;
          break;
        }
        mbar_expect_tx(k_full(st), C::KBYTES);
        const int32_t krow = (int32_t)(wk.kbase + (int64_t)(wk.kt_begin + j) * kTileK);
        for (int kc = 0; kc < C::KC; ++kc)
          tma_load_2d(sbase + C::OFF_K + st * C::KBYTES + kc * kTileK * 128, &kmap,
                      kc * (128 / C::ESZ), krow, k_full(st));
        ++issued;
      }
      // leave no copy in flight behind us
      for (int j = max(0, issued - NK); j < issued; ++j)
        mbar_wait(k_full(j % NK), (j / NK) & 1, R.status);
      mbar_wait(q_full, 0, R.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(q_full, 0, R.status);
      int job = 0;
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int st = j % NK;
        if (!mbar_wait(k_full(st), (j / NK) & 1, R.status) || *abort_flag) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_base = sbase + C::OFF_K + st * C::KBYTES;
        for (int g = 0; g < NG; ++g, ++job) {
          const int slot = job % C::NS;
          if (!mbar_wait(s_empty(slot), ((job / C::NS) & 1) ^ 1, R.status) || *abort_flag) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t b_base = sbase + C::OFF_Q + g * C::KC * C::N * 128;
          const uint32_t d = tmem + slot * C::N;
#pragma unroll
          for (int kk = 0; kk < C::KSTEPS; ++kk) {
            const int kc = kk / 4, sub = (kk % 4) * 32;
            const uint64_t da = desc_sw128(a_base + kc * kTileK * 128 + sub, 1024);
            const uint64_t db = desc_sw128(b_base + kc * C::N * 128 + sub, 1024);
            if constexpr (DT == DSA_BF16)
              mma_bf16(d, da, db, C::IDESC, kk > 0 ? 1u : 0u);
            else
              mma_e4m3(d, da, db, C::IDESC, kk > 0 ? 1u : 0u);
          }
          mma_commit(s_full(slot));
        }
        if (!ok) break;
        mma_commit(k_empty(st));
      }
      if (!ok) {
        *abort_flag = 1;
        mma_commit(drain);
        mbar_wait(drain, 0, R.status);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int et = tid - 64;           // 0..767
    const int quad = warp & 3;         // TMEM lane quadrant this warp may read
    const int set = et >> 7;           // warps 2-5: set 0, 6-9: set 1, ... 22-25: set 5
    for (int i = et; i < C::QB * kHI; i += kEpiThreadsP) {
      const int qi = i / kHI, h = i - qi * kHI;
      const int32_t tq = wk.t0 + qi;
      float v = 0.f;
      if (qi < wk.nq && tq >= wk.qvalid_lo && tq < wk.qvalid_hi) {
        const int64_t qr = wk.qrow0 + qi;
        v = __ldg(w + qr * kHI + h);
        if (q_scale) v *= __ldg(q_scale + qr * kHI + h);
      }
      wq[i] = v;
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreadsP) : "memory");
    // Unit u = (accumulator u / G, query u % G); set `set` takes units set,
    // set + 6, ...  G < 6, so a set reads each accumulator at most once.
    static_assert(G < kEpiSetsP, "one unit of an accumulator per set");
    const int n_units = n_tiles * NG * G;
    for (int u = set; u < n_units; u += kEpiSetsP) {
      const int job = u / G, qq = u - job * G;
      const int j = job / NG, g = job - j * NG;
      const int slot = job % C::NS;
      const int32_t s = (wk.kt_begin + j) * kTileK + quad * 32 + lane;
      // the key scale is fetched before the wait, which hides its latency
      const float ks = (DT == DSA_E4M3 && k_scale && s < wk.len) ? __ldg(k_scale + wk.kbase + s) : 1.f;
      // warp-uniform: the tcgen05 loads below need the whole warp
      if (!__all_sync(0xffffffffu,
                      mbar_wait(s_full(slot), (job / C::NS) & 1, R.status) && !*abort_flag)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const int qi = g * G + qq;
      const float4* wr = reinterpret_cast<const float4*>(wq + qi * kHI);
      const uint32_t ta = tmem + ((uint32_t)(quad * 32) << 16) + slot * C::N + qq * kHI;
      uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        float v[32];
        tmem_ld32(ta + 32 * half, v);
#pragma unroll
        for (int h4 = 0; h4 < 8; ++h4) {
          const float4 w4 = wr[8 * half + h4];
          acc[(2 * h4) & 3] = fma2(fmaxf(v[4 * h4], 0.f), fmaxf(v[4 * h4 + 1], 0.f), w4.x, w4.y,
                                   acc[(2 * h4) & 3]);
          acc[(2 * h4 + 1) & 3] = fma2(fmaxf(v[4 * h4 + 2], 0.f), fmaxf(v[4 * h4 + 3], 0.f),
                                       w4.z, w4.w, acc[(2 * h4 + 1) & 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_empty(slot));
      const float sum = (lo32(acc[0]) + hi32(acc[0])) + (lo32(acc[1]) + hi32(acc[1])) +
                        ((lo32(acc[2]) + hi32(acc[2])) + (lo32(acc[3]) + hi32(acc[3])));
      const int32_t tq = wk.t0 + qi;
      if (tq >= wk.qvalid_lo && tq < wk.qvalid_hi && s < R.max_len) {
        float* o = scores + (int64_t)(wk.qrow0 + qi - row0) * ld;
        if (s <= tq)
          o[s] = sum * ks;
        else if (fill)
          o[s] = -INFINITY;
      }
    }
    // -inf beyond the last scored tile (unit call only)
    if (fill) {
      for (int qi = 0; qi < C::QB; ++qi) {
        const int32_t tq = wk.t0 + qi;
        if (qi >= wk.nq || tq < wk.qvalid_lo || tq >= wk.qvalid_hi) continue;
        float* o = scores + (int64_t)(wk.qrow0 + qi - row0) * ld;
        const int32_t from = wk.kt_end * kTileK;
        for (int s = from + et; s < R.max_len; s += kEpiThreadsP) o[s] = -INFINITY;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TCOLS);
  }
}


// ---------------------------------------------------------------------------
// Decode: one query per sequence against its whole cache.  A persistent grid
// (one CTA per SM) cuts the concatenated key tiles of all rows into equal
// contiguous ranges, one per CTA; a range may cross row boundaries, and the
// key stream keeps flowing across them (the query block and head weights of
// the next row load into the other of two buffers while the current row is
// scored).  Equal ranges keep every SM streaming keys until the end, where a
// grid of per-row chunks paid a prologue and a pipeline ramp per chunk and
// left the last wave ragged.
// SEL: the fused filter of the decode path; it adds the segment histogram
// (8 KB) and the segment's candidate counter.
using SelB = sel::Blk<kEpiThreads, 4, 64>;  // the 512 epilogue threads, named barrier 4
template <int DT, int NK, bool SEL = false>
struct DecCfg {
  using C = Cfg<DT, 1, 1, NK>;
  static constexpr int OFF_Q = 0;                         // [2][64 x ROWB] query blocks
  static constexpr int OFF_K = 2 * C::QBYTES;             // [NK][128 x ROWB] key ring
  static constexpr int OFF_W = OFF_K + NK * C::KBYTES;    // [2][64] head weights
  static constexpr int OFF_SCAN = OFF_W + 2 * kHI * 4;    // block-scan scratch
  static constexpr int OFF_BAR = OFF_SCAN + 32 * 8 + 32;
  // k_full/k_empty [NK], s_full/s_empty [NS], q_full/q_empty [2], drain
  static constexpr int NBAR = 2 * NK + 2 * C::NS + 4 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int OFF_SSM = (OFF_MISC + 32 + 15) / 16 * 16;  // sel::Smem (histogram first)
  static constexpr int SSM_BYTES = SEL ? ((int)sizeof(sel::Smem<SelB::NW>) + 15) / 16 * 16 : 0;
  static constexpr int OFF_SCNT = OFF_SSM + SSM_BYTES;     // the segment's candidate count
  static constexpr int SMEM = OFF_SCNT + (SEL ? 16 : 0) + 1024;
  static_assert(C::QBYTES % 1024 == 0 && C::KBYTES % 1024 == 0, "1024-byte operand alignment");
  static_assert(C::NS % kEpiSets == 0, "a TMEM slot always belongs to the same epilogue set");
};

// The bin that holds the k-th best of the scores a histogram has counted (0
// while it holds fewer than k): one warp.  Each lane sums 64 bins (16-byte
// loads), a suffix scan over the lanes finds the lane whose bins hold the
// k-th best, and a second scan over that lane's bins, two per lane, finds
// the bin.  The histogram may be read while others still add to it; the
// counts read are then at most the true ones, which can only lower the bin.
__device__ __noinline__ uint32_t kth_bin(const uint32_t* hist, int k, int lane) {
  const uint4* h4 = reinterpret_cast<const uint4*>(hist) + lane * 16;
  uint32_t own = 0;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint4 v = h4[i];
    own += (v.x + v.y) + (v.z + v.w);
  }
  uint32_t suf = own;  // this lane and the lanes above it (higher bins)
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_down_sync(0xffffffffu, suf, o);
    if (lane + o < 32) suf += v;
  }
  const uint32_t kk = (uint32_t)k;
  const uint32_t hit = __ballot_sync(0xffffffffu, suf - own < kk && kk <= suf);
  if (!hit) return 0u;
  const int L = __ffs(hit) - 1;
  const uint32_t need = kk - __shfl_sync(0xffffffffu, suf - own, L);  // 1 .. lane L's count
  // lane L's 64 bins, two per lane (bins 2j, 2j+1 of the 64), counted from the top
  const uint2 c = reinterpret_cast<const uint2*>(hist + L * 64)[lane];
  const uint32_t pair = c.x + c.y;
  uint32_t sp = pair;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_down_sync(0xffffffffu, sp, o);
    if (lane + o < 32) sp += v;
  }
  const uint32_t above = sp - pair;  // in higher bins of lane L's 64
  const bool in_hi = above < need && need <= above + c.y;
  const bool in_lo = !in_hi && above + c.y < need && need <= sp;
  const uint32_t bh = __ballot_sync(0xffffffffu, in_hi || in_lo);
  if (!bh) return 0u;  // (cannot happen: counts only grow between the two reads)
  const int j = __ffs(bh) - 1;
  const uint32_t hi_bit = __shfl_sync(0xffffffffu, in_hi ? 1u : 0u, j);
  return (uint32_t)(L * 64 + 2 * j) + hi_bit;
}

// Key tiles of decode row r (0 when the row has no candidates).
__device__ __forceinline__ int32_t dec_row_tiles(const Rows& R, int32_t r) {
  const RowInfo ri = row_info(R, r);
  return ri.t < 0 ? 0 : (ri.t + kTileK) / kTileK;
}

// Inclusive sum over the block of one value per thread (kThreads threads);
// `total` receives the block's sum.  Uses 18 int64 words of `scr`.
__device__ __forceinline__ int64_t block_incl_scan(int64_t v, int64_t* scr, int64_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t u = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += u;
  }
  if (lane == 31) scr[warp] = v;
  __syncthreads();
  int64_t before = 0, all = 0;
  for (int i = 0; i < kThreads / 32; ++i) {
    const int64_t s = scr[i];
    if (i < warp) before += s;
    all += s;
  }
  __syncthreads();
  total = all;
  return v + before;
}

// One CTA's walk over its tile range: local row r, key tiles [kb, ke) of it,
// and the tiles of the range that come after this segment.
struct SegWalk {
  int32_t r, kb, ke;
  int64_t left;
};

__device__ __forceinline__ SegWalk seg_first(const Rows& R, int32_t row0, int32_t r, int32_t off,
                                             int64_t n) {
  SegWalk s;
  s.r = r;
  s.kb = off;
  const int64_t take = min((int64_t)(dec_row_tiles(R, row0 + r) - off), n);
  s.ke = off + (int32_t)take;
  s.left = n - take;
  return s;
}

__device__ __forceinline__ bool seg_next(const Rows& R, int32_t row0, int32_t nrows, SegWalk& s) {
  while (s.left > 0 && ++s.r < nrows) {
    const int32_t nt = dec_row_tiles(R, row0 + s.r);
    if (nt == 0) continue;
    const int64_t take = min((int64_t)nt, s.left);
    s.kb = 0;
    s.ke = (int32_t)take;
    s.left -= take;
    return true;
  }
  return false;
}

// SEL (the fused top-k of dsa_forward's decode path): instead of writing
// score rows, each score is counted in a histogram of this CTA's segment and
// kept, as (rank key, position) in its row's candidate list, only when its
// bin reaches the row's running threshold: the bin of the k-th best score
// among those counted so far, in this segment or -- shared through a global
// maximum -- in another CTA's segment of the same row.  The k-th best of any
// subset of a row is at most the row's k-th best, so no score that can be
// among the row's k best is dropped ("GLM sparse attention", threshold
// figure: the cut-off is the k-th best score).  A segment over the row's key
// tiles [kb, ke) appends to its own part of the row's list, entries
// kb*128 .. ke*128 (so no list overflows and no two CTAs share a counter),
// and at its end records its count and adds its histogram into the row's;
// select_rows_kernel then picks each row's k best from its segments' lists.
//   cand  [nrows][cap]        candidates (cap >= max_len)
//   rstate[nrows]             per row: running threshold bin (zero at launch)
//   segcnt[nrows][cap / 128]  per row and first tile of a segment: its
//                             candidate count (zero at launch)
//   rhist [nrows][kBins]      per row: histogram of all its scores (zero at launch)
template <int DT, int NK, bool SEL = false>
__global__ void __launch_bounds__(kThreads, 1)
    indexer_decode_kernel(const __grid_constant__ CUtensorMap qmap,
                          const __grid_constant__ CUtensorMap kmap, Rows R, int32_t row0,
                          int32_t nrows, const float* __restrict__ w,
                          const float* __restrict__ q_scale, const float* __restrict__ k_scale,
                          float* __restrict__ scores, int64_t ld, int fill,
                          uint64_t* __restrict__ cand, int64_t cap, uint32_t* __restrict__ rstate,
                          uint32_t* __restrict__ segcnt, uint32_t* __restrict__ rhist, int k) {
  using D = DecCfg<DT, NK, SEL>;
  using C = typename D::C;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  float* wq = reinterpret_cast<float*>(smem + D::OFF_W);
  int64_t* scr = reinterpret_cast<int64_t*>(smem + D::OFF_SCAN);
  const uint32_t bar0 = sbase + D::OFF_BAR;
  auto k_full = [&](int i) { return bar0 + 8u * i; };
  auto k_empty = [&](int i) { return bar0 + 8u * (NK + i); };
  auto s_full = [&](int i) { return bar0 + 8u * (2 * NK + i); };
  auto s_empty = [&](int i) { return bar0 + 8u * (2 * NK + C::NS + i); };
  auto q_full = [&](int b) { return bar0 + 8u * (2 * NK + 2 * C::NS + b); };
  auto q_empty = [&](int b) { return bar0 + 8u * (2 * NK + 2 * C::NS + 2 + b); };
  const uint32_t drain = bar0 + 8u * (2 * NK + 2 * C::NS + 4);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + D::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + D::OFF_MISC + 4);
  volatile int32_t* s_first = reinterpret_cast<volatile int32_t*>(smem + D::OFF_MISC + 8);
  auto* ssm = reinterpret_cast<sel::Smem<SelB::NW>*>(smem + D::OFF_SSM);
  uint32_t* const rthr = rstate;  // [nrows] running threshold bin
  uint32_t* const scnt = reinterpret_cast<uint32_t*>(smem + D::OFF_SCNT);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t G = gridDim.x;

  // -inf past the last tile of each row (unit call only); row r's tail is
  // written by CTA r mod G, its tiles by whichever CTA scores them
  if (fill) {
    for (int64_t r = blockIdx.x; r < nrows; r += G) {
      const int32_t from = min(dec_row_tiles(R, row0 + (int32_t)r) * kTileK, R.max_len);
      float* o = scores + r * ld;
      for (int32_t s = from + tid; s < R.max_len; s += kThreads) o[s] = -INFINITY;
    }
  }

  // ---- this CTA's share of the concatenated key tiles: [T0, T1)
  int64_t total = 0;
  for (int32_t r0 = 0; r0 < nrows; r0 += kThreads) {
    const int32_t r = r0 + tid;
    int64_t blk;
    block_incl_scan(r < nrows ? dec_row_tiles(R, row0 + r) : 0, scr, blk);
    total += blk;
  }
  const int64_t T0 = total * blockIdx.x / G, T1 = total * (blockIdx.x + 1) / G;
  if (T0 >= T1) return;
  if (tid == 0) s_first[0] = -1;
  int64_t base = 0;
  for (int32_t r0 = 0; r0 < nrows; r0 += kThreads) {
    const int32_t r = r0 + tid;
    const int32_t n = r < nrows ? dec_row_tiles(R, row0 + r) : 0;
    int64_t blk;
    const int64_t excl = base + block_incl_scan(n, scr, blk) - n;
    if (n > 0 && excl <= T0 && T0 < excl + n) {
      s_first[0] = r;
      s_first[1] = (int32_t)(T0 - excl);
    }
    base += blk;
  }
  __syncthreads();
  const int32_t first_row = s_first[0], first_off = s_first[1];
  if (first_row < 0) return;  // offsets changed under us; nothing sensible to do
  const SegWalk start = seg_first(R, row0, first_row, first_off, T1 - T0);

  if (tid == 0) {
    for (int i = 0; i < NK; ++i) {
      mbar_init(k_full(i), 1);
      mbar_init(k_empty(i), 1);
    }
    for (int i = 0; i < C::NS; ++i) {
      mbar_init(s_full(i), 1);
      mbar_init(s_empty(i), 4);  // the four warps of the set that owns the slot
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(q_full(b), 1);
      mbar_init(q_empty(b), 1 + kEpiThreads / 32);  // MMA commit + every epilogue warp
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if constexpr (SEL) {
    for (int i = tid; i < sel::kBins; i += kThreads) ssm->hist[i] = 0;
    if (tid == 0) *scnt = 0;
  }
  if (warp == 1) {
    tmem_alloc(sbase + D::OFF_MISC, C::TCOLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // The whole warp stages the head weights of each row; lane 0 issues
    // the TMA loads of the query block and the key tiles.
    if (lane == 0) {
      tma_prefetch(&qmap);
      tma_prefetch(&kmap);
    }
    SegWalk sg = start;
    int si = 0, q_issued = 0;
    int64_t gt = 0, issued = 0;
    bool ok = true;
    do {
      const int qb = si & 1;
      // buffer qb is free once the MMAs and the epilogue of segment si - 2 are done
      if (si >= 2) {
        int free_ok = 1;
        if (lane == 0)
          free_ok = mbar_wait(q_empty(qb), ((si - 2) >> 1) & 1, R.status) && !*abort_flag;
        if (!__shfl_sync(0xffffffffu, free_ok, 0)) {
          ok = false;
          break;
        }
      }
      const int64_t qr = (int64_t)row0 + sg.r;  // global query row
      for (int h = lane; h < kHI; h += 32) {
        float v = __ldg(w + qr * kHI + h);
        if (q_scale) v *= __ldg(q_scale + qr * kHI + h);
        wq[qb * kHI + h] = v;
      }
      __syncwarp();
      int lane_ok = 1;
      if (lane == 0) {
        const RowInfo ri = row_info(R, (int32_t)qr);
        mbar_expect_tx(q_full(qb), C::QBYTES);
        for (int kc = 0; kc < C::KC; ++kc)
          tma_load_2d(sbase + D::OFF_Q + qb * C::QBYTES + kc * C::N * 128, &qmap,
                      kc * (128 / C::ESZ), (int32_t)qr * kHI, q_full(qb));
        ++q_issued;
        for (int j = sg.kb; j < sg.ke; ++j, ++gt) {
          const int st = (int)(gt % NK);
          if (!mbar_wait(k_empty(st), (int)((gt / NK) & 1) ^ 1, R.status) || *abort_flag) {
            lane_ok = 0;
            break;
          }
          mbar_expect_tx(k_full(st), C::KBYTES);
          const int32_t krow = (int32_t)(ri.kbase + (int64_t)j * kTileK);
          for (int kc = 0; kc < C::KC; ++kc)
            tma_load_2d(sbase + D::OFF_K + st * C::KBYTES + kc * kTileK * 128, &kmap,
                        kc * (128 / C::ESZ), krow, k_full(st));
          ++issued;
        }
      }
      ok = __shfl_sync(0xffffffffu, lane_ok, 0) != 0;
      ++si;
    } while (ok && seg_next(R, row0, nrows, sg));
    if (!ok) *abort_flag = 1;
    if (lane == 0) {
      // leave no copy in flight behind us
      for (int64_t j = max((int64_t)0, issued - NK); j < issued; ++j)
        mbar_wait(k_full((int)(j % NK)), (int)((j / NK) & 1), R.status);
      for (int s2 = max(0, q_issued - 2); s2 < q_issued; ++s2)
        mbar_wait(q_full(s2 & 1), (s2 >> 1) & 1, R.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      SegWalk sg = start;
      int si = 0;
      int64_t gt = 0;
      bool ok = true;
      do {
        const int qb = si & 1;
        if (!mbar_wait(q_full(qb), (si >> 1) & 1, R.status) || *abort_flag) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t b_base = sbase + D::OFF_Q + qb * C::QBYTES;
        for (int j = sg.kb; j < sg.ke; ++j, ++gt) {
          const int st = (int)(gt % NK), slot = (int)(gt % C::NS);
          if (!mbar_wait(k_full(st), (int)((gt / NK) & 1), R.status) ||
              !mbar_wait(s_empty(slot), (int)((gt / C::NS) & 1) ^ 1, R.status) || *abort_flag) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = sbase + D::OFF_K + st * C::KBYTES;
          const uint32_t d = tmem + slot * C::N;
#pragma unroll
          for (int kk = 0; kk < C::KSTEPS; ++kk) {
            const int kc = kk / 4, sub = (kk % 4) * 32;
            const uint64_t da = desc_sw128(a_base + kc * kTileK * 128 + sub, 1024);
            const uint64_t db = desc_sw128(b_base + kc * C::N * 128 + sub, 1024);
            if constexpr (DT == DSA_BF16)
              mma_bf16(d, da, db, C::IDESC, kk > 0 ? 1u : 0u);
            else
              mma_e4m3(d, da, db, C::IDESC, kk > 0 ? 1u : 0u);
          }
          mma_commit(s_full(slot));
          mma_commit(k_empty(st));
        }
        if (!ok) break;
        mma_commit(q_empty(qb));
        ++si;
      } while (seg_next(R, row0, nrows, sg));
      if (!ok) {
        *abort_flag = 1;
        mma_commit(drain);
        mbar_wait(drain, 0, R.status);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Set `set` (four warps, one per TMEM lane quadrant) takes every fourth
    // accumulator: with a single query per accumulator this keeps all
    // sixteen warps busy.
    const int et = tid - 64, quad = warp & 3, set = et >> 7;
    SegWalk sg = start;
    int si = 0;
    int64_t gt = 0;
    bool ok = true;
    do {
      const int qb = si & 1;
      // warp-uniform outcome of each wait: the tcgen05 loads below need the
      // whole warp, so a lane that gave up takes the others with it
      bool seg_ok =
          __all_sync(0xffffffffu, mbar_wait(q_full(qb), (si >> 1) & 1, R.status) && !*abort_flag);
      const RowInfo ri = row_info(R, row0 + sg.r);
      if (seg_ok) {
        const float4* wr = reinterpret_cast<const float4*>(wq + qb * kHI);
        float* o = scores + (int64_t)sg.r * ld;
        // this set's accumulators in the segment: tiles j0, j0 + 4, ...; the key
        // scales of the next one are fetched while this one is summed (the MMAs
        // run ahead, so the scale load would otherwise stand alone in the way)
        const int64_t gt0 = gt;
        const int j0 = sg.kb + (int)((set - (int)(gt0 % kEpiSets) + kEpiSets) % kEpiSets);
        auto key_scale = [&](int j) {
          const int32_t s = j * kTileK + quad * 32 + lane;
          return (DT == DSA_E4M3 && k_scale && j < sg.ke && s <= ri.t)
                     ? __ldg(k_scale + ri.kbase + s)
                     : 1.f;
        };
        float ks_next = key_scale(j0);
        gt = gt0 + (sg.ke - sg.kb);
        // fused selection: this warp's copy of the row's threshold bin, raised
        // from the segment histogram every fourth unit and shared through the
        // row's global maximum
        uint32_t thr_w = 0, units = 0;
        if constexpr (SEL) thr_w = __ldcg(rthr + sg.r);
        for (int j = j0; j < sg.ke; j += kEpiSets) {
          const int64_t gj = gt0 + (j - sg.kb);
          const int slot = (int)(gj % C::NS);
          const int32_t s = j * kTileK + quad * 32 + lane;
          const float ks = ks_next;
          ks_next = key_scale(j + kEpiSets);
          if (!__all_sync(0xffffffffu, mbar_wait(s_full(slot), (int)((gj / C::NS) & 1), R.status) &&
                                           !*abort_flag)) {
            seg_ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t ta = tmem + ((uint32_t)(quad * 32) << 16) + slot * C::N;
          // (the fused filter reads the 64 head scores 32 at a time: fewer live registers)
          const float sum = SEL ? relu_wsum_halves(ta, wr) : relu_wsum(ta, wr);
          if constexpr (SEL) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(s_empty(slot));
            const float x = sum * ks;
            const bool valid = s <= ri.t;
            const uint32_t b = sel::score_bin(x);
            if (valid) atomicAdd(&ssm->hist[b], 1u);
            const bool keep = valid && b >= thr_w;
            uint32_t cs;
            if (sel::warp_append(keep, scnt, cs) && keep)
              cand[(int64_t)sg.r * cap + (int64_t)sg.kb * kTileK + cs] =
                  sel::pack_cand(sel::rank_key(x), s);
            ++units;
            if ((units & 7) == 0) {  // this segment's k-th best so far, shared with the row
              const uint32_t bk = kth_bin(ssm->hist, k, lane);
              if (lane == 0 && bk > thr_w) atomicMax(rthr + sg.r, bk);  // no wait for it
              thr_w = max(thr_w, bk);
            }
            if ((units & 15) == 0) {  // other segments' thresholds, now and then
              uint32_t g = 0;
              if (lane == 0) g = __ldcg(rthr + sg.r);
              thr_w = max(thr_w, __shfl_sync(0xffffffffu, g, 0));
            }
          } else {
            if (s < R.max_len) {
              if (s <= ri.t)
                o[s] = sum * ks;
              else if (fill)
                o[s] = -INFINITY;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(s_empty(slot));
          }
        }
        if (seg_ok) {
          __syncwarp();
          if (lane == 0) mbar_arrive(q_empty(qb));
        }
      }
      if constexpr (SEL) {
        // every epilogue thread comes here once per segment: the segment's
        // scores are all counted and filtered (or someone gave up)
        if (!seg_ok) *abort_flag = 1;
        seg_ok = bar_red_and<4, kEpiThreads>(seg_ok);
        if (seg_ok) {
          // the segment's count and histogram into the row's, then fresh ones
          uint32_t* const rh = rhist + (int64_t)sg.r * sel::kBins;
          for (int i = et; i < sel::kBins; i += kEpiThreads) {
            const uint32_t c = ssm->hist[i];
            if (c) atomicAdd(rh + i, c);
            ssm->hist[i] = 0;
          }
          if (et == 0) {
            segcnt[(int64_t)sg.r * (cap / kTileK) + sg.kb] = *scnt;
            *scnt = 0;
          }
          asm volatile("bar.sync 4, %0;" ::"n"(kEpiThreads) : "memory");
        }
      }
      ok = seg_ok;
      if (!ok) break;
      ++si;
    } while (seg_next(R, row0, nrows, sg));
    if (!ok) *abort_flag = 1;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TCOLS);
  }
}

}  // namespace

bool make_tmap_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize,
                  uint64_t cols, uint64_t rows, uint32_t box_cols, uint32_t box_rows) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  if (!encode) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !p)
      return false;
    encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * (uint64_t)esize};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return encode(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool indexer_tc_supported(int dtype, int H_I, int D_I) {
  return (dtype == DSA_BF16 || dtype == DSA_E4M3) && H_I == kHI && D_I == kDI;
}

template <int DT, int G, int NG, int NK>
static dsa_status_t launch_cfg(const Rows& R, int32_t row0, int32_t nrows, const void* q_idx,
                               const float* q_scale, const float* w, const void* k_idx,
                               const float* k_scale, float* scores, int64_t ld, bool fill,
                               cudaStream_t st) {
  using C = Cfg<DT, G, NG, NK>;
  CUtensorMap qmap, kmap;
  const CUtensorMapDataType tdt =
      DT == DSA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const uint32_t box_cols = 128 / C::ESZ;
  if (!make_tmap_2d(&qmap, q_idx, tdt, C::ESZ, kDI, (uint64_t)R.n_q * kHI, box_cols, C::N) ||
      !make_tmap_2d(&kmap, k_idx, tdt, C::ESZ, kDI, (uint64_t)R.n_k, box_cols, kTileK))
    return DSA_ERR_CUDA;
  auto kfn = indexer_tc_kernel<DT, G, NG, NK>;
  if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) !=
      cudaSuccess)
    return DSA_ERR_CUDA;
  const int32_t span = nrows < R.max_len ? nrows : R.max_len;
  const dim3 grid((span + C::QB - 1) / C::QB + 1, R.B);
  kfn<<<grid, kThreadsP, C::SMEM, st>>>(qmap, kmap, R, row0, nrows, w, q_scale, k_scale, scores,
                                       ld, fill ? 1 : 0);
  return launch_status();
}

// The decode kernel; SEL = the fused selection (cand / rstate / idx / k used).
template <int DT, int NK, bool SEL = false>
static dsa_status_t launch_decode(const Rows& R, int32_t row0, int32_t nrows, const void* q_idx,
                                  const float* q_scale, const float* w, const void* k_idx,
                                  const float* k_scale, float* scores, int64_t ld, bool fill,
                                  cudaStream_t st, uint64_t* cand = nullptr, int64_t cap = 0,
                                  uint32_t* rstate = nullptr, uint32_t* segcnt = nullptr,
                                  uint32_t* rhist = nullptr, int k = 0) {
  using D = DecCfg<DT, NK, SEL>;
  using C = typename D::C;
  CUtensorMap qmap, kmap;
  const CUtensorMapDataType tdt =
      DT == DSA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const uint32_t box_cols = 128 / C::ESZ;
  if (!make_tmap_2d(&qmap, q_idx, tdt, C::ESZ, kDI, (uint64_t)R.n_q * kHI, box_cols, C::N) ||
      !make_tmap_2d(&kmap, k_idx, tdt, C::ESZ, kDI, (uint64_t)R.n_k, box_cols, kTileK))
    return DSA_ERR_CUDA;
  auto kfn = indexer_decode_kernel<DT, NK, SEL>;
  if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, D::SMEM) !=
      cudaSuccess)
    return DSA_ERR_CUDA;
  kfn<<<num_sms(), kThreads, D::SMEM, st>>>(qmap, kmap, R, row0, nrows, w, q_scale, k_scale,
                                            scores, ld, fill ? 1 : 0, cand, cap, rstate, segcnt,
                                            rhist, k);
  return launch_status();
}

bool indexer_select_supported(const Rows& R, int dtype, int H_I, int D_I, int k) {
  // (the selection kernel takes rows of up to 1024 key tiles)
  return R.mode == DSA_DECODE && indexer_tc_supported(dtype, H_I, D_I) && k >= 1 &&
         k <= 16384 && R.max_len <= 1024 * kTileK;
}

// Workspace of the fused path: the candidate lists ([nrows][cap], cap =
// max_len rounded up to whole key tiles), then per row its threshold, segment
// counts and histogram (zeroed before each launch).
static int64_t select_cap(const Rows& R) { return ((int64_t)R.max_len + kTileK - 1) / kTileK * kTileK; }
static size_t select_state_words(const Rows& R, int32_t nrows) {
  return (size_t)nrows * (1 + (size_t)(select_cap(R) / kTileK) + sel::kBins);
}

size_t indexer_select_workspace(const Rows& R, int32_t nrows) {
  if (nrows <= 0) return 0;
  const size_t cand = (size_t)nrows * (size_t)select_cap(R) * sizeof(uint64_t);
  return (cand + 255) / 256 * 256 + select_state_words(R, nrows) * sizeof(uint32_t);
}

dsa_status_t launch_indexer_select(const Rows& R, int32_t row0, int32_t nrows, int dtype,
                                   int H_I, int D_I, const void* q_idx, const float* q_scale,
                                   const float* w, const void* k_idx, const float* k_scale, int k,
                                   int32_t* idx, void* ws, size_t ws_bytes, cudaStream_t st) {
  if (!indexer_select_supported(R, dtype, H_I, D_I, k)) return DSA_ERR_UNSUPPORTED;
  if (nrows <= 0) return DSA_OK;
  if (!ws || ws_bytes < indexer_select_workspace(R, nrows)) return DSA_ERR_WORKSPACE;
  const int64_t cap = select_cap(R);
  uint64_t* cand = reinterpret_cast<uint64_t*>(ws);
  const size_t cbytes = ((size_t)nrows * (size_t)cap * sizeof(uint64_t) + 255) / 256 * 256;
  uint32_t* rstate = reinterpret_cast<uint32_t*>(reinterpret_cast<char*>(ws) + cbytes);
  uint32_t* segcnt = rstate + nrows;
  uint32_t* rhist = segcnt + (size_t)nrows * (cap / kTileK);
  if (cudaMemsetAsync(rstate, 0, select_state_words(R, nrows) * sizeof(uint32_t), st) !=
      cudaSuccess)
    return DSA_ERR_CUDA;
  dsa_status_t s =
      dtype == DSA_BF16
          ? launch_decode<DSA_BF16, 5, true>(R, row0, nrows, q_idx, q_scale, w, k_idx, k_scale,
                                             nullptr, 0, false, st, cand, cap, rstate, segcnt,
                                             rhist, k)
          : launch_decode<DSA_E4M3, 12, true>(R, row0, nrows, q_idx, q_scale, w, k_idx, k_scale,
                                              nullptr, 0, false, st, cand, cap, rstate, segcnt,
                                              rhist, k);
  if (s) return s;
  return launch_select_rows(R, row0, nrows, cand, cap, segcnt, rhist, k, idx, st);
}

dsa_status_t launch_indexer_tc(const Rows& R, int32_t row0, int32_t nrows, int dtype, int H_I,
                               int D_I, const void* q_idx, const float* q_scale, const float* w,
                               const void* k_idx, const float* k_scale, float* scores, int64_t ld,
                               bool fill, cudaStream_t st) {
  if (!indexer_tc_supported(dtype, H_I, D_I)) return DSA_ERR_UNSUPPORTED;
  if (nrows <= 0) return DSA_OK;
  const bool decode = R.mode == DSA_DECODE;
  if (dtype == DSA_BF16) {
    if (decode)
      return launch_decode<DSA_BF16, 6>(R, row0, nrows, q_idx, q_scale, w, k_idx, k_scale, scores,
                                        ld, fill, st);
    return launch_cfg<DSA_BF16, 4, 2, 2>(R, row0, nrows, q_idx, q_scale, w, k_idx,
                                                k_scale, scores, ld, fill, st);
  }
  if (decode)
    return launch_decode<DSA_E4M3, 12>(R, row0, nrows, q_idx, q_scale, w, k_idx, k_scale, scores,
                                       ld, fill, st);
  return launch_cfg<DSA_E4M3, 4, 2, 4>(R, row0, nrows, q_idx, q_scale, w, k_idx, k_scale,
                                              scores, ld, fill, st);
}

}  // namespace dsa
