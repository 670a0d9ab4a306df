// Sparse MLA attention on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// For query row r, head h and the selected positions S_r (k slots, -1 = empty):
//   z[h,s] = sm_scale * <q[r,h,0:576], C[s,0:576]>
//   o[r,h] = sum_s softmax_S(z[h,:])_s * C[s,0:512],   lse = log sum_s exp z
// ("GLM sparse attention", MLA passage: one cached latent row (512 latent +
// 64 rotary) per token, scored by the absorbed query of every head, so one
// gathered row serves all 128 heads; a full softmax over the selected rows;
// these rows lie anywhere in the cache, so the gather sets the pace.)
//
// TMEM holds 128 lanes x 512 fp32 columns, exactly the size of the 128 x 512
// output accumulator.  Each query row therefore runs on two CTAs, one per
// half of the 512 value columns.  Both compute the full 576-d scores of every
// tile (the QK product is done twice) and make identical softmax decisions;
// nothing is exchanged between them.  Measured on B200 with 2-CTA clusters on
// two SMs, distributed shared memory moves only 3-10 bytes/cycle per SM
// (remote loads, remote stores and bulk copies alike), so exchanging a 32 KB
// partial-score tile per 64 selected rows would cost more than recomputing
// the 9.4 MFLOP of QK on the tensor cores.
//
// Per CTA:
//   TMEM columns   0..191  query dims 0..383 of every head (bf16 pairs, the
//                          .ts MMA form reads A from TMEM)
//                192..255  the 64-column score tile (fp32)
//                256..511  this CTA's 256 output columns (fp32)
//   shared memory: query dims 384..575 (three 128-byte-swizzled K-major
//   atoms), two stages of 64 gathered cache rows (nine atoms of 64 dims,
//   K-major for QK, MN-major for PV), and the tile's probabilities P (bf16,
//   K-major) for PV.
// The query row arrives by TMA (nine 16 KB boxes, one per 64-dim atom of
// all heads): dims 384..575 straight into their operand atoms, dims 0..383
// staged in the not yet used gather stages, from which the softmax threads
// move them into TMEM.  (Loaded by each softmax thread from its own head's
// row, the query took about 20K cycles of a CTA's start.)
// The gather: 224 producer threads publish each tile's indices and fetch its
// QK-only atoms, the 256 softmax threads its value atoms (bf16 cache), all
// with 16-byte cp.async, eight lanes per 128-byte segment, straight into the
// swizzled layout the MMA reads (an empty slot -1 is zero-filled).
// Measured on B200 (scattered 128-byte rows, L2-resident source, 208 KB of
// shared memory per CTA): cp.async from 7 warps sustains 20 B/cycle per SM,
// from 15 warps 27; TMA tile::gather4 from 8 issuing threads 28, and
// cp.async and gather4 issued together stay at 28 (one limit for both).
// Inside this kernel, gather4 from lane 0 of the 7 producer warps was slower
// than cp.async (6.2 against 5.0 ms on 4096 prefill rows): one thread issues
// a gather4 only about every 120 cycles.
//
// Warp roles (512 threads per CTA):
//   warps 0-6   gather producer (indices -> shared memory, cp.async of the
//               QK-only atoms; of every atom for an e4m3 cache, via registers)
//   warp 7      TMEM allocator and MMA issuer (one thread, issues whichever of
//               QK(next tile) and PV(oldest tile with P ready) can go)
//   warps 8-15  softmax, two warpgroups: a thread owns one head (its TMEM
//               lane) and half of each tile's 64 rows.  Online softmax in the
//               log2 domain with a lazy rescale (the reference max moves only
//               when a new score exceeds it by more than 2^8); P to shared
//               memory as bf16; the denominator sums the fp32 probabilities;
//               cp.async of the next tile's value atoms (bf16 cache); final
//               normalisation and store of this CTA's output columns.
// Decode rows are split over several CTA pairs; each split writes a
// normalised partial output and its log-sum-exp, merged by
// attn_combine_kernel.
#include <cudaTypedefs.h>

#include <cstdint>

#include "kernels.cuh"
#include "sm100.cuh"

namespace dsa {

using namespace sm100;

namespace {

constexpr int kH = 128, kDK = 576, kDV = 512;
constexpr int kNT = 64;                        // selected rows per tile
constexpr int kAtoms = kDK / 64;               // 9 swizzle atoms per gathered row
constexpr int kProducers = 224;                // warps 0-6
constexpr int kMmaWarp = 7;
constexpr int kSoftmax0 = 256;                 // first softmax thread (warps 8-15)
constexpr int kSoftmaxThreads = 256;
constexpr int kThreads = kSoftmax0 + kSoftmaxThreads;  // 512
constexpr int kAtomBytes = kNT * 128;          // 8192: one 64-dim atom of a tile
constexpr int kCBytes = kAtoms * kAtomBytes;   // 73728 per stage
constexpr int kStages = 2;
// A stage is filled and released in two groups of atoms: the 5 atoms only QK
// reads (group A, free once the QK steps over them retire) and the 4 atoms of
// this CTA's value columns (group V, read by QK and PV, free once PV retires).
constexpr int kAtomsA = 5, kAtomsV = 4;
constexpr int kChunksA = kNT * kAtomsA * 8;    // 2560 16-byte chunks
constexpr int kChunksV = kNT * kAtomsV * 8;    // 2048
constexpr int kIdxRing = 8;                    // tiles whose indices are held
// e4m3 cache: a 16-byte load brings 16 codes, two 16-byte bf16 chunks of the
// swizzled operand, so each group takes half as many loads as chunks.
constexpr int kLoadsA = kChunksA / 2, kLoadsV = kChunksV / 2;  // 1280, 1024
constexpr int kQTmemDims = 384;                // query dims held in TMEM
constexpr int kQSmemAtoms = (kDK - kQTmemDims) / 64;  // 3 atoms in shared memory
constexpr int kQAtomBytes = kH * 128;          // 16384
constexpr int kPBytes = kH * 128;              // P: 128 heads x 64 rows bf16
constexpr int OFF_C = 0;
constexpr int OFF_Q = OFF_C + kStages * kCBytes;
constexpr int OFF_P = OFF_Q + kQSmemAtoms * kQAtomBytes;
constexpr int OFF_IDX = OFF_P + kPBytes;                 // [ring][64] int32
constexpr int OFF_MASK = OFF_IDX + kIdxRing * kNT * 4;   // [ring][2] uint32 validity bits
constexpr int OFF_HMAX = OFF_MASK + kIdxRing * 2 * 4;    // [2 tiles][2 warpgroups][128] float
constexpr int OFF_KSC = OFF_HMAX + 2 * 2 * kH * 4;       // [ring][64] fp32 cache scales (e4m3)
constexpr int OFF_BAR = OFF_KSC + kIdxRing * kNT * 4;
constexpr int kNumBars = 23;
constexpr int OFF_MISC = OFF_BAR + kNumBars * 8;
// The dynamic window starts 1024-aligned (right after the driver's reserved
// kilobyte, with no static shared memory); the kernel checks it.
constexpr int kSmem = OFF_MISC + 16;
static_assert(kSmem <= 232448, "shared memory");
static_assert(OFF_Q % 1024 == 0 && OFF_P % 1024 == 0 && OFF_BAR % 8 == 0, "alignment");
// TMEM columns
constexpr uint32_t TM_Q = 0;     // query dims 0..383 of all heads, bf16 pairs (192 cols)
constexpr uint32_t TM_S = 192;   // 64-column score tile
constexpr uint32_t TM_O = 256;   // 256-column output accumulator
constexpr uint32_t IDESC_QK = idesc(1, 128, kNT);
// PV MMA width: 256 (one MMA per 16 rows of the tile for this CTA's value
// columns).  Four N = 64 MMAs instead (the QK MMAs are N = 64; a probe stream
// that mixed N = 64 and N = 256 MMAs took about twice the time of its parts)
// measured 3% slower in this kernel.
constexpr int kPvN = 256;
constexpr uint32_t IDESC_PV = idesc(1, 128, kPvN, false, true);
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescale = 8.0f;  // log2 headroom before the reference max moves

enum {
  B_QREADY = 0,   // the query is in TMEM and shared memory (every softmax thread)
  B_AFULL = 1,    // [2] group-A rows landed, indices published (producers)
  B_VFULL = 3,    // [2] group-V rows landed (producers)
  B_AEMPTY = 5,   // [2] QK steps over group A retired
  B_VEMPTY = 7,   // [2] PV of the stage retired
  B_SFULL = 9,    // QK retired
  B_SEMPTY = 10,  // scores read (every softmax thread)
  B_PFULL = 11,   // P stored (every softmax thread)
  B_PVDONE = 12,  // PV retired
  B_DRAIN = 13,
  B_IDX = 14,     // [kIdxRing] the tile's indices, mask and scales are in the ring (producers)
  B_QLOAD = 22    // the query row landed (TMA transaction bytes)
};
static_assert(B_IDX + kIdxRing <= B_QLOAD && B_QLOAD < kNumBars, "barrier count");

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

// Orders this thread's generic-proxy shared-memory writes before later
// async-proxy reads (the MMA reading the query and P operands).
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 16 bytes of read-only global memory, not kept in L1.
__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// 16 e4m3 codes (dims 16c .. 16c+15 of a 64-dim atom row) -> the two 16-byte
// bf16 chunks 2c, 2c+1 of that row at `rowp`, in the 128-byte swizzle.
__device__ __forceinline__ void store_codes(uint8_t* rowp, int c, int row, const uint4& x) {
  uint4 a, b;
  e4m3x4_to_bf16x4(x.x, a.x, a.y);
  e4m3x4_to_bf16x4(x.y, a.z, a.w);
  e4m3x4_to_bf16x4(x.z, b.x, b.y);
  e4m3x4_to_bf16x4(x.w, b.z, b.w);
  *reinterpret_cast<uint4*>(rowp + (((2 * c) ^ (row & 7)) << 4)) = a;
  *reinterpret_cast<uint4*>(rowp + (((2 * c + 1) ^ (row & 7)) << 4)) = b;
}

// Diagnostic build only (-DDSA_ATTN_TRACE, libdsa_trace.so; stage_bench.py
// --trace prints the table): clock64 stamps of each tile's events on the two
// CTAs of one row -- the MMA thread's issue of each work item, the softmax
// thread's waits, producer thread 0's copies.  The product library compiles
// the stamps to nothing.
#ifdef DSA_ATTN_TRACE
constexpr int kTraceTiles = 64, kTraceEvents = 16;
__device__ long long g_attn_trace[2 * kTraceTiles * kTraceEvents];
__device__ long long g_attn_trace_t0[2];
__device__ int g_attn_trace_item = -1;
#define DSA_STAMP(n, f)                                                                \
  do {                                                                                 \
    if (tslot >= 0 && (n) >= 0 && (n) < kTraceTiles)                                   \
      g_attn_trace[(tslot * kTraceTiles + (n)) * kTraceEvents + (f)] = clock64();      \
  } while (0)
#else
#define DSA_STAMP(n, f) \
  do {                  \
  } while (0)
#endif

struct Split {
  int nsplit, tiles_per_split;
  int packed;  // the row's valid indices come first, at most t + 1 of them
};

// Fixed scratch for callers that cannot allocate device memory (see
// launch_attn_tc_static): the split partials of one call, 20 MiB, room for
// 79 (query row, split) blocks of 128 x 513 floats.
constexpr size_t kPartialBytes = size_t(kH) * (kDV + 1) * sizeof(float);
constexpr size_t kStaticScratchBytes = size_t(20) << 20;
constexpr int kScratchPairs = int((kStaticScratchBytes - 256) / kPartialBytes);
static __device__ __align__(256) float g_attn_scratch[kStaticScratchBytes / sizeof(float)];

// Decode rows are few: split each row's tiles over several CTA pairs (two
// CTAs per pair, one CTA per SM).  Only splits that keep every pair in ONE
// wave are taken: a second wave costs a whole split's tiles for the pairs
// that spill into it.  Among those, the estimate is tiles per split plus the
// merge (each (row, split) block's 256 KiB of fp32 partials go out to memory
// and back, about 1/48 of a gathered tile's time).  The pair count is capped
// by the fixed scratch, so both attention entry points plan alike.
inline Split plan_split(int32_t nrows, int k) {
  const int tiles = k > 0 ? (k + kNT - 1) / kNT : 1;
  int pairs = num_sms() / 2;
  if (pairs > kScratchPairs) pairs = kScratchPairs;
  Split best{1, tiles};
  int64_t best_cost = int64_t(tiles) * 48;
  for (int want = 2; want <= tiles && (int64_t)nrows * want <= pairs; ++want) {
    const int tps = (tiles + want - 1) / want, ns = (tiles + tps - 1) / tps;
    if (ns != want) continue;  // same plan as a smaller split
    const int64_t cost = int64_t(tps) * 48 + (int64_t)nrows * ns;
    if (cost < best_cost) {
      best_cost = cost;
      best = Split{ns, tps};
    }
  }
  return best;
}

// FP8: the cache holds e4m3 codes [n_k, 576] with one fp32 scale per token
// (kv_scale).  The codes are gathered through registers and written to the
// same swizzled bf16 operand, exactly converted; the MMAs are the bf16 ones.
// The token's scale multiplies its score column and its probability in the
// PV operand (P' = p * scale); the softmax denominator sums p.
// qmap: the queries as a [n_q * 128, 576] bf16 map, 64 x 128 boxes, 128-byte
// swizzle (one box = one K-major operand atom of all heads).
template <bool FP8>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap qmap, const void* __restrict__ kv,
                   const float* __restrict__ kv_scale, Rows R,
                   int32_t row0, const int32_t* __restrict__ idx, int k, float scale2, Split sp,
                   uint16_t* __restrict__ out, float* __restrict__ lse,
                   float* __restrict__ part_o, float* __restrict__ part_lse) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  const uint32_t sb = smem_u32(smem);
  if (sb & 1023u) {  // the swizzled operand layouts need 1024-byte alignment
    if (threadIdx.x == 0) raise_status(R, kErrLayout);
    return;
  }
  int32_t* sidx = reinterpret_cast<int32_t*>(smem + OFF_IDX);
  uint32_t* vmask = reinterpret_cast<uint32_t*>(smem + OFF_MASK);
  float* hmax = reinterpret_cast<float*>(smem + OFF_HMAX);
  float* ksc = reinterpret_cast<float*>(smem + OFF_KSC);
  auto bar = [&](int i) { return sb + OFF_BAR + 8u * i; };
  constexpr int kRowBytes = FP8 ? kDK : kDK * 2;  // one cached token
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int half = blockIdx.x & 1;  // this CTA's output columns 256*half ..
#ifdef DSA_ATTN_TRACE
  const int tslot = (int)(blockIdx.x >> 1) == g_attn_trace_item ? half : -1;
  if (threadIdx.x == 0 && tslot >= 0) g_attn_trace_t0[tslot] = clock64();
#endif
  const int item = blockIdx.x >> 1;
  const int32_t rloc = item / sp.nsplit, split = item % sp.nsplit;
  const int32_t r = row0 + rloc;
  const RowInfo ri = row_info(R, r);
  const int slot_lo = split * sp.tiles_per_split * kNT;
  // (packed indices: the slots after min(t + 1, k) are all empty)
  const int slot_end = sp.packed ? min(k, max(ri.t + 1, 0)) : k;
  const int slot_hi = min(slot_end, slot_lo + sp.tiles_per_split * kNT);
  const int ntiles = slot_hi > slot_lo ? (slot_hi - slot_lo + kNT - 1) / kNT : 0;

  if (tid == 0) {
    mbar_init(bar(B_QREADY), kSoftmaxThreads);
    for (int i = 0; i < kStages; ++i) {
      // per producer: an arrive after the index store and a cp.async arrive
      mbar_init(bar(B_AFULL + i), 2 * kProducers);
      // group V: a cp.async arrive per softmax thread (bf16) or an arrive per producer (e4m3)
      mbar_init(bar(B_VFULL + i), FP8 ? kProducers : kSoftmaxThreads);
      mbar_init(bar(B_AEMPTY + i), 1);
      mbar_init(bar(B_VEMPTY + i), 1);
    }
    mbar_init(bar(B_SFULL), 1);
    for (int i = 0; i < kIdxRing; ++i) mbar_init(bar(B_IDX + i), kProducers);
    mbar_init(bar(B_SEMPTY), kSoftmaxThreads);
    mbar_init(bar(B_PFULL), kSoftmaxThreads);
    mbar_init(bar(B_PVDONE), 1);
    mbar_init(bar(B_DRAIN), 1);
    mbar_init(bar(B_QLOAD), 1);
    *abort_flag = 0;
    fence_mbar_init();
    // The query row by TMA, nine atoms of 128 heads x 64 dims: dims 384..575
    // straight into their operand atoms, dims 0..383 staged in the gather
    // stages (unused until the softmax threads have moved them into TMEM).
    tma_prefetch(&qmap);
    mbar_expect_tx(bar(B_QLOAD), (uint32_t)(kH * kDK * 2));
    for (int a = 0; a < kAtoms; ++a) {
      const uint32_t dst = a < kQTmemDims / 64 ? sb + OFF_C + a * kQAtomBytes
                                               : sb + OFF_Q + (a - kQTmemDims / 64) * kQAtomBytes;
      tma_load_2d(dst, &qmap, 64 * a, r * kH, bar(B_QLOAD));
    }
  }
  if (warp == kMmaWarp) {
    tmem_alloc(sb + OFF_MISC, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const char* kvb = reinterpret_cast<const char*>(kv) + ri.kbase * kRowBytes;
  // bf16 cache: issues 16-byte chunk i of atom group A or V (eight lanes per
  // 128-byte segment of a row, a warp four consecutive segments) of the tile
  // whose indices are in ring slot `ring` into stage st.
  auto issue = [&](int st, int ring, int i, bool group_a) {
    const int ch = i & 7, seg = i >> 3;
    int row, atom;
    if (group_a) {  // the five atoms only QK reads
      row = seg / kAtomsA;
      const int ai = seg - row * kAtomsA;
      atom = ai < 4 ? 4 * (half ^ 1) + ai : 8;
    } else {  // this CTA's value columns
      row = seg >> 2;
      atom = 4 * half + (seg & 3);
    }
    const int32_t s = sidx[ring * kNT + row];
    const char* src = s >= 0 ? kvb + (int64_t)s * kRowBytes + atom * 128 + ch * 16
                             : reinterpret_cast<const char*>(kv);
    const uint32_t nbytes = s >= 0 ? 16u : 0u;  // 0: zero-fill
    const uint32_t dst = sb + OFF_C + st * kCBytes + atom * kAtomBytes + row * 128 +
                         ((uint32_t)(ch ^ (row & 7)) << 4);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(nbytes)
                 : "memory");
  };

  if (warp < kMmaWarp) {
    // ------------------------------------------------------------ gather producer
    auto load_idx = [&](int n) -> int32_t {
      const int slot = slot_lo + n * kNT + tid;
      int32_t s = slot < slot_hi ? __ldg(idx + (int64_t)rloc * k + slot) : -1;
      // candidates are the causal positions 0..t (t < L_b); a later one is bad data
      if (s < -1 || s > ri.t) {
        if (s != -1 && ri.t >= 0) raise_status(R, kErrBadIndex);
        s = -1;
      }
      return s;
    };
    // the scale of cache row s of this sequence (e4m3 cache), 0 for an empty slot
    auto load_scale = [&](int32_t s) -> float {
      return (FP8 && s >= 0) ? __ldg(kv_scale + ri.kbase + s) : 0.f;
    };
    // Threads 0..63 own the index (and scale) of tile row tid.
    int32_t pre = (tid < kNT && ntiles > 0) ? load_idx(0) : -1;
    float pre_sc = load_scale(pre);
    // Publishes the indices (and mask and scales) of tile n into ring slot
    // n % kIdxRing (threads 0..63 hold them in pre / pre_sc), then loads tile
    // n+1's into pre / pre_sc.
    auto publish = [&](int n) {
      const int ring = n % kIdxRing;
      if (tid < kNT) {
        sidx[ring * kNT + tid] = pre;
        if (FP8) ksc[ring * kNT + tid] = pre_sc;
        const uint32_t bits = __ballot_sync(0xffffffffu, pre >= 0);
        if (lane == 0) vmask[ring * 2 + warp] = bits;
      }
      mbar_arrive(bar(B_AFULL + n % kStages));  // publishes indices to the MMA issuer
      mbar_arrive(bar(B_IDX + ring));           // ... and indices, mask, scales to the softmax
      asm volatile("bar.sync 2, %0;" ::"n"(kProducers) : "memory");  // producers see them
      if (tid < kNT) {  // overlaps the copies below
        pre = n + 1 < ntiles ? load_idx(n + 1) : -1;
        pre_sc = load_scale(pre);
      }
    };
    if constexpr (FP8) {
      // Codes go through registers (converted on the way into the swizzled
      // bf16 operand), software-pipelined: tile n+1's loads are in flight
      // while tile n waits for its stage, which QK(n-2) and PV(n-2) release.
      constexpr int JA = (kLoadsA + kProducers - 1) / kProducers;
      constexpr int JV = (kLoadsV + kProducers - 1) / kProducers;
      uint4 xa[JA], xv[JV];
      auto load = [&](int n) {
        const int ring = n % kIdxRing;
#pragma unroll
        for (int j = 0; j < JA; ++j) {
          const int i = tid + kProducers * j, c = i & 3, seg = i >> 2, row = seg / kAtomsA;
          const int ai = seg - row * kAtomsA, atom = ai < 4 ? 4 * (half ^ 1) + ai : 8;
          const int32_t s = i < kLoadsA ? sidx[ring * kNT + row] : -1;
          xa[j] = s >= 0 ? ld_nc_v4(kvb + (int64_t)s * kRowBytes + atom * 64 + c * 16)
                         : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int j = 0; j < JV; ++j) {  // 16 codes per load: quarter c of segment (row, atom)
          const int i = tid + kProducers * j, c = i & 3, seg = i >> 2, row = seg >> 2;
          const int atom = 4 * half + (seg & 3);
          const int32_t s = i < kLoadsV ? sidx[ring * kNT + row] : -1;
          xv[j] = s >= 0 ? ld_nc_v4(kvb + (int64_t)s * kRowBytes + atom * 64 + c * 16)
                         : make_uint4(0, 0, 0, 0);
        }
      };
      if (ntiles > 0) {
        publish(0);
        load(0);
      }
      for (int n = 0; n < ntiles; ++n) {
        const int st = n % kStages;
        const uint32_t par = ((n / kStages) & 1) ^ 1;
        // (the first tile also waits until the staged query has left the stages)
        bool ok = (n > 0 || mbar_wait(bar(B_QREADY), 0, R.status)) &&
                  mbar_wait(bar(B_AEMPTY + st), par, R.status) &&
                  mbar_wait(bar(B_VEMPTY + st), par, R.status) && !*abort_flag;
        if (!bar_and<2, kProducers>(ok)) {
          *abort_flag = 1;
          break;
        }
#pragma unroll
        for (int j = 0; j < JA; ++j) {
          const int i = tid + kProducers * j, c = i & 3, seg = i >> 2, row = seg / kAtomsA;
          const int ai = seg - row * kAtomsA, atom = ai < 4 ? 4 * (half ^ 1) + ai : 8;
          if (i < kLoadsA)
            store_codes(smem + OFF_C + st * kCBytes + atom * kAtomBytes + row * 128, c, row,
                        xa[j]);
        }
        fence_async_smem();
        mbar_arrive(bar(B_AFULL + st));
#pragma unroll
        for (int j = 0; j < JV; ++j) {
          const int i = tid + kProducers * j, c = i & 3, seg = i >> 2, row = seg >> 2;
          const int atom = 4 * half + (seg & 3);
          if (i < kLoadsV)
            store_codes(smem + OFF_C + st * kCBytes + atom * kAtomBytes + row * 128, c, row,
                        xv[j]);
        }
        fence_async_smem();
        mbar_arrive(bar(B_VFULL + st));
        if (n + 1 < ntiles) {
          publish(n + 1);
          load(n + 1);
        }
      }
    } else {
      for (int n = 0; n < ntiles; ++n) {
        const int st = n % kStages, ring = n % kIdxRing;
        const uint32_t par = ((n / kStages) & 1) ^ 1;
        // group A of the stage is free once QK(n-2) read it (and, for the
        // first tile, once the staged query has left the stages)
        bool ok = (n > 0 || mbar_wait(bar(B_QREADY), 0, R.status)) &&
                  mbar_wait(bar(B_AEMPTY + st), par, R.status) && !*abort_flag;
        if (tid == 0) DSA_STAMP(n, 10);
        if (!bar_and<2, kProducers>(ok)) {
          *abort_flag = 1;
          break;
        }
        publish(n);
#pragma unroll
        for (int j = 0; j < (kChunksA + kProducers - 1) / kProducers; ++j)
          if (tid + kProducers * j < kChunksA) issue(st, ring, tid + kProducers * j, true);
        asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(
                         bar(B_AFULL + st))
                     : "memory");
        if (tid == 0) DSA_STAMP(n, 11);
        // (group V, this CTA's value columns, is fetched by the softmax
        // threads once PV(n-2) has released it)
      }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(bar(B_QREADY), 0, R.status);
      // Three kinds of work, issued as soon as they can go (bf16 cache: QK-B
      // first, then PV, then QK-A):
      //   QK-A(n): the 20 K steps over group A (rows landed, score tile free)
      //   QK-B(n): the 16 K steps over group V, then S(n) is complete
      //   PV(n):   P(n) stored
      // Splitting QK lets PV(n-1) slip in between QK-A(n) and QK-B(n) when
      // group V of tile n is late, and group A of a stage is released as soon
      // as its QK steps retire.  With QK-B(n) ahead of PV(n-1) when both can
      // go, S(n) completes earlier and PV(n-1) runs while the softmax threads
      // read it (measured 4.29 against 4.58 ms on 4096 prefill rows, together
      // with the softmax-side fetch of group V).
      // Polling uses the non-blocking test: try_wait may suspend the thread
      // while another of the three could already go.
      int na = 0, nb = 0, np = 0;
      // Descriptors advance by adding byte offsets / 16 to the start address
      // field (no carry: shared addresses stay below 256 KB).
      const uint64_t dq0 = desc_sw128(sb + OFF_Q, 1024);
      const uint64_t dp0 = desc_sw128(sb + OFF_P, 1024);
      const uint32_t ts = tmem + TM_S;
      // One QK K step over dims 64*atom + 16*sub of the stage whose
      // descriptor is db: A from TMEM for dims < 384, else from the query
      // atoms in shared memory.  `atom` and `sub` are compile-time after
      // unrolling, so a step is a handful of instructions.
      auto qk_step = [&](uint64_t db, int atom, int sub, uint32_t acc) {
        const uint64_t bdesc = db + (uint64_t)((atom * kAtomBytes + sub * 32) >> 4);
        if (atom < kQTmemDims / 64)
          mma_bf16_ts(ts, tmem + TM_Q + 32 * atom + 8 * sub, bdesc, IDESC_QK, acc);
        else
          mma_bf16(ts,
                   dq0 + (uint64_t)(((atom - kQTmemDims / 64) * kQAtomBytes + sub * 32) >> 4),
                   bdesc, IDESC_QK, acc);
      };
      long long t0 = clock64();
      while (ok && np < ntiles) {
        if (*abort_flag) {
          ok = false;
          break;
        }
        bool progressed = false;
        auto qkb_go = [&] {
          return nb < na && mbar_test(bar(B_VFULL + nb % kStages), (nb / kStages) & 1);
        };
        auto pv_go = [&] { return np < nb && mbar_test(bar(B_PFULL), np & 1); };
        // (bf16 cache: the score tile's release is the usual holdup of QK-A,
        // tested first)
        auto qka_go = [&] {
          if (na != nb || na >= ntiles) return false;
          const uint32_t afull = bar(B_AFULL + na % kStages), apar = (na / kStages) & 1;
          return FP8 ? mbar_test(afull, apar) && mbar_test(bar(B_SEMPTY), (na & 1) ^ 1)
                     : mbar_test(bar(B_SEMPTY), (na & 1) ^ 1) && mbar_test(afull, apar);
        };
        auto do_qkb = [&] {
          DSA_STAMP(nb, 2);
          fence_async_smem();  // rows written by cp.async (generic proxy)
          tc_fence_after();
          const uint64_t db = desc_sw128(sb + OFF_C + (nb % kStages) * kCBytes, 1024);
          if (half) {
#pragma unroll
            for (int a = 0; a < kAtomsV; ++a)
#pragma unroll
              for (int sub = 0; sub < 4; ++sub) qk_step(db, 4 + a, sub, 1u);
          } else {
#pragma unroll
            for (int a = 0; a < kAtomsV; ++a)
#pragma unroll
              for (int sub = 0; sub < 4; ++sub) qk_step(db, a, sub, 1u);
          }
          mma_commit(bar(B_SFULL));
          DSA_STAMP(nb, 3);
          ++nb;
          progressed = true;
        };
        auto do_pv = [&] {
          DSA_STAMP(np, 4);
          tc_fence_after();
          // this CTA's value columns: atoms 4*half .. 4*half+3 of the stage
          const uint64_t dv = desc_sw128_mn(
              sb + OFF_C + (np % kStages) * kCBytes + 4 * half * kAtomBytes, kAtomBytes, 1024);
#pragma unroll
          for (int kk = 0; kk < kNT / 16; ++kk)
#pragma unroll
            for (int a = 0; a < 256 / kPvN; ++a)  // 64-column blocks are atoms kAtomBytes apart
              mma_bf16(tmem + TM_O + kPvN * a, dp0 + (uint64_t)(kk * 2),
                       dv + (uint64_t)(kk * 128 + a * (kPvN / 64) * (kAtomBytes >> 4)), IDESC_PV,
                       (np > 0 || kk > 0) ? 1u : 0u);
          mma_commit(bar(B_PVDONE));
          mma_commit(bar(B_VEMPTY + np % kStages));
          DSA_STAMP(np, 5);
          ++np;
          progressed = true;
        };
        auto do_qka = [&] {
          DSA_STAMP(na, 0);
          fence_async_smem();  // rows written by cp.async (generic proxy)
          tc_fence_after();
          const uint64_t db = desc_sw128(sb + OFF_C + (na % kStages) * kCBytes, 1024);
          // group A atoms: the other latent half (4*(half^1) .. +3), then rotary (8)
          if (half) {
#pragma unroll
            for (int a = 0; a < kAtomsA; ++a)
#pragma unroll
              for (int sub = 0; sub < 4; ++sub)
                qk_step(db, a < 4 ? a : 8, sub, (a > 0 || sub > 0) ? 1u : 0u);
          } else {
#pragma unroll
            for (int a = 0; a < kAtomsA; ++a)
#pragma unroll
              for (int sub = 0; sub < 4; ++sub)
                qk_step(db, a < 4 ? 4 + a : 8, sub, (a > 0 || sub > 0) ? 1u : 0u);
          }
          mma_commit(bar(B_AEMPTY + na % kStages));
          DSA_STAMP(na, 1);
          ++na;
          progressed = true;
        };
        // bf16 cache: QK-B first, and what usually follows an issue is tested
        // right after it, without another trip round the loop (4.04 against
        // 4.29 ms on 4096 prefill rows).  e4m3 cache: PV first (its value
        // atoms come from the producers, behind group A), one item per trip
        // (chaining measured 5.06 against 4.95 ms there).
        if constexpr (FP8) {
          if (pv_go())
            do_pv();
          else if (qkb_go())
            do_qkb();
          else if (qka_go())
            do_qka();
        } else {
          auto qkb_then_pv = [&] {
            do_qkb();
            if (pv_go()) do_pv();
          };
          if (qkb_go()) {
            qkb_then_pv();
          } else if (pv_go()) {
            do_pv();
          } else if (qka_go()) {
            do_qka();
            if (qkb_go()) qkb_then_pv();
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
    // tile for the head of its TMEM lane.
    const int wg = (warp - kSoftmax0 / 32) >> 2;
    const int quad = warp & 3;
    const int h = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    {
      // query dims 0..383 -> TMEM columns 0..191 (warpgroup wg: 192 dims),
      // read from the atoms the TMA staged in the gather stages
      const bool q_ok = mbar_wait(bar(B_QLOAD), 0, R.status);
      if (!q_ok) *abort_flag = 1;
      if (q_ok) {
#pragma unroll
        for (int part = 0; part < 4; ++part) {  // 4 x 48 dims = 4 x 24 columns
          uint32_t w24[24];
#pragma unroll
          for (int v = 0; v < 6; ++v) {
            const int d = 192 * wg + 48 * part + 8 * v, a = d >> 6, ch = (d >> 3) & 7;
            const uint4 x = *reinterpret_cast<const uint4*>(
                smem + OFF_C + a * kQAtomBytes + h * 128 + ((ch ^ (h & 7)) << 4));
            w24[4 * v] = x.x;
            w24[4 * v + 1] = x.y;
            w24[4 * v + 2] = x.z;
            w24[4 * v + 3] = x.w;
          }
          const uint32_t ta = tmem + lane_off + TM_Q + 96 * wg + 24 * part;
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
      }
      tc_fence_before();
      mbar_arrive(bar(B_QREADY));  // the staged atoms are read: the stages are free
    }
    // bf16 cache: group V of tile m (this CTA's value atoms, 2048 chunks, 8 per
    // thread), once PV(m-2) has freed the stage and the producers have
    // published m's indices.  Tile m+1's goes out in tile m's iteration right
    // after the wait for PV(m-1), the release of its stage, which that
    // iteration waits for anyway before storing P(m).  The producers thus only
    // fetch group A, and the copies are issued by 15 warps instead of 7
    // (probe: 27 against 20 B/cycle per SM).  For an e4m3 cache the producers
    // fetch both groups.
    auto fetch_v = [&](int m) -> bool {
      if constexpr (FP8) {
        return true;
      } else {
        const int st = m % kStages, ring = m % kIdxRing;
        const bool w = mbar_wait(bar(B_VEMPTY + st), ((m / kStages) & 1) ^ 1, R.status) &&
                       mbar_wait(bar(B_IDX + ring), (m / kIdxRing) & 1, R.status);
        if (w) {
#pragma unroll
          for (int j = 0; j < kChunksV / kSoftmaxThreads; ++j)
            issue(st, ring, (tid - kSoftmax0) + kSoftmaxThreads * j, false);
        }
        asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(
                         bar(B_VFULL + st))
                     : "memory");
        if (tid == kSoftmax0) DSA_STAMP(m, 12);
        return w;
      }
    };
    static_assert(kChunksV % kSoftmaxThreads == 0, "group V split");
    // tile 0's value atoms go where the staged query was: after every
    // softmax thread has read it
    if constexpr (!FP8) {
      if (ntiles > 0 && !(mbar_wait(bar(B_QREADY), 0, R.status) && fetch_v(0))) *abort_flag = 1;
    }
    // row h of P: this warpgroup's 32 rows are 16-byte chunks 4wg .. 4wg+3
    uint8_t* const prow = smem + OFF_P + h * 128;
    float m2 = -INFINITY, l = 0.f;
    bool ok = true;
    for (int n = 0; ok && n < ntiles; ++n) {
      float s[32];
      // S(n) retired; then the tile's validity bits and scales are visible
      // (B_IDX: the producers published them; they cannot publish tile
      // n + kIdxRing into this slot before this thread has read S(n+1), so
      // the parity names tile n's phase)
      bool w_ok = __all_sync(0xffffffffu,
                             mbar_wait(bar(B_SFULL), n & 1, R.status) &&
                                 mbar_wait(bar(B_IDX + n % kIdxRing), (n / kIdxRing) & 1,
                                           R.status) &&
                                 !*abort_flag);
      if (tid == kSoftmax0) DSA_STAMP(n, 6);
      if (w_ok) {
        tc_fence_after();
        tmem_ld32(tmem + lane_off + TM_S + 32 * wg, s);
        tc_fence_before();
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) s[j] = 0.f;
      }
      const uint32_t bits = vmask[(n % kIdxRing) * 2 + wg];
      mbar_arrive(bar(B_SEMPTY));  // the MMA may overwrite the score tile
      if (tid == kSoftmax0) DSA_STAMP(n, 7);
      // this warpgroup's 32 rows of the tile: their cache scales (e4m3); the
      // ring entry stays until the producers refill it four tiles on
      const float* const tsc = ksc + (n % kIdxRing) * kNT + 32 * wg;
      float hm = -INFINITY;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float sc = FP8 ? scale2 * tsc[j] : scale2;
        s[j] = ((bits >> j) & 1u) ? s[j] * sc : -INFINITY;
        hm = fmaxf(hm, s[j]);
      }
      float* const hm_buf = hmax + (n & 1) * (2 * kH);  // two tiles in flight
      hm_buf[wg * kH + h] = hm;
      if (!bar_and<1, kSoftmaxThreads>(w_ok)) {  // half maxima visible
        ok = false;
        break;
      }
      const float mt = fmaxf(hm, hm_buf[(wg ^ 1) * kH + h]);  // same value in both warpgroups
      // P of tile n-1 is consumed and O is final up to tile n-1 once PV(n-1) retired
      const bool t_ok = n == 0 || __all_sync(0xffffffffu,
                                             mbar_wait(bar(B_PVDONE), (n - 1) & 1, R.status));
      if (tid == kSoftmax0) DSA_STAMP(n, 8);
      if constexpr (!FP8) {
        if (n + 1 < ntiles && !fetch_v(n + 1)) *abort_flag = 1;
      }
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
        const float p0 = ex2(s[2 * j] - mref);
        const float p1 = ex2(s[2 * j + 1] - mref);
        if (FP8)  // the PV operand carries each token's cache scale: P' = p * scale
          pw[j] = pack_bf16(p0 * tsc[2 * j], p1 * tsc[2 * j + 1]);
        else
          pw[j] = pack_bf16(p0, p1);  // bf16 only as the MMA operand
        lsum += p0 + p1;              // the denominator keeps fp32 probabilities
      }
      if (t_ok) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
          *reinterpret_cast<uint4*>(prow + (((4 * wg + c) ^ (h & 7)) << 4)) =
              make_uint4(pw[4 * c], pw[4 * c + 1], pw[4 * c + 2], pw[4 * c + 3]);
      }
      l += lsum;
      if (!t_ok) *abort_flag = 1;  // seen by everyone at the next barrier reduction
      fence_async_smem();          // P stores before the PV MMA reads them
      tc_fence_before();           // a rescale's TMEM stores before the PV MMA
      mbar_arrive(bar(B_PFULL));
      if (tid == kSoftmax0) DSA_STAMP(n, 9);
    }
    if (!ok) *abort_flag = 1;
    asm volatile("cp.async.wait_all;" ::: "memory");
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
      const int col = half * 256 + c32 * 32;
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
    if (half == 0 && wg == 0) {
      if (final_out) {
        if (lse) lse[(int64_t)r * kH + h] = lse_v;
      } else {
        part_lse[((int64_t)rloc * sp.nsplit + split) * kH + h] = lse_v;
      }
    }
  }

  // the query load has landed before the CTA may exit (it has, unless a wait
  // above gave up)
  if (tid == 0) mbar_wait(bar(B_QLOAD), 0, R.status);
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
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

}  // namespace

bool attn_tc_supported(int H, int D_K, int D_V) { return H == kH && D_K == kDK && D_V == kDV; }

size_t attn_tc_workspace(int32_t nrows, int k, int H, int D_V) {
  if (nrows <= 0) return 0;
  const Split sp = plan_split(nrows, k);
  if (sp.nsplit == 1) return 0;
  return (size_t)nrows * sp.nsplit * kH * (kDV + 1) * sizeof(float) + 256;
}

dsa_status_t launch_attn_tc(const Rows& R, int32_t row0, int32_t nrows, const uint16_t* q,
                            const void* kv, const float* kv_scale, const int32_t* idx, int k,
                            float sm_scale, uint16_t* out, float* lse, void* ws, size_t ws_bytes,
                            cudaStream_t st, bool packed) {
  if (nrows <= 0) return DSA_OK;
  Split sp = plan_split(nrows, k);
  sp.packed = packed ? 1 : 0;
  float *part_o = nullptr, *part_lse = nullptr;
  if (sp.nsplit > 1) {
    if (!ws || ws_bytes < attn_tc_workspace(nrows, k, kH, kDV)) return DSA_ERR_WORKSPACE;
    part_o = reinterpret_cast<float*>(ws);
    part_lse = part_o + (size_t)nrows * sp.nsplit * kH * kDV;
  }
  // the queries as [n_q * 128, 576] (row coordinates r * 128 are 32-bit)
  if ((int64_t)R.n_q * kH >= INT32_MAX) return DSA_ERR_INVALID_ARGUMENT;
  CUtensorMap qmap;
  if (!make_tmap_2d(&qmap, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kDK, (uint64_t)R.n_q * kH, 64,
                    kH))
    return DSA_ERR_CUDA;
  auto kfn = kv_scale ? attn_tc_kernel<true> : attn_tc_kernel<false>;
  if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) != cudaSuccess)
    return DSA_ERR_CUDA;
  const dim3 grid(2 * nrows * sp.nsplit);
  kfn<<<grid, kThreads, kSmem, st>>>(qmap, kv, kv_scale, R, row0, idx, k, sm_scale * kLog2e, sp,
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
    static std::mutex lock;  // concurrent first calls from several host threads
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return DSA_ERR_CUDA;
    std::lock_guard<std::mutex> hold(lock);
    if (!addr[dev]) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_attn_scratch) != cudaSuccess || !p) return DSA_ERR_CUDA;
      addr[dev] = p;
    }
    scratch = addr[dev];
  }
  return launch_attn_tc(R, row0, nrows, q, kv, nullptr, idx, k, sm_scale, out, lse, scratch, need,
                        st);
}

}  // namespace dsa

#ifdef DSA_ATTN_TRACE
// Diagnostic build only: selects the traced row (grid item, -1: none) and
// copies the stamps out ([2][64][16] then the two CTA start stamps).
extern "C" int dsa_attn_trace_select(int item) {
  return (int)cudaMemcpyToSymbol(dsa::g_attn_trace_item, &item, sizeof(int));
}
extern "C" int dsa_attn_trace_copy(long long* host) {
  int e = (int)cudaMemcpyFromSymbol(host, dsa::g_attn_trace, sizeof(dsa::g_attn_trace));
  if (e) return e;
  return (int)cudaMemcpyFromSymbol(host + 2 * dsa::kTraceTiles * dsa::kTraceEvents,
                                   dsa::g_attn_trace_t0, sizeof(dsa::g_attn_trace_t0));
}
#endif
