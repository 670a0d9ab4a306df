// Selection primitives shared by the top-k kernels and the fused indexer
// selection (not part of the ABI).
//
// Scores become 32-bit keys whose unsigned order is the float order (NaN
// ranks as -inf, -0 == +0), and a 2048-bin histogram over a monotone bin of
// the score finds the bin that holds the k-th best; the members of that bin
// are ranked by (key, then the lower position) -- the tie rule of
// "Sparse Attention Architecture Evolution in LLMs", Top-K Selection.
//
// Block-level routines take a Blk<NT, BAR, T0> policy: NT threads starting at
// thread T0 of the CTA take part, synchronised by __syncthreads() (BAR == 0)
// or by the named barrier BAR over those NT threads.
#pragma once

#include "common.cuh"

namespace dsa {
namespace sel {

constexpr int kBins = 2048;
constexpr int kCand = 2048;  // candidate buffer (keys + positions)

template <int NT_, int BAR_, int T0_>
struct Blk {
  static constexpr int NT = NT_, BAR = BAR_, T0 = T0_, NW = NT / 32;
  static_assert(NT % 32 == 0 && T0 % 32 == 0, "whole warps");
  __device__ static __forceinline__ int tid() { return (int)threadIdx.x - T0; }
  __device__ static __forceinline__ void sync() {
    if constexpr (BAR == 0)
      __syncthreads();
    else
      asm volatile("bar.sync %0, %1;" ::"n"(BAR), "n"(NT) : "memory");
  }
};

__device__ __forceinline__ uint32_t rank_key(float x) {
  uint32_t u = __float_as_uint(x);
  if ((u & 0x7fffffffu) > 0x7f800000u) u = 0xff800000u;  // NaN -> -inf
  if (u == 0x80000000u) u = 0u;                          // -0 -> +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Bin of a score, 0 .. 2047, non-decreasing in the score: the magnitude
// bits >> 18 are (exponent, top 5 mantissa bits), clamped to the 1024 steps
// of 2^-16 .. 2^16; negative scores mirror below 1024.  -0 counts as +0 and
// NaN as -inf (bin 0).
constexpr int kMagBase = (111 << 5);  // exponent 111 = 2^-16, mantissa step 0
__device__ __forceinline__ uint32_t score_bin(float x) {
  const uint32_t w = __float_as_uint(x), a = w & 0x7fffffffu;
  const bool neg = w > 0x80000000u || a > 0x7f800000u;
  const int mb = min(max((int)(a >> 18) - kMagBase, 0), 1023);
  return neg ? (uint32_t)(1023 - mb) : (uint32_t)(1024 + mb);
}
// The floats of bin b form the closed interval [lo, hi].  Bin 0 holds -inf
// (and NaN, which no float comparison admits); callers handle it apart.
__device__ __forceinline__ void bin_bounds(uint32_t b, float& lo, float& hi) {
  const int mb = b >= 1024 ? (int)b - 1024 : 1023 - (int)b;
  const uint32_t a_lo = mb == 0 ? 0u : (uint32_t)(kMagBase + mb) << 18;
  const uint32_t a_hi = mb == 1023 ? 0x7f800000u : ((uint32_t)(kMagBase + mb + 1) << 18) - 1u;
  if (b >= 1024) {
    lo = __uint_as_float(a_lo);
    hi = __uint_as_float(a_hi);
  } else {
    lo = -__uint_as_float(a_hi);
    hi = mb == 0 ? -__uint_as_float(1u) : -__uint_as_float(a_lo);  // zeros sit in bin 1024
  }
}

template <int NW>
struct Smem {
  uint32_t hist[kBins];
  uint32_t warp_tot[NW];
  uint32_t sel_bin;
  uint32_t sel_above;
  uint32_t n_out;   // positions written so far
  uint32_t n_cand;  // members of bin b1 seen in pass 2
  uint32_t kmin, kmax;  // candidate key range (ranking)
};

// Given hist[0..nbins) and the number `need` of elements still to take,
// finds bin b with above(b) < need <= above(b) + hist[b], where above(b) is
// the count in bins > b.  Result in sm.sel_bin / sm.sel_above.
template <class B>
__device__ void find_bin(Smem<B::NW>& sm, int nbins, uint32_t need) {
  const int tid = B::tid(), lane = tid & 31, warp = tid >> 5;
  constexpr int kThreads = B::NT, kWarps = B::NW;
  const int per = nbins / kThreads;  // contiguous bins per thread
  if (tid == 0) {  // (a need above the histogram's total finds no bin: bin 0, nothing above)
    sm.sel_bin = 0;
    sm.sel_above = 0;
  }
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
  B::sync();
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
  B::sync();
}

// Warp-aggregated append: every lane with `pred` gets a distinct slot of
// *ctr.  All 32 lanes must call it.
__device__ __forceinline__ uint32_t warp_append(bool pred, uint32_t* ctr, uint32_t& slot) {
  const uint32_t mask = __ballot_sync(0xffffffffu, pred);
  if (!mask) return 0;
  const int lane = threadIdx.x & 31, leader = __ffs(mask) - 1;
  uint32_t base = 0;
  if (lane == leader) base = atomicAdd(ctr, (uint32_t)__popc(mask));
  base = __shfl_sync(0xffffffffu, base, leader);
  slot = base + __popc(mask & ((1u << lane) - 1u));
  return mask;
}

// Order of candidates: a larger key first, then (the tie rule) the lower
// position.  Positions are distinct, so no two candidates compare equal.
__device__ __forceinline__ uint64_t cand_order(uint32_t key, int32_t pos) {
  return ((uint64_t)key << 32) | (uint64_t)(0xffffffffu - (uint32_t)pos);
}

__device__ __forceinline__ uint32_t warp_sum(uint32_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Writes the `need` best of m <= kCand candidates (key, position) to
// dst[0 .. need) in any order.  The candidates' keys span [kmin, kmax]; a
// histogram of (key - kmin) >> shift over kBins buckets (monotone in the key)
// finds the bucket sb that holds the need-th best.  Candidates in buckets
// above sb go out at once; the members of sb (typically one or two) move to
// the front of the candidate arrays and are ranked by the candidate order,
// one warp per member with its lanes sharing the comparisons, the best of
// them filling the remaining slots.  All threads of the CTA call it.
template <class B>
__device__ void rank_candidates(Smem<B::NW>& sm, uint32_t* ckey, int32_t* cpos, int m,
                                uint32_t need, int32_t* dst) {
  constexpr int kThreads = B::NT, kWarps = B::NW;
  constexpr int R = kCand / kThreads;
  const int tid = B::tid(), lane = tid & 31, warp = tid >> 5;
  uint32_t key[R];
  int32_t pos[R];
  uint32_t lo = 0xffffffffu, hi = 0u;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int j = tid + r * kThreads;
    key[r] = j < m ? ckey[j] : 0u;
    pos[r] = j < m ? cpos[j] : 0;
    if (j < m) {
      lo = min(lo, key[r]);
      hi = max(hi, key[r]);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if (tid == 0) {
    sm.kmin = 0xffffffffu;
    sm.kmax = 0u;
    sm.n_out = 0;
    sm.n_cand = 0;
  }
  for (int i = tid; i < kBins; i += kThreads) sm.hist[i] = 0;
  B::sync();
  if (lane == 0) {
    atomicMin(&sm.kmin, lo);
    atomicMax(&sm.kmax, hi);
  }
  B::sync();
  const uint32_t kmin = sm.kmin, span = sm.kmax - kmin;
  const int bits = span ? 32 - __clz(span) : 0;  // bits of the span
  const int shift = bits > 11 ? bits - 11 : 0;   // (span >> shift) < 2048 buckets
#pragma unroll
  for (int r = 0; r < R; ++r)
    if (tid + r * kThreads < m) atomicAdd(&sm.hist[(key[r] - kmin) >> shift], 1u);
  B::sync();
  find_bin<B>(sm, kBins, need);  // ends with a barrier: every candidate is in registers
  const uint32_t sb = sm.sel_bin, need2 = need - sm.sel_above;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const bool ok = tid + r * kThreads < m;
    const uint32_t b = (key[r] - kmin) >> shift;
    const bool up = ok && b > sb, in = ok && b == sb;
    uint32_t slot;
    if (warp_append(up, &sm.n_out, slot) && up) dst[slot] = pos[r];
    if (warp_append(in, &sm.n_cand, slot) && in) {
      ckey[slot] = key[r];
      cpos[slot] = pos[r];
    }
  }
  B::sync();
  const int c = (int)sm.n_cand;
  const uint32_t base_out = sm.n_out;  // == sm.sel_above
  for (int j = warp; j < c; j += kWarps) {
    const uint64_t oj = cand_order(ckey[j], cpos[j]);
    uint32_t better = 0;
    for (int l = lane; l < c; l += 32) better += cand_order(ckey[l], cpos[l]) > oj ? 1u : 0u;
    better = warp_sum(better);
    if (lane == 0 && better < need2) dst[base_out + better] = cpos[j];
  }
}


// The float whose rank key is `key` (inverse of rank_key on the values it
// produces: NaN has already become -inf and -0 has become +0).
__device__ __forceinline__ float key_float(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// Candidate entry of a list: the score's rank key in the high word, its
// position in the low word.
__device__ __forceinline__ uint64_t pack_cand(uint32_t key, int32_t pos) {
  return ((uint64_t)key << 32) | (uint32_t)pos;
}

// Radix select of one 11- or 10-bit digit over the entries get(0 .. m-1)
// that `member` admits: histogram of digit (v >> shift) & mask in sm.hist,
// then find_bin for `need`.  The caller folds the digit into its prefix.
template <class B, class Get, class Member, class Value>
__device__ void radix_level(Smem<B::NW>& sm, const Get& get, uint32_t m, int shift,
                            uint32_t width, uint32_t need, Member member, Value value) {
  const int tid = B::tid();
  for (int i = tid; i < kBins; i += B::NT) sm.hist[i] = 0;
  B::sync();
  for (uint32_t i = tid; i < m; i += B::NT) {
    const uint64_t c = get(i);
    if (member(c)) atomicAdd(&sm.hist[(value(c) >> shift) & ((1u << width) - 1u)], 1u);
  }
  B::sync();
  find_bin<B>(sm, 1 << width, need);
}

// Exact top-k of a candidate list: the k best of the entries get(0 .. m-1)
// by key, ties to the lower position, written to out[0, k) in any order (-1
// padded when m < k).  The list must hold every score of the row that can be
// among its k best (then the result is the row's top-k).
// have_hist: sm.hist already holds the bin histogram of the whole row (of
// which the list holds at least every score in the bins from the k-th best's
// up), else it is built from the list.  ckey / cpos: kCand entries of shared
// scratch.  All NT threads of B call it.
template <class B, class Get>
__device__ void select_list(Smem<B::NW>& sm, const Get& ld, uint32_t m, int k, int32_t* out,
                            uint32_t* ckey, int32_t* cpos, bool have_hist = false) {
  constexpr int RB = 8;  // candidates each thread loads per round (in flight together)
  const int tid = B::tid();
  if (m <= (uint32_t)k) {
    for (int i = tid; i < k; i += B::NT) out[i] = (uint32_t)i < m ? (int32_t)(uint32_t)ld(i) : -1;
    return;
  }
  // pass 1: the bin b1 that holds the k-th best
  if (!have_hist) {
    for (int i = tid; i < kBins; i += B::NT) sm.hist[i] = 0;
    B::sync();
    for (uint32_t base = 0; base < m; base += B::NT * RB) {
      uint64_t c[RB];
#pragma unroll
      for (int r = 0; r < RB; ++r) {
        const uint32_t i = base + tid + B::NT * r;
        c[r] = i < m ? ld(i) : 0ull;
      }
#pragma unroll
      for (int r = 0; r < RB; ++r)
        if (base + tid + B::NT * r < m)
          atomicAdd(&sm.hist[score_bin(key_float((uint32_t)(c[r] >> 32)))], 1u);
    }
  }
  if (tid == 0) {
    sm.n_out = 0;
    sm.n_cand = 0;
  }
  B::sync();
  find_bin<B>(sm, kBins, (uint32_t)k);
  const uint32_t b1 = sm.sel_bin, above1 = sm.sel_above, in_b1 = sm.hist[b1];
  B::sync();
  // pass 2: above b1 -> out; members of b1 -> the buffer when they fit
  const bool collect = in_b1 <= (uint32_t)kCand;
  const uint32_t mbase = (m + 31u) & ~31u;  // whole warps in every trip
  for (uint32_t base = 0; base < mbase; base += B::NT * RB) {  // uniform trip count
    uint64_t cr[RB];
#pragma unroll
    for (int r = 0; r < RB; ++r) {
      const uint32_t i = base + tid + B::NT * r;
      cr[r] = i < m ? ld(i) : 0ull;
    }
#pragma unroll
    for (int r = 0; r < RB; ++r) {
      const uint32_t i = base + tid + B::NT * r;
      const uint64_t c = cr[r];
      const uint32_t key = (uint32_t)(c >> 32), b = i < m ? score_bin(key_float(key)) : 0u;
      const bool gt = i < m && b > b1, eq = collect && i < m && b == b1;
      uint32_t slot;
      if (warp_append(gt, &sm.n_out, slot) && gt && slot < (uint32_t)k)
        out[slot] = (int32_t)(uint32_t)c;
      if (warp_append(eq, &sm.n_cand, slot) && eq && slot < (uint32_t)kCand) {
        ckey[slot] = key;
        cpos[slot] = (int32_t)(uint32_t)c;
      }
    }
  }
  B::sync();
  if (collect) {
    const uint32_t nc = sm.n_cand < in_b1 ? sm.n_cand : in_b1;  // equal for a valid list
    rank_candidates<B>(sm, ckey, cpos, (int)nc, (uint32_t)k - above1, out + above1);
    return;
  }
  // b1 overflows the buffer: radix levels over its members' keys find the
  // k-th best key tau, then the positions of the members equal to tau
  // (ties: the lowest positions) by radix levels over their positions
  auto in_b1f = [&](uint64_t c) { return score_bin(key_float((uint32_t)(c >> 32))) == b1; };
  auto keyf = [](uint64_t c) { return (uint32_t)(c >> 32); };
  // digits of 11, 11 and 10 bits, from the top
  auto dshift = [](int lvl) { return lvl == 0 ? 21 : lvl == 1 ? 10 : 0; };
  auto dwidth = [](int lvl) { return lvl == 2 ? 10u : 11u; };
  uint32_t prefix = 0, c_gt = above1;
#pragma unroll 1
  for (int lvl = 0; lvl < 3; ++lvl) {
    const int hi = dshift(lvl) + (int)dwidth(lvl);
    const uint32_t pre = prefix;
    radix_level<B>(sm, ld, m, dshift(lvl), dwidth(lvl), (uint32_t)k - c_gt,
                   [&](uint64_t c) { return in_b1f(c) && (hi >= 32 || (keyf(c) >> hi) == pre); },
                   keyf);
    prefix = (prefix << dwidth(lvl)) | sm.sel_bin;
    c_gt += sm.sel_above;
    B::sync();
  }
  const uint32_t tau = prefix, need_eq = (uint32_t)k - c_gt;  // >= 1
  // positions of the members equal to tau: the need_eq-th lowest, p_cut
  // (radix levels from the top digit: a position's order is reversed so that
  // find_bin, which counts from the top, counts the lowest positions first)
  auto eqf = [&](uint64_t c) { return (uint32_t)(c >> 32) == tau; };
  auto rpos = [](uint64_t c) { return ~(uint32_t)c; };  // larger = lower position
  uint32_t pprefix = 0, p_gt = 0;  // p_gt: equal members at lower positions than the range
#pragma unroll 1
  for (int lvl = 0; lvl < 3; ++lvl) {
    const int hi = dshift(lvl) + (int)dwidth(lvl);
    const uint32_t pre = pprefix;
    radix_level<B>(sm, ld, m, dshift(lvl), dwidth(lvl), need_eq - p_gt,
                   [&](uint64_t c) { return eqf(c) && (hi >= 32 || (rpos(c) >> hi) == pre); },
                   rpos);
    pprefix = (pprefix << dwidth(lvl)) | sm.sel_bin;
    p_gt += sm.sel_above;
    B::sync();
  }
  const uint32_t rcut = pprefix;  // rpos of the need_eq-th lowest position
  // members above tau, and those equal to tau at a position no higher than the cut
  if (tid == 0) sm.n_out = above1;
  B::sync();
  for (uint32_t base = 0; base < mbase; base += B::NT) {
    const uint32_t i = base + tid;
    const uint64_t c = i < m ? ld(i) : 0ull;
    const uint32_t key = (uint32_t)(c >> 32);
    const bool take = i < m && in_b1f(c) && (key > tau || (key == tau && rpos(c) >= rcut));
    uint32_t slot;
    if (warp_append(take, &sm.n_out, slot) && take && slot < (uint32_t)k)
      out[slot] = (int32_t)(uint32_t)c;
  }
  B::sync();
}

}  // namespace sel
}  // namespace dsa
