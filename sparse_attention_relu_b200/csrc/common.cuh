// Internal helpers shared by the libdsa kernels (not part of the ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/dsa.h"

namespace dsa {

// Bits of the per-device status word (see dsa_device_status).
enum : unsigned {
  kErrTimeout = 1u,     // a bounded wait ran out
  kErrBadOffsets = 2u,  // kv_offsets not monotone / out of range
  kErrBadIndex = 4u,    // an index outside [0, L_b) (other than -1)
  kErrLayout = 8u,      // shared memory not laid out as a kernel requires
};

// Description of the query rows, passed by value to every kernel.
struct Rows {
  unsigned* status;     // this device's status word (see dsa_device_status)
  const int32_t* offs;  // [B+1] device
  const int32_t* qoffs;  // [B+1] device, CHUNKED only (query rows of each sequence)
  int32_t B;
  int32_t mode;  // DSA_PREFILL / DSA_DECODE
  int32_t max_len;
  int32_t n_q;
  int64_t n_k;
};

__device__ __forceinline__ void raise_status(const Rows& R, unsigned bits) {
  atomicOr(R.status, bits);
}

struct RowInfo {
  int64_t kbase;  // first cache row of the sequence
  int32_t t;      // query position inside the sequence (-1: no candidates)
  int32_t len;    // sequence length
  int32_t seq;
};

// Locates query row r.  Offsets that break the layout contract make the row
// empty (t = -1) and raise kErrBadOffsets.
__device__ __forceinline__ RowInfo row_info(const Rows& R, int32_t r) {
  RowInfo ri{0, -1, 0, 0};
  if (R.mode == DSA_CHUNKED) {
    // largest b with qoffs[b] <= r; query i of b sits at L_b - C_b + i
    int32_t lo = 0, hi = R.B - 1;
    while (lo < hi) {
      int32_t mid = (lo + hi + 1) >> 1;
      if (__ldg(R.qoffs + mid) <= r) lo = mid; else hi = mid - 1;
    }
    const int32_t q0 = __ldg(R.qoffs + lo), q1 = __ldg(R.qoffs + lo + 1);
    const int32_t o0 = __ldg(R.offs + lo), o1 = __ldg(R.offs + lo + 1);
    if (q0 < 0 || q1 < q0 || r < q0 || r >= q1 || q1 > R.n_q || o0 < 0 || o1 < o0 ||
        (int64_t)o1 > R.n_k || o1 - o0 > R.max_len || q1 - q0 > o1 - o0) {
      raise_status(R, kErrBadOffsets);
      return ri;
    }
    ri.kbase = o0;
    ri.len = o1 - o0;
    ri.t = ri.len - (q1 - q0) + (r - q0);
    ri.seq = lo;
    return ri;
  }
  if (R.mode == DSA_DECODE) {
    int32_t b = r;
    int32_t o0 = __ldg(R.offs + b), o1 = __ldg(R.offs + b + 1);
    if (o0 < 0 || o1 < o0 || (int64_t)o1 > R.n_k || o1 - o0 > R.max_len) {
      raise_status(R, kErrBadOffsets);
      return ri;
    }
    ri.kbase = o0;
    ri.len = o1 - o0;
    ri.t = ri.len - 1;
    ri.seq = b;
    return ri;
  }
  // prefill: largest b with offs[b] <= r
  int32_t lo = 0, hi = R.B - 1;
  while (lo < hi) {
    int32_t mid = (lo + hi + 1) >> 1;
    if (__ldg(R.offs + mid) <= r) lo = mid; else hi = mid - 1;
  }
  int32_t o0 = __ldg(R.offs + lo), o1 = __ldg(R.offs + lo + 1);
  if (o0 < 0 || o1 < o0 || r < o0 || r >= o1 || (int64_t)o1 > R.n_k || o1 - o0 > R.max_len) {
    raise_status(R, kErrBadOffsets);
    return ri;
  }
  ri.kbase = o0;
  ri.len = o1 - o0;
  ri.t = r - o0;
  ri.seq = lo;
  return ri;
}

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
  return __uint_as_float(((uint32_t)b) << 16);
}

// Four e4m3 codes (c0 in the low byte of w) -> bf16 pairs {c0, c1}, {c2, c3},
// exactly: each code's exponent and mantissa bits move into a bf16 with the
// exponent bias of e4m3's unbiased field (a bf16 subnormal when the code is
// subnormal), and one exact multiplication by 2^120 rebiases 7 -> 127 for
// normal and subnormal codes alike.  (The NaN codes S.1111.111 come out as
// +-480; the cache holds none.)
__device__ __forceinline__ void e4m3x4_to_bf16x4(uint32_t w, uint32_t& lo, uint32_t& hi) {
  uint32_t a, b;
  asm("prmt.b32 %0, %1, 0, 0x4140;" : "=r"(a) : "r"(w));  // c0, c1 in the low bytes of halves
  asm("prmt.b32 %0, %1, 0, 0x4342;" : "=r"(b) : "r"(w));  // c2, c3
  a = ((a << 4) & 0x07F007F0u) | ((a << 8) & 0x80008000u);
  b = ((b << 4) & 0x07F007F0u) | ((b << 8) & 0x80008000u);
  const uint32_t k2p120 = 0x7B807B80u;  // bf16x2 {2^120, 2^120}
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(lo) : "r"(a), "r"(k2p120));
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(hi) : "r"(b), "r"(k2p120));
}

// Host-side launch error helper.
inline dsa_status_t launch_status() {
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// SM count of the current device, looked up once per device (the lock makes
// concurrent first calls from several host threads safe).
inline int num_sms() {
  static int count[64] = {};
  static std::mutex lock;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  std::lock_guard<std::mutex> hold(lock);
  if (!count[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    count[dev] = n;
  }
  return count[dev];
}

}  // namespace dsa
