// C ABI of libdsa: argument validation and the orchestration of the stages.
// The semantics of each call are documented in include/dsa.h.
#include <math.h>
#include <stdlib.h>

#include <mutex>

#include "kernels.cuh"
#include "sm100.cuh"

namespace dsa {

namespace {

// The per-device status word.  Kernels receive its device address in Rows.
__device__ unsigned g_status = 0;

// Its device address, looked up once per device with that device current;
// the lock makes concurrent first calls from several host threads safe.
unsigned* status_word() {
  static unsigned* addr[64] = {};
  static std::mutex lock;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> hold(lock);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return nullptr;
    addr[dev] = (unsigned*)p;
  }
  return addr[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// One thread waits, through the bounded wait every kernel uses, on an
// mbarrier that nothing arrives on; after `limit` cycles the wait gives up
// and raises kErrTimeout.  Nothing is in flight when it returns.
__global__ void wait_timeout_selftest(unsigned* status, long long limit) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = (uint32_t)__cvta_generic_to_shared(&bar);
  sm100::mbar_init(b, 1);
  sm100::fence_mbar_init();
  sm100::mbar_wait_for(b, 0, status, limit);
}

// Checks the layout; fills the device-side row description.
dsa_status_t check_layout(const dsa_layout_t* L, Rows* R) {
  if (!L) return DSA_ERR_INVALID_ARGUMENT;
  if (L->mode != DSA_PREFILL && L->mode != DSA_DECODE && L->mode != DSA_CHUNKED)
    return DSA_ERR_INVALID_ARGUMENT;
  if (L->batch < 0 || L->max_len < 0 || L->n_q < 0 || L->n_k < 0) return DSA_ERR_INVALID_ARGUMENT;
  if (L->batch > 0 && (!L->kv_offsets || !aligned16(L->kv_offsets)))
    return DSA_ERR_INVALID_ARGUMENT;
  if (L->n_k >= (int64_t(1) << 31)) return DSA_ERR_UNSUPPORTED;  // int32 offsets
  if (L->mode == DSA_PREFILL) {
    if (L->n_q != L->n_k) return DSA_ERR_INVALID_ARGUMENT;
  } else if (L->mode == DSA_DECODE) {
    if (L->n_q != L->batch) return DSA_ERR_INVALID_ARGUMENT;
  } else {  // CHUNKED: every query is a cache row of its sequence
    if (L->batch > 0 && (!L->q_offsets || !aligned16(L->q_offsets)))
      return DSA_ERR_INVALID_ARGUMENT;
    if ((int64_t)L->n_q > L->n_k) return DSA_ERR_INVALID_ARGUMENT;
  }
  if (L->n_q > 0 && (L->batch == 0 || L->max_len == 0)) return DSA_ERR_INVALID_ARGUMENT;
  R->status = nullptr;  // filled by device_rows() once every argument passed
  R->offs = L->kv_offsets;
  R->qoffs = L->mode == DSA_CHUNKED ? L->q_offsets : nullptr;
  R->B = L->batch;
  R->mode = L->mode;
  R->max_len = L->max_len;
  R->n_q = L->n_q;
  R->n_k = L->n_k;
  return DSA_OK;
}

// Last step before launching: the device address of the status word.
dsa_status_t device_rows(Rows* R) {
  R->status = status_word();
  return R->status ? DSA_OK : DSA_ERR_CUDA;
}

bool ptr_ok(const void* p, bool needed) { return !needed || (p && aligned16(p)); }

dsa_status_t check_indexer(const Rows& R, const void* q_idx, const float* q_scale,
                           const float* w, const void* k_idx, const float* k_scale, int dtype,
                           int H_I, int D_I) {
  if (dtype != DSA_F32 && dtype != DSA_BF16 && dtype != DSA_E4M3) return DSA_ERR_INVALID_ARGUMENT;
  if (H_I < 1 || D_I < 1 || H_I > 128 || D_I > 256) return DSA_ERR_INVALID_ARGUMENT;
  if ((int64_t)H_I * D_I > 16384 && !indexer_tc_supported(dtype, H_I, D_I))
    return DSA_ERR_UNSUPPORTED;
  const bool rows = R.n_q > 0;
  if (!ptr_ok(q_idx, rows) || !ptr_ok(w, rows) || !ptr_ok(k_idx, R.n_k > 0))
    return DSA_ERR_INVALID_ARGUMENT;
  if (dtype == DSA_E4M3) {
    if (!ptr_ok(q_scale, rows) || !ptr_ok(k_scale, R.n_k > 0)) return DSA_ERR_INVALID_ARGUMENT;
  } else if (q_scale || k_scale) {
    return DSA_ERR_INVALID_ARGUMENT;
  }
  // row strides of the 16-byte vector / TMA paths
  const int esz = dtype == DSA_F32 ? 4 : dtype == DSA_BF16 ? 2 : 1;
  if ((D_I * esz) % 16) return DSA_ERR_INVALID_ARGUMENT;
  return DSA_OK;
}

// kv_dtype: DSA_BF16, or DSA_E4M3 with kv_scale [n_k] (the per-token scales).
dsa_status_t check_attn(const Rows& R, const void* q, const void* kv, int kv_dtype,
                        const float* kv_scale, int k, int H, int D_K, int D_V, float sm_scale,
                        const void* out, const float* lse) {
  if (k < 1 || k > 16384) return DSA_ERR_INVALID_ARGUMENT;
  if (H < 1 || H > 128 || D_K < 8 || D_K > 1024 || D_K % 8 || D_V < 8 || D_V > D_K || D_V % 8)
    return DSA_ERR_INVALID_ARGUMENT;
  if (kv_dtype == DSA_E4M3) {
    if (D_K % 16 || !ptr_ok(kv_scale, R.n_k > 0)) return DSA_ERR_INVALID_ARGUMENT;
  } else if (kv_dtype != DSA_BF16 || kv_scale) {
    return DSA_ERR_INVALID_ARGUMENT;
  }
  if (!isfinite(sm_scale)) return DSA_ERR_INVALID_ARGUMENT;
  const bool rows = R.n_q > 0;
  if (!ptr_ok(q, rows) || !ptr_ok(kv, R.n_k > 0) || !ptr_ok(out, rows))
    return DSA_ERR_INVALID_ARGUMENT;
  if (lse && !aligned16(lse)) return DSA_ERR_INVALID_ARGUMENT;
  return DSA_OK;
}

dsa_status_t run_indexer(const Rows& R, int32_t row0, int32_t nrows, int dtype, int H_I, int D_I,
                         const void* q_idx, const float* q_scale, const float* w,
                         const void* k_idx, const float* k_scale, float* scores, bool fill,
                         cudaStream_t st) {
  if (indexer_tc_supported(dtype, H_I, D_I))
    return launch_indexer_tc(R, row0, nrows, dtype, H_I, D_I, q_idx, q_scale, w, k_idx, k_scale,
                             scores, R.max_len, fill, st);
  return launch_indexer_simt(R, row0, nrows, dtype, H_I, D_I, q_idx, q_scale, w, k_idx, k_scale,
                             scores, R.max_len, fill, st);
}

size_t attn_ws(int32_t nrows, int k, int H, int D_K, int D_V) {
  return attn_tc_supported(H, D_K, D_V) ? attn_tc_workspace(nrows, k, H, D_V) : 0;
}

// kv_scale != NULL: an e4m3 cache with per-token scales, else bf16.
// packed: idx is the chain's own top-k output (valid indices first, at most
// t + 1 per row), whose empty trailing tiles the tensor-core kernel skips.
dsa_status_t run_attn(const Rows& R, int32_t row0, int32_t nrows, const void* q, const void* kv,
                      const float* kv_scale, const int32_t* idx, int k, int H, int D_K, int D_V,
                      float sm_scale, void* out, float* lse, void* ws, size_t ws_bytes,
                      cudaStream_t st, bool packed = false) {
  if (attn_tc_supported(H, D_K, D_V))
    return launch_attn_tc(R, row0, nrows, (const uint16_t*)q, kv, kv_scale, idx, k, sm_scale,
                          (uint16_t*)out, lse, ws, ws_bytes, st, packed);
  return launch_attn_simt(R, row0, nrows, (const uint16_t*)q, kv, kv_scale, idx, k, H, D_K, D_V,
                          sm_scale, (uint16_t*)out, lse, st);
}

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Prefill slabs hold at most this many bytes of scores.
constexpr size_t kSlabBytes = size_t(1) << 30;

int32_t slab_rows(const Rows& R) {
  if (R.n_q == 0) return 0;
  size_t row_bytes = (size_t)R.max_len * 4;
  size_t rows = kSlabBytes / (row_bytes ? row_bytes : 1);
  if (rows < 1) rows = 1;
  if (rows > (size_t)R.n_q) rows = R.n_q;
  return (int32_t)rows;
}

// The fused decode selection (indexer and top-k in one kernel, no score rows)
// is built and tested but not yet faster than the separate top-k kernel, so
// dsa_forward takes it only when the environment variable
// DSA_FUSED_DECODE_SELECT is 1 at the call (and at the workspace query: the
// two plans differ in size).
bool fused_decode_select() {
  const char* v = getenv("DSA_FUSED_DECODE_SELECT");
  return v && v[0] == '1' && v[1] == 0;
}

struct ForwardPlan {
  int32_t slab;
  bool fused;  // decode: indexer and top-k in one kernel, no score rows
  size_t off_scores, off_idx, off_attn, total;
};

// slab_cap > 0 caps the rows per slab below the scores bound.  Decode rows
// (tensor-core indexer) take the fused indexer + selection: the workspace then
// holds the rows' candidate lists instead of their scores.
ForwardPlan plan_forward(const Rows& R, const dsa_forward_args_t* a, bool own_idx,
                         int32_t slab_cap = 0) {
  ForwardPlan p{};
  p.slab = slab_rows(R);
  if (slab_cap > 0 && slab_cap < p.slab) p.slab = slab_cap;
  p.fused = fused_decode_select() &&
            indexer_select_supported(R, a->idx_dtype, a->H_I, a->D_I, a->k);
  size_t o = 0;
  p.off_scores = o;
  o = align_up(o + (p.fused ? indexer_select_workspace(R, p.slab)
                            : (size_t)p.slab * R.max_len * 4));
  p.off_idx = o;
  if (own_idx) o = align_up(o + (size_t)p.slab * a->k * 4);
  p.off_attn = o;
  o = align_up(o + attn_ws(p.slab, a->k, a->H, a->D_K, a->D_V));
  p.total = o;
  return p;
}

// The two copy streams of dsa_forward_host (host to device, device to host),
// one pair per device, created on first use and kept for the process.  The
// lock makes the first use from several host threads create one pair.
dsa_status_t copy_streams(cudaStream_t* h2d, cudaStream_t* d2h) {
  static cudaStream_t made[64][2] = {};
  static std::mutex lock;
  std::lock_guard<std::mutex> hold(lock);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return DSA_ERR_CUDA;
  for (int i = 0; i < 2; ++i)
    if (!made[dev][i] &&
        cudaStreamCreateWithFlags(&made[dev][i], cudaStreamNonBlocking) != cudaSuccess)
      return DSA_ERR_CUDA;
  *h2d = made[dev][0];
  *d2h = made[dev][1];
  return DSA_OK;
}

// Host-side arguments of dsa_forward_host: the same shapes and scalars as the
// device ones; every per-query input present (q_scale exactly when e4m3); a
// key-side input may be NULL (its device copy is current).
dsa_status_t check_host(const Rows& R, const dsa_forward_args_t* h, const dsa_forward_args_t* d,
                        const void* host_out, const float* host_lse, const float* dev_lse) {
  if (h->idx_dtype != d->idx_dtype || h->H_I != d->H_I || h->D_I != d->D_I || h->H != d->H ||
      h->D_K != d->D_K || h->D_V != d->D_V || h->k != d->k || !(h->sm_scale == d->sm_scale) ||
      h->kv_dtype != d->kv_dtype)
    return DSA_ERR_INVALID_ARGUMENT;
  if (d->kv_dtype != DSA_E4M3 && h->kv_scale) return DSA_ERR_INVALID_ARGUMENT;
  const bool rows = R.n_q > 0, e4m3 = d->idx_dtype == DSA_E4M3;
  if (rows && (!h->q_idx || !h->w || !h->q || !host_out || (e4m3 && !h->q_scale)))
    return DSA_ERR_INVALID_ARGUMENT;
  if (!e4m3 && (h->q_scale || h->k_scale)) return DSA_ERR_INVALID_ARGUMENT;
  if (host_lse && !dev_lse) return DSA_ERR_INVALID_ARGUMENT;
  return DSA_OK;
}

// Events of one dsa_forward_host call, destroyed on return (a recorded event
// that has not completed is released by the runtime once it completes; waits
// already enqueued on it are unaffected).
struct CallEvents {
  cudaEvent_t e[5] = {};
  bool ok = true;
  CallEvents() {
    for (auto& x : e)
      if (cudaEventCreateWithFlags(&x, cudaEventDisableTiming) != cudaSuccess) ok = false;
  }
  ~CallEvents() {
    for (auto& x : e)
      if (x) cudaEventDestroy(x);
  }
};

dsa_status_t sparse_mla_attn(const dsa_layout_t* layout, const void* q, const void* kv,
                             int kv_dtype, const float* kv_scale, const int32_t* idx, int32_t k,
                             int32_t H, int32_t D_K, int32_t D_V, float sm_scale, void* out,
                             float* lse, void* workspace, size_t ws_bytes, void* stream) {
  Rows R;
  dsa_status_t s = check_layout(layout, &R);
  if (s) return s;
  if ((s = check_attn(R, q, kv, kv_dtype, kv_scale, k, H, D_K, D_V, sm_scale, out, lse)))
    return s;
  if (!ptr_ok(idx, R.n_q > 0)) return DSA_ERR_INVALID_ARGUMENT;
  const size_t need = attn_ws(R.n_q, k, H, D_K, D_V);
  if (need && (!workspace || ws_bytes < need || !aligned16(workspace))) return DSA_ERR_WORKSPACE;
  if (R.n_q == 0) return DSA_OK;
  if ((s = device_rows(&R))) return s;
  return run_attn(R, 0, R.n_q, q, kv, kv_scale, idx, k, H, D_K, D_V, sm_scale, out, lse,
                  workspace, ws_bytes, (cudaStream_t)stream);
}

}  // namespace
}  // namespace dsa

using namespace dsa;

extern "C" {

int32_t dsa_abi_version(void) { return 4; }

const char* dsa_status_string(dsa_status_t s) {
  switch (s) {
    case DSA_OK: return "ok";
    case DSA_ERR_INVALID_ARGUMENT: return "invalid argument";
    case DSA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case DSA_ERR_WORKSPACE: return "workspace missing or too small";
    case DSA_ERR_CUDA: return "CUDA error";
    case DSA_ERR_TIMEOUT: return "a bounded device wait ran out";
    case DSA_ERR_DEVICE_DATA: return "device data (offsets or indices) out of range";
  }
  return "unknown status";
}

dsa_status_t dsa_device_status(void* stream) {
  cudaStream_t st = (cudaStream_t)stream;
  unsigned v = 0, zero = 0;
  if (cudaStreamSynchronize(st) != cudaSuccess) return DSA_ERR_CUDA;
  if (cudaMemcpyFromSymbolAsync(&v, g_status, sizeof v, 0, cudaMemcpyDeviceToHost, st) !=
      cudaSuccess)
    return DSA_ERR_CUDA;
  if (cudaMemcpyToSymbolAsync(g_status, &zero, sizeof zero, 0, cudaMemcpyHostToDevice, st) !=
      cudaSuccess)
    return DSA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return DSA_ERR_CUDA;
  if (v & kErrTimeout) return DSA_ERR_TIMEOUT;
  if (v) return DSA_ERR_DEVICE_DATA;
  return DSA_OK;
}

dsa_status_t dsa_selftest_wait_timeout(int64_t cycles, void* stream) {
  if (cycles < 0 || cycles > (int64_t)sm100::kSpinLimit) return DSA_ERR_INVALID_ARGUMENT;
  unsigned* status = status_word();
  if (!status) return DSA_ERR_CUDA;
  wait_timeout_selftest<<<1, 1, 0, (cudaStream_t)stream>>>(status, (long long)cycles);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

dsa_status_t dsa_indexer_scores(const dsa_layout_t* layout, const void* q_idx,
                                const float* q_scale, const float* w, const void* k_idx,
                                const float* k_scale, int32_t dtype, int32_t H_I, int32_t D_I,
                                float* scores, void* stream) {
  Rows R;
  dsa_status_t s = check_layout(layout, &R);
  if (s) return s;
  if ((s = check_indexer(R, q_idx, q_scale, w, k_idx, k_scale, dtype, H_I, D_I))) return s;
  if (!ptr_ok(scores, R.n_q > 0)) return DSA_ERR_INVALID_ARGUMENT;
  if (R.n_q == 0) return DSA_OK;
  if ((s = device_rows(&R))) return s;
  return run_indexer(R, 0, R.n_q, dtype, H_I, D_I, q_idx, q_scale, w, k_idx, k_scale, scores,
                     true, (cudaStream_t)stream);
}

dsa_status_t dsa_topk(const dsa_layout_t* layout, const float* scores, int32_t k, int32_t* idx,
                      void* stream) {
  Rows R;
  dsa_status_t s = check_layout(layout, &R);
  if (s) return s;
  if (k < 1 || k > 16384) return DSA_ERR_INVALID_ARGUMENT;
  if (!ptr_ok(scores, R.n_q > 0) || !ptr_ok(idx, R.n_q > 0)) return DSA_ERR_INVALID_ARGUMENT;
  if (R.n_q == 0) return DSA_OK;
  if ((s = device_rows(&R))) return s;
  return launch_topk(R, 0, R.n_q, scores, R.max_len, k, idx, (cudaStream_t)stream);
}

size_t dsa_sparse_mla_attn_workspace_size(const dsa_layout_t* layout, int32_t k, int32_t H,
                                          int32_t D_K, int32_t D_V) {
  Rows R;
  if (check_layout(layout, &R)) return 0;
  return attn_ws(R.n_q, k, H, D_K, D_V);
}


dsa_status_t dsa_sparse_mla_attn(const dsa_layout_t* layout, const void* q, const void* kv,
                                 const int32_t* idx, int32_t k, int32_t H, int32_t D_K,
                                 int32_t D_V, float sm_scale, void* out, float* lse,
                                 void* workspace, size_t ws_bytes, void* stream) {
  return sparse_mla_attn(layout, q, kv, DSA_BF16, nullptr, idx, k, H, D_K, D_V, sm_scale, out, lse,
                         workspace, ws_bytes, stream);
}

dsa_status_t dsa_sparse_mla_attn_e4m3(const dsa_layout_t* layout, const void* q, const void* kv,
                                      const float* kv_scale, const int32_t* idx, int32_t k,
                                      int32_t H, int32_t D_K, int32_t D_V, float sm_scale,
                                      void* out, float* lse, void* workspace, size_t ws_bytes,
                                      void* stream) {
  return sparse_mla_attn(layout, q, kv, DSA_E4M3, kv_scale, idx, k, H, D_K, D_V, sm_scale, out,
                         lse, workspace, ws_bytes, stream);
}

dsa_status_t dsa_sparse_mla_attn_noalloc(const dsa_layout_t* layout, const void* q,
                                         const void* kv, const int32_t* idx, int32_t k, int32_t H,
                                         int32_t D_K, int32_t D_V, float sm_scale, void* out,
                                         float* lse, void* stream) {
  Rows R;
  dsa_status_t s = check_layout(layout, &R);
  if (s) return s;
  if ((s = check_attn(R, q, kv, DSA_BF16, nullptr, k, H, D_K, D_V, sm_scale, out, lse))) return s;
  if (!ptr_ok(idx, R.n_q > 0)) return DSA_ERR_INVALID_ARGUMENT;
  if (attn_tc_supported(H, D_K, D_V) &&
      attn_tc_workspace(R.n_q, k, H, D_V) > attn_tc_static_scratch_bytes())
    return DSA_ERR_WORKSPACE;
  if (R.n_q == 0) return DSA_OK;
  if ((s = device_rows(&R))) return s;
  if (attn_tc_supported(H, D_K, D_V))
    return launch_attn_tc_static(R, 0, R.n_q, (const uint16_t*)q, (const uint16_t*)kv, idx, k,
                                 sm_scale, (uint16_t*)out, lse, (cudaStream_t)stream);
  return launch_attn_simt(R, 0, R.n_q, (const uint16_t*)q, kv, nullptr, idx, k, H, D_K, D_V,
                          sm_scale, (uint16_t*)out, lse, (cudaStream_t)stream);
}

size_t dsa_forward_workspace_size(const dsa_layout_t* layout, const dsa_forward_args_t* a) {
  Rows R;
  if (!a || check_layout(layout, &R)) return 0;
  return plan_forward(R, a, true).total;
}

dsa_status_t dsa_forward_timed(const dsa_layout_t* layout, const dsa_forward_args_t* a,
                               void* out, float* lse, int32_t* idx_out, void* workspace,
                               size_t ws_bytes, void* stream, void* const* events,
                               int32_t n_events, int32_t* kinds, int32_t* n_launched) {
  Rows R;
  dsa_status_t s = check_layout(layout, &R);
  if (s) return s;
  if (!a) return DSA_ERR_INVALID_ARGUMENT;
  if ((s = check_indexer(R, a->q_idx, a->q_scale, a->w, a->k_idx, a->k_scale, a->idx_dtype,
                         a->H_I, a->D_I)))
    return s;
  if ((s = check_attn(R, a->q, a->kv, a->kv_dtype, a->kv_scale, a->k, a->H, a->D_K, a->D_V,
                      a->sm_scale, out, lse)))
    return s;
  if (idx_out && !aligned16(idx_out)) return DSA_ERR_INVALID_ARGUMENT;
  if (n_events > 0 && !events) return DSA_ERR_INVALID_ARGUMENT;
  const ForwardPlan p = plan_forward(R, a, idx_out == nullptr);
  if (!workspace || ws_bytes < p.total || !aligned16(workspace)) return DSA_ERR_WORKSPACE;
  if (n_launched) *n_launched = 0;
  if (R.n_q == 0) return DSA_OK;
  if ((s = device_rows(&R))) return s;
  cudaStream_t st = (cudaStream_t)stream;
  int32_t launched = 0;
  auto mark = [&](int32_t kind) -> dsa_status_t {
    if (launched + 1 < n_events &&
        cudaEventRecord((cudaEvent_t)events[launched + 1], st) != cudaSuccess)
      return DSA_ERR_CUDA;
    if (kinds && launched + 1 < n_events) kinds[launched] = kind;
    ++launched;
    if (n_launched) *n_launched = launched;
    return DSA_OK;
  };
  if (n_events > 0 && cudaEventRecord((cudaEvent_t)events[0], st) != cudaSuccess)
    return DSA_ERR_CUDA;
  char* ws = (char*)workspace;
  float* scores = (float*)(ws + p.off_scores);
  for (int32_t r0 = 0; r0 < R.n_q; r0 += p.slab) {
    const int32_t nr = (R.n_q - r0) < p.slab ? (R.n_q - r0) : p.slab;
    int32_t* idx = idx_out ? idx_out + (int64_t)r0 * a->k : (int32_t*)(ws + p.off_idx);
    if (p.fused) {  // indexer and top-k in one kernel
      if ((s = launch_indexer_select(R, r0, nr, a->idx_dtype, a->H_I, a->D_I, a->q_idx,
                                     a->q_scale, a->w, a->k_idx, a->k_scale, a->k, idx, scores,
                                     p.off_idx - p.off_scores, st)))
        return s;
      if ((s = mark(0))) return s;
    } else {
      if ((s = run_indexer(R, r0, nr, a->idx_dtype, a->H_I, a->D_I, a->q_idx, a->q_scale, a->w,
                           a->k_idx, a->k_scale, scores, false, st)))
        return s;
      if ((s = mark(0))) return s;
      if ((s = launch_topk(R, r0, nr, scores, R.max_len, a->k, idx, st))) return s;
      if ((s = mark(1))) return s;
    }
    // (idx is this chain's own top-k output: packed)
    if ((s = run_attn(R, r0, nr, a->q, a->kv, a->kv_scale, idx, a->k, a->H, a->D_K, a->D_V,
                      a->sm_scale, out,
                      lse, ws + p.off_attn, p.total - p.off_attn, st, true)))
      return s;
    if ((s = mark(2))) return s;
  }
  return DSA_OK;
}

dsa_status_t dsa_forward(const dsa_layout_t* layout, const dsa_forward_args_t* a, void* out,
                         float* lse, int32_t* idx_out, void* workspace, size_t ws_bytes,
                         void* stream) {
  return dsa_forward_timed(layout, a, out, lse, idx_out, workspace, ws_bytes, stream, nullptr, 0,
                           nullptr, nullptr);
}

size_t dsa_forward_host_workspace_size(const dsa_layout_t* layout, const dsa_forward_args_t* a,
                                       int32_t rows_per_slab) {
  Rows R;
  if (!a || rows_per_slab < 0 || check_layout(layout, &R)) return 0;
  return plan_forward(R, a, true, rows_per_slab).total;
}

dsa_status_t dsa_forward_host(const dsa_layout_t* layout, const dsa_forward_args_t* host,
                              const dsa_forward_args_t* dev, void* host_out, float* host_lse,
                              void* dev_out, float* dev_lse, int32_t rows_per_slab,
                              void* workspace, size_t ws_bytes, void* stream) {
  Rows R;
  dsa_status_t s = check_layout(layout, &R);
  if (s) return s;
  if (!host || !dev || rows_per_slab < 0) return DSA_ERR_INVALID_ARGUMENT;
  const dsa_forward_args_t* a = dev;
  if ((s = check_indexer(R, a->q_idx, a->q_scale, a->w, a->k_idx, a->k_scale, a->idx_dtype,
                         a->H_I, a->D_I)))
    return s;
  if ((s = check_attn(R, a->q, a->kv, a->kv_dtype, a->kv_scale, a->k, a->H, a->D_K, a->D_V,
                      a->sm_scale, dev_out,
                      dev_lse)))
    return s;
  if ((s = check_host(R, host, dev, host_out, host_lse, dev_lse))) return s;
  const ForwardPlan p = plan_forward(R, a, true, rows_per_slab);
  if (!workspace || ws_bytes < p.total || !aligned16(workspace)) return DSA_ERR_WORKSPACE;
  if (R.n_q == 0) return DSA_OK;
  if ((s = device_rows(&R))) return s;
  cudaStream_t st = (cudaStream_t)stream, hs = nullptr, ds = nullptr;
  if ((s = copy_streams(&hs, &ds))) return s;
  CallEvents ev;
  if (!ev.ok) return DSA_ERR_CUDA;
  const cudaEvent_t start = ev.e[0], in = ev.e[1], done = ev.e[2], end = ev.e[3],
                    in_q = ev.e[4];
  // bytes of one row of each array
  const size_t esz = a->idx_dtype == DSA_F32 ? 4 : a->idx_dtype == DSA_BF16 ? 2 : 1;
  const size_t qi_row = (size_t)a->H_I * a->D_I * esz, hv_row = (size_t)a->H_I * 4,
               q_row = (size_t)a->H * a->D_K * 2, out_row = (size_t)a->H * a->D_V * 2,
               lse_row = (size_t)a->H * 4;
  // bytes [off, off + n) of src to dst on cs; nothing when either side is absent
  auto copy = [](const void* dst, const void* src, size_t off, size_t n, cudaStream_t cs) {
    return !dst || !src || !n ||
           cudaMemcpyAsync((char*)dst + off, (const char*)src + off, n, cudaMemcpyDefault, cs) ==
               cudaSuccess;
  };
  char* ws = (char*)workspace;
  float* scores = (float*)(ws + p.off_scores);
  int32_t* idx = (int32_t*)(ws + p.off_idx);
  // the copies start after what `stream` holds (the previous call included)
  bool ok = cudaEventRecord(start, st) == cudaSuccess &&
            cudaStreamWaitEvent(hs, start, 0) == cudaSuccess &&
            cudaStreamWaitEvent(ds, start, 0) == cudaSuccess;
  // the key side first: any slab may read any cache row
  ok = ok && copy(a->k_idx, host->k_idx, 0, (size_t)R.n_k * a->D_I * esz, hs) &&
       copy(a->k_scale, host->k_scale, 0, (size_t)R.n_k * 4, hs) &&
       copy(a->kv, host->kv, 0, (size_t)R.n_k * a->D_K * (a->kv_dtype == DSA_E4M3 ? 1 : 2), hs) &&
       copy(a->kv_scale, host->kv_scale, 0, (size_t)R.n_k * 4, hs);
  for (int32_t r0 = 0; ok && r0 < R.n_q; r0 += p.slab) {
    const int32_t nr = (R.n_q - r0) < p.slab ? (R.n_q - r0) : p.slab;
    const size_t r = (size_t)r0, n = (size_t)nr;
    // slab i's query rows go up while slab i-1 computes and slab i-2's results come down;
    // the indexer's inputs first, under their own event, so that the indexer and the
    // top-k run while the attention's (larger) queries are still on the way
    ok = copy(a->q_idx, host->q_idx, r * qi_row, n * qi_row, hs) &&
         copy(a->q_scale, host->q_scale, r * hv_row, n * hv_row, hs) &&
         copy(a->w, host->w, r * hv_row, n * hv_row, hs) && cudaEventRecord(in, hs) == cudaSuccess &&
         copy(a->q, host->q, r * q_row, n * q_row, hs) &&
         cudaEventRecord(in_q, hs) == cudaSuccess && cudaStreamWaitEvent(st, in, 0) == cudaSuccess;
    if (!ok) break;
    if (p.fused) {
      if ((s = launch_indexer_select(R, r0, nr, a->idx_dtype, a->H_I, a->D_I, a->q_idx,
                                     a->q_scale, a->w, a->k_idx, a->k_scale, a->k, idx, scores,
                                     p.off_idx - p.off_scores, st)))
        break;
    } else {
      if ((s = run_indexer(R, r0, nr, a->idx_dtype, a->H_I, a->D_I, a->q_idx, a->q_scale, a->w,
                           a->k_idx, a->k_scale, scores, false, st)))
        break;
      if ((s = launch_topk(R, r0, nr, scores, R.max_len, a->k, idx, st))) break;
    }
    if (cudaStreamWaitEvent(st, in_q, 0) != cudaSuccess) {
      ok = false;
      break;
    }
    if ((s = run_attn(R, r0, nr, a->q, a->kv, a->kv_scale, idx, a->k, a->H, a->D_K, a->D_V,
                      a->sm_scale,
                      dev_out, dev_lse, ws + p.off_attn, p.total - p.off_attn, st, true)))
      break;
    ok = cudaEventRecord(done, st) == cudaSuccess &&
         cudaStreamWaitEvent(ds, done, 0) == cudaSuccess &&
         copy(host_out, dev_out, r * out_row, n * out_row, ds) &&
         copy(host_lse, dev_lse, r * lse_row, n * lse_row, ds);
  }
  // join, on every path: `stream` goes on only after both copy streams drained
  const bool joined = cudaEventRecord(in, hs) == cudaSuccess &&
                      cudaStreamWaitEvent(st, in, 0) == cudaSuccess &&
                      cudaEventRecord(end, ds) == cudaSuccess &&
                      cudaStreamWaitEvent(st, end, 0) == cudaSuccess;
  if (s) return s;
  return ok && joined ? DSA_OK : DSA_ERR_CUDA;
}

}  // extern "C"
