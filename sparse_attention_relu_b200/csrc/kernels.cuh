// Internal launchers of libdsa (not part of the ABI).
//
// Row conventions: query-row arrays (q_idx, q_scale, w, q, out, lse) are
// indexed by the absolute query row r; per-slab arrays (scores, idx) point
// at the slab's first row `row0` and are indexed by r - row0.
#pragma once

#include "common.cuh"

namespace dsa {

// Generic indexer (any dtype, H_I * D_I <= 16384, D_I <= 256).
dsa_status_t launch_indexer_simt(const Rows& R, int32_t row0, int32_t nrows, int dtype, int H_I,
                                 int D_I, const void* q_idx, const float* q_scale,
                                 const float* w, const void* k_idx, const float* k_scale,
                                 float* scores, int64_t ld, bool fill_masked, cudaStream_t st);

// Tensor-core indexer (bf16 / e4m3, H_I = 64, D_I = 128).  Returns
// DSA_ERR_UNSUPPORTED when the shape does not fit it.
dsa_status_t launch_indexer_tc(const Rows& R, int32_t row0, int32_t nrows, int dtype, int H_I,
                               int D_I, const void* q_idx, const float* q_scale, const float* w,
                               const void* k_idx, const float* k_scale, float* scores, int64_t ld,
                               bool fill_masked, cudaStream_t st);
bool indexer_tc_supported(int dtype, int H_I, int D_I);

// Decode indexer with the top-k fused in (no score rows are written): each
// row's scores are filtered against a running threshold into a candidate list
// in the workspace, and the row's k best are selected from it into idx
// [nrows, k] (the semantics of launch_topk).
bool indexer_select_supported(const Rows& R, int dtype, int H_I, int D_I, int k);
size_t indexer_select_workspace(const Rows& R, int32_t nrows);
dsa_status_t launch_indexer_select(const Rows& R, int32_t row0, int32_t nrows, int dtype,
                                   int H_I, int D_I, const void* q_idx, const float* q_scale,
                                   const float* w, const void* k_idx, const float* k_scale, int k,
                                   int32_t* idx, void* ws, size_t ws_bytes, cudaStream_t st);

// The k best of each row from the fused decode indexer's candidate lists
// (cand [nrows][cap] in segments, segment counts segcnt [nrows][cap / 128],
// row histograms rhist [nrows][2048]).
dsa_status_t launch_select_rows(const Rows& R, int32_t row0, int32_t nrows, const uint64_t* cand,
                                int64_t cap, const uint32_t* segcnt, const uint32_t* rhist, int k,
                                int32_t* idx, cudaStream_t st);

// Radix top-k, one CTA per row.
dsa_status_t launch_topk(const Rows& R, int32_t row0, int32_t nrows, const float* scores,
                         int64_t ld, int k, int32_t* idx, cudaStream_t st);

// Generic sparse MLA attention (H <= 128, D_V <= D_K <= 1024, multiples of 8);
// the cache as for launch_attn_tc.
dsa_status_t launch_attn_simt(const Rows& R, int32_t row0, int32_t nrows, const uint16_t* q,
                              const void* kv, const float* kv_scale, const int32_t* idx, int k,
                              int H, int D_K, int D_V, float sm_scale, uint16_t* out, float* lse,
                              cudaStream_t st);

// Tensor-core sparse MLA attention (H = 128, D_K = 576, D_V = 512).  kv is a
// bf16 cache, or (kv_scale != NULL) e4m3 codes with one fp32 scale per token.
bool attn_tc_supported(int H, int D_K, int D_V);
size_t attn_tc_workspace(int32_t nrows, int k, int H, int D_V);
// packed: each row's valid indices come first and number at most t + 1 (the
// top-k's output), so the tiles after slot min(t + 1, k) hold no index and are
// skipped; otherwise every one of the k slots is scanned.
dsa_status_t launch_attn_tc(const Rows& R, int32_t row0, int32_t nrows, const uint16_t* q,
                            const void* kv, const float* kv_scale, const int32_t* idx, int k,
                            float sm_scale, uint16_t* out, float* lse, void* ws, size_t ws_bytes,
                            cudaStream_t st, bool packed = false);

// As launch_attn_tc, with the split partials in a fixed static device array
// (DSA_ERR_WORKSPACE when the call needs more than it holds).
size_t attn_tc_static_scratch_bytes();
dsa_status_t launch_attn_tc_static(const Rows& R, int32_t row0, int32_t nrows, const uint16_t* q,
                                   const uint16_t* kv, const int32_t* idx, int k, float sm_scale,
                                   uint16_t* out, float* lse, cudaStream_t st);

}  // namespace dsa
