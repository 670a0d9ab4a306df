/*
 * dsa.h -- C ABI of libdsa.so, the B200 (sm_100a) hot path of DeepSeek Sparse
 * Attention: lightning indexer -> per-query top-k -> sparse MLA attention.
 *
 * The method (three stages: score every earlier token cheaply, keep the k
 * best, run exact attention on the survivors):
 *   "Linear and Sparse Attention" (yuxiangdai.com), "DeepSeek Sparse Attention";
 *   "GLM sparse attention" (thethings.ai), two-stage paragraph and MLA passage;
 *   "DeepSeek Sparse Attention" (divagr.pages.dev), "Step through token selection".
 *
 * Conventions shared by every call
 *  - Tensor arguments are DEVICE pointers owned by the caller; the library
 *    never allocates device memory, frees or synchronises (dsa_device_status
 *    excepted).  Scratch memory comes only through the caller's `workspace`.
 *    dsa_forward_host alone also takes HOST pointers (its `host` block and
 *    results), and creates two copy streams per device on first use and a
 *    few events per call.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call
 *    only enqueues work on it and returns.
 *  - Arguments are validated on the host before anything is launched; a
 *    failure returns DSA_ERR_INVALID_ARGUMENT / DSA_ERR_UNSUPPORTED /
 *    DSA_ERR_WORKSPACE and leaves every output untouched.  A failed launch
 *    returns DSA_ERR_CUDA.
 *  - Conditions only the device can see (offsets that are not monotone or
 *    exceed n_k, an index outside its causal range, a bounded wait that ran out)
 *    make the kernels skip the affected row or tile and raise a bit in a
 *    per-device status word, read and cleared by dsa_device_status().
 *  - Every device pointer passed must be 16-byte aligned (host pointers may
 *    have any alignment).
 *  - Index outputs are LOCAL positions inside the query's own sequence.
 *  - bf16 tensors are passed as raw 16-bit storage, e4m3 as raw bytes
 *    (OCP FP8 E4M3 "fn": no infinities, S.1111.111 = NaN).
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARGUMENT = 1, /* null pointer, bad size, misalignment */
  DSA_ERR_UNSUPPORTED = 2,      /* a valid shape or dtype this build does not run */
  DSA_ERR_WORKSPACE = 3,        /* workspace NULL or smaller than *_workspace_size() */
  DSA_ERR_CUDA = 4,             /* a CUDA runtime call or launch failed */
  DSA_ERR_TIMEOUT = 5,          /* device status: a bounded wait ran out */
  DSA_ERR_DEVICE_DATA = 6       /* device status: bad offsets or index values were skipped */
} dsa_status_t;

typedef enum { DSA_F32 = 0, DSA_BF16 = 1, DSA_E4M3 = 2 } dsa_dtype_t;

typedef enum { DSA_PREFILL = 0, DSA_DECODE = 1, DSA_CHUNKED = 2 } dsa_mode_t;

/*
 * Ragged layout shared by every call.
 *
 * The caches hold B sequences back to back; sequence b owns cache rows
 * kv_offsets[b] .. kv_offsets[b+1]-1, so its length is
 * L_b = kv_offsets[b+1] - kv_offsets[b].
 *  - PREFILL: every cache row is also a query row (self-attention over the
 *    prompt); n_q == n_k, query row r of sequence b sits at local position
 *    t = r - kv_offsets[b] and sees positions 0..t.
 *  - DECODE: one query per sequence, n_q == B; query row b sits at position
 *    t = L_b - 1 (the cache already holds the new token) and sees 0..t.
 *  - CHUNKED: a prefill of new tokens against a cache that already holds
 *    earlier ones (chunked prefill with a prefix cache).  Sequence b owns
 *    query rows q_offsets[b] .. q_offsets[b+1]-1, C_b of them, its LAST C_b
 *    positions: query i sits at t = L_b - C_b + i and sees 0..t (the cache
 *    already holds the chunk's own tokens).  n_q == q_offsets[B].  PREFILL is
 *    the case C_b = L_b, DECODE the case C_b = 1.  q_offsets must be
 *    non-decreasing with C_b <= L_b; a sequence that breaks this is skipped
 *    on the device and reported as DSA_ERR_DEVICE_DATA.
 * The candidate set of a query is s <= t, the causal lower triangle
 * ("GLM sparse attention", 56-token causal figure; the diagonal included).
 */
typedef struct {
  int32_t mode;              /* dsa_mode_t */
  int32_t batch;             /* B >= 0 */
  const int32_t* kv_offsets; /* DEVICE [B+1], kv_offsets[0] = 0, non-decreasing */
  int32_t max_len;           /* >= every L_b; the row stride of score arrays */
  int32_t n_q;               /* query rows (see above) */
  int64_t n_k;               /* cache rows = kv_offsets[B] */
  const int32_t* q_offsets;  /* CHUNKED only: DEVICE [B+1], q_offsets[0] = 0; else unused */
} dsa_layout_t;

/*
 * Stage 1, lightning indexer ("GLM sparse attention", ReLU paragraph;
 * "Sparse Attention Architecture Evolution in LLMs", Indexer section):
 *
 *   scores[r, s] = sum_{j < H_I} w[r, j] * ReLU( <q_idx[r, j, :], k_idx[kbase + s, :]> )
 *
 * for s <= t(r), and -inf for t(r) < s < max_len.  Each head's similarity is
 * clipped at zero before the weighted head sum; there is no other scale.
 *  q_idx   [n_q, H_I, D_I]  dtype (f32, bf16 or e4m3)
 *  q_scale [n_q, H_I] fp32  e4m3 only (NULL otherwise): dequantised
 *          q = code * q_scale[r, j]; must be > 0 (it is folded into w)
 *  w       [n_q, H_I] fp32
 *  k_idx   [n_k, D_I]       dtype
 *  k_scale [n_k] fp32       e4m3 only (NULL otherwise); must be > 0
 *  scores  [n_q, max_len] fp32, written in full
 * Products accumulate in fp32.  Supported: f32 any H_I <= 128, D_I <= 256;
 * bf16/e4m3 any H_I <= 128, D_I <= 256 (H_I = 64, D_I = 128 runs on the
 * tensor cores).
 */
dsa_status_t dsa_indexer_scores(const dsa_layout_t* layout, const void* q_idx,
                                const float* q_scale, const float* w, const void* k_idx,
                                const float* k_scale, int32_t dtype, int32_t H_I, int32_t D_I,
                                float* scores, void* stream);

/*
 * Stage 2, top-k selection ("Sparse Attention Architecture Evolution in
 * LLMs", Top-K Selection; "GLM sparse attention", threshold figure: the
 * cut-off is the k-th best score):
 *
 * For query row r with n = t(r)+1 candidates, idx[r, :] receives the k
 * positions of largest scores[r, 0:n]; ties go to the lower position; -0 and
 * +0 are equal; NaN ranks as -inf.  If n <= k every position 0..n-1 is
 * written and the remaining slots are -1.  The order inside a row is
 * unspecified (a set).  Columns >= n of `scores` are never read.
 *  scores [n_q, max_len] fp32, idx [n_q, k] int32, 1 <= k <= 16384.
 */
dsa_status_t dsa_topk(const dsa_layout_t* layout, const float* scores, int32_t k, int32_t* idx,
                      void* stream);

/*
 * Stage 3, sparse MLA attention ("GLM sparse attention", MLA passage: one
 * latent row per token, read by every head as in multi-query attention, and
 * a full softmax over the selected tokens, the attention itself not
 * approximated; "DeepSeek Sparse Attention" (divagr.pages.dev), "the risk":
 * a token left out of the selection adds nothing to the output):
 *
 *   z[h, s]  = sm_scale * <q[r, h, 0:D_K], kv[kbase + s, 0:D_K]>
 *   out[r,h] = sum_{s in S_r} softmax_S(z[h, :])_s * kv[kbase + s, 0:D_V]
 *   lse[r,h] = log sum_{s in S_r} exp(z[h, s])          (natural log)
 *
 * S_r = the entries of idx[r, 0:k] that are >= 0 (-1 marks an empty slot);
 * entries must be distinct causal positions, 0 <= s <= t(r) (so < L_b); an
 * entry outside that range is skipped like -1 and raises
 * DSA_ERR_DEVICE_DATA.  q is the absorbed query (rope part
 * already rotated), kv a row of latent (first D_V columns, also the value)
 * followed by the rotary key.  A row with no selected position gets out = 0
 * and lse = -inf.
 *  q   [n_q, H, D_K] bf16, kv [n_k, D_K] bf16, idx [n_q, k] int32
 *  out [n_q, H, D_V] bf16, lse [n_q, H] fp32 (may be NULL)
 * Products accumulate in fp32.  H = 128, D_K = 576, D_V = 512 runs on the
 * tensor cores; other shapes (H <= 128, D_V <= D_K <= 1024, multiples of 8)
 * on the generic path.
 */
dsa_status_t dsa_sparse_mla_attn(const dsa_layout_t* layout, const void* q, const void* kv,
                                 const int32_t* idx, int32_t k, int32_t H, int32_t D_K,
                                 int32_t D_V, float sm_scale, void* out, float* lse,
                                 void* workspace, size_t ws_bytes, void* stream);

/* Workspace bytes dsa_sparse_mla_attn (and dsa_sparse_mla_attn_e4m3) need
 * for this layout and shape. */
size_t dsa_sparse_mla_attn_workspace_size(const dsa_layout_t* layout, int32_t k, int32_t H,
                                          int32_t D_K, int32_t D_V);

/*
 * Stage 3 over an FP8 MLA cache.  "GLM sparse attention" (ReLU paragraph)
 * gives FP8 as the indexer's precision; this call applies the same storage
 * format to the cached latent + rotary rows, halving the bytes each selected
 * token costs to gather (576 instead of 1152 at D_K = 576):
 *
 *   C[s, d] = code(kv[kbase + s, d]) * kv_scale[kbase + s]
 *
 * with code() the exact value of an OCP e4m3 byte, and then exactly the
 * attention of dsa_sparse_mla_attn on that C (the value is C[s, 0:D_V]).
 *  kv       [n_k, D_K] e4m3 codes (raw bytes; the NaN codes are not allowed)
 *  kv_scale [n_k] fp32, one scale per cached token
 * q, idx, out, lse, workspace and every error: as dsa_sparse_mla_attn; D_K
 * must be a multiple of 16.  The codes are decoded exactly to bf16 on the
 * device and the MMAs are the bf16 ones: each score is multiplied by its
 * token's scale, and the PV operand holds p * scale (rounded to bf16, like p
 * in dsa_sparse_mla_attn); the softmax denominator sums the fp32 p.
 */
dsa_status_t dsa_sparse_mla_attn_e4m3(const dsa_layout_t* layout, const void* q, const void* kv,
                                      const float* kv_scale, const int32_t* idx, int32_t k,
                                      int32_t H, int32_t D_K, int32_t D_V, float sm_scale,
                                      void* out, float* lse, void* workspace, size_t ws_bytes,
                                      void* stream);

/*
 * dsa_sparse_mla_attn for callers that cannot allocate device memory.
 *
 * The pages have no counterpart to this entry point; it exists for the
 * library's users.  Some callers cannot call cudaMalloc or any allocating
 * routine: code that runs while a CUDA graph is being captured with a strict
 * capture mode, code inside a framework whose memory pool owns the whole
 * device, or plug-ins that are handed tensors but no allocator.  This call
 * takes the same arguments as dsa_sparse_mla_attn minus the workspace: the
 * decode split partials go to a fixed 20 MiB array that the library owns
 * on every GPU where it is loaded, held until the process exits.
 *  - Capacity: 79 (query row, split) blocks of 128 heads x 513 floats.  The
 *    split plan of both attention entry points keeps every CTA pair in one
 *    wave (74 pairs on a 148-SM B200) and never uses more blocks than that,
 *    so no call is refused for size.  DSA_ERR_WORKSPACE here would mean a
 *    plan beyond the array, which the planner does not produce.
 *  - Nothing needs zeroing: every call writes each partial it later reads.
 *  - The array is shared by all calls on a device and keeps the last call's
 *    contents: calls whose executions overlap on the GPU (different streams,
 *    no ordering between them) race on it and must be serialised.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current); make that first call
 *    before any stream capture.
 * Results equal those of dsa_sparse_mla_attn on the same inputs.
 */
dsa_status_t dsa_sparse_mla_attn_noalloc(const dsa_layout_t* layout, const void* q,
                                         const void* kv, const int32_t* idx, int32_t k, int32_t H,
                                         int32_t D_K, int32_t D_V, float sm_scale, void* out,
                                         float* lse, void* stream);

/* Inputs of the whole chain (each field as in the stage calls above). */
typedef struct {
  int32_t idx_dtype; /* dsa_dtype_t of q_idx / k_idx */
  int32_t H_I, D_I;
  const void* q_idx;
  const float* q_scale;
  const float* w;
  const void* k_idx;
  const float* k_scale;
  int32_t H, D_K, D_V;
  float sm_scale;
  const void* q;
  const void* kv;
  int32_t k;            /* top-k budget */
  int32_t kv_dtype;     /* DSA_BF16, or DSA_E4M3 (then kv holds codes, see below) */
  const float* kv_scale; /* DSA_E4M3: [n_k] fp32 per-token cache scales
                            (dsa_sparse_mla_attn_e4m3); NULL for bf16 */
} dsa_forward_args_t;

/* Workspace bytes dsa_forward needs (scores slab, indices, attention partials). */
size_t dsa_forward_workspace_size(const dsa_layout_t* layout, const dsa_forward_args_t* args);

/*
 * The whole hot path (prefill, chunked or decode): indexer -> top-k -> sparse MLA
 * attention, enqueued on one stream.  Query rows run in slabs so that only a
 * slab of scores is ever held (in the workspace): as many rows as fit 1 GiB
 * of fp32 scores at max_len per row (4096 rows at 64K context).
 *  out [n_q, H, D_V] bf16; lse [n_q, H] fp32 or NULL;
 *  idx_out [n_q, k] int32 or NULL (then the indices live in the workspace).
 * Decode with the environment variable DSA_FUSED_DECODE_SELECT set to "1" at
 * the call runs the indexer with the top-k fused in (per-row candidate lists
 * against a running threshold, no score rows; the same indices as the
 * separate kernels).  Off by default: it is slower.  The workspace size
 * depends on it, so query dsa_forward_workspace_size under the same setting.
 */
dsa_status_t dsa_forward(const dsa_layout_t* layout, const dsa_forward_args_t* args, void* out,
                         float* lse, int32_t* idx_out, void* workspace, size_t ws_bytes,
                         void* stream);

/*
 * dsa_forward with a timeline: events[0] (a cudaEvent_t created by the
 * caller) is recorded on `stream` before the first kernel and events[i+1]
 * right after the i-th kernel launch, for i < n_events - 1; kinds[i] gets
 * that kernel's stage (0 indexer, 1 top-k, 2 attention, 3 split combine) and
 * *n_launched the number of kernels enqueued (kinds / n_launched may be
 * NULL).  For measurement; results are those of dsa_forward.
 */
dsa_status_t dsa_forward_timed(const dsa_layout_t* layout, const dsa_forward_args_t* args,
                               void* out, float* lse, int32_t* idx_out, void* workspace,
                               size_t ws_bytes, void* stream, void* const* events,
                               int32_t n_events, int32_t* kinds, int32_t* n_launched);

/*
 * dsa_forward for inputs and results in host memory, pipelined over slabs of
 * query rows: slab i's query rows are copied up (on a copy stream of the
 * library's own) while slab i-1 computes on `stream` and slab i-2's output
 * is copied down (on a second copy stream), so the two PCIe directions and
 * the kernels overlap.  A slab's indexer inputs (q_idx, q_scale, w) go up
 * first, so its indexer and top-k start while its attention queries (q) are
 * still on the way.  The kernels and their arguments are those of
 * dsa_forward, and so are the results, up to the rounding order of the
 * attention sums (the order of a row's selected indices is unspecified, as
 * for dsa_topk, so two calls of either entry point may differ in the last
 * bits).
 *  host: the arguments with host pointers (pinned memory for the copies to
 *        overlap; pageable memory gives the same results, serialised).
 *        q_idx, w, q (and q_scale for e4m3) are required when n_q > 0.
 *        k_idx, k_scale, kv may each be NULL: `dev`'s copy is then taken as
 *        current (a cache kept in HBM across calls); otherwise all n_k rows
 *        are copied before the first slab.  Scalars must equal dev's.
 *  dev:  the same arguments with full-size device buffers (checked as in
 *        dsa_forward); the call writes the host inputs into them.
 *  host_out [n_q, H, D_V] bf16, host_lse [n_q, H] fp32 or NULL: the results;
 *  dev_out / dev_lse: full-size device buffers they pass through (dev_lse
 *        required when host_lse is given).
 *  rows_per_slab: 0 for dsa_forward's slabs (bounded by 1 GiB of scores),
 *        else at most that many rows per slab.
 *  workspace: dsa_forward_host_workspace_size(layout, dev, rows_per_slab)
 *        bytes, 16-byte aligned.
 * Ordering: the copies start after the work `stream` holds at the call, and
 * `stream` continues only after the last result reached host memory, so a
 * synchronisation of `stream` makes host_out / host_lse readable.  With
 * n_q = 0 nothing is copied or launched.  Calls from several host threads
 * are correct; their copies share the device's two copy streams, so they
 * take turns on PCIe.  Errors: those of dsa_forward, and
 * DSA_ERR_INVALID_ARGUMENT for host arguments that break the above.  After
 * DSA_ERR_CUDA, copies may still be in flight: synchronise the device.
 */
size_t dsa_forward_host_workspace_size(const dsa_layout_t* layout, const dsa_forward_args_t* args,
                                       int32_t rows_per_slab);
dsa_status_t dsa_forward_host(const dsa_layout_t* layout, const dsa_forward_args_t* host,
                              const dsa_forward_args_t* dev, void* host_out, float* host_lse,
                              void* dev_out, float* dev_lse, int32_t rows_per_slab,
                              void* workspace, size_t ws_bytes, void* stream);

/*
 * Synchronises `stream`, then returns and clears this device's status word:
 * DSA_OK, DSA_ERR_TIMEOUT or DSA_ERR_DEVICE_DATA (DSA_ERR_CUDA if the
 * synchronisation itself failed).  The word is shared by every stream of the
 * device.
 */
dsa_status_t dsa_device_status(void* stream);

/*
 * Self-test of the failure path every kernel shares: one thread waits on a
 * barrier that nothing completes, using the same bounded wait as the
 * kernels, but giving up after `cycles` clock cycles (0 .. the kernels' own
 * limit of 2e9) instead of the kernels' limit.  The wait then raises the
 * timeout bit, so the next dsa_device_status() returns DSA_ERR_TIMEOUT and
 * the device stays usable.  No copy, MMA or other work is in flight when the
 * wait gives up.  Not part of the method; it exists so that tests can see a
 * wait run out without faulting or hanging the GPU.
 * Returns DSA_ERR_INVALID_ARGUMENT for `cycles` outside that range,
 * DSA_ERR_CUDA if the launch fails.
 */
dsa_status_t dsa_selftest_wait_timeout(int64_t cycles, void* stream);

/* Static description of a status code. */
const char* dsa_status_string(dsa_status_t status);

/* ABI version, bumped on any signature change (4: the FP8 MLA cache, fields
 * kv_dtype / kv_scale of dsa_forward_args_t). */
int32_t dsa_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H_ */
