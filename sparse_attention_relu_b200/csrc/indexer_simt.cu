// Generic lightning indexer on the CUDA cores.
//
//   I[t, s] = sum_j w[t, j] * ReLU(<q_I[t, j, :], k_I[s, :]>),  s <= t
//
// ("GLM sparse attention", ReLU paragraph: each head's similarity is clipped
// at zero before the weighted sum.)  Used for fp32 inputs and for indexer
// shapes the tensor-core kernel does not take.  One CTA scores one query row
// against a tile of keys; the query row and the key tile are staged in
// shared memory as fp32, the key tile padded by one word per row so that the
// 32 lanes (one key each) read distinct banks.
//
// fp8 scales: the dequantised similarity of head j is
// q_scale[t,j] * k_scale[s] * <q8, k8>, and for positive scales
// a * ReLU(x) = ReLU(a * x), so q_scale folds into w and k_scale multiplies
// the finished sum.
#include <cuda_fp8.h>

#include "kernels.cuh"

namespace dsa {

template <int DT>
__device__ __forceinline__ float load_val(const void* p, int64_t i) {
  if constexpr (DT == DSA_F32) {
    return __ldg(reinterpret_cast<const float*>(p) + i);
  } else if constexpr (DT == DSA_BF16) {
    return bf16_bits_to_f32(__ldg(reinterpret_cast<const uint16_t*>(p) + i));
  } else {
    __nv_fp8_e4m3 v;
    v.__x = __ldg(reinterpret_cast<const unsigned char*>(p) + i);
    return static_cast<float>(v);
  }
}

template <int DT, int KT>
__global__ void __launch_bounds__(128) indexer_simt_kernel(Rows R, int32_t row0, int H_I, int D_I,
                                                           const void* q_idx, const float* q_scale,
                                                           const float* w, const void* k_idx,
                                                           const float* k_scale, float* scores,
                                                           int64_t ld, int fill) {
  extern __shared__ float sm[];
  float* qs = sm;                 // [H_I][D_I]
  float* ws = qs + H_I * D_I;     // [H_I]
  float* ks = ws + H_I;           // [KT][D_I + 1]
  const int tid = threadIdx.x;
  const int32_t r = row0 + blockIdx.x;
  const RowInfo ri = row_info(R, r);
  float* out = scores + (int64_t)blockIdx.x * ld;
  const int s0 = blockIdx.y * KT;
  if (s0 > ri.t) {  // the whole tile lies above the diagonal
    if (fill)
      for (int s = s0 + tid; s < min(s0 + KT, R.max_len); s += blockDim.x) out[s] = -INFINITY;
    return;
  }
  for (int i = tid; i < H_I * D_I; i += blockDim.x)
    qs[i] = load_val<DT>(q_idx, (int64_t)r * H_I * D_I + i);
  for (int j = tid; j < H_I; j += blockDim.x)
    ws[j] = __ldg(w + (int64_t)r * H_I + j) * (q_scale ? __ldg(q_scale + (int64_t)r * H_I + j) : 1.f);
  const int nk = min(KT, ri.t + 1 - s0);
  for (int i = tid; i < nk * D_I; i += blockDim.x) {
    int kk = i / D_I, d = i - kk * D_I;
    ks[kk * (D_I + 1) + d] = load_val<DT>(k_idx, (ri.kbase + s0 + kk) * D_I + d);
  }
  __syncthreads();
  for (int kk = tid; kk < KT; kk += blockDim.x) {
    int s = s0 + kk;
    if (s >= R.max_len) break;
    if (kk < nk) {
      const float* kr = ks + kk * (D_I + 1);
      float acc = 0.f;
      for (int j = 0; j < H_I; ++j) {
        const float* qj = qs + j * D_I;
        float dot = 0.f;
        for (int d = 0; d < D_I; ++d) dot = fmaf(qj[d], kr[d], dot);
        acc = fmaf(ws[j], fmaxf(dot, 0.f), acc);
      }
      if (k_scale) acc *= __ldg(k_scale + ri.kbase + s);
      out[s] = acc;
    } else if (fill) {
      out[s] = -INFINITY;
    }
  }
}

template <int DT>
static dsa_status_t launch_dt(const Rows& R, int32_t row0, int32_t nrows, int H_I, int D_I,
                              const void* q_idx, const float* q_scale, const float* w,
                              const void* k_idx, const float* k_scale, float* scores, int64_t ld,
                              bool fill, cudaStream_t st) {
  if (nrows <= 0 || R.max_len <= 0) return DSA_OK;
  if (D_I <= 128) {
    constexpr int KT = 128;
    size_t smem = sizeof(float) * ((size_t)H_I * D_I + H_I + (size_t)KT * (D_I + 1));
    auto kfn = indexer_simt_kernel<DT, KT>;
    if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return DSA_ERR_CUDA;
    dim3 grid(nrows, (R.max_len + KT - 1) / KT);
    kfn<<<grid, 128, smem, st>>>(R, row0, H_I, D_I, q_idx, q_scale, w, k_idx, k_scale, scores, ld,
                                 fill ? 1 : 0);
  } else {
    constexpr int KT = 64;
    size_t smem = sizeof(float) * ((size_t)H_I * D_I + H_I + (size_t)KT * (D_I + 1));
    auto kfn = indexer_simt_kernel<DT, KT>;
    if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return DSA_ERR_CUDA;
    dim3 grid(nrows, (R.max_len + KT - 1) / KT);
    kfn<<<grid, 128, smem, st>>>(R, row0, H_I, D_I, q_idx, q_scale, w, k_idx, k_scale, scores, ld,
                                 fill ? 1 : 0);
  }
  return launch_status();
}

dsa_status_t launch_indexer_simt(const Rows& R, int32_t row0, int32_t nrows, int dtype, int H_I,
                                 int D_I, const void* q_idx, const float* q_scale,
                                 const float* w, const void* k_idx, const float* k_scale,
                                 float* scores, int64_t ld, bool fill_masked, cudaStream_t st) {
  switch (dtype) {
    case DSA_F32:
      return launch_dt<DSA_F32>(R, row0, nrows, H_I, D_I, q_idx, q_scale, w, k_idx, k_scale,
                                scores, ld, fill_masked, st);
    case DSA_BF16:
      return launch_dt<DSA_BF16>(R, row0, nrows, H_I, D_I, q_idx, q_scale, w, k_idx, k_scale,
                                 scores, ld, fill_masked, st);
    case DSA_E4M3:
      return launch_dt<DSA_E4M3>(R, row0, nrows, H_I, D_I, q_idx, q_scale, w, k_idx, k_scale,
                                 scores, ld, fill_masked, st);
    default:
      return DSA_ERR_UNSUPPORTED;
  }
}

}  // namespace dsa
