// Generic sparse MLA attention on the CUDA cores.
//
// For query row r and head h, over the selected positions S_r:
//   z_s = sm_scale * <q[r,h,0:D_K], C[s,0:D_K]>,  out = softmax(z) . C[S_r, 0:D_V]
// ("GLM sparse attention", MLA passage: the cached latent row is read by
// every head, as in multi-query attention; the softmax is exact over the
// survivors.)  Used for shapes the tensor-core kernel does not take (the
// tiny 8-head, 80/64 configuration among them).
//
// One CTA = one query row x a group of 16 heads.  The selected rows arrive
// in chunks of 32 index slots: the chunk's latent rows are gathered with
// 16-byte loads into shared memory as fp32 (rows padded by one word, so a
// warp with one lane per row reads 32 banks); a warp scores two heads with
// one lane per row and runs the online softmax; then every thread updates
// its slice of the 16 x D_V output accumulator held in registers.
#include "kernels.cuh"

namespace dsa {

namespace {

constexpr int kHG = 16;       // heads per CTA
constexpr int kChunk = 32;    // index slots per chunk
constexpr int kThreads = 256;

// FP8: the cache holds e4m3 codes with one fp32 scale per token (kv_scale);
// a gathered row is decoded exactly and multiplied by its scale in fp32.
template <int VPT, bool FP8>  // output columns per thread: D_V <= 16 * VPT
__global__ void __launch_bounds__(kThreads) attn_simt_kernel(Rows R, int32_t row0,
                                                             const uint16_t* __restrict__ q,
                                                             const void* __restrict__ kv,
                                                             const float* __restrict__ kv_scale,
                                                             const int32_t* __restrict__ idx, int k,
                                                             int H, int D_K, int D_V, float sm_scale,
                                                             uint16_t* __restrict__ out,
                                                             float* __restrict__ lse) {
  extern __shared__ float smf[];
  float* qs = smf;                              // [kHG][D_K]
  float* cs = qs + kHG * D_K;                   // [kChunk][D_K + 1]
  float* ps = cs + kChunk * (D_K + 1);          // [kHG][kChunk]
  float* alpha = ps + kHG * kChunk;             // [kHG]
  float* lsum = alpha + kHG;                    // [kHG]
  float* mrow = lsum + kHG;                     // [kHG]
  int* sel = reinterpret_cast<int*>(mrow + kHG);  // [kChunk]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int32_t r = row0 + blockIdx.x;
  const int h0 = blockIdx.y * kHG;
  const RowInfo ri = row_info(R, r);
  const int32_t* irow = idx + (int64_t)blockIdx.x * k;

  for (int i = tid; i < kHG * D_K; i += kThreads) {
    int hh = i / D_K, d = i - hh * D_K;
    qs[i] = (h0 + hh < H) ? bf16_bits_to_f32(q[((int64_t)r * H + h0 + hh) * D_K + d]) : 0.f;
  }
  // softmax state of heads 2*warp, 2*warp+1 (replicated in every lane)
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  // output accumulator: head tid / 16, columns (tid % 16) + 16 * i
  const int oh = tid >> 4, oc = tid & 15;
  float acc[VPT];
#pragma unroll
  for (int i = 0; i < VPT; ++i) acc[i] = 0.f;

  const int nvec = FP8 ? D_K / 16 : D_K / 8;  // 16-byte vectors per cached row
  for (int c0 = 0; c0 < k; c0 += kChunk) {
    if (tid < kChunk) {
      int s = (c0 + tid < k) ? __ldg(irow + c0 + tid) : -1;
      // candidates are the causal positions 0..t (t < L_b); a later one is bad data
      if (s < -1 || s > ri.t) {
        if (s != -1 && ri.t >= 0) raise_status(R, kErrBadIndex);
        s = -1;
      }
      sel[tid] = s;
    }
    __syncthreads();
    for (int i = tid; i < kChunk * nvec; i += kThreads) {
      int rr = i / nvec, vv = i - rr * nvec;
      int s = sel[rr];
      float* dst = cs + rr * (D_K + 1) + vv * 8;
      if (FP8) {
        float* d16 = cs + rr * (D_K + 1) + vv * 16;
        if (s >= 0) {
          const uint8_t* row = reinterpret_cast<const uint8_t*>(kv) + (ri.kbase + s) * D_K;
          const uint4 v = __ldg(reinterpret_cast<const uint4*>(row) + vv);
          const float sc = __ldg(kv_scale + ri.kbase + s);
          const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            uint32_t lo, hi;
            e4m3x4_to_bf16x4(w4[e], lo, hi);
            d16[4 * e] = __uint_as_float(lo << 16) * sc;
            d16[4 * e + 1] = __uint_as_float(lo & 0xffff0000u) * sc;
            d16[4 * e + 2] = __uint_as_float(hi << 16) * sc;
            d16[4 * e + 3] = __uint_as_float(hi & 0xffff0000u) * sc;
          }
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) d16[e] = 0.f;
        }
      } else if (s >= 0) {
        const uint16_t* row = reinterpret_cast<const uint16_t*>(kv) + (ri.kbase + s) * D_K;
        uint4 v = __ldg(reinterpret_cast<const uint4*>(row) + vv);
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          dst[2 * e] = __uint_as_float(w4[e] << 16);
          dst[2 * e + 1] = __uint_as_float(w4[e] & 0xffff0000u);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) dst[e] = 0.f;
      }
    }
    __syncthreads();
    // scores and online softmax: warp -> heads 2w, 2w+1; lane -> slot
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int hh = 2 * warp + u;
      const float* qh = qs + hh * D_K;
      const float* cr = cs + lane * (D_K + 1);
      float dot = 0.f;
      for (int d = 0; d < D_K; ++d) dot = fmaf(qh[d], cr[d], dot);
      float z = sel[lane] >= 0 ? dot * sm_scale : -INFINITY;
      float mc = z;
      for (int off = 16; off; off >>= 1) mc = fmaxf(mc, __shfl_xor_sync(0xffffffffu, mc, off));
      const float m_new = fmaxf(m_run[u], mc);
      float p = 0.f, a = 1.f;
      if (m_new != -INFINITY) {
        p = __expf(z - m_new);
        a = __expf(m_run[u] - m_new);
      }
      float ps_sum = p;
      for (int off = 16; off; off >>= 1) ps_sum += __shfl_xor_sync(0xffffffffu, ps_sum, off);
      l_run[u] = l_run[u] * a + ps_sum;
      m_run[u] = m_new;
      ps[hh * kChunk + lane] = p;
      if (lane == 0) alpha[hh] = a;
    }
    __syncthreads();
    {
      const float a = alpha[oh];
      const float* pr = ps + oh * kChunk;
#pragma unroll
      for (int i = 0; i < VPT; ++i) {
        const int col = oc + 16 * i;
        if (col < D_V) {
          float v = acc[i] * a;
          for (int j = 0; j < kChunk; ++j) v = fmaf(pr[j], cs[j * (D_K + 1) + col], v);
          acc[i] = v;
        }
      }
    }
    __syncthreads();
  }
  if (lane == 0) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      lsum[2 * warp + u] = l_run[u];
      mrow[2 * warp + u] = m_run[u];
    }
  }
  __syncthreads();
  const int h = h0 + oh;
  if (h < H) {
    const float l = lsum[oh];
    const float inv = l > 0.f ? 1.f / l : 0.f;
    __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(out) + ((int64_t)r * H + h) * D_V;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int col = oc + 16 * i;
      if (col < D_V) o[col] = __float2bfloat16_rn(acc[i] * inv);
    }
    if (lse && oc == 0) lse[(int64_t)r * H + h] = l > 0.f ? mrow[oh] + logf(l) : -INFINITY;
  }
}

template <int VPT>
dsa_status_t launch_v(const Rows& R, int32_t row0, int32_t nrows, const uint16_t* q,
                      const void* kv, const float* kv_scale, const int32_t* idx, int k, int H,
                      int D_K, int D_V, float sm_scale, uint16_t* out, float* lse,
                      cudaStream_t st) {
  size_t smem = sizeof(float) * ((size_t)kHG * D_K + (size_t)kChunk * (D_K + 1) +
                                 kHG * kChunk + 3 * kHG) +
                sizeof(int) * kChunk;
  auto kfn = kv_scale ? attn_simt_kernel<VPT, true> : attn_simt_kernel<VPT, false>;
  if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return DSA_ERR_CUDA;
  dim3 grid(nrows, (H + kHG - 1) / kHG);
  kfn<<<grid, kThreads, smem, st>>>(R, row0, q, kv, kv_scale, idx, k, H, D_K, D_V, sm_scale, out,
                                    lse);
  return launch_status();
}

}  // namespace

dsa_status_t launch_attn_simt(const Rows& R, int32_t row0, int32_t nrows, const uint16_t* q,
                              const void* kv, const float* kv_scale, const int32_t* idx, int k,
                              int H, int D_K, int D_V, float sm_scale, uint16_t* out, float* lse,
                              cudaStream_t st) {
  if (nrows <= 0) return DSA_OK;
  if (kv_scale && D_K % 16) return DSA_ERR_UNSUPPORTED;  // 16-byte vectors of e4m3 codes
  const int vpt = (D_V + 15) / 16;
#define DSA_LAUNCH_V(n) \
  launch_v<n>(R, row0, nrows, q, kv, kv_scale, idx, k, H, D_K, D_V, sm_scale, out, lse, st)
  if (vpt <= 4) return DSA_LAUNCH_V(4);
  if (vpt <= 8) return DSA_LAUNCH_V(8);
  if (vpt <= 16) return DSA_LAUNCH_V(16);
  if (vpt <= 32) return DSA_LAUNCH_V(32);
  if (vpt <= 64) return DSA_LAUNCH_V(64);
#undef DSA_LAUNCH_V
  return DSA_ERR_UNSUPPORTED;
}

}  // namespace dsa
