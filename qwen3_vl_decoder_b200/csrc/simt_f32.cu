// fp32 path of the layer on CUDA cores (FFMA, no TF32): the same steps as
// the bf16 tensor-core path, for workloads that keep every value in fp32.
// TF32 is excluded on purpose: its 10-bit mantissa moves the residual far
// beyond a 1e-5 relative tolerance.
#include "q3vl_device.cuh"
#include "q3vl_internal.h"

namespace q3vl {
namespace {

constexpr int TM = 64, TN = 64, TK = 16;

// C[M, N] = A[M, K] B[N, K]^T, then per element:
// v = acc * row_scale[r] + bias[c] + resid[r, c] + ds_slab[ds_map[r], c].
__global__ void __launch_bounds__(256)
gemm_f32_kernel(const float* __restrict__ A, const float* __restrict__ B, int64_t M, int64_t N,
                int64_t K, float* __restrict__ out, int64_t ldo, const float* __restrict__ row_scale,
                const float* __restrict__ bias, const float* __restrict__ resid,
                const float* __restrict__ ds_slab, const int32_t* __restrict__ ds_map) {
  __shared__ float As[TK][TM + 4];
  __shared__ float Bs[TK][TN + 4];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const int64_t m0 = int64_t(blockIdx.y) * TM, n0 = int64_t(blockIdx.x) * TN;
  float acc[4][4] = {};
  for (int64_t k0 = 0; k0 < K; k0 += TK) {
    for (int e = threadIdx.x; e < TM * TK; e += 256) {
      const int mm = e / TK, kk = e % TK;
      const int64_t gm = m0 + mm, gk = k0 + kk;
      As[kk][mm] = (gm < M && gk < K) ? A[gm * K + gk] : 0.f;
      const int64_t gn = n0 + mm;
      Bs[kk][mm] = (gn < N && gk < K) ? B[gn * K + gk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { a[i] = As[kk][ty * 4 + i]; b[i] = Bs[kk][tx * 4 + i]; }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t r = m0 + ty * 4 + i;
    if (r >= M) continue;
    const float s = row_scale ? row_scale[r] : 1.f;
    const int32_t dk = ds_map ? ds_map[r] : -1;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t c = n0 + tx * 4 + j;
      if (c >= N) continue;
      float v = acc[i][j] * s;
      if (bias) v += bias[c];
      if (resid) v += resid[r * ldo + c];
      if (dk >= 0 && ds_slab) v += ds_slab[int64_t(dk) * N + c];
      out[r * ldo + c] = v;
    }
  }
}

// Per-head RMSNorm then split-half MRoPE, in place, one warp per (row,
// head) over the q and k heads (cortiq qwen3te.rs `Qwen3Encoder::norm_rope`).
// Lane l holds columns l, l+32, l+64, l+96, so both rotation pairs
// (l, l+64) and (l+32, l+96) are in-thread.
__global__ void qk_norm_rope_f32_kernel(float* __restrict__ qkv, int64_t S, int64_t ld, int nh,
                                        int nkv, const float* __restrict__ qn,
                                        const float* __restrict__ kn,
                                        const float2* __restrict__ cs, float eps) {
  const int64_t w = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int heads = nh + nkv;
  if (w >= S * heads) return;
  const int64_t r = w / heads;
  const int hh = static_cast<int>(w % heads);
  float* x = qkv + r * ld + int64_t(hh) * kHeadDim;
  const float* gain = hh < nh ? qn : kn;
  float v[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) v[t] = x[lane + 32 * t];
  const float ss = warp_sum(v[0] * v[0] + v[1] * v[1] + v[2] * v[2] + v[3] * v[3]);
  const float rn = 1.0f / sqrtf(ss / kHeadDim + eps);
#pragma unroll
  for (int t = 0; t < 4; ++t) v[t] = v[t] * rn * gain[lane + 32 * t];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const float2 c = cs[r * kHalf + lane + 32 * t];
    const float a = v[t], b = v[t + 2];
    v[t] = a * c.x - b * c.y;
    v[t + 2] = a * c.y + b * c.x;
  }
#pragma unroll
  for (int t = 0; t < 4; ++t) x[lane + 32 * t] = v[t];
}

// act[r, c] = silu(s_r * (A W_gu^T)[r, g(c)]) * (s_r * (A W_gu^T)[r, g(c) + 128]),
// g(c) = (c / 128) * 256 + c % 128: gate and up accumulate side by side in
// one CTA, so no [S, 2I] intermediate is stored.
__global__ void __launch_bounds__(256)
gemm_swiglu_f32_kernel(const float* __restrict__ A, const float* __restrict__ B, int64_t M,
                       int64_t I, int64_t K, const float* __restrict__ row_scale,
                       float* __restrict__ act) {
  __shared__ float As[TK][TM + 4];
  __shared__ float Gs[TK][TN + 4];
  __shared__ float Us[TK][TN + 4];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const int64_t m0 = int64_t(blockIdx.y) * TM, c0 = int64_t(blockIdx.x) * TN;  // act columns
  float ag[4][4] = {}, au[4][4] = {};
  for (int64_t k0 = 0; k0 < K; k0 += TK) {
    for (int e = threadIdx.x; e < TM * TK; e += 256) {
      const int mm = e / TK, kk = e % TK;
      const int64_t gm = m0 + mm, gk = k0 + kk;
      As[kk][mm] = (gm < M && gk < K) ? A[gm * K + gk] : 0.f;
      const int64_t c = c0 + mm;
      const int64_t gr = (c / 128) * 256 + c % 128;
      const bool okc = c < I && gk < K;
      Gs[kk][mm] = okc ? B[gr * K + gk] : 0.f;
      Us[kk][mm] = okc ? B[(gr + 128) * K + gk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float a[4], g[4], u[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = As[kk][ty * 4 + i]; g[i] = Gs[kk][tx * 4 + i]; u[i] = Us[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          ag[i][j] = fmaf(a[i], g[j], ag[i][j]);
          au[i][j] = fmaf(a[i], u[j], au[i][j]);
        }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t r = m0 + ty * 4 + i;
    if (r >= M) continue;
    const float s = row_scale[r];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t c = c0 + tx * 4 + j;
      if (c < I) act[r * I + c] = silu_f(ag[i][j] * s) * (au[i][j] * s);
    }
  }
}

// Causal GQA attention, one warp per (query row, head), online softmax in
// fp32; lane l holds dims l, l+32, l+64, l+96.
__global__ void attention_f32_kernel(const float* __restrict__ qkv, int64_t S, int64_t ld,
                                     int nh, int nkv, float* __restrict__ o, int64_t ldo) {
  const int64_t w = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= S * nh) return;
  const int64_t p = w / nh;
  const int h = static_cast<int>(w % nh);
  const int g = h / (nh / nkv);
  const float* q = qkv + p * ld + int64_t(h) * kHeadDim;
  const int64_t kc = int64_t(nh) * kHeadDim + int64_t(g) * kHeadDim;
  const int64_t vc = int64_t(nh + nkv) * kHeadDim + int64_t(g) * kHeadDim;
  const float scale = 1.0f / sqrtf(static_cast<float>(kHeadDim));
  float qv[4], acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int t = 0; t < 4; ++t) qv[t] = q[lane + 32 * t];
  float m = -INFINITY, l = 0.f;
  for (int64_t j = 0; j <= p; ++j) {
    const float* k = qkv + j * ld + kc;
    const float* v = qkv + j * ld + vc;
    float d = 0.f;
#pragma unroll
    for (int t = 0; t < 4; ++t) d = fmaf(qv[t], k[lane + 32 * t], d);
    const float s = warp_sum(d) * scale;
    const float m_new = fmaxf(m, s);
    const float alpha = expf(m - m_new), e = expf(s - m_new);
    l = l * alpha + e;
#pragma unroll
    for (int t = 0; t < 4; ++t) acc[t] = acc[t] * alpha + e * v[lane + 32 * t];
    m = m_new;
  }
  float* dst = o + p * ldo + int64_t(h) * kHeadDim;
#pragma unroll
  for (int t = 0; t < 4; ++t) dst[lane + 32 * t] = acc[t] / l;
}

}  // namespace

cudaError_t launch_gemm_f32(Epi epi, const GemmArgs& a, cudaStream_t st) {
  (void)epi;
  dim3 grid(static_cast<unsigned>((a.N + TN - 1) / TN), static_cast<unsigned>((a.M + TM - 1) / TM));
  gemm_f32_kernel<<<grid, 256, 0, st>>>(
      static_cast<const float*>(a.A), static_cast<const float*>(a.B), a.M, a.N, a.K,
      static_cast<float*>(a.out), a.ldo, a.row_scale, a.bias, static_cast<const float*>(a.resid),
      static_cast<const float*>(a.ds_slab), a.ds_map);
  return counted_launch(1);
}

cudaError_t launch_qk_norm_rope_f32(const q3vl_config& c, float* qkv, int64_t S,
                                    const float* q_norm, const float* k_norm, const float* cs,
                                    cudaStream_t st) {
  const int64_t warps = S * (c.n_heads + c.n_kv_heads);
  qk_norm_rope_f32_kernel<<<static_cast<unsigned>((warps * 32 + 255) / 256), 256, 0, st>>>(
      qkv, S, qkv_dim(c), c.n_heads, c.n_kv_heads, q_norm, k_norm,
      reinterpret_cast<const float2*>(cs), static_cast<float>(c.rms_eps));
  return counted_launch(1);
}

cudaError_t launch_gemm_swiglu_f32(const float* A, const float* B, int64_t M, int64_t I, int64_t K,
                                   const float* row_scale, float* act, cudaStream_t st) {
  dim3 grid(static_cast<unsigned>((I + TN - 1) / TN), static_cast<unsigned>((M + TM - 1) / TM));
  gemm_swiglu_f32_kernel<<<grid, 256, 0, st>>>(A, B, M, I, K, row_scale, act);
  return counted_launch(1);
}

cudaError_t launch_attention_f32(const q3vl_config& c, const float* qkv, int64_t S, float* o,
                                 cudaStream_t st) {
  const int64_t warps = S * c.n_heads;
  attention_f32_kernel<<<static_cast<unsigned>((warps * 32 + 255) / 256), 256, 0, st>>>(
      qkv, S, qkv_dim(c), c.n_heads, c.n_kv_heads, o, q_dim(c));
  return counted_launch(1);
}

}  // namespace q3vl
