// Positions (P0), MRoPE cos/sin table (P1), RMSNorm row statistic (P2/P7),
// final RMSNorm (P10), DeepStack row map, weight packing, the device error
// record and the wait-timeout self-test.
//
// Memory-bound kernels read and write with 128-bit vectors, one warp per
// row, and reduce with warp shuffles.
#include <mutex>

#include "q3vl_device.cuh"
#include "q3vl_internal.h"

namespace q3vl {

// Per-device error record [code, where]; see q3vl_device_status().
__device__ int32_t g_error_record[2];

int32_t* device_error_ptr() {
  static std::mutex mu;
  static int32_t* cache[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (cache[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_error_record) != cudaSuccess) return nullptr;
    cache[dev] = static_cast<int32_t*>(p);
  }
  return cache[dev];
}

// ---------------------------------------------------------------------------
// P0: positions. inferencelayer vision.rs `mrope_positions` (token form) and
// cortiq qwen3te.rs `Qwen3Encoder::mrope_positions` (span form).
//
// One block walks the prompt in chunks. With c(i) = number of image tokens
// before token i, a text token's counter is (i - c) plus the advances of
// the grids completed before it; image token i belongs to grid g with
// gstart[g] <= c < gstart[g+1] and sits at k = c - gstart[g] in it, i.e. at
// frame k / (rows cols), row (k mod rows cols) / cols, column k mod cols.
// ---------------------------------------------------------------------------
constexpr int kMaxGrids = 4096;
constexpr int kPosThreads = 1024;
constexpr int kPosItems = 4;

__device__ __forceinline__ void pos_fail(int32_t* info, int32_t code) {
  atomicCAS(info, 0, code);
}

__global__ void __launch_bounds__(kPosThreads)
positions_kernel(const uint8_t* __restrict__ tt, int64_t S, const int32_t* __restrict__ grids,
                 int n_grids, int32_t* __restrict__ pos, int32_t* __restrict__ info) {
  __shared__ int32_t gstart[kMaxGrids + 1];  // image-token index where grid g starts
  __shared__ int32_t gadv[kMaxGrids + 1];    // counter advance of grids before g
  __shared__ int32_t warp_tot[32];
  __shared__ int32_t s_carry;
  __shared__ int32_t s_max[32];
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  griddep_wait();
  griddep_launch_dependents();

  if (tid == 0) {
    info[0] = 0;
    s_carry = 0;
  }
  __syncthreads();  // the status word is cleared before any check can fail
  for (int g = tid; g < n_grids; g += kPosThreads) {
    const int t = grids[3 * g], r = grids[3 * g + 1], c = grids[3 * g + 2];
    const bool ok = t >= 1 && r >= 1 && c >= 1 && int64_t(t) * r * c <= S;
    if (!ok) pos_fail(info, Q3VL_EGRID);
    gstart[g + 1] = ok ? t * r * c : 0;  // t frames of r x c tokens
    gadv[g + 1] = ok ? max(r, c) : 0;    // the counter moves by the longer side only
  }
  __syncthreads();
  if (tid == 0) {
    gstart[0] = 0;
    gadv[0] = 0;
    int64_t a = 0, b = 0;
    for (int g = 1; g <= n_grids; ++g) {
      a += gstart[g];
      b += gadv[g];
      if (a > S) a = S + 1;  // more image tokens than the prompt holds: flagged below
      gstart[g] = static_cast<int32_t>(a);
      gadv[g] = static_cast<int32_t>(b > S ? S : b);
    }
  }
  __syncthreads();
  const int32_t total_img = gstart[n_grids];
  int32_t my_max = -1;

  for (int64_t base = 0; base < S; base += int64_t(kPosThreads) * kPosItems) {
    uint8_t t[kPosItems];
    int cnt = 0;
#pragma unroll
    for (int u = 0; u < kPosItems; ++u) {
      const int64_t i = base + int64_t(tid) * kPosItems + u;
      t[u] = i < S ? tt[i] : 0;
      cnt += (t[u] != 0);
    }
    // block exclusive scan of cnt
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) warp_tot[wid] = incl;
    __syncthreads();
    if (wid == 0) {
      int w = warp_tot[lane];
      int wi = w;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o) wi += v;
      }
      warp_tot[lane] = wi - w;  // exclusive prefix of warp totals
    }
    __syncthreads();
    int32_t c = s_carry + warp_tot[wid] + (incl - cnt);
#pragma unroll
    for (int u = 0; u < kPosItems; ++u) {
      const int64_t i = base + int64_t(tid) * kPosItems + u;
      if (i >= S) break;
      int32_t p0, p1, p2;
      if (t[u] == 0) {
        // grids completed before i: count of g with gstart[g+1] <= c
        int lo = 0, hi = n_grids;
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          if (gstart[mid + 1] <= c) lo = mid + 1; else hi = mid;
        }
        p0 = p1 = p2 = static_cast<int32_t>(i - c) + gadv[lo];
        my_max = max(my_max, p0);
      } else if (t[u] != 1 || c >= total_img) {
        pos_fail(info, Q3VL_EGRID);
        p0 = p1 = p2 = 0;
        ++c;
      } else {
        // grid g: largest g with gstart[g] <= c
        int lo = 0, hi = n_grids - 1;
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (gstart[mid] <= c) lo = mid; else hi = mid - 1;
        }
        const int g = lo;
        const int32_t k = c - gstart[g];
        if (k > 0 && tt[i - 1] != 1) pos_fail(info, Q3VL_EGRID);  // run broken by text
        const int32_t rows = max(grids[3 * g + 1], 1), cols = max(grids[3 * g + 2], 1);
        const int32_t frame = k / (rows * cols), rem = k % (rows * cols);
        const int32_t b = static_cast<int32_t>(i - k) - gstart[g] + gadv[g];
        p0 = b + frame;
        p1 = b + rem / cols;
        p2 = b + rem % cols;
        my_max = max(my_max, max(p0, max(p1, p2)));
        ++c;
      }
      pos[i] = p0;
      pos[S + i] = p1;
      pos[2 * S + i] = p2;
    }
    __syncthreads();
    if (tid == kPosThreads - 1) s_carry = c;
    __syncthreads();
  }
  const int32_t m = __reduce_max_sync(0xffffffffu, my_max);
  if (lane == 0) s_max[wid] = m;
  __syncthreads();
  if (tid == 0) {
    int32_t mm = -1;
    for (int w = 0; w < kPosThreads / 32; ++w) mm = max(mm, s_max[w]);
    if (s_carry != total_img) pos_fail(info, Q3VL_EGRID);  // grids left over / run cut short
    info[1] = mm + 1;
  }
}

cudaError_t launch_positions(const uint8_t* tt, int64_t S, const int32_t* grids, int n_grids,
                             int32_t* pos, int32_t* info, cudaStream_t st) {
  const cudaError_t e =
      launch_pdl_plain(positions_kernel, dim3(1), dim3(kPosThreads), 0, st, tt, S, grids, n_grids,
                       pos, info);
  if (e != cudaSuccess) return e;
  return counted_launch(1);
}

// ---------------------------------------------------------------------------
// P1: cos/sin table. cortiq qwen3te.rs `Qwen3Encoder::norm_rope`: slot i
// rotates by pos[axis(i)] * theta^(-2i/hd); the angle is formed in fp64.
// ---------------------------------------------------------------------------
__global__ void rope_table_kernel(const int32_t* __restrict__ pos, int64_t S, double theta,
                                  int sec_h, int sec_w, float2* __restrict__ cs) {
  __shared__ double freq[kHalf];
  if (threadIdx.x < kHalf) freq[threadIdx.x] = pow(theta, -2.0 * threadIdx.x / kHeadDim);
  __syncthreads();
  const int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= S * kHalf) return;
  const int64_t p = idx / kHalf;
  const int i = static_cast<int>(idx % kHalf);
  int axis = 0;
  if (i % 3 == 1 && i < 3 * sec_h) axis = 1;
  else if (i % 3 == 2 && i < 3 * sec_w) axis = 2;
  const double ang = static_cast<double>(pos[axis * S + p]) * freq[i];
  double s, c;
  sincos(ang, &s, &c);
  cs[idx] = make_float2(static_cast<float>(c), static_cast<float>(s));
}

cudaError_t launch_rope_table(const q3vl_config& c, const int32_t* pos, int64_t S, float* cs,
                              cudaStream_t st) {
  const int64_t n = S * kHalf;
  const int th = 256;
  rope_table_kernel<<<static_cast<unsigned>((n + th - 1) / th), th, 0, st>>>(
      pos, S, c.rope_theta, c.mrope_section[1], c.mrope_section[2],
      reinterpret_cast<float2*>(cs));
  return counted_launch(1);
}

// ---------------------------------------------------------------------------
// P2/P7: inv_rms[r] = 1 / sqrt(mean(x_r^2) + eps), cortiq qwen3te.rs
// `rms_norm_into`. One warp per row, 16-byte loads.
// ---------------------------------------------------------------------------
template <typename T>
__device__ __forceinline__ float sumsq16(const uint4& v);

template <>
__device__ __forceinline__ float sumsq16<float>(const uint4& v) {
  const float a = __uint_as_float(v.x), b = __uint_as_float(v.y), c = __uint_as_float(v.z),
              d = __uint_as_float(v.w);
  return a * a + b * b + c * c + d * d;
}

template <>
__device__ __forceinline__ float sumsq16<__nv_bfloat16>(const uint4& v) {
  float s = 0.f;
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 f = unpack_bf16x2(w[j]);
    s += f.x * f.x + f.y * f.y;
  }
  return s;
}

// Sum of squares of one row, read by a warp in batches of 16 16-byte vectors
// per lane, all requested before any is used so the loads overlap.
template <typename T>
__device__ __forceinline__ float row_sumsq(const uint4* __restrict__ p, int64_t nvec, int lane) {
  constexpr int kBatch = 16;
  float s = 0.f;
  for (int64_t base = 0; base < nvec; base += 32 * kBatch) {
    uint4 v[kBatch];
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int64_t i = base + b * 32 + lane;
      v[b] = i < nvec ? __ldg(p + i) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int b = 0; b < kBatch; ++b) s += sumsq16<T>(v[b]);
  }
  return warp_sum(s);
}

template <typename T>
__global__ void rowstat_kernel(const T* __restrict__ x, int64_t S, int64_t width, float eps,
                               float* __restrict__ inv) {
  const int64_t row = int64_t(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= S) return;
  const float s = row_sumsq<T>(reinterpret_cast<const uint4*>(x + row * width),
                               width * int64_t(sizeof(T)) / 16, lane);
  if (lane == 0) inv[row] = 1.0f / sqrtf(s / static_cast<float>(width) + eps);
}

cudaError_t launch_rowstat(const q3vl_config& c, const void* x, int64_t S, int64_t width,
                           float* inv, cudaStream_t st) {
  const int warps = 8;
  const unsigned blocks = static_cast<unsigned>((S + warps - 1) / warps);
  if (c.dtype == Q3VL_DTYPE_BF16)
    rowstat_kernel<__nv_bfloat16><<<blocks, warps * 32, 0, st>>>(
        static_cast<const __nv_bfloat16*>(x), S, width, static_cast<float>(c.rms_eps), inv);
  else
    rowstat_kernel<float><<<blocks, warps * 32, 0, st>>>(static_cast<const float*>(x), S, width,
                                                         static_cast<float>(c.rms_eps), inv);
  return counted_launch(1);
}

// ---------------------------------------------------------------------------
// The cos/sin table in the slot-major layout the bf16 QKV epilogue reads:
// float4 number t * S + p holds (cos, sin) of slots 2t and 2t + 1 at
// position p, so the 32 threads of a warp (32 consecutive rows) read 512
// contiguous bytes per slot pair. From the position-major [S][64][2] table.
// ---------------------------------------------------------------------------
__global__ void rope_slot_major_kernel(const float4* __restrict__ cs, int64_t S,
                                       float4* __restrict__ out) {
  const int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= S * (kHalf / 2)) return;
  const int64_t t = idx / S, pp = idx % S;
  out[t * S + pp] = cs[pp * (kHalf / 2) + t];
}

cudaError_t launch_rope_slot_major(const float* cs, int64_t S, float* out, cudaStream_t st) {
  const int64_t n = S * (kHalf / 2);
  rope_slot_major_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(
      reinterpret_cast<const float4*>(cs), S, reinterpret_cast<float4*>(out));
  return counted_launch(1);
}

// ---------------------------------------------------------------------------
// The bf16 layer's prologue in one launch: P2 (the input row statistic, a
// warp per row) in the first blocks, P1 (the cos/sin table, written
// slot-major as above) in the last table_blocks blocks, and the stream-K
// flags of the GEMMs set to zero by the first table block. Launched as a programmatic dependent: it waits for the previous
// kernel in the stream (the positions, or the previous layer) before reading
// pos or x, and lets the QKV GEMM start its prologue early.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
layer_prologue_kernel(const int32_t* __restrict__ pos, int64_t S, double theta, int sec_h,
                      int sec_w, float2* __restrict__ cs, int table_blocks,
                      const __nv_bfloat16* __restrict__ x, int64_t width, float eps,
                      float* __restrict__ inv, int32_t* __restrict__ flags, int n_flags) {
  griddep_wait();
  griddep_launch_dependents();
  // the row-statistic blocks come first, so the 21 MB pass over x starts at
  // once on every SM and the table blocks fill in behind it
  const int stat_blocks = static_cast<int>(gridDim.x) - table_blocks;
  if (static_cast<int>(blockIdx.x) >= stat_blocks) {
    const int tb = static_cast<int>(blockIdx.x) - stat_blocks;
    __shared__ double freq[kHalf];
    if (threadIdx.x < kHalf) freq[threadIdx.x] = pow(theta, -2.0 * threadIdx.x / kHeadDim);
    if (tb == 0)
      for (int i = threadIdx.x; i < n_flags; i += blockDim.x) flags[i] = 0;
    __syncthreads();
    // slot-major: consecutive threads take consecutive positions of one slot
    const int64_t idx = int64_t(tb) * blockDim.x + threadIdx.x;
    if (idx >= S * kHalf) return;
    const int i = static_cast<int>(idx / S);
    const int64_t pp = idx % S;
    int axis = 0;
    if (i % 3 == 1 && i < 3 * sec_h) axis = 1;
    else if (i % 3 == 2 && i < 3 * sec_w) axis = 2;
    const double ang = static_cast<double>(pos[axis * S + pp]) * freq[i];
    double sn, c;
    sincos(ang, &sn, &c);
    cs[(int64_t(i >> 1) * S + pp) * 2 + (i & 1)] =
        make_float2(static_cast<float>(c), static_cast<float>(sn));
    return;
  }
  if (x == nullptr) return;
  const int64_t row = int64_t(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= S) return;
  const float sq = row_sumsq<__nv_bfloat16>(reinterpret_cast<const uint4*>(x + row * width),
                                            width * 2 / 16, lane);
  if (lane == 0) inv[row] = 1.0f / sqrtf(sq / static_cast<float>(width) + eps);
}

cudaError_t launch_layer_prologue(const q3vl_config& c, const int32_t* pos, int64_t S, float* cs,
                                  const void* x, float* inv, int32_t* flags, int n_flags,
                                  cudaStream_t st) {
  const int th = 256;
  const int table_blocks = static_cast<int>((S * kHalf + th - 1) / th);
  const int rows_per_block = th / 32;
  const int stat_blocks = x != nullptr ? static_cast<int>((S + rows_per_block - 1) / rows_per_block)
                                       : 0;
  const cudaError_t e = launch_pdl_plain(
      layer_prologue_kernel, dim3(table_blocks + stat_blocks), dim3(th), 0, st, pos, S,
      c.rope_theta, c.mrope_section[1], c.mrope_section[2], reinterpret_cast<float2*>(cs),
      table_blocks, static_cast<const __nv_bfloat16*>(x), static_cast<int64_t>(c.hidden),
      static_cast<float>(c.rms_eps), inv, flags, n_flags);
  if (e != cudaSuccess) return e;
  return counted_launch(1);
}

// ---------------------------------------------------------------------------
// P10: x <- x * inv_rms(x) * g in place.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint4 scale16(const uint4& v, float inv, const uint4& g, float) {
  uint4 o;
  o.x = __float_as_uint(__uint_as_float(v.x) * inv * __uint_as_float(g.x));
  o.y = __float_as_uint(__uint_as_float(v.y) * inv * __uint_as_float(g.y));
  o.z = __float_as_uint(__uint_as_float(v.z) * inv * __uint_as_float(g.z));
  o.w = __float_as_uint(__uint_as_float(v.w) * inv * __uint_as_float(g.w));
  return o;
}

__device__ __forceinline__ uint4 scale16(const uint4& v, float inv, const uint4& g,
                                         __nv_bfloat16) {
  const uint32_t a[4] = {v.x, v.y, v.z, v.w}, b[4] = {g.x, g.y, g.z, g.w};
  uint32_t o[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 f = unpack_bf16x2(a[j]), w = unpack_bf16x2(b[j]);
    o[j] = pack_bf16x2(f.x * inv * w.x, f.y * inv * w.y);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

template <typename T>
__global__ void final_norm_kernel(T* __restrict__ x, int64_t S, int64_t width, float eps,
                                  const T* __restrict__ gain) {
  const int64_t row = int64_t(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= S) return;
  uint4* p = reinterpret_cast<uint4*>(x + row * width);
  const uint4* g = reinterpret_cast<const uint4*>(gain);
  const int64_t nvec = width * sizeof(T) / 16;
  const float s = row_sumsq<T>(p, nvec, lane);
  const float inv = 1.0f / sqrtf(s / static_cast<float>(width) + eps);
#pragma unroll 4
  for (int64_t v = lane; v < nvec; v += 32) p[v] = scale16(p[v], inv, __ldg(g + v), T());
}

cudaError_t launch_final_norm(const q3vl_config& c, void* x, int64_t S, const void* gain,
                              cudaStream_t st) {
  const int warps = 8;
  const unsigned blocks = static_cast<unsigned>((S + warps - 1) / warps);
  const float eps = static_cast<float>(c.rms_eps);
  if (c.dtype == Q3VL_DTYPE_BF16)
    final_norm_kernel<__nv_bfloat16><<<blocks, warps * 32, 0, st>>>(
        static_cast<__nv_bfloat16*>(x), S, c.hidden, eps,
        static_cast<const __nv_bfloat16*>(gain));
  else
    final_norm_kernel<float><<<blocks, warps * 32, 0, st>>>(static_cast<float*>(x), S, c.hidden,
                                                            eps, static_cast<const float*>(gain));
  return counted_launch(1);
}

// ---------------------------------------------------------------------------
// DeepStack row map: map[r] = k for r = rows[k], else -1 (hf2q
// qwen3vl_text/forward.rs: positions must be inside the sequence).
// ---------------------------------------------------------------------------
__global__ void fill_i32_kernel(int32_t* p, int64_t n, int32_t v) {
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < n) p[i] = v;
}

__global__ void deepstack_map_kernel(const int32_t* __restrict__ rows, int n_img, int64_t S,
                                     int32_t* __restrict__ map, int32_t* err) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= n_img) return;
  const int32_t r = rows[k];
  if (r < 0 || r >= S) {
    record_error(err, Q3VL_ERANGE, kWhereDeepstackMap);
    return;
  }
  if (atomicCAS(map + r, -1, k) != -1) record_error(err, Q3VL_ERANGE, kWhereDeepstackMap);
}

cudaError_t launch_deepstack_map(const int32_t* rows, int n_img, int64_t S, int32_t* map,
                                 cudaStream_t st) {
  fill_i32_kernel<<<static_cast<unsigned>((S + 255) / 256), 256, 0, st>>>(map, S, -1);
  if (n_img > 0)
    deepstack_map_kernel<<<(n_img + 255) / 256, 256, 0, st>>>(rows, n_img, S, map,
                                                               device_error_ptr());
  return counted_launch(1 + (n_img > 0 ? 1 : 0));
}

// ---------------------------------------------------------------------------
// Token embedding gather with the soft-token splice (hf2q
// qwen3vl_text/forward.rs, `forward_text_prefill_logits_last` step 1):
// x[p] = table[tokens[p]], except rows with map[p] = k >= 0, which take
// soft[k]. One warp per row, 16-byte copies. A token id outside the table
// records Q3VL_ERANGE and leaves the row zero.
// ---------------------------------------------------------------------------
__global__ void embed_kernel(const uint4* __restrict__ table, int64_t vocab,
                             const int32_t* __restrict__ tokens, int64_t S,
                             const uint4* __restrict__ soft, const int32_t* __restrict__ map,
                             int64_t row_vecs, uint4* __restrict__ x, int32_t* err) {
  const int64_t row = int64_t(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= S) return;
  const uint4* src = nullptr;
  const int32_t k = map != nullptr ? map[row] : -1;
  if (k >= 0) {
    src = soft + int64_t(k) * row_vecs;
  } else {
    const int32_t tok = tokens[row];
    if (tok >= 0 && tok < vocab) src = table + int64_t(tok) * row_vecs;
    else if (lane == 0) record_error(err, Q3VL_ERANGE, kWhereEmbed);
  }
  uint4* dst = x + row * row_vecs;
  for (int64_t v = lane; v < row_vecs; v += 32)
    dst[v] = src != nullptr ? __ldg(src + v) : make_uint4(0, 0, 0, 0);
}

cudaError_t launch_embed(const q3vl_config& c, const void* table, int64_t vocab,
                         const int32_t* tokens, int64_t S, const void* soft, const int32_t* map,
                         void* x, cudaStream_t st) {
  const int64_t row_vecs = int64_t(c.hidden) * int64_t(elem_bytes(c)) / 16;
  const int warps = 8;
  embed_kernel<<<static_cast<unsigned>((S + warps - 1) / warps), warps * 32, 0, st>>>(
      static_cast<const uint4*>(table), vocab, tokens, S, static_cast<const uint4*>(soft), map,
      row_vecs, static_cast<uint4*>(x), device_error_ptr());
  return counted_launch(1);
}

// ---------------------------------------------------------------------------
// Weight packing (one-time).
// ---------------------------------------------------------------------------
enum PackMode : int { kConcat3 = 0, kInterleaveGU = 1, kCopy = 2 };

template <typename T>
__device__ __forceinline__ float ld_f(const T* p, int64_t i) {
  return static_cast<float>(p[i]);
}
template <>
__device__ __forceinline__ float ld_f<__nv_bfloat16>(const __nv_bfloat16* p, int64_t i) {
  return __bfloat162float(p[i]);
}
__device__ __forceinline__ void st_f(float* p, int64_t i, float v) { p[i] = v; }
__device__ __forceinline__ void st_f(__nv_bfloat16* p, int64_t i, float v) {
  p[i] = __float2bfloat16_rn(v);
}

template <typename T>
__global__ void pack_rows_kernel(T* __restrict__ out, int64_t rows, int64_t cols, int mode,
                                 const T* s0, const T* s1, const T* s2, int64_t r0, int64_t r1,
                                 const T* gain) {
  const int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= rows * cols) return;
  const int64_t n = idx / cols, k = idx % cols;
  const T* src;
  int64_t sr;
  if (mode == kConcat3) {
    if (n < r0) { src = s0; sr = n; }
    else if (n < r0 + r1) { src = s1; sr = n - r0; }
    else { src = s2; sr = n - r0 - r1; }
  } else if (mode == kInterleaveGU) {
    const int64_t blk = n / 256, r = n % 256;
    src = r < 128 ? s0 : s1;
    sr = blk * 128 + (r < 128 ? r : r - 128);
  } else {
    src = s0;
    sr = n;
  }
  float v = ld_f(src, sr * cols + k);
  if (gain != nullptr) v *= ld_f(gain, k);
  st_f(out, idx, v);
}

template <typename T>
__global__ void to_f32_concat_kernel(float* __restrict__ out, const T* a, int64_t na, const T* b,
                                     int64_t nb, const T* c, int64_t nc) {
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < na) out[i] = ld_f(a, i);
  else if (i < na + nb) out[i] = ld_f(b, i - na);
  else if (i < na + nb + nc) out[i] = ld_f(c, i - na - nb);
}

template <typename T>
static cudaError_t pack_typed(const q3vl_config& c, const q3vl_raw_weights& w, char* base,
                              cudaStream_t st) {
  const PackLayout L = pack_layout(c);
  const int64_t H = c.hidden, Dq = q_dim(c), Dkv = kv_dim(c), I = c.intermediate;
  auto T_ = [](const void* p) { return static_cast<const T*>(p); };
  auto grid = [](int64_t n) { return static_cast<unsigned>((n + 255) / 256); };
  const int64_t Nt = Dq + 2 * Dkv;
  pack_rows_kernel<T><<<grid(Nt * H), 256, 0, st>>>(reinterpret_cast<T*>(base + L.w_qkv), Nt, H,
                                                    kConcat3, T_(w.wq), T_(w.wk), T_(w.wv), Dq,
                                                    Dkv, T_(w.attn_norm));
  if (c.has_qkv_bias)
    to_f32_concat_kernel<T><<<grid(Nt), 256, 0, st>>>(reinterpret_cast<float*>(base + L.b_qkv),
                                                      T_(w.bq), Dq, T_(w.bk), Dkv, T_(w.bv), Dkv);
  to_f32_concat_kernel<T><<<1, 256, 0, st>>>(reinterpret_cast<float*>(base + L.q_norm),
                                             T_(w.q_norm), kHeadDim, nullptr, 0, nullptr, 0);
  to_f32_concat_kernel<T><<<1, 256, 0, st>>>(reinterpret_cast<float*>(base + L.k_norm),
                                             T_(w.k_norm), kHeadDim, nullptr, 0, nullptr, 0);
  pack_rows_kernel<T><<<grid(H * Dq), 256, 0, st>>>(reinterpret_cast<T*>(base + L.w_o), H, Dq,
                                                    kCopy, T_(w.wo), nullptr, nullptr, 0, 0,
                                                    nullptr);
  pack_rows_kernel<T><<<grid(2 * I * H), 256, 0, st>>>(reinterpret_cast<T*>(base + L.w_gu),
                                                       2 * I, H, kInterleaveGU, T_(w.wg),
                                                       T_(w.wu), nullptr, 0, 0,
                                                       T_(w.ffn_norm));
  pack_rows_kernel<T><<<grid(H * I), 256, 0, st>>>(reinterpret_cast<T*>(base + L.w_down), H, I,
                                                   kCopy, T_(w.wd), nullptr, nullptr, 0, 0,
                                                   nullptr);
  return counted_launch((c.has_qkv_bias ? 7 : 6));
}

cudaError_t launch_pack(const q3vl_config& c, const q3vl_raw_weights& raw, void* packed,
                        cudaStream_t st) {
  char* base = static_cast<char*>(packed);
  if (c.dtype == Q3VL_DTYPE_BF16) return pack_typed<__nv_bfloat16>(c, raw, base, st);
  return pack_typed<float>(c, raw, base, st);
}

// ---------------------------------------------------------------------------
// Self-test of the bounded wait: an mbarrier nothing arrives at.
// ---------------------------------------------------------------------------
__global__ void selftest_timeout_kernel(uint64_t limit_ns, int32_t* err) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_mbar_init();
  mbar_wait(&bar, 0, err, kWhereSelftest, nullptr, limit_ns);
}

cudaError_t launch_selftest_timeout(uint32_t timeout_us, cudaStream_t st) {
  selftest_timeout_kernel<<<1, 32, 0, st>>>(uint64_t(timeout_us) * 1000ull, device_error_ptr());
  return counted_launch(1);
}

}  // namespace q3vl
