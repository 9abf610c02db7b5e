// Persistent tcgen05 GEMM for sm_100a on CTA pairs: C[M, N] = A[M, K] B[N, K]^T,
// bf16 inputs, fp32 accumulation in tensor memory, fused epilogues.
//
// A cluster of two CTAs computes one 256 x BN tile with tcgen05.mma
// cta_group::2: each CTA stages its own 128 rows of A and BN/2 rows of B per
// 64-wide k-block (TMA, 128-byte swizzle, no multicast), so each SM moves half
// the B operand a single-CTA 128 x BN tile would need. The even CTA issues the
// MMAs; its commits arrive on both CTAs' barriers.
//
// Roles per CTA (192 threads):
//   warp 0    one thread issues the TMA loads into a ring of stages; the
//             completion of both CTAs' loads is counted on the even CTA's
//             barrier;
//   warp 1    allocates TMEM (pair allocation); on the even CTA one thread
//             issues the MMAs into one of two TMEM accumulators;
//   warps 2-5 epilogue: thread = accumulator row of this CTA (tcgen05.ld
//             32x32b), apply the fused epilogue, write bf16 into a swizzled
//             shared-memory tile, TMA-store it. The residual tile is
//             TMA-loaded into the same buffer ahead of the accumulator.
// Two accumulators let the epilogue of tile i overlap the main loop of tile
// i + 1. Tiles are visited M-fastest so concurrently running pairs share the
// same weight (B) panels in L2.
//
// Epilogues (cortiq qwen3te.rs `Qwen3Encoder::encode_with_images` and
// `Qwen3Encoder::norm_rope`; hf2q qwen3vl_text/forward.rs module doc for
// the bias-before-norm order):
//   kQkv      v = inv_rms[r] * acc + b; q/k heads: per-head RMSNorm with the
//             q_norm / k_norm gain, then split-half MRoPE from the cos/sin
//             table (slot-major, so a warp's loads are contiguous); v heads:
//             v only.
//   kResidual out = resid + acc (+ DeepStack slab row ds_map[r]).
//   kSwiGLU   out = silu(s*g) * (s*u), s = inv_rms[r] (fast exp / divide); B's 256-row block
//             holds 128 gate rows then the 128 matching up rows.
//   kPlain    out = acc.
#include "q3vl_device.cuh"
#include "q3vl_internal.h"

namespace q3vl {
namespace {

constexpr int BM = 128;   // accumulator rows per CTA (256 per CTA pair)
constexpr int BK = 64;
constexpr int kThreads = 192;

template <int BN>
struct Cfg {
  static constexpr int kStages = BN == 256 ? 5 : 6;
  static constexpr int kABytes = BM * BK * 2;           // this CTA's 128 rows of A
  static constexpr int kBBytes = (BN / 2) * BK * 2;     // this CTA's BN/2 rows of B
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kOutBytes = BM * BN * 2;         // bf16 epilogue tile
  static constexpr int kTmemCols = 2 * BN;
  static constexpr size_t kSmem = 1024 + size_t(kStages) * kStageBytes + kOutBytes + 256;
};
static_assert(Cfg<256>::kSmem <= 232448, "shared memory budget");
static_assert(Cfg<128>::kSmem <= 232448, "shared memory budget");

struct Params {
  int64_t M, N, K;
  int64_t ldo;
  const float* row_scale;
  const float* bias;
  const float* q_norm;
  const float* k_norm;
  const float2* cos_sin;
  int64_t q_cols, k_cols;
  float eps;
  const __nv_bfloat16* ds_slab;
  const int32_t* ds_map;
  int32_t* err;
  // schedule over pair tiles (see WorkIter)
  int64_t dp_tiles, sk_units;
  int sk_pairs;   // pairs sk_first .. sk_first+sk_pairs-1 share the stream-K units
  int sk_first;
  int kb_per_tile;
  int m_fastest;  // tile order: 1 = M index fastest (A stays in L2), 0 = N fastest (B stays)
  // stream-K scratch: one fp32 128 x BN partial tile and one flag per CTA
  float* sk_partials;
  int32_t* sk_flags;
  int sk_slots;   // CTA slots of partials and flags (checked by debug builds)
  // row statistics between GEMMs (see GemmArgs)
  float* rowsq_out;
  const float* rowsq_in;
  int rowsq_n;
  float rowsq_width;
};

// Work schedule over 256 x BN pair tiles, shared by the roles of both CTAs of
// a pair. Each pair first works through its stream-K range, then its
// data-parallel tiles:
//   tiles [0, dp_tiles): data parallel; pair c takes tiles c, c + G, ... over
//     their whole K range;
//   tiles [dp_tiles, T): stream-K; their U = (T - dp_tiles) * KB k-block
//     units are cut into Gs = sk_pairs equal contiguous ranges, pair
//     sk_first + i (i < Gs) taking units [i U / Gs, (i + 1) U / Gs).
// A stream-K tile split across pairs is finished by the pair holding its
// first k-block, which reaches it last (at the end of its stream-K range).
// The pairs holding its later k-blocks reach them first (at the start of
// their ranges): each of their CTAs leaves its fp32 partial rows in its own
// scratch slot and raises its flag; the finisher adds the partials in pair
// order (deterministic) before the fused epilogue. Running the stream-K part
// first lets these longer epilogues overlap the data-parallel main loops.
enum Role : int { kFull = 0, kFinisher = 1, kContributor = 2 };

struct Work {
  int64_t tile;
  int kb0, kb1, role;
};

struct WorkIter {
  int64_t dp_t, dp_tiles, stride;
  int64_t u, u1, sk_base;
  int KB;
  __device__ WorkIter(const Params& p, int c, int G)
      : dp_t(c), dp_tiles(p.dp_tiles), stride(G),
        u(in_sk(p, c) ? p.sk_units * (c - p.sk_first) / p.sk_pairs : 0),
        u1(in_sk(p, c) ? p.sk_units * (c - p.sk_first + 1) / p.sk_pairs : 0), sk_base(p.dp_tiles),
        KB(p.kb_per_tile) {}
  __device__ static bool in_sk(const Params& p, int c) {
    return c >= p.sk_first && c < p.sk_first + p.sk_pairs;
  }
  __device__ bool next(Work& w) {
    if (u < u1) {
      const int64_t t = u / KB;
      const int64_t end = min(u1, (t + 1) * KB);
      w.tile = sk_base + t;
      w.kb0 = static_cast<int>(u - t * KB);
      w.kb1 = static_cast<int>(end - t * KB);
      w.role = w.kb0 > 0 ? kContributor : (w.kb1 == KB ? kFull : kFinisher);
      u = end;
      return true;
    }
    if (dp_t < dp_tiles) {
      w.tile = dp_t; w.kb0 = 0; w.kb1 = KB; w.role = kFull;
      dp_t += stride;
      return true;
    }
    return false;
  }
};

// Row-tile and column-tile index of pair tile t.
__device__ __forceinline__ void tile_mn(const Params& p, int64_t t, int64_t num_m, int64_t num_n,
                                        int64_t& m, int64_t& n) {
  if (p.m_fastest) { m = t % num_m; n = t / num_m; }
  else { n = t % num_n; m = t / num_n; }
}

// Owner pair of stream-K unit u: the largest c with c U / G <= u.
__device__ __forceinline__ int sk_owner(int64_t u, int64_t U, int G) {
  return static_cast<int>(((u + 1) * G - 1) / U);
}

__device__ __forceinline__ int ld_acquire(const int32_t* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release(int32_t* p, int v) {
  asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Named barrier over the four epilogue warps of this CTA.
__device__ __forceinline__ void epilogue_sync() { asm volatile("barrier.sync 1, 128;" ::: "memory"); }

// Byte offset, in the swizzled bf16 epilogue tile, of 16-byte unit u (8
// columns) of 32-column chunk cc of row r. The tile is BN/64 TMA boxes of
// 128 rows x 64 columns (16 KB each) with the 128-byte swizzle: unit k of a
// row sits at k ^ (r mod 8).
__device__ __forceinline__ uint32_t out_off(int r, int cc, int u) {
  return static_cast<uint32_t>((cc >> 1) * 16384 + r * 128 +
                               (((((cc & 1) << 2) + u) ^ (r & 7)) << 4));
}

__device__ __forceinline__ void stage_bf16x32(uint8_t* tile, int r, int cc, const float* v) {
#pragma unroll
  for (int u = 0; u < 4; ++u)
    *reinterpret_cast<uint4*>(tile + out_off(r, cc, u)) =
        make_uint4(pack_bf16x2(v[8 * u + 0], v[8 * u + 1]), pack_bf16x2(v[8 * u + 2], v[8 * u + 3]),
                   pack_bf16x2(v[8 * u + 4], v[8 * u + 5]), pack_bf16x2(v[8 * u + 6], v[8 * u + 7]));
}

// stage_bf16x32 that also returns the sum of squares of the rounded values.
__device__ __forceinline__ float stage_bf16x32_ss(uint8_t* tile, int r, int cc, const float* v) {
  float ss = 0.f;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    uint32_t w[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const __nv_bfloat162 b = __floats2bfloat162_rn(v[8 * u + 2 * t], v[8 * u + 2 * t + 1]);
      const float2 f = __bfloat1622float2(b);
      ss = fmaf(f.x, f.x, fmaf(f.y, f.y, ss));
      w[t] = *reinterpret_cast<const uint32_t*>(&b);
    }
    *reinterpret_cast<uint4*>(tile + out_off(r, cc, u)) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  return ss;
}

__device__ __forceinline__ void add_staged_bf16x32(const uint8_t* tile, int r, int cc, float* v) {
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const uint4 q = *reinterpret_cast<const uint4*>(tile + out_off(r, cc, u));
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const float2 f = unpack_bf16x2(w[t]);
      v[8 * u + 2 * t] += f.x;
      v[8 * u + 2 * t + 1] += f.y;
    }
  }
}

__device__ __forceinline__ void add_bf16x32(float* v, const __nv_bfloat16* src) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint4 u = __ldg(s + j);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const float2 f = unpack_bf16x2(w[t]);
      v[8 * j + 2 * t] += f.x;
      v[8 * j + 2 * t + 1] += f.y;
    }
  }
}

// Layout of a stream-K partial tile in its scratch slot: the float4 holding
// accumulator columns [32 cc + 4 j, 32 cc + 4 j + 4) of row rr is float4
// number (cc * 8 + j) * BM + rr, so each warp-wide store or load of one
// (cc, j) covers 32 consecutive float4 (512 contiguous bytes).
__device__ __forceinline__ size_t part_f4(int cc, int j, int rr) {
  return (static_cast<size_t>(cc) * 8 + j) * BM + rr;
}

// Loads accumulator columns [32 cc, 32 cc + 32) of this thread's row from
// TMEM and adds the fp32 partial rows of n_part contributor slots (slot i at
// part + i * slot_stride floats). The partials are requested kGroup slots at
// a time, all before any of them is used, so n_part slots cost about
// n_part / kGroup round trips to L2 instead of n_part.
template <int BN, int kGroup>
__device__ __forceinline__ void load_chunk(uint32_t taddr, int cc, int rr, const float* part,
                                           int n_part, size_t slot_stride, float* v) {
  float4 q[kGroup][8];
#pragma unroll
  for (int u = 0; u < kGroup; ++u)
    if (u < n_part) {
      const float4* src = reinterpret_cast<const float4*>(part + u * slot_stride);
#pragma unroll
      for (int j = 0; j < 8; ++j) q[u][j] = __ldcg(src + part_f4(cc, j, rr));
    }
  uint32_t r[32];
  tmem_ld32(taddr, r);
  tmem_ld_wait();
#pragma unroll
  for (int t = 0; t < 32; ++t) v[t] = __uint_as_float(r[t]);
  for (int i0 = 0; i0 < n_part; i0 += kGroup) {
    if (i0 > 0) {
#pragma unroll
      for (int u = 0; u < kGroup; ++u)
        if (i0 + u < n_part) {
          const float4* src = reinterpret_cast<const float4*>(part + (i0 + u) * slot_stride);
#pragma unroll
          for (int j = 0; j < 8; ++j) q[u][j] = __ldcg(src + part_f4(cc, j, rr));
        }
    }
#pragma unroll
    for (int u = 0; u < kGroup; ++u)
      if (i0 + u < n_part) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          v[4 * j] += q[u][j].x; v[4 * j + 1] += q[u][j].y;
          v[4 * j + 2] += q[u][j].z; v[4 * j + 3] += q[u][j].w;
        }
      }
  }
}

// 1 / rms of row `row`: from the per-tile sums of squares of the previous
// GEMM's epilogue (rowsq_in, summed in tile order) or the given row scale.
// The partial sums are requested eight at a time before any is added, so the
// sum costs a few L2 round trips, not one per tile.
__device__ __forceinline__ float row_inv_rms(const Params& p, int64_t row) {
  if (p.rowsq_in == nullptr) return p.row_scale[row];
  const float* rs = p.rowsq_in + row * p.rowsq_n;
  float ss = 0.f;
  for (int t0 = 0; t0 < p.rowsq_n; t0 += 8) {
    float q[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) q[u] = t0 + u < p.rowsq_n ? __ldg(rs + t0 + u) : 0.f;
#pragma unroll
    for (int u = 0; u < 8; ++u) ss += q[u];
  }
  return 1.0f / sqrtf(ss / p.rowsq_width + p.eps);
}

// One 128-column head of the QKV epilogue for this thread's row (row scale
// s), staged as chunks [cc0, cc0 + 4) of the epilogue tile. Every global
// read (bias, norm gain, cos/sin) is issued eight float4 at a time ahead of
// its use, so a head costs a dozen round trips to L1/L2 rather than a
// hundred.
template <int BN>
__device__ __forceinline__ void qkv_head(uint32_t taddr, int cc0, int rr, const float* part,
                                         int n_part, size_t slot_stride, int64_t row, bool valid,
                                         float s, int64_t c0, const Params& p, uint8_t* tile) {
  float v[128];
  if (n_part == 0) {
    // all four TMEM loads in flight at once, one wait (the raw fp32 bits land
    // in v directly)
#pragma unroll
    for (int j = 0; j < 4; ++j)
      tmem_ld32(taddr + 32 * j, *reinterpret_cast<uint32_t(*)[32]>(v + 32 * j));
    tmem_ld_wait();
  } else {
#pragma unroll
    for (int j = 0; j < 4; ++j)
      load_chunk<BN, 1>(taddr + 32 * j, cc0 + j, rr, part, n_part, slot_stride, v + 32 * j);
  }
  if (valid) {
#pragma unroll
    for (int t = 0; t < 128; ++t) v[t] *= s;
    if (p.bias != nullptr) {
      const float4* b = reinterpret_cast<const float4*>(p.bias + c0);
#pragma unroll
      for (int t0 = 0; t0 < 32; t0 += 4) {
        float4 bb[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) bb[u] = __ldg(b + t0 + u);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int t = t0 + u;
          v[4 * t] += bb[u].x; v[4 * t + 1] += bb[u].y;
          v[4 * t + 2] += bb[u].z; v[4 * t + 3] += bb[u].w;
        }
      }
    }
    const bool is_q = c0 < p.q_cols;
    const bool is_k = !is_q && c0 < p.q_cols + p.k_cols;
    if (is_q || is_k) {
      float ss = 0.f;
#pragma unroll
      for (int t = 0; t < 128; ++t) ss += v[t] * v[t];
      const float rn = 1.0f / sqrtf(ss * (1.0f / 128.0f) + p.eps);
      const float4* g = reinterpret_cast<const float4*>(is_q ? p.q_norm : p.k_norm);
#pragma unroll
      for (int t0 = 0; t0 < 32; t0 += 4) {
        float4 gg[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) gg[u] = __ldg(g + t0 + u);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int t = t0 + u;
          v[4 * t] *= rn * gg[u].x; v[4 * t + 1] *= rn * gg[u].y;
          v[4 * t + 2] *= rn * gg[u].z; v[4 * t + 3] *= rn * gg[u].w;
        }
      }
      // slot-major table: one warp reads 32 consecutive rows' float4 per slot pair
      const float4* cs = reinterpret_cast<const float4*>(p.cos_sin) + row;
#pragma unroll
      for (int t0 = 0; t0 < 32; t0 += 4) {
        float4 q[4];  // (cos_i, sin_i, cos_{i+1}, sin_{i+1}), i = 2t
#pragma unroll
        for (int u = 0; u < 4; ++u) q[u] = __ldg(cs + int64_t(t0 + u) * p.M);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = 2 * (t0 + u);
          const float a0 = v[i], b0 = v[i + 64], a1 = v[i + 1], b1 = v[i + 65];
          v[i] = a0 * q[u].x - b0 * q[u].y;
          v[i + 64] = a0 * q[u].y + b0 * q[u].x;
          v[i + 1] = a1 * q[u].z - b1 * q[u].w;
          v[i + 65] = a1 * q[u].w + b1 * q[u].z;
        }
      }
    }
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) stage_bf16x32(tile, rr, cc0 + j, v + 32 * j);
}

template <int BN, int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const __grid_constant__ CUtensorMap tmOut, const __grid_constant__ CUtensorMap tmRes,
               Params p) {
  using C = Cfg<BN>;
  constexpr int S = C::kStages;
  constexpr bool kRes = EPI == static_cast<int>(Epi::kResidual);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* smA = smem;
  uint8_t* smB = smem + S * C::kABytes;
  uint8_t* tile = smem + S * C::kStageBytes;  // bf16 epilogue tile (1024-aligned)
  uint64_t* full = reinterpret_cast<uint64_t*>(tile + C::kOutBytes);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* res_full = drain + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(res_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool lead_cta = rank == 0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) { mbar_init(full + s, 1); mbar_init(empty + s, 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(tfull + b, 1); mbar_init(tempty + b, 2); }
    mbar_init(drain, 1);
    mbar_init(res_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmOut);
    if (kRes) tma_prefetch_desc(&tmRes);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, C::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int64_t num_m = (p.M + 2 * BM - 1) / (2 * BM);
  const int64_t num_n = p.N / BN;
  const int G = static_cast<int>(gridDim.x >> 1);
  const int c = static_cast<int>(blockIdx.x >> 1);

  // Programmatic dependent launch: the next kernel in the stream may start
  // its own prologue once every CTA of this grid got here.
  griddep_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0;
      uint32_t issued = 0, last_ph = 0;  // per-stage bit masks
      WorkIter it(p, c, G);
      Work w;
      bool ok = true;
      bool have = it.next(w);
      // The weights (B) do not depend on the previous kernel in the stream:
      // the first stages' B boxes are requested before waiting for it, the A
      // boxes (this layer's activations) after.
      int pre = 0;
      if (have) {
        int64_t tm, tn;
        tile_mn(p, w.tile, num_m, num_n, tm, tn);
        const int32_t n0 = static_cast<int32_t>(tn * BN + rank * (BN / 2));
        pre = w.kb1 - w.kb0 < S ? w.kb1 - w.kb0 : S;
        for (int i = 0; i < pre; ++i) {
          const uint32_t fb = map_to_cta(smem_u32(full + i), 0);
          if (lead_cta) mbar_arrive_expect_tx(full + i, 2 * C::kStageBytes);
          tma_load_2d_pair(smB + i * C::kBBytes, &tmB, fb, (w.kb0 + i) * BK, n0);
        }
      }
      griddep_wait();
      bool first = true;
      while (ok && have) {
        int64_t tm, tn;
        tile_mn(p, w.tile, num_m, num_n, tm, tn);
        const int32_t m0 = static_cast<int32_t>(tm * 2 * BM + rank * BM);
        const int32_t n0 = static_cast<int32_t>(tn * BN + rank * (BN / 2));
        for (int kb = w.kb0; kb < w.kb1; ++kb) {
          const uint32_t fb = map_to_cta(smem_u32(full + stage), 0);
          if (first && kb - w.kb0 < pre) {
            // B already requested; stage `stage` is in its first use
            tma_load_2d_pair(smA + stage * C::kABytes, &tmA, fb, kb * BK, m0);
          } else {
            if (!mbar_wait<true>(empty + stage, ph ^ 1, p.err, kWhereGemmProducer, abort_flag)) {
              ok = false;
              break;
            }
            // both CTAs' loads complete on the even CTA's barrier
            if (lead_cta) mbar_arrive_expect_tx(full + stage, 2 * C::kStageBytes);
            tma_load_2d_pair(smA + stage * C::kABytes, &tmA, fb, kb * BK, m0);
            tma_load_2d_pair(smB + stage * C::kBBytes, &tmB, fb, kb * BK, n0);
          }
          issued |= 1u << stage;
          last_ph = (last_ph & ~(1u << stage)) | (ph << stage);
          if (++stage == S) { stage = 0; ph ^= 1; }
        }
        first = false;
        have = ok && it.next(w);
      }
      // Every issued load must land before the pair exits (the even CTA's
      // barrier counts both CTAs' bytes; the final cluster barrier holds the
      // odd CTA until then).
      if (lead_cta)
        for (int s = 0; s < S; ++s)
          if (issued & (1u << s))
            mbar_wait<true>(full + s, (last_ph >> s) & 1u, p.err, kWhereGemmDrain, nullptr);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      if (lead_cta) {
        constexpr uint32_t idesc = idesc_bf16_f32(2 * BM, BN, false, false);
        int stage = 0;
        uint32_t ph = 0;
        int acc_i = 0;
        WorkIter it(p, c, G);
        Work w;
        bool ok = true;
        while (ok && it.next(w)) {
          const int buf = acc_i & 1;
          if (!mbar_wait<true>(tempty + buf, ((acc_i >> 1) & 1) ^ 1, p.err, kWhereGemmMma, abort_flag))
            break;
          tc_fence_after();
          const uint32_t d = tmem_base + buf * BN;
          for (int kb = w.kb0; kb < w.kb1; ++kb) {
            if (!mbar_wait<true>(full + stage, ph, p.err, kWhereGemmMma, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint32_t a0 = smem_u32(smA + stage * C::kABytes);
            const uint32_t b0 = smem_u32(smB + stage * C::kBBytes);
#pragma unroll
            for (int k = 0; k < BK / 16; ++k)
              umma_bf16_ss_pair(d, sdesc_sw128(a0 + 32 * k, 16, 1024),
                                sdesc_sw128(b0 + 32 * k, 16, 1024), idesc,
                                (kb > w.kb0 || k > 0) ? 1u : 0u);
            umma_commit_pair(empty + stage, 0x3);
            if (++stage == S) { stage = 0; ph ^= 1; }
          }
          if (!ok) break;
          umma_commit_pair(tfull + buf, 0x3);
          ++acc_i;
        }
        // All issued MMAs complete before either CTA releases its TMEM.
        umma_commit_pair(drain, 0x3);
      }
      mbar_wait<true>(drain, 0, p.err, kWhereGemmDrain, nullptr);
    }
  } else {
    griddep_wait();  // the epilogue reads and writes this layer's activations
    const int quarter = warp & 3;
    const int rr = quarter * 32 + lane;
    const bool el = warp == 2 && lane == 0;  // epilogue leader
    const uint32_t lane_field = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tempty_lead = map_to_cta(smem_u32(tempty), 0);
    const size_t slot_floats = static_cast<size_t>(BM) * BN;
    int acc_i = 0;
    uint32_t res_ph = 0;
    bool pending = false;
    WorkIter it(p, c, G);
    Work w;
    while (it.next(w)) {
      const int buf = acc_i & 1;
      int64_t tm, tn;
      tile_mn(p, w.tile, num_m, num_n, tm, tn);
      const int64_t row0 = tm * 2 * BM + rank * BM;
      const int64_t row = row0 + rr;
      const int64_t n0 = tn * BN;
      const bool valid = row < p.M;
      const bool stores = w.role != kContributor;
      // the epilogue tile is free once the previous TMA store has read it
      if (el && pending) {
        bulk_wait_read_all();
        pending = false;
      }
      epilogue_sync();
      const bool need_res = kRes && stores;
      if (need_res && el) {
        mbar_arrive_expect_tx(res_full, C::kOutBytes);
#pragma unroll
        for (int b = 0; b < BN / 64; ++b)
          tma_load_2d(tile + b * 16384, &tmRes, res_full, static_cast<int32_t>(n0 + 64 * b),
                      static_cast<int32_t>(row0));
      }
      bool ok = mbar_wait<true>(tfull + buf, (acc_i >> 1) & 1, p.err, kWhereGemmEpilogue, abort_flag);
      if (need_res) {
        ok = ok && mbar_wait<true>(res_full, res_ph, p.err, kWhereGemmEpilogue, abort_flag);
        res_ph ^= 1;
      }
      if (!ok) *abort_flag = 1;
      // all four epilogue warps take the same decision, so none is left
      // waiting alone at a named barrier
      epilogue_sync();
      if (*abort_flag) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + buf * BN + lane_field;
      if (w.role == kContributor) {
        // leave this CTA's fp32 partial rows in its slot, then raise its flag
        float* slot = p.sk_partials + static_cast<size_t>(blockIdx.x) * slot_floats;
        const bool slot_ok =
            dcheck(static_cast<int>(blockIdx.x) < p.sk_slots, p.err, kWhereDbgGemmScratch);
#pragma unroll 1
        for (int cc = 0; slot_ok && cc < BN / 32; ++cc) {
          uint32_t r[32];
          tmem_ld32(tbase + 32 * cc, r);
          tmem_ld_wait();
          float4* dst = reinterpret_cast<float4*>(slot);
#pragma unroll
          for (int j = 0; j < 8; ++j)
            __stcg(dst + part_f4(cc, j, rr),
                   make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                               __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3])));
        }
        __threadfence();
        epilogue_sync();
        if (el && slot_ok) st_release(p.sk_flags + blockIdx.x, 1);
      } else {
        const float* part = nullptr;
        int n_part = 0;
        const size_t slot_stride = 2 * slot_floats;  // same-rank CTAs of consecutive pairs
        if (w.role == kFinisher) {
          // contributors: the pairs owning k-blocks [kb1, KB) of this tile
          const int64_t t_rel = w.tile - p.dp_tiles;
          const int c_last =
              p.sk_first + sk_owner((t_rel + 1) * p.kb_per_tile - 1, p.sk_units, p.sk_pairs);
          const int first = 2 * (c + 1) + static_cast<int>(rank);
          part = p.sk_partials + static_cast<size_t>(first) * slot_floats;
          n_part = c_last - c;
          if (!dcheck(2 * c_last + static_cast<int>(rank) < p.sk_slots, p.err,
                      kWhereDbgGemmScratch))
            n_part = 0;
          if (el) {
            for (int cp = c + 1; cp <= c + n_part; ++cp) {
              int32_t* flag = p.sk_flags + 2 * cp + rank;
              const uint64_t t0 = globaltimer_ns();
              while (ld_acquire(flag) != 1) {
                if (*abort_flag) break;
                if (globaltimer_ns() - t0 > kWaitLimitNs) {
                  record_error(p.err, Q3VL_ETIMEOUT, kWhereGemmEpilogue);
                  *abort_flag = 1;
                  break;
                }
              }
              *flag = 0;  // ready for the next launch on this workspace
            }
          }
          epilogue_sync();
        }
        if constexpr (EPI == static_cast<int>(Epi::kQkv)) {
          const float s = valid ? row_inv_rms(p, row) : 0.f;
#pragma unroll 1
          for (int hh = 0; hh < BN / 128; ++hh)
            qkv_head<BN>(tbase + 128 * hh, 4 * hh, rr, part, n_part, slot_stride, row, valid, s,
                         n0 + 128 * hh, p, tile);
        } else if constexpr (EPI == static_cast<int>(Epi::kSwiGLU)) {
          const float s = valid ? row_inv_rms(p, row) : 0.f;
#pragma unroll 1
          for (int cc = 0; cc < 4; ++cc) {
            float g[32], u[32];
            load_chunk<BN, 2>(tbase + 32 * cc, cc, rr, part, n_part, slot_stride, g);
            load_chunk<BN, 2>(tbase + 128 + 32 * cc, cc + 4, rr, part, n_part, slot_stride, u);
            float v[32];
#pragma unroll
            for (int t = 0; t < 32; ++t) v[t] = silu_fast(g[t] * s) * (u[t] * s);
            stage_bf16x32(tile, rr, cc, v);
          }
        } else {
          const int32_t dsk = (kRes && valid && p.ds_map != nullptr) ? p.ds_map[row] : -1;
          float ss = 0.f;
#pragma unroll 1
          for (int cc = 0; cc < BN / 32; ++cc) {
            float v[32];
            load_chunk<BN, 4>(tbase + 32 * cc, cc, rr, part, n_part, slot_stride, v);
            if constexpr (kRes) {
              add_staged_bf16x32(tile, rr, cc, v);
              if (dsk >= 0) add_bf16x32(v, p.ds_slab + int64_t(dsk) * p.N + n0 + 32 * cc);
            }
            if (p.rowsq_out != nullptr) ss += stage_bf16x32_ss(tile, rr, cc, v);
            else stage_bf16x32(tile, rr, cc, v);
          }
          if (p.rowsq_out != nullptr && valid &&
              dcheck(tn < p.rowsq_n, p.err, kWhereDbgGemmRowsq))
            p.rowsq_out[row * p.rowsq_n + tn] = ss;
        }
        fence_proxy_async_smem();
      }
      tc_fence_before();
      epilogue_sync();
      if (el) {
        // this CTA's accumulator rows are read: hand the buffer back
        if (lead_cta) mbar_arrive(tempty + buf);
        else mbar_arrive_cluster(tempty_lead + buf * sizeof(uint64_t));
        if (stores && row0 < p.M) {
          constexpr int kOutCols = EPI == static_cast<int>(Epi::kSwiGLU) ? BN / 2 : BN;
          const int64_t oc0 = EPI == static_cast<int>(Epi::kSwiGLU) ? n0 / 2 : n0;
#pragma unroll
          for (int b = 0; b < kOutCols / 64; ++b)
            tma_store_2d(&tmOut, tile + b * 16384, static_cast<int32_t>(oc0 + 64 * b),
                         static_cast<int32_t>(row0));
          bulk_commit_group();
          pending = true;
        }
      }
      ++acc_i;
    }
    if (el) bulk_wait_all();
  }
  tc_fence_before();
  cluster_sync();  // no CTA of the pair leaves while the other may touch its memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::kTmemCols);
  }
}

// Host-side schedule over pair tiles. Whole waves of tiles run data
// parallel. The tiles of a last, partial wave (rem < G of them) are each
// split along K into s = G / rem equal ranges (ranges of at least 16
// k-blocks) run by rem * s pairs (stream-K over exactly those tiles), so
// that wave costs about 1/s of a tile instead of a whole one. Longer ranges
// mean fewer partials for the finisher to add. On the 4B layer this gives
// QKV and gate/up 2 ways, the o-projection 4 and down 6; measured there, the
// o-projection took 65.0 us at 4 ways against 67.2 at 6 and 66.9 at 3, down
// 141.6 at 6 against 142.7 at 4, and QKV was slower above 2. Every pair of a wave starts its tiles at k-block 0 and moves
// through K at the same pace, so the pairs running at one time read the same
// k-slab of the operand panels and L2 serves the repeats. Problems smaller
// than one wave split each tile into ranges of at least 8 k-blocks.
struct HostSched {
  int pairs;
  int sk_pairs;
  int64_t dp_tiles, sk_units;
};

HostSched make_sched(int64_t tiles, int kb, int max_pairs) {
  HostSched h{};
  const int64_t G = max_pairs;
  const int64_t full = tiles / G, rem = tiles % G;
  int64_t s = rem > 0 ? G / rem : 1;
  const int64_t s_max = full == 0 ? kb / 8 : kb / 16;
  if (s > s_max) s = s_max;
  if (s < 1) s = 1;
  if (rem == 0 || s == 1) {
    // data parallel: whole tiles, round robin over the pairs
    h.pairs = static_cast<int>(tiles < G ? tiles : G);
    h.dp_tiles = tiles;
    h.sk_units = 0;
    h.sk_pairs = 1;
    return h;
  }
  h.dp_tiles = full * G;
  h.sk_units = rem * kb;
  h.sk_pairs = static_cast<int>(rem * s);
  h.pairs = static_cast<int>(full > 0 ? G : h.sk_pairs);
  return h;
}

template <int BN, int EPI>
cudaError_t launch_bn(const GemmArgs& a, Params p, cudaStream_t st) {
  using C = Cfg<BN>;
  constexpr int kOutDiv = EPI == static_cast<int>(Epi::kSwiGLU) ? 2 : 1;
  CUtensorMap tmA, tmB, tmOut, tmRes;
  if (!make_tmap_bf16(&tmA, a.A, a.M, a.K, a.K, BK, BM)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16(&tmB, a.B, a.N, a.K, a.K, BK, BN / 2)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16(&tmOut, a.out, a.M, a.N / kOutDiv, a.ldo, 64, BM))
    return cudaErrorInvalidValue;
  if (EPI == static_cast<int>(Epi::kResidual)) {
    if (!make_tmap_bf16(&tmRes, a.resid, a.M, a.N, a.ldo, 64, BM)) return cudaErrorInvalidValue;
  } else {
    tmRes = tmOut;
  }
  auto kern = gemm_tc_kernel<BN, EPI>;
  cudaError_t e = smem_attr_at_least(reinterpret_cast<const void*>(kern), C::kSmem);
  if (e != cudaSuccess) return e;
  // Stream-K finishers wait on other pairs, so every pair of the grid must be
  // resident at once: the grid never exceeds the co-resident cluster count.
  int n = 0;
  e = max_active_clusters(reinterpret_cast<const void*>(kern), kThreads, C::kSmem, 2, &n);
  if (e != cudaSuccess) return e;
  const int max_clusters = n > 0 ? (n < sm_count() / 2 ? n : sm_count() / 2) : 1;
  const int64_t tiles = ((a.M + 2 * BM - 1) / (2 * BM)) * (a.N / BN);
  const HostSched h = make_sched(tiles, static_cast<int>(a.K / BK), max_clusters);
  const int grid = 2 * h.pairs;
  if (h.sk_units > 0 &&
      (a.sk_partials == nullptr || a.sk_flags == nullptr || grid > a.sk_slots ||
       size_t(BM) * BN * sizeof(float) > a.sk_slot_bytes))
    return cudaErrorInvalidValue;
  p.dp_tiles = h.dp_tiles;
  p.sk_units = h.sk_units;
  p.sk_pairs = h.sk_pairs;
  p.kb_per_tile = static_cast<int>(a.K / BK);
  // keep the smaller operand resident in L2 while the larger one streams
  p.m_fastest = a.M <= a.N ? 1 : 0;
  // The QKV GEMM gives its stream-K ranges to the last pairs: their last
  // data-parallel tiles are V columns (N runs slowest in its tile order),
  // whose epilogue is the short one, so the pairs with the extra range do not
  // also end on a q/k tile's norm and rotation.
  p.sk_first = (EPI == static_cast<int>(Epi::kQkv) && h.sk_units > 0 && p.m_fastest)
                   ? h.pairs - h.sk_pairs : 0;
  e = launch_pdl_plain(kern, dim3(grid), dim3(kThreads), C::kSmem, st, tmA, tmB, tmOut, tmRes, p);
  if (e != cudaSuccess) return e;
  return counted_launch(1);
}

}  // namespace

cudaError_t launch_gemm_tc(Epi epi, const GemmArgs& a, cudaStream_t st) {
  Params p{};
  p.M = a.M; p.N = a.N; p.K = a.K;
  p.ldo = a.ldo;
  p.row_scale = a.row_scale; p.bias = a.bias; p.q_norm = a.q_norm; p.k_norm = a.k_norm;
  p.cos_sin = reinterpret_cast<const float2*>(a.cos_sin);
  p.q_cols = a.q_cols; p.k_cols = a.k_cols; p.eps = a.eps;
  p.ds_slab = static_cast<const __nv_bfloat16*>(a.ds_slab);
  p.ds_map = a.ds_map;
  p.err = device_error_ptr();
  p.sk_partials = a.sk_partials;
  p.sk_flags = a.sk_flags;
  p.sk_slots = a.sk_slots;
  p.rowsq_out = a.rowsq_out;
  p.rowsq_in = a.rowsq_in;
  p.rowsq_n = a.rowsq_n;
  p.rowsq_width = a.rowsq_width;
  if (a.K % BK != 0 || a.N % 128 != 0 || a.M <= 0) return cudaErrorInvalidValue;
  const bool use256 = a.N % 256 == 0;
  switch (epi) {
    case Epi::kQkv:
      return use256 ? launch_bn<256, 0>(a, p, st) : launch_bn<128, 0>(a, p, st);
    case Epi::kResidual:
      return use256 ? launch_bn<256, 1>(a, p, st) : launch_bn<128, 1>(a, p, st);
    case Epi::kSwiGLU:
      if (a.N % 256 != 0) return cudaErrorInvalidValue;
      return launch_bn<256, 2>(a, p, st);
    case Epi::kPlain:
      return use256 ? launch_bn<256, 3>(a, p, st) : launch_bn<128, 3>(a, p, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace q3vl
