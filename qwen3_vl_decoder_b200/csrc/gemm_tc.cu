// Persistent tcgen05 GEMM for sm_100a: C[M, N] = A[M, K] * B[N, K]^T, bf16
// inputs, fp32 accumulation in tensor memory, fused epilogues.
//
// Roles (192 threads, one CTA per SM):
//   warp 0    one thread issues TMA loads of A (128 x 64) and B (BN x 64)
//             tiles, 128-byte swizzled, into a ring of shared-memory stages;
//   warp 1    allocates TMEM; one thread issues tcgen05.mma (M=128, N=BN,
//             K=16) into one of two TMEM accumulators and commits to
//             mbarriers;
//   warps 2-5 epilogue: thread = accumulator row (tcgen05.ld 32x32b), apply
//             the fused epilogue, store bf16 to global memory.
// Two accumulators let the epilogue of tile i overlap the main loop of tile
// i + 1. Tiles are visited M-fastest so concurrently running CTAs share the
// same weight (B) panels in L2.
//
// Epilogues (cortiq qwen3te.rs `Qwen3Encoder::encode_with_images` and
// `Qwen3Encoder::norm_rope`; hf2q qwen3vl_text/forward.rs module doc for
// the bias-before-norm order):
//   kQkv      v = inv_rms[r] * acc + b; q/k heads: per-head RMSNorm with the
//             q_norm / k_norm gain, then split-half MRoPE from the cos/sin
//             table; v heads: v only.
//   kResidual out = resid + acc (+ DeepStack slab row ds_map[r]).
//   kSwiGLU   out = silu(s*g) * (s*u), s = inv_rms[r]; B's 256-row block
//             holds 128 gate rows then the 128 matching up rows.
//   kPlain    out = acc.
#include "q3vl_device.cuh"
#include "q3vl_internal.h"

namespace q3vl {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int kThreads = 192;

template <int BN>
struct Cfg {
  static constexpr int kStages = BN == 256 ? 4 : 6;
  static constexpr int kABytes = BM * BK * 2;
  static constexpr int kBBytes = BN * BK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTmemCols = 2 * BN;
  static constexpr size_t kSmem = 1024 + size_t(kStages) * kStageBytes + 256;
};

struct Params {
  int64_t M, N, K;
  __nv_bfloat16* out;
  int64_t ldo;
  const float* row_scale;
  const float* bias;
  const float* q_norm;
  const float* k_norm;
  const float2* cos_sin;
  int64_t q_cols, k_cols;
  float eps;
  const __nv_bfloat16* resid;
  const __nv_bfloat16* ds_slab;
  const int32_t* ds_map;
  int32_t* err;
  // schedule (see Sched)
  int64_t dp_tiles, sk_units;
  int kb_per_tile;
  // stream-K scratch: one fp32 partial tile per CTA and one flag per CTA
  float* sk_partials;
  int32_t* sk_flags;
};

// Work schedule shared by the three roles of a CTA. Each CTA first works
// through its stream-K range, then its data-parallel tiles:
//   tiles [0, dp_tiles): data parallel; CTA c takes tiles c, c + G, ... over
//     their whole K range;
//   tiles [dp_tiles, T): stream-K; their U = (T - dp_tiles) * KB k-block
//     units are cut into G equal contiguous ranges, CTA c taking units
//     [c U / G, (c + 1) U / G).
// A stream-K tile split across CTAs is finished by the CTA holding its first
// k-block, which reaches it last (at the end of its stream-K range). The
// CTAs holding its later k-blocks reach them first (at the start of their
// ranges): they leave fp32 partial sums in their own scratch slot and raise
// their flag; the finisher adds the partials in CTA order (deterministic)
// before the fused epilogue. Running the stream-K part first lets these
// longer epilogues overlap the data-parallel main loops that follow.
enum Role : int { kFull = 0, kFinisher = 1, kContributor = 2 };

struct Work {
  int64_t tile;
  int kb0, kb1, role;
};

struct WorkIter {
  int64_t dp_t, dp_tiles, stride;  // data-parallel part
  int64_t u, u1, sk_base;          // stream-K part (units relative to tile dp_tiles)
  int KB;
  __device__ WorkIter(const Params& p, int c, int G)
      : dp_t(c), dp_tiles(p.dp_tiles), stride(G), u(p.sk_units * c / G),
        u1(p.sk_units * (c + 1) / G), sk_base(p.dp_tiles), KB(p.kb_per_tile) {}
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

// Owner CTA of stream-K unit u: the largest c with c U / G <= u.
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

// Named barrier over the four epilogue warps only.
__device__ __forceinline__ void epilogue_sync() { asm volatile("barrier.sync 1, 128;" ::: "memory"); }

// Loads accumulator columns [32 cc, 32 cc + 32) of this thread's row from
// TMEM and adds the partial sums of n_part contributor slots (fp32).
template <int BN>
__device__ __forceinline__ void load_chunk(uint32_t taddr, int cc, int rr, const float* part,
                                           int n_part, float* v) {
  // the first contributor's partial is requested before the TMEM load so the
  // two latencies overlap
  float4 q0[8];
  const size_t off = (static_cast<size_t>(cc) * BM + rr) * 32;
  if (n_part > 0) {
    const float4* src = reinterpret_cast<const float4*>(part + off);
#pragma unroll
    for (int j = 0; j < 8; ++j) q0[j] = __ldcg(src + j);
  }
  uint32_t r[32];
  tmem_ld32(taddr, r);
  tmem_ld_wait();
#pragma unroll
  for (int t = 0; t < 32; ++t) v[t] = __uint_as_float(r[t]);
  if (n_part > 0) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      v[4 * j] += q0[j].x; v[4 * j + 1] += q0[j].y; v[4 * j + 2] += q0[j].z; v[4 * j + 3] += q0[j].w;
    }
  }
  for (int i = 1; i < n_part; ++i) {
    const float4* src = reinterpret_cast<const float4*>(part + static_cast<size_t>(i) * (BM * BN) + off);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float4 q = __ldcg(src + j);
      v[4 * j] += q.x; v[4 * j + 1] += q.y; v[4 * j + 2] += q.z; v[4 * j + 3] += q.w;
    }
  }
}

__device__ __forceinline__ void store_bf16x32(__nv_bfloat16* dst, const float* v) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    d[j] = make_uint4(pack_bf16x2(v[8 * j + 0], v[8 * j + 1]), pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                      pack_bf16x2(v[8 * j + 4], v[8 * j + 5]), pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
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

// One 128-column head of the QKV epilogue for this thread's row.
template <int BN>
__device__ __forceinline__ void qkv_head(uint32_t taddr, int cc0, int rr, const float* part,
                                         int n_part, int64_t row, bool valid, int64_t c0,
                                         const Params& p) {
  float v[128];
#pragma unroll
  for (int j = 0; j < 4; ++j) load_chunk<BN>(taddr + 32 * j, cc0 + j, rr, part, n_part, v + 32 * j);
  if (!valid) return;
  const float s = p.row_scale[row];
#pragma unroll
  for (int t = 0; t < 128; ++t) v[t] *= s;
  if (p.bias != nullptr) {
    const float4* b = reinterpret_cast<const float4*>(p.bias + c0);
#pragma unroll
    for (int t = 0; t < 32; ++t) {
      const float4 bb = __ldg(b + t);
      v[4 * t] += bb.x; v[4 * t + 1] += bb.y; v[4 * t + 2] += bb.z; v[4 * t + 3] += bb.w;
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
    for (int t = 0; t < 32; ++t) {
      const float4 gg = __ldg(g + t);
      v[4 * t] *= rn * gg.x; v[4 * t + 1] *= rn * gg.y;
      v[4 * t + 2] *= rn * gg.z; v[4 * t + 3] *= rn * gg.w;
    }
    const float4* cs = reinterpret_cast<const float4*>(p.cos_sin + row * 64);
#pragma unroll
    for (int t = 0; t < 32; ++t) {
      const float4 q = __ldg(cs + t);  // (cos_i, sin_i, cos_{i+1}, sin_{i+1}), i = 2t
      const int i = 2 * t;
      const float a0 = v[i], b0 = v[i + 64], a1 = v[i + 1], b1 = v[i + 65];
      v[i] = a0 * q.x - b0 * q.y;
      v[i + 64] = a0 * q.y + b0 * q.x;
      v[i + 1] = a1 * q.z - b1 * q.w;
      v[i + 65] = a1 * q.w + b1 * q.z;
    }
  }
  __nv_bfloat16* dst = p.out + row * p.ldo + c0;
#pragma unroll
  for (int j = 0; j < 4; ++j) store_bf16x32(dst + 32 * j, v + 32 * j);
}

template <int BN, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               Params p) {
  using C = Cfg<BN>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* smA = smem;
  uint8_t* smB = smem + S * C::kABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * C::kStageBytes);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) { mbar_init(full + s, 1); mbar_init(empty + s, 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(tfull + b, 1); mbar_init(tempty + b, 128); }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int64_t num_m = (p.M + BM - 1) / BM;
  const int G = static_cast<int>(gridDim.x);
  const int c = static_cast<int>(blockIdx.x);

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0;
      uint32_t issued = 0, last_ph = 0;  // per-stage bit masks
      WorkIter it(p, c, G);
      Work w;
      bool ok = true;
      while (ok && it.next(w)) {
        const int32_t m0 = static_cast<int32_t>((w.tile % num_m) * BM);
        const int32_t n0 = static_cast<int32_t>((w.tile / num_m) * BN);
        for (int kb = w.kb0; kb < w.kb1; ++kb) {
          if (!mbar_wait(empty + stage, ph ^ 1, p.err, kWhereGemmProducer, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(full + stage, C::kStageBytes);
          tma_load_2d(smA + stage * C::kABytes, &tmA, full + stage, kb * BK, m0);
          tma_load_2d(smB + stage * C::kBBytes, &tmB, full + stage, kb * BK, n0);
          issued |= 1u << stage;
          last_ph = (last_ph & ~(1u << stage)) | (ph << stage);
          if (++stage == S) { stage = 0; ph ^= 1; }
        }
      }
      // Every issued load must land before the block exits.
      for (int s = 0; s < S; ++s)
        if (issued & (1u << s))
          mbar_wait(full + s, (last_ph >> s) & 1u, p.err, kWhereGemmDrain, nullptr);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, false, false);
      int stage = 0;
      uint32_t ph = 0;
      int acc_i = 0;
      WorkIter it(p, c, G);
      Work w;
      bool ok = true;
      while (ok && it.next(w)) {
        const int buf = acc_i & 1;
        if (!mbar_wait(tempty + buf, ((acc_i >> 1) & 1) ^ 1, p.err, kWhereGemmMma, abort_flag))
          break;
        tc_fence_after();
        const uint32_t d = tmem_base + buf * BN;
        for (int kb = w.kb0; kb < w.kb1; ++kb) {
          if (!mbar_wait(full + stage, ph, p.err, kWhereGemmMma, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smA + stage * C::kABytes);
          const uint32_t b0 = smem_u32(smB + stage * C::kBBytes);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            umma_bf16_ss(d, sdesc_sw128(a0 + 32 * k, 16, 1024), sdesc_sw128(b0 + 32 * k, 16, 1024),
                         idesc, (kb > w.kb0 || k > 0) ? 1u : 0u);
          umma_commit(empty + stage);
          if (++stage == S) { stage = 0; ph ^= 1; }
        }
        if (!ok) break;
        umma_commit(tfull + buf);
        ++acc_i;
      }
      // All issued MMAs complete before TMEM is released.
      umma_commit(drain);
      mbar_wait(drain, 0, p.err, kWhereGemmDrain, nullptr);
    }
  } else {
    const int quarter = warp & 3;
    const int rr = quarter * 32 + lane;
    const bool leader = warp == 2 && lane == 0;
    const uint32_t lane_field = static_cast<uint32_t>(quarter * 32) << 16;
    int acc_i = 0;
    WorkIter it(p, c, G);
    Work w;
    while (it.next(w)) {
      const int buf = acc_i & 1;
      bool ok = mbar_wait(tfull + buf, (acc_i >> 1) & 1, p.err, kWhereGemmEpilogue, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const int64_t row = (w.tile % num_m) * BM + rr;
      const int64_t n0 = (w.tile / num_m) * BN;
      const bool valid = row < p.M;
      const uint32_t tbase = tmem_base + buf * BN + lane_field;
      if (w.role == kContributor) {
        // leave the fp32 partial tile in this CTA's slot, then raise the flag
        float* slot = p.sk_partials + static_cast<size_t>(c) * (BM * BN);
#pragma unroll 1
        for (int cc = 0; cc < BN / 32; ++cc) {
          uint32_t r[32];
          tmem_ld32(tbase + 32 * cc, r);
          tmem_ld_wait();
          float4* dst = reinterpret_cast<float4*>(slot + (static_cast<size_t>(cc) * BM + rr) * 32);
#pragma unroll
          for (int j = 0; j < 8; ++j)
            __stcg(dst + j, make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                        __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3])));
        }
        __threadfence();
        epilogue_sync();
        if (leader) st_release(p.sk_flags + c, 1);
      } else {
        const float* part = nullptr;
        int n_part = 0;
        if (w.role == kFinisher) {
          // contributors: the CTAs owning k-blocks [kb1, KB) of this tile
          const int64_t t_rel = w.tile - p.dp_tiles;
          const int c_last = sk_owner((t_rel + 1) * p.kb_per_tile - 1, p.sk_units, G);
          part = p.sk_partials + static_cast<size_t>(c + 1) * (BM * BN);
          n_part = c_last - c;
          if (leader) {
            for (int cp = c + 1; cp <= c_last; ++cp) {
              const uint64_t t0 = globaltimer_ns();
              while (ld_acquire(p.sk_flags + cp) != 1) {
                if (*abort_flag) break;
                if (globaltimer_ns() - t0 > kWaitLimitNs) {
                  record_error(p.err, Q3VL_ETIMEOUT, kWhereGemmEpilogue);
                  *abort_flag = 1;
                  break;
                }
              }
              p.sk_flags[cp] = 0;  // ready for the next launch on this workspace
            }
          }
          epilogue_sync();
        }
        if constexpr (EPI == static_cast<int>(Epi::kQkv)) {
#pragma unroll 1
          for (int hh = 0; hh < BN / 128; ++hh)
            qkv_head<BN>(tbase + 128 * hh, 4 * hh, rr, part, n_part, row, valid, n0 + 128 * hh, p);
        } else if constexpr (EPI == static_cast<int>(Epi::kSwiGLU)) {
          const float s = valid ? p.row_scale[row] : 0.f;
#pragma unroll 1
          for (int cc = 0; cc < 4; ++cc) {
            float g[32], u[32];
            load_chunk<BN>(tbase + 32 * cc, cc, rr, part, n_part, g);
            load_chunk<BN>(tbase + 128 + 32 * cc, cc + 4, rr, part, n_part, u);
            if (valid) {
              float v[32];
#pragma unroll
              for (int t = 0; t < 32; ++t) v[t] = silu_f(g[t] * s) * (u[t] * s);
              store_bf16x32(p.out + row * p.ldo + n0 / 2 + 32 * cc, v);
            }
          }
        } else {
          constexpr bool kRes = EPI == static_cast<int>(Epi::kResidual);
          const int32_t dsk = (kRes && valid && p.ds_map != nullptr) ? p.ds_map[row] : -1;
          // residual chunks are requested one chunk ahead of their use
          uint4 res[4];
          const uint4* rsrc = reinterpret_cast<const uint4*>(p.resid + row * p.ldo + n0);
          if (kRes && valid) {
#pragma unroll
            for (int j = 0; j < 4; ++j) res[j] = __ldg(rsrc + j);
          }
#pragma unroll 1
          for (int cc = 0; cc < BN / 32; ++cc) {
            uint4 cur[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) cur[j] = res[j];
            if (kRes && valid && cc + 1 < BN / 32) {
#pragma unroll
              for (int j = 0; j < 4; ++j) res[j] = __ldg(rsrc + 4 * (cc + 1) + j);
            }
            float v[32];
            load_chunk<BN>(tbase + 32 * cc, cc, rr, part, n_part, v);
            if (valid) {
              const int64_t col = n0 + 32 * cc;
              if constexpr (kRes) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                  const uint32_t wds[4] = {cur[j].x, cur[j].y, cur[j].z, cur[j].w};
#pragma unroll
                  for (int t = 0; t < 4; ++t) {
                    const float2 f = unpack_bf16x2(wds[t]);
                    v[8 * j + 2 * t] += f.x;
                    v[8 * j + 2 * t + 1] += f.y;
                  }
                }
                if (dsk >= 0) add_bf16x32(v, p.ds_slab + int64_t(dsk) * p.N + col);
              }
              store_bf16x32(p.out + row * p.ldo + col, v);
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(tempty + buf);
      ++acc_i;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// Host-side schedule: data-parallel waves, and stream-K over the remainder
// when the last wave would leave many SMs idle.
struct HostSched {
  int grid;
  int64_t dp_tiles, sk_units;
};

HostSched make_sched(int64_t tiles, int kb, int sms) {
  HostSched h{};
  const int64_t rem = tiles % sms;
  if (rem == 0 || (tiles >= sms && rem * 100 >= 92LL * sms)) {
    h.grid = static_cast<int>(tiles < sms ? tiles : sms);
    h.dp_tiles = tiles;
    h.sk_units = 0;
    return h;
  }
  const int64_t waves = tiles / sms;
  h.dp_tiles = waves > 0 ? (waves - 1) * sms : 0;
  h.sk_units = (tiles - h.dp_tiles) * kb;
  int64_t g = sms;
  if (tiles < sms) {
    // small problems: whole tiles, or at least 8 k-blocks per CTA
    const int64_t by_units = (h.sk_units + 7) / 8;
    g = tiles > by_units ? tiles : by_units;
    if (g > sms) g = sms;
  }
  if (g > h.sk_units) g = h.sk_units;
  h.grid = static_cast<int>(g);
  return h;
}

template <int BN, int EPI>
cudaError_t launch_bn(const GemmArgs& a, Params p, cudaStream_t st) {
  using C = Cfg<BN>;
  CUtensorMap tmA, tmB;
  if (!make_tmap_bf16(&tmA, a.A, a.M, a.K, a.K, BK, BM)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16(&tmB, a.B, a.N, a.K, a.K, BK, BN)) return cudaErrorInvalidValue;
  auto kern = gemm_tc_kernel<BN, EPI>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(C::kSmem));
  if (e != cudaSuccess) return e;
  const int64_t tiles = ((a.M + BM - 1) / BM) * (a.N / BN);
  const HostSched h = make_sched(tiles, static_cast<int>(a.K / BK), sm_count());
  if (h.sk_units > 0 &&
      (a.sk_partials == nullptr || a.sk_flags == nullptr || h.grid > a.sk_slots ||
       size_t(BM) * BN * sizeof(float) > a.sk_slot_bytes))
    return cudaErrorInvalidValue;
  p.dp_tiles = h.dp_tiles;
  p.sk_units = h.sk_units;
  p.kb_per_tile = static_cast<int>(a.K / BK);
  kern<<<h.grid, kThreads, C::kSmem, st>>>(tmA, tmB, p);
  return counted_launch(1);
}

}  // namespace

cudaError_t launch_gemm_tc(Epi epi, const GemmArgs& a, cudaStream_t st) {
  Params p{};
  p.M = a.M; p.N = a.N; p.K = a.K;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.ldo = a.ldo;
  p.row_scale = a.row_scale; p.bias = a.bias; p.q_norm = a.q_norm; p.k_norm = a.k_norm;
  p.cos_sin = reinterpret_cast<const float2*>(a.cos_sin);
  p.q_cols = a.q_cols; p.k_cols = a.k_cols; p.eps = a.eps;
  p.resid = static_cast<const __nv_bfloat16*>(a.resid);
  p.ds_slab = static_cast<const __nv_bfloat16*>(a.ds_slab);
  p.ds_map = a.ds_map;
  p.err = device_error_ptr();
  p.sk_partials = a.sk_partials;
  p.sk_flags = a.sk_flags;
  if (a.K % BK != 0 || a.N % 128 != 0 || a.M <= 0) return cudaErrorInvalidValue;
  // 128 x 256 tiles: a 128-wide N tile makes a single-CTA tcgen05.mma
  // shared-memory-bandwidth bound; stream-K absorbs the wave quantization.
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
