// Causal GQA flash attention on tcgen05 tensor cores (sm_100a), head_dim 128.
//
// o[p, h] = sum_{j <= p} softmax_j(q_p,h . k_j,g / sqrt(128)) v_j,g with
// g = h / (nh / nkv) (cortiq qwen3te.rs, the per-pair loop and
// `Qwen3Encoder::attention_gemm`), computed with an online softmax so no
// S x S matrix exists.
//
// One CTA = one 128-row query tile of one head; CTAs are ordered longest
// (last query tile) first, and the query heads of one KV group are
// neighbours so their K/V tiles are shared through L2. Causality skips every
// key tile past the diagonal; the diagonal tile is masked in registers.
//
// Roles (192 threads):
//   warp 0    one thread: TMA loads of Q (once), K and V tiles (two-stage
//             rings), 128-byte swizzled.
//   warp 1    one thread: S_j = Q K_j^T into one of two TMEM buffers, and
//             O += P_j V_j into the TMEM accumulator (V as an MN-major
//             operand, no transpose pass).
//   warps 2-5 softmax: thread = query row; reads S_j with tcgen05.ld, keeps
//             the running max m and sum l in registers, rescales O in TMEM
//             when m grows, writes P_j (bf16) to shared memory in the
//             swizzled K-major layout the MMA reads, and at the end writes
//             O / l.
#include "q3vl_device.cuh"
#include "q3vl_internal.h"

namespace q3vl {
namespace {

constexpr int kThreads = 192;
constexpr int kTile = 128;               // query rows per CTA and keys per tile
constexpr int kBlockBytes = 128 * 64 * 2;  // one [128 x 64] bf16 swizzle block
constexpr int kTileBytes = 2 * kBlockBytes;  // [128 x 128] bf16
constexpr size_t kSmem = 1024 + 6 * size_t(kTileBytes) + 256;  // Q, K[2], V[2], P

struct Params {
  int64_t S;
  int nh, nkv, num_qt;
  int32_t k_col0, v_col0;
  __nv_bfloat16* o;
  int64_t ldo;
  float scale_log2;  // log2(e) / sqrt(128)
  int32_t* err;
};

__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm, Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* sQ = smem;
  uint8_t* sK = smem + kTileBytes;      // 2 stages
  uint8_t* sV = smem + 3 * kTileBytes;  // 2 stages
  uint8_t* sP = smem + 5 * kTileBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 6 * kTileBytes);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;   // [2]
  uint64_t* k_empty = bars + 3;  // [2]
  uint64_t* v_full = bars + 5;   // [2]
  uint64_t* v_empty = bars + 7;  // [2]
  uint64_t* s_full = bars + 9;   // [2]
  uint64_t* p_full = bars + 11;
  uint64_t* o_done = bars + 12;
  uint64_t* drain = bars + 13;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 14);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = p.num_qt - 1 - static_cast<int>(blockIdx.x / p.nh);
  const int h = static_cast<int>(blockIdx.x % p.nh);
  const int g = h / (p.nh / p.nkv);
  const int n_kv = qt + 1;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(k_full + s, 1); mbar_init(k_empty + s, 1);
      mbar_init(v_full + s, 1); mbar_init(v_empty + s, 1);
      mbar_init(s_full + s, 1);
    }
    mbar_init(p_full, 128);
    mbar_init(o_done, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // programmatic dependent launch: let the next kernel start its prologue,
  // and wait for the QKV projection before reading q, k and v
  griddep_launch_dependents();
  const uint32_t tO = tmem + 256;

  if (warp == 0) {
    if (lane == 0) {
      griddep_wait();
      mbar_arrive_expect_tx(q_full, kTileBytes);
      tma_load_2d(sQ, &tm, q_full, h * 128, qt * kTile);
      tma_load_2d(sQ + kBlockBytes, &tm, q_full, h * 128 + 64, qt * kTile);
      int nk_issued = 0, nv_issued = 0;
      for (int j = 0; j < n_kv; ++j) {
        const int s = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (!mbar_wait(k_empty + s, ph ^ 1, p.err, kWhereAttnProducer, abort_flag)) break;
        mbar_arrive_expect_tx(k_full + s, kTileBytes);
        tma_load_2d(sK + s * kTileBytes, &tm, k_full + s, p.k_col0 + g * 128, j * kTile);
        tma_load_2d(sK + s * kTileBytes + kBlockBytes, &tm, k_full + s, p.k_col0 + g * 128 + 64,
                    j * kTile);
        ++nk_issued;
        if (!mbar_wait(v_empty + s, ph ^ 1, p.err, kWhereAttnProducer, abort_flag)) break;
        mbar_arrive_expect_tx(v_full + s, kTileBytes);
        tma_load_2d(sV + s * kTileBytes, &tm, v_full + s, p.v_col0 + g * 128, j * kTile);
        tma_load_2d(sV + s * kTileBytes + kBlockBytes, &tm, v_full + s, p.v_col0 + g * 128 + 64,
                    j * kTile);
        ++nv_issued;
      }
      // Every issued load must land before the block exits: the last two
      // loads of each ring are the only ones whose completion may be unseen.
      mbar_wait(q_full, 0, p.err, kWhereAttnDrain, nullptr);
      for (int j = nk_issued - 2; j < nk_issued; ++j)
        if (j >= 0) mbar_wait(k_full + (j & 1), (j >> 1) & 1, p.err, kWhereAttnDrain, nullptr);
      for (int j = nv_issued - 2; j < nv_issued; ++j)
        if (j >= 0) mbar_wait(v_full + (j & 1), (j >> 1) & 1, p.err, kWhereAttnDrain, nullptr);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, 128, false, true);
      const uint32_t q0 = smem_u32(sQ), p0 = smem_u32(sP);
      bool ok = mbar_wait(q_full, 0, p.err, kWhereAttnMma, abort_flag);
      auto issue_s = [&](int j) -> bool {
        const int s = j & 1;
        if (!mbar_wait(k_full + s, (j >> 1) & 1, p.err, kWhereAttnMma, abort_flag)) return false;
        tc_fence_after();
        const uint32_t k0 = smem_u32(sK + s * kTileBytes);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kBlockBytes + (kk & 3) * 32;
          umma_bf16_ss(tmem + s * 128, sdesc_sw128(q0 + off, 16, 1024),
                       sdesc_sw128(k0 + off, 16, 1024), idesc_s, kk > 0);
        }
        umma_commit(s_full + s);
        umma_commit(k_empty + s);
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 0; ok && j < n_kv; ++j) {
        if (j + 1 < n_kv && !issue_s(j + 1)) break;
        if (!mbar_wait(p_full, j & 1, p.err, kWhereAttnMma, abort_flag)) break;
        tc_fence_after();
        const int s = j & 1;
        if (!mbar_wait(v_full + s, (j >> 1) & 1, p.err, kWhereAttnMma, abort_flag)) break;
        tc_fence_after();
        const uint32_t v0 = smem_u32(sV + s * kTileBytes);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          umma_bf16_ss(tO, sdesc_sw128(p0 + (kk >> 2) * kBlockBytes + (kk & 3) * 32, 16, 1024),
                       sdesc_sw128(v0 + kk * 2048, kBlockBytes, 1024), idesc_o, (j | kk) != 0);
        }
        umma_commit(o_done);
        umma_commit(v_empty + s);
      }
      umma_commit(drain);
      mbar_wait(drain, 0, p.err, kWhereAttnDrain, nullptr);
    }
  } else {
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_field = static_cast<uint32_t>(quarter * 32) << 16;
    const int64_t qpos = int64_t(qt) * kTile + r;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      ok = mbar_wait(s_full + (j & 1), (j >> 1) & 1, p.err, kWhereAttnSoftmax, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      float x[128];
      {
        uint32_t raw[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tmem + (j & 1) * 128 + lane_field + 32 * c, raw[c]);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int t = 0; t < 32; ++t) x[32 * c + t] = __uint_as_float(raw[c][t]) * p.scale_log2;
      }
      if (j == qt) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c > r) x[c] = -INFINITY;
      }
      float mx = x[0];
#pragma unroll
      for (int c = 1; c < 128; ++c) mx = fmaxf(mx, x[c]);
      const float m_new = fmaxf(m, mx);
      const float alpha = exp2f(m - m_new);
      float rs = 0.f;
      uint32_t pk[64];
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const __nv_bfloat162 b =
            __floats2bfloat162_rn(exp2f(x[2 * c] - m_new), exp2f(x[2 * c + 1] - m_new));
        const float2 f = __bfloat1622float2(b);
        rs += f.x + f.y;
        pk[c] = *reinterpret_cast<const uint32_t*>(&b);
      }
      if (j > 0) {
        // P_{j-1} V_{j-1} must be done before O is rescaled and P is reused.
        ok = mbar_wait(o_done, (j - 1) & 1, p.err, kWhereAttnSoftmax, abort_flag);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(0xffffffffu, m_new > m)) {
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            tmem_ld32(tO + lane_field + 32 * c, o);
            tmem_ld_wait();
#pragma unroll
            for (int t = 0; t < 32; ++t) o[t] = __float_as_uint(__uint_as_float(o[t]) * alpha);
            tmem_st32(tO + lane_field + 32 * c, o);
          }
          tmem_st_wait();
        }
      }
      l = l * alpha + rs;
      m = m_new;
      // P row r, 128-byte swizzle: 16-byte chunk c8 of row r sits at c8 ^ (r % 8).
#pragma unroll
      for (int cc = 0; cc < 16; ++cc) {
        const int off = (cc >> 3) * kBlockBytes + r * 128 + (((cc & 7) ^ (r & 7)) << 4);
        *reinterpret_cast<uint4*>(sP + off) =
            make_uint4(pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    griddep_wait();  // before this kernel's global stores
    if (ok) {
      ok = mbar_wait(o_done, (n_kv - 1) & 1, p.err, kWhereAttnSoftmax, abort_flag);
      if (__all_sync(0xffffffffu, ok)) {
        tc_fence_after();
        const float inv_l = 1.0f / l;
        __nv_bfloat16* dst = p.o + qpos * p.ldo + h * 128;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + lane_field + 32 * c, o);
          tmem_ld_wait();
          if (qpos < p.S && dcheck((h + 1) * 128 <= p.ldo, p.err, kWhereDbgAttnStore)) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * c);
#pragma unroll
            for (int t = 0; t < 4; ++t)
              d4[t] = make_uint4(
                  pack_bf16x2(__uint_as_float(o[8 * t]) * inv_l, __uint_as_float(o[8 * t + 1]) * inv_l),
                  pack_bf16x2(__uint_as_float(o[8 * t + 2]) * inv_l, __uint_as_float(o[8 * t + 3]) * inv_l),
                  pack_bf16x2(__uint_as_float(o[8 * t + 4]) * inv_l, __uint_as_float(o[8 * t + 5]) * inv_l),
                  pack_bf16x2(__uint_as_float(o[8 * t + 6]) * inv_l, __uint_as_float(o[8 * t + 7]) * inv_l));
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// Two query heads per CTA (the heads 2m, 2m+1 of one KV group, same 128 query
// rows), so every K/V tile loaded serves both. The MMA warp interleaves the
// two heads: while softmax warpgroup A works on S_A(j) the tensor core runs
// S_B(j), and while softmax B works the tensor core runs P_A(j) V(j) and
// S_A(j+1). P_X(j) is written back as bf16 into the first 64 TMEM columns of
// S_X (two per 32-bit column) and read from there as the A operand of the
// P V product; tcgen05.mma operations of one thread run in issue order, so
// S_X(j+1), issued after P_X(j) V(j), overwrites those columns only after
// they were read. The running max is raised lazily: O and l are rescaled
// only when a row's max grows by more than 2^8, so P entries stay <= 256.
//
// Roles (320 threads): warp 0 TMA, warp 1 MMA, warps 2-5 softmax of head A,
// warps 6-9 softmax of head B (thread = query row).
// TMEM: S_A [0,128), S_B [128,256), O_A [256,384), O_B [384,512).
// ---------------------------------------------------------------------------
// Row max of the raw (unscaled) scores of one 128-column tile held in
// registers (diagonal tile: keys past the query row excluded).
template <bool kDiag>
__device__ __forceinline__ float row_max_regs(const uint32_t* sr, int r) {
  // eight independent partial maxima keep the dependency chains short; on
  // the diagonal tile the columns past r enter as -inf
  auto v = [&](int c) {
    const float x = __uint_as_float(sr[c]);
    return kDiag && c > r ? -INFINITY : x;
  };
  float pm[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) pm[q] = fmaxf(v(q), v(q + 8));
#pragma unroll
  for (int c = 16; c < 128; c += 16)
#pragma unroll
    for (int q = 0; q < 8; ++q) pm[q] = fmax3(pm[q], v(c + q), v(c + q + 8));
  return fmaxf(fmaxf(fmax3(pm[0], pm[1], pm[2]), fmax3(pm[3], pm[4], pm[5])), fmaxf(pm[6], pm[7]));
}

// 2^x for a pair of fp32 values on the FMA pipe (the special-function unit
// delivers 16 exponentials per clock per SM, an eighth of the FMA rate, and
// a 128-key tile needs 16384 of them per head). x = j + f with j the nearest
// integer (the 1.5 * 2^23 shift puts it in the low mantissa bits) and
// f in [-1/2, 1/2]; 2^f is a degree-3 polynomial fitted to minimise the
// relative error on that interval (max 7.5e-5, far below the bf16 rounding
// of P); 2^j enters by adding j to the exponent field. x is clamped at -126
// so the exponent stays in range (2^-126 stands for every smaller value).
__device__ __forceinline__ uint64_t exp2_poly_x2(uint64_t x2) {
  float x0, x1;
  f2_unpack(x2, x0, x1);
  const uint64_t X = f2_pack(fmaxf(x0, -126.0f), fmaxf(x1, -126.0f));
  const uint64_t T = f2_add(X, f2_pack(12582912.0f, 12582912.0f));     // 1.5 * 2^23 + j
  const uint64_t J = f2_add(T, f2_pack(-12582912.0f, -12582912.0f));   // j
  const uint64_t F = f2_fma(J, f2_pack(-1.0f, -1.0f), X);              // f = x - j
  uint64_t P = f2_fma(F, f2_pack(0.0551716685f, 0.0551716685f), f2_pack(0.24261114f, 0.24261114f));
  P = f2_fma(P, F, f2_pack(0.69326097f, 0.69326097f));
  P = f2_fma(P, F, f2_pack(0.99992806f, 0.99992806f));
  float p0, p1, t0, t1;
  f2_unpack(P, p0, p1);
  f2_unpack(T, t0, t1);
  // the low 9 bits of T hold j in two's complement; shifted into the
  // exponent field they add j to 2^f's exponent
  return f2_pack(__uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23)),
                 __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23)));
}

// P = 2^(s*sc - m) for the 128 columns of a score row held in registers,
// written as packed bf16 pairs into the first 64 TMEM columns of the same S
// buffer; returns the fp32 row sum. The scale-and-shift and the running sum
// run as packed f32x2 operations. Of every 16 pairs, kPoly take 2^x from
// exp2_poly_x2 and the rest from ex2.approx, so the FMA pipe shares the
// exponentials with the special-function unit that otherwise bounds the tile.
template <bool kDiag, int kPoly>
__device__ __forceinline__ float exp_regs(const uint32_t* sr, uint32_t tS, int r, float sc, float m) {
  const uint64_t sc2 = f2_pack(sc, sc), nm2 = f2_pack(-m, -m);
  uint64_t acc[4];  // four independent running sums of pairs
#pragma unroll
  for (int q = 0; q < 4; ++q) acc[q] = f2_pack(0.f, 0.f);
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) {
    uint32_t pk[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      const int c0 = 32 * cc + 2 * t;
      const uint64_t xx = f2_fma(f2_pack(__uint_as_float(sr[c0]), __uint_as_float(sr[c0 + 1])), sc2, nm2);
      float e0, e1;
      if (t >= 16 - kPoly) {
        f2_unpack(exp2_poly_x2(xx), e0, e1);
      } else {
        float x0, x1;
        f2_unpack(xx, x0, x1);
        e0 = ex2_approx(x0);
        e1 = ex2_approx(x1);
      }
      if (kDiag) {
        if (c0 > r) e0 = 0.f;
        if (c0 + 1 > r) e1 = 0.f;
      }
      acc[t & 3] = f2_add(acc[t & 3], f2_pack(e0, e1));
      const __nv_bfloat162 b2 = __floats2bfloat162_rn(e0, e1);
      pk[t] = *reinterpret_cast<const uint32_t*>(&b2);
    }
    tmem_st16(tS + 16 * cc, pk);
  }
  float a0, a1;
  f2_unpack(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), a0, a1);
  return a0 + a1;
}

constexpr int kThreads2 = 320;
// Q_A, Q_B, K[2], V[2], 4 KB per softmax warp for the output box it stores
// by TMA, and the barriers
constexpr int kStageBytes2 = 32 * 128;
constexpr size_t kSmem2 = 1024 + 6 * size_t(kTileBytes) + 256 + 8 * size_t(kStageBytes2);
static_assert(kSmem2 <= 232448, "shared memory budget");
constexpr float kRescaleLog2 = 8.0f;
// Pairs of every 16 whose exponentials run on the FMA pipe. Measured on the
// 4B layer at S = 4096: 0 -> 137.7 us, 2 -> 141.8, 4 -> 135.7, 6 -> 145.9
// (more spill under the 168-register cap of a 320-thread CTA).
constexpr int kPolyPairs = 4;

// Persistent: one CTA per SM walks work items (query tile qt, head pair h0);
// item k has qt = num_qt - 1 - k / pairs, so items come longest first, and
// CTA c takes items c, 2G-1-c, 2G+c, 4G-1-c, ... (G CTAs, a snake that
// evens out the causal tile counts). Across items the pipeline keeps going:
// the TMA warp loads the next item's Q as soon as the last S of the current
// item has read Q; the MMA warp issues each head's first S product of the
// next item right behind that head's last P V of the current item (once that
// Q and the first K tile have arrived) and signals the head's finished O on a
// barrier of its own, so one head's softmax warps write their output and go
// on while the other head finishes; only the next item's first P V of a head
// waits for that head's softmax warps to have read its O out of TMEM.
// Barrier phases run on counters across items: per CTA item index ii and
// per CTA tile index t (a tile = one key tile of one item).
template <int kPoly>
__global__ void __launch_bounds__(kThreads2, 1)
attn2_tc_kernel(const __grid_constant__ CUtensorMap tm, const __grid_constant__ CUtensorMap tmo,
                Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* sQ = smem;                   // [2] heads
  uint8_t* sK = smem + 2 * kTileBytes;  // [2] stages
  uint8_t* sV = smem + 4 * kTileBytes;  // [2] stages
  uint8_t* s_out = smem + 6 * kTileBytes;  // [8 softmax warps][32 rows x 128 B], 128-byte swizzle
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_out + 8 * kStageBytes2);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;   // [2]
  uint64_t* k_empty = bars + 3;  // [2]
  uint64_t* v_full = bars + 5;   // [2]
  uint64_t* v_empty = bars + 7;  // [2]
  uint64_t* s_full = bars + 9;   // [2] per head
  uint64_t* p_full = bars + 11;  // [2] per head
  uint64_t* o_final = bars + 13;  // [2] per head
  uint64_t* drain = bars + 15;
  uint64_t* q_empty = bars + 16;
  uint64_t* o_free = bars + 17;  // [2] per head
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 19);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pairs = p.nh / 2;
  const int n_items = p.num_qt * pairs;
  const int G = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
  // the ii-th item of this CTA, or -1 past the end
  auto item_of = [&](int ii) -> int {
    const int k = (ii >> 1) * 2 * G + ((ii & 1) ? 2 * G - 1 - c : c);
    return k < n_items ? k : -1;
  };

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(k_full + s, 1); mbar_init(k_empty + s, 1);
      mbar_init(v_full + s, 1); mbar_init(v_empty + s, 1);
      mbar_init(s_full + s, 1); mbar_init(p_full + s, 128);
      mbar_init(o_free + s, 128);
      mbar_init(o_final + s, 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm);
    tma_prefetch_desc(&tmo);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // programmatic dependent launch: let the next kernel start its prologue,
  // and wait for the QKV projection before reading q, k and v
  griddep_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      // The TMA warp waits with the suspend-time hint (fewer issue slots
      // taken from the softmax warps: the 32B shape at S = 1064 39.4 ->
      // 37.4 us); the MMA warp polls plainly, its wake-up is on each head's
      // critical path (with the hint: 133.9 -> 141.8 us on the 4B layer).
      griddep_wait();
      int nk_issued = 0, nv_issued = 0, nq_issued = 0;
      bool ok = true;
      for (int ii = 0, k = item_of(0); ok && k >= 0; k = item_of(++ii)) {
        const int qt = p.num_qt - 1 - k / pairs, h0 = 2 * (k % pairs);
        const int g = h0 / (p.nh / p.nkv);
        // Q is free once the previous item's last S products completed
        if (ii > 0 && !mbar_wait<true>(q_empty, (ii - 1) & 1, p.err, kWhereAttnProducer, abort_flag)) break;
        mbar_arrive_expect_tx(q_full, 2 * kTileBytes);
        for (int x = 0; x < 2; ++x) {
          tma_load_2d(sQ + x * kTileBytes, &tm, q_full, (h0 + x) * 128, qt * kTile);
          tma_load_2d(sQ + x * kTileBytes + kBlockBytes, &tm, q_full, (h0 + x) * 128 + 64,
                      qt * kTile);
        }
        ++nq_issued;
        for (int j = 0; j <= qt; ++j) {
          const int t = nk_issued, s = t & 1;
          const uint32_t ph = (t >> 1) & 1;
          if (!mbar_wait<true>(k_empty + s, ph ^ 1, p.err, kWhereAttnProducer, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(k_full + s, kTileBytes);
          tma_load_2d(sK + s * kTileBytes, &tm, k_full + s, p.k_col0 + g * 128, j * kTile);
          tma_load_2d(sK + s * kTileBytes + kBlockBytes, &tm, k_full + s, p.k_col0 + g * 128 + 64,
                      j * kTile);
          ++nk_issued;
          if (!mbar_wait<true>(v_empty + s, ph ^ 1, p.err, kWhereAttnProducer, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(v_full + s, kTileBytes);
          tma_load_2d(sV + s * kTileBytes, &tm, v_full + s, p.v_col0 + g * 128, j * kTile);
          tma_load_2d(sV + s * kTileBytes + kBlockBytes, &tm, v_full + s, p.v_col0 + g * 128 + 64,
                      j * kTile);
          ++nv_issued;
        }
      }
      // every issued load lands before the block exits: the last Q and the
      // last two loads of each ring are the only ones whose completion may be
      // unseen
      if (nq_issued > 0) mbar_wait(q_full, (nq_issued - 1) & 1, p.err, kWhereAttnDrain, nullptr);
      for (int t = nk_issued - 2; t < nk_issued; ++t)
        if (t >= 0) mbar_wait(k_full + (t & 1), (t >> 1) & 1, p.err, kWhereAttnDrain, nullptr);
      for (int t = nv_issued - 2; t < nv_issued; ++t)
        if (t >= 0) mbar_wait(v_full + (t & 1), (t >> 1) & 1, p.err, kWhereAttnDrain, nullptr);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, 128, false, true);
      // The issuing thread shares its SM sub-partition with two softmax
      // warps, and each head's chain waits for its 16 products to be issued:
      // the descriptors are formed once and advanced by constant offsets
      // (the start-address field holds the address / 16; every address stays
      // below 256 KB, so the sum never carries out of the field).
      const uint64_t dq0 = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dk0 = sdesc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dv0 = sdesc_sw128(smem_u32(sV), kBlockBytes, 1024);
      auto issue_s = [&](int x, int t) {
        const uint64_t dq = dq0 + static_cast<uint64_t>((x * kTileBytes) >> 4);
        const uint64_t dk = dk0 + static_cast<uint64_t>(((t & 1) * kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t off = ((kk >> 2) * kBlockBytes + (kk & 3) * 32) >> 4;
          umma_bf16_ss(tmem + x * 128, dq + off, dk + off, idesc_s, kk > 0);
        }
        umma_commit(s_full + x);
      };
      auto issue_pv = [&](int x, int j, int t) {
        const uint64_t dv = dv0 + static_cast<uint64_t>(((t & 1) * kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_bf16_ts(tmem + 256 + x * 128, tmem + x * 128 + kk * 8, dv + ((kk * 2048) >> 4), idesc_o,
                       (j | kk) != 0);
      };
      bool ok = true;
      int t0 = 0;  // this CTA's tile index of the item's first key tile
      // The first item's first score products; every later item's follow
      // the previous item's last P V of the same head (below).
      if (item_of(0) >= 0) {
        ok = mbar_wait(q_full, 0, p.err, kWhereAttnMma, abort_flag) &&
             mbar_wait(k_full + 0, 0, p.err, kWhereAttnMma, abort_flag);
        if (ok) {
          tc_fence_after();
          issue_s(0, 0);
          issue_s(1, 0);
          umma_commit(k_empty + 0);
          if (p.num_qt - item_of(0) / pairs == 1) umma_commit(q_empty);
        }
      }
      for (int ii = 0, k = item_of(0); ok && k >= 0; k = item_of(++ii)) {
        const int n_kv = p.num_qt - k / pairs;
        const int kn = item_of(ii + 1), tn = t0 + n_kv;  // the next item and its first tile
        for (int j = 0; j < n_kv; ++j) {
          const int t = t0 + j, s = t & 1;
          const bool more = j + 1 < n_kv;
          if (!mbar_wait(v_full + s, (t >> 1) & 1, p.err, kWhereAttnMma, abort_flag)) { ok = false; break; }
          // the next K tile has usually landed by now: checking it here keeps
          // the wait off the stretch between P_A and S_A(j+1)
          bool k_next = !more || mbar_try_wait(smem_u32(k_full + (s ^ 1)), ((t + 1) >> 1) & 1);
          if (!mbar_wait(p_full + 0, t & 1, p.err, kWhereAttnMma, abort_flag)) { ok = false; break; }
          // the first P V of an item overwrites O: the previous item's O_A
          // must have been read out
          if (j == 0 && ii > 0 &&
              !mbar_wait(o_free + 0, (ii - 1) & 1, p.err, kWhereAttnMma, abort_flag)) { ok = false; break; }
          tc_fence_after();
          issue_pv(0, j, t);
          if (more) {
            if (!k_next) {
              if (!mbar_wait(k_full + (s ^ 1), ((t + 1) >> 1) & 1, p.err, kWhereAttnMma, abort_flag)) {
                ok = false;
                break;
              }
              tc_fence_after();
            }
            issue_s(0, t + 1);
          } else {
            // head A's O is complete once this P V is; the next item's
            // first S_A follows it (S_A overwrites P_A only after this P V,
            // issued before it, has read P_A: in-order execution), so head
            // A's softmax warps start the next item while head B finishes
            umma_commit(o_final + 0);
            if (kn >= 0) {
              if (!mbar_wait(q_full, (ii + 1) & 1, p.err, kWhereAttnMma, abort_flag) ||
                  !mbar_wait(k_full + (tn & 1), (tn >> 1) & 1, p.err, kWhereAttnMma, abort_flag)) {
                ok = false;
                break;
              }
              tc_fence_after();
              issue_s(0, tn);
            }
          }
          if (!mbar_wait(p_full + 1, t & 1, p.err, kWhereAttnMma, abort_flag)) { ok = false; break; }
          if (j == 0 && ii > 0 &&
              !mbar_wait(o_free + 1, (ii - 1) & 1, p.err, kWhereAttnMma, abort_flag)) { ok = false; break; }
          tc_fence_after();
          issue_pv(1, j, t);
          umma_commit(v_empty + s);
          if (more) {
            issue_s(1, t + 1);
            umma_commit(k_empty + (s ^ 1));
            if (j + 2 == n_kv) umma_commit(q_empty);  // the item's last S products
          } else {
            umma_commit(o_final + 1);
            if (kn >= 0) {
              issue_s(1, tn);
              umma_commit(k_empty + (tn & 1));
              if (p.num_qt - kn / pairs == 1) umma_commit(q_empty);  // the next item's only tile
            }
          }
        }
        t0 += n_kv;
      }
      if (!ok) *abort_flag = 1;
      umma_commit(drain);
      mbar_wait(drain, 0, p.err, kWhereAttnDrain, nullptr);
    }
  } else {
    const int x = (warp - 2) >> 2;  // head of this warpgroup
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_field = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + x * 128 + lane_field;
    const uint32_t tO = tmem + 256 + x * 128 + lane_field;
    const float sc = p.scale_log2;
    griddep_wait();  // before this kernel's global stores
    bool ok = true;
    int t = 0;  // this CTA's running tile index
    for (int ii = 0, k = item_of(0); ok && k >= 0; k = item_of(++ii)) {
      const int qt = p.num_qt - 1 - k / pairs, h0 = 2 * (k % pairs);
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j <= qt; ++j, ++t) {
        ok = mbar_wait(s_full + x, t & 1, p.err, kWhereAttnSoftmax, abort_flag);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
        const bool diag = j == qt;
        // the whole score row in registers: one batch of TMEM loads, one wait
        uint32_t sr[128];
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) tmem_ld32(tS + 32 * cc, *reinterpret_cast<uint32_t(*)[32]>(sr + 32 * cc));
        tmem_ld_wait();
        // row max of the raw (unscaled) scores; the scale is positive
        const float mx = diag ? row_max_regs<true>(sr, r) : row_max_regs<false>(sr, r);
        const float m_new = fmaxf(m, mx * sc);
        const bool grow = m_new > m + kRescaleLog2;
        const float alpha = grow ? ex2_approx(m - m_new) : 1.0f;
        if (grow) m = m_new;
        // the warp's rescale decision before the exponentials, so nothing
        // but the stores is left between them and the arrival
        const bool rescale = j > 0 && __any_sync(0xffffffffu, grow);
        // P = 2^(s*scale - m) as bf16 into the first 64 columns of S
        const float rs = diag ? exp_regs<true, kPoly>(sr, tS, r, sc, m)
                              : exp_regs<false, kPoly>(sr, tS, r, sc, m);
        l = l * alpha + rs;
        if (rescale) {
          // O_X(j-1) is complete: S_X(j) was issued after P_X(j-1) V(j-1).
#pragma unroll 1
          for (int c4 = 0; c4 < 4; ++c4) {
            uint32_t o[32];
            tmem_ld32(tO + 32 * c4, o);
            tmem_ld_wait();
#pragma unroll
            for (int u = 0; u < 32; ++u) o[u] = __float_as_uint(__uint_as_float(o[u]) * alpha);
            tmem_st32(tO + 32 * c4, o);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(p_full + x);
      }
      if (!ok) break;
      ok = mbar_wait(o_final + x, ii & 1, p.err, kWhereAttnSoftmax, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      const float inv_l = 1.0f / l;
      uint32_t o[4][32];
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) tmem_ld32(tO + 32 * c4, o[c4]);
      tmem_ld_wait();
      // O is in registers: the next item's first P V may overwrite it
      tc_fence_before();
      mbar_arrive(o_free + x);
      // The warp's 32 rows go out by TMA, 64 columns at a time: each thread
      // writes its row's 128 bytes into the warp's staging box in the
      // 128-byte swizzle the tensor map expects, and one lane issues the
      // bulk store. The warps move on to the next item at once; the stores of
      // all CTAs, which finish their items at about the same time, drain in
      // the background (as 16-byte stores into 32 rows 8 KB apart they held
      // the softmax warps ~4,000 cycles per item).
      uint8_t* stg = s_out + (warp - 2) * kStageBytes2;
      const bool cols_ok = dcheck(((h0 + x) + 1) * 128 <= p.ldo, p.err, kWhereDbgAttnStore);
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        // the box is free once the previous bulk store has read it
        if (lane == 0) bulk_wait_read_all();
        __syncwarp();
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint32_t* ov = o[2 * hf + (u >> 2)] + 8 * (u & 3);
          *reinterpret_cast<uint4*>(stg + lane * 128 + ((u ^ (lane & 7)) << 4)) = make_uint4(
              pack_bf16x2(__uint_as_float(ov[0]) * inv_l, __uint_as_float(ov[1]) * inv_l),
              pack_bf16x2(__uint_as_float(ov[2]) * inv_l, __uint_as_float(ov[3]) * inv_l),
              pack_bf16x2(__uint_as_float(ov[4]) * inv_l, __uint_as_float(ov[5]) * inv_l),
              pack_bf16x2(__uint_as_float(ov[6]) * inv_l, __uint_as_float(ov[7]) * inv_l));
        }
        fence_proxy_async_smem();
        __syncwarp();
        // rows past S are clipped by the tensor map; a box wholly past it
        // is not issued
        const int32_t y0 = qt * kTile + quarter * 32;
        if (lane == 0 && cols_ok && y0 < p.S) {
          tma_store_2d(&tmo, stg, (h0 + x) * 128 + 64 * hf, y0);
          bulk_commit_group();
        }
      }
    }
  }
  if (warp >= 2 && lane == 0) bulk_wait_all();  // this warp's output stores complete
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

cudaError_t launch_attention_tc(const q3vl_config& c, const void* qkv, int64_t S, void* o,
                                cudaStream_t st) {
  const int64_t Ntot = qkv_dim(c);
  CUtensorMap tm;
  if (!make_tmap_bf16(&tm, qkv, S, Ntot, Ntot, 64, 128)) return cudaErrorInvalidValue;
  Params p;
  p.S = S;
  p.nh = c.n_heads;
  p.nkv = c.n_kv_heads;
  p.num_qt = static_cast<int>((S + kTile - 1) / kTile);
  p.k_col0 = static_cast<int32_t>(q_dim(c));
  p.v_col0 = static_cast<int32_t>(q_dim(c) + kv_dim(c));
  p.o = static_cast<__nv_bfloat16*>(o);
  p.ldo = q_dim(c);
  p.scale_log2 = 1.4426950408889634f / sqrtf(128.0f);
  p.err = device_error_ptr();
  if ((p.nh / p.nkv) % 2 == 0) {
    // two query heads of one KV group per CTA
    // the output, [S, nh * 128] with row stride ldo, in 64-column x 32-row boxes
    CUtensorMap tmo;
    if (!make_tmap_bf16(&tmo, o, S, q_dim(c), p.ldo, 64, 32)) return cudaErrorInvalidValue;
    auto kern = attn2_tc_kernel<kPolyPairs>;
    cudaError_t e = smem_attr_at_least(reinterpret_cast<const void*>(kern), kSmem2);
    if (e != cudaSuccess) return e;
    const int64_t items = int64_t(p.num_qt) * (p.nh / 2);
    const unsigned grid = static_cast<unsigned>(items < sm_count() ? items : sm_count());
    e = launch_pdl_plain(kern, dim3(grid), dim3(kThreads2), kSmem2, st, tm, tmo, p);
    if (e != cudaSuccess) return e;
    return counted_launch(1);
  }
  cudaError_t e = smem_attr_at_least(reinterpret_cast<const void*>(attn_tc_kernel), kSmem);
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>(int64_t(p.num_qt) * p.nh);
  e = launch_pdl_plain(attn_tc_kernel, dim3(grid), dim3(kThreads), kSmem, st, tm, p);
  if (e != cudaSuccess) return e;
  return counted_launch(1);
}

}  // namespace q3vl
