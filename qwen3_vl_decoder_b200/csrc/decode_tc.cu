// One-token-per-sequence decode on sm_100a: the KV cache writes of the
// prefill, the skinny projections (tcgen05, swap-AB, split-K; also the LM
// head's), the attention over the cache (tcgen05, split over the sequence),
// and the step that advances positions and lengths.
//
// Why a decoded token needs no re-run of the prompt: hf2q
// qwen3vl_text/forward.rs, module doc "Why no KV cache yet" (the generation
// loop may re-run the prefill over prompt + decoded tokens and keep the last
// row; the cache keeps the earlier rows' K/V instead). The per-token
// arithmetic is the prefill's (cortiq-engine qwen3te.rs,
// `Qwen3Encoder::encode_with_images` loop body; `Qwen3Encoder::norm_rope`;
// `rms_norm_into`; `silu`).
//
// Projections. With B <= 256 tokens the layer streams each weight matrix
// once, so the work is bound by HBM, not by the tensor cores. The weight
// matrix is the MMA's M operand (128 rows per tile, or 256 for gate/up whose
// packed rows interleave 128 gate and 128 up rows) and the tokens are its N
// operand (B rounded up to 16; TMA fills the missing rows with zeros), so
// one 128 x NB x 64 MMA consumes one 16 KB weight box. The K range of each
// row tile is split over up to 8 CTAs (about two CTAs per SM stream
// weights) that form one thread-block cluster: each CTA leaves its fp32
// partial tile in its shared memory, and after a cluster barrier the CTAs
// share out the tokens, each summing the partials of its tokens over DSMEM
// in split order and running the epilogue of the prefill's step: 1/rms,
// bias, per-head RMSNorm and MRoPE with the K/V rows written into the cache
// (QKV); residual add and the row sum of squares for the next norm
// (o-projection, down); SiLU(g) * u (gate/up); plain fp32 rows (the LM
// head's logits). The weights of a projection do not depend on the previous
// kernel, so each projection is launched as a programmatic dependent of it
// and starts streaming its weights before that kernel has finished.
#include "q3vl_device.cuh"
#include "q3vl_internal.h"

namespace q3vl {

namespace {

constexpr int kDecThreads = 192;     // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr int kDecMaxB = 256;
constexpr int kBK = 64;              // K elements per stage (one 128-byte row)
constexpr int kDecMaxSplits = 8;     // portable cluster size

__device__ __forceinline__ float bf16_to_f(__nv_bfloat16 v) { return __bfloat162float(v); }

struct DecGemmParams {
  int B, NB, R;          // tokens, MMA N (B rounded up to 16), 128-row blocks per tile
  int n_k, splits, stages;  // splits = cluster size (<= kDecMaxSplits)
  int32_t* err;
  // epilogue
  int64_t N;             // output columns (kQkv: q columns nh*128; kSwiGLU: I)
  __nv_bfloat16* out;    // [B][N]
  float* out_f32;        // [B][N] (kPlain)
  const __nv_bfloat16* resid;  // [B][N] (kResidual)
  float* rowsq_out;      // [B][N/128] (kResidual) or null
  const float* rowsq_in; // [B][rowsq_n] (kQkv, kSwiGLU) or null
  int rowsq_n;
  float rowsq_width;
  const float* inv;      // [B] 1/rms when rowsq_in is null
  float eps;
  const float* bias;     // [Ntot] or null (kQkv)
  const float* q_norm;   // [128] (kQkv)
  const float* k_norm;   // [128] (kQkv)
  const float2* cs;      // [B][64] (cos, sin) (kQkv)
  int n_heads, n_kv;
  __nv_bfloat16* k_cache;  // [n_seq][cap][nkv*128] (kQkv)
  __nv_bfloat16* v_cache;
  int64_t cap;
  int n_seq;
  const int32_t* seq;    // [B]
  const int32_t* len;    // [B]
};

// 1/rms of token j, by the whole warp: from the previous kernel's per-block
// row sums of squares (the lanes load them at once and add them in a fixed
// tree), or the precomputed 1/rms.
__device__ __forceinline__ float dec_row_scale(const DecGemmParams& p, int j, int lane) {
  if (p.rowsq_in != nullptr) {
    float ss = 0.f;
    for (int t = lane; t < p.rowsq_n; t += 32) ss += p.rowsq_in[j * p.rowsq_n + t];
    ss = warp_sum(ss);
    return 1.0f / sqrtf(ss / p.rowsq_width + p.eps);
  }
  return p.inv[j];
}

__device__ __forceinline__ bool dec_token_valid(const DecGemmParams& p, int j, int& slot,
                                                int& row) {
  slot = p.seq[j];
  row = p.len[j];
  return slot >= 0 && slot < p.n_seq && row >= 0 && static_cast<int64_t>(row) < p.cap;
}

// The global inputs of one token's epilogue (lane l's features l + 32 i):
// the 1/rms s (kQkv, kSwiGLU); bias and q/k-norm gain (kQkv) or the
// residual (kResidual) in a and b; the token's cos/sin pairs (kQkv).
struct DecEpiIn {
  float s;
  float a[4], b[4];
  float2 cs[2];
};

// Loads them. Everything it reads is final once griddepcontrol.wait has
// returned, so an epilogue warp that knows its token does this while the
// MMAs still run.
template <int EPI>
__device__ __forceinline__ void dec_epilogue_load(const DecGemmParams& p, int tile, int j, int lane,
                                                  DecEpiIn& in) {
  const int64_t c0 = int64_t(tile) * 128;
  if constexpr (EPI == static_cast<int>(Epi::kQkv)) {
    const bool is_q = tile < p.n_heads, is_k = !is_q && tile < p.n_heads + p.n_kv;
    const float* gsrc = is_q ? p.q_norm : p.k_norm;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      in.a[i] = p.bias != nullptr ? p.bias[c0 + lane + 32 * i] : 0.f;
      in.b[i] = (is_q || is_k) ? gsrc[lane + 32 * i] : 0.f;
    }
#pragma unroll
    for (int i = 0; i < 2; ++i)
      in.cs[i] = (is_q || is_k) ? p.cs[j * 64 + lane + 32 * i] : make_float2(1.f, 0.f);
    in.s = dec_row_scale(p, j, lane);
  } else if constexpr (EPI == static_cast<int>(Epi::kResidual)) {
    const bool ok = dcheck(j < p.B && c0 + 128 <= p.N, p.err, kWhereDbgDecodeStore);
    const __nv_bfloat16* r = p.resid + int64_t(j) * p.N + c0;
#pragma unroll
    for (int i = 0; i < 4; ++i) in.a[i] = ok ? bf16_to_f(r[lane + 32 * i]) : 0.f;
  } else if constexpr (EPI == static_cast<int>(Epi::kSwiGLU)) {
    in.s = dec_row_scale(p, j, lane);
  }
}

// Final epilogue of one token j of row tile `tile`, one warp: lane l holds
// features l + 32 i (i < 4) of each 128-row block r; `in` holds the loaded
// inputs of that token.
template <int EPI>
__device__ __forceinline__ void dec_epilogue_token(const DecGemmParams& p, int tile, int j,
                                                   int lane, float (&v)[2][4], const DecEpiIn& in) {
  if constexpr (EPI == static_cast<int>(Epi::kQkv)) {
    const int64_t c0 = int64_t(tile) * 128;
    const bool is_q = tile < p.n_heads, is_k = !is_q && tile < p.n_heads + p.n_kv;
#pragma unroll
    for (int i = 0; i < 4; ++i) v[0][i] = v[0][i] * in.s + in.a[i];
    if (is_q || is_k) {
      float ss = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) ss += v[0][i] * v[0][i];
      ss = warp_sum(ss);
      const float rn = 1.0f / sqrtf(ss * (1.0f / 128.0f) + p.eps);
#pragma unroll
      for (int i = 0; i < 4; ++i) v[0][i] *= rn * in.b[i];
      // split-half rotation: feature f pairs with f + 64 (i with i + 2)
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const float2 q = in.cs[i];
        const float a = v[0][i], b = v[0][i + 2];
        v[0][i] = a * q.x - b * q.y;
        v[0][i + 2] = a * q.y + b * q.x;
      }
    }
    if (is_q) {
      if (!dcheck(j < p.B && c0 + 128 <= p.N, p.err, kWhereDbgDecodeStore)) return;
      __nv_bfloat16* o = p.out + int64_t(j) * p.N + c0;
#pragma unroll
      for (int i = 0; i < 4; ++i) o[lane + 32 * i] = __float2bfloat16_rn(v[0][i]);
    } else {
      int slot, row;
      if (!dec_token_valid(p, j, slot, row)) {
        if (lane == 0) record_error(p.err, Q3VL_ERANGE, kWhereDecodeRange);
        return;
      }
      const int g = is_k ? tile - p.n_heads : tile - p.n_heads - p.n_kv;
      if (!dcheck(g >= 0 && g < p.n_kv && slot >= 0 && slot < p.n_seq && row >= 0 &&
                      row < p.cap, p.err, kWhereDbgDecodeStore))
        return;
      const int64_t dkv = int64_t(p.n_kv) * 128;
      __nv_bfloat16* dst = (is_k ? p.k_cache : p.v_cache) +
                           (int64_t(slot) * p.cap + row) * dkv + int64_t(g) * 128;
#pragma unroll
      for (int i = 0; i < 4; ++i) dst[lane + 32 * i] = __float2bfloat16_rn(v[0][i]);
    }
  } else if constexpr (EPI == static_cast<int>(Epi::kResidual)) {
    const int64_t c0 = int64_t(tile) * 128;
    if (!dcheck(j < p.B && c0 + 128 <= p.N, p.err, kWhereDbgDecodeStore)) return;
    __nv_bfloat16* o = p.out + int64_t(j) * p.N + c0;
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat16 ob = __float2bfloat16_rn(in.a[i] + v[0][i]);
      o[lane + 32 * i] = ob;
      const float f = bf16_to_f(ob);
      ss += f * f;
    }
    if (p.rowsq_out != nullptr) {
      ss = warp_sum(ss);
      if (lane == 0) p.rowsq_out[int64_t(j) * (p.N / 128) + tile] = ss;
    }
  } else if constexpr (EPI == static_cast<int>(Epi::kPlain)) {
    // fp32 rows of N outputs (the last tile may run past N)
    float* o = p.out_f32 + int64_t(j) * p.N + int64_t(tile) * 128;
    const int64_t left = p.N - int64_t(tile) * 128;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (lane + 32 * i < left) o[lane + 32 * i] = v[0][i];
  } else {  // kSwiGLU: block 0 = gate rows, block 1 = the matching up rows
    if (!dcheck(j < p.B && (int64_t(tile) + 1) * 128 <= p.N, p.err, kWhereDbgDecodeStore)) return;
    __nv_bfloat16* o = p.out + int64_t(j) * p.N + int64_t(tile) * 128;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      o[lane + 32 * i] = __float2bfloat16_rn(silu_fast(v[0][i] * in.s) * (v[1][i] * in.s));
  }
}

template <int EPI>
__global__ void __launch_bounds__(kDecThreads, 2)
decode_gemm_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                   DecGemmParams p) {
  constexpr int R = EPI == static_cast<int>(Epi::kSwiGLU) ? 2 : 1;
  constexpr uint32_t kABytes = 16384u * R;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const int S = p.stages;
  const uint32_t b_bytes = static_cast<uint32_t>(p.NB) * 128u;
  uint8_t* smA = smem;
  uint8_t* smB = smem + size_t(S) * kABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smB + size_t(S) * b_bytes);
  uint64_t* empty = full + S;
  uint64_t* acc_full = empty + S;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = static_cast<int>(blockIdx.x) / p.splits;
  const int split = static_cast<int>(blockIdx.x) % p.splits;
  const int k_lo = static_cast<int>(int64_t(split) * p.n_k / p.splits);
  const int k_hi = static_cast<int>(int64_t(split + 1) * p.n_k / p.splits);
  const int n = k_hi - k_lo;
  uint32_t tcols = 32;
  while (tcols < static_cast<uint32_t>(p.NB * R)) tcols <<= 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) { mbar_init(full + s, 1); mbar_init(empty + s, 1); }
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
  }
  if (warp == 1) {
    // At most a few dozen columns per CTA for small batches; if an earlier
    // grid still holds this SM's TMEM the allocation waits for it to finish.
    tmem_alloc(tmem_slot, tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_launch_dependents();
  // the first token this warp finishes in the split sum below
  const int pre_j = warp >= 2 ? split + (warp - 2) * p.splits : p.B;
  DecEpiIn pre{};

  if (warp == 0) {
    if (lane == 0) {
      const int32_t row0 = tile * 128 * R;
      const int pre = n < S ? n : S;
      // The weights do not depend on the previous kernel: stream the first
      // stages' boxes before waiting for it.
      for (int i = 0; i < pre; ++i) {
        mbar_arrive_expect_tx(full + i, kABytes + b_bytes);
        tma_load_2d(smA + size_t(i) * kABytes, &tmW, full + i, (k_lo + i) * kBK, row0);
      }
      griddep_wait();
      for (int i = 0; i < pre; ++i)
        tma_load_2d(smB + size_t(i) * b_bytes, &tmX, full + i, (k_lo + i) * kBK, 0);
      int issued = pre;
      for (int i = pre; i < n; ++i) {
        const int s = i % S;
        if (!mbar_wait(empty + s, ((i / S) - 1) & 1, p.err, kWhereDecodeProducer, abort_flag))
          break;
        mbar_arrive_expect_tx(full + s, kABytes + b_bytes);
        tma_load_2d(smA + size_t(s) * kABytes, &tmW, full + s, (k_lo + i) * kBK, row0);
        tma_load_2d(smB + size_t(s) * b_bytes, &tmX, full + s, (k_lo + i) * kBK, 0);
        issued = i + 1;
      }
      // every issued load lands before the CTA may exit
      for (int i = issued - S > 0 ? issued - S : 0; i < issued; ++i)
        mbar_wait(full + (i % S), (i / S) & 1, p.err, kWhereDecodeProducer, nullptr);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t d = tmem_base;
      const uint32_t idesc = idesc_bf16_f32(128, p.NB, false, false);
      bool ok = true;
      for (int i = 0; i < n; ++i) {
        const int s = i % S;
        if (!mbar_wait(full + s, (i / S) & 1, p.err, kWhereDecodeMma, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a0 = smem_u32(smA + size_t(s) * kABytes);
        const uint32_t b0 = smem_u32(smB + size_t(s) * b_bytes);
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          const uint64_t bd = sdesc_sw128(b0 + kk * 32, 16, 1024);
#pragma unroll
          for (int r = 0; r < R; ++r)
            umma_bf16_ss(d + r * p.NB, sdesc_sw128(a0 + r * 16384 + kk * 32, 16, 1024), bd, idesc,
                         (i | kk) != 0 ? 1u : 0u);
        }
        umma_commit(empty + s);
      }
      if (ok) umma_commit(acc_full);
      else *abort_flag = 1;
    }
    __syncwarp();
  } else {
    // epilogue warps: wait for the accumulator (TMEM lanes 32 q .. 32 q + 31
    // of warp q = warp % 4 are this tile's weight rows, columns are tokens),
    // loading the inputs of this warp's first token meanwhile
    griddep_wait();
    if (pre_j < p.B) dec_epilogue_load<EPI>(p, tile, pre_j, lane, pre);
    bool ok = true;
    if (lane == 0) ok = mbar_wait(acc_full, 0, p.err, kWhereDecodeEpilogue, abort_flag);
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    if (!ok) *abort_flag = 1;
  }
  // Split sum over the cluster: the splits of a row tile are one cluster.
  // Each CTA leaves its fp32 partial tile in its own (drained) stage ring;
  // after a cluster barrier CTA `split` finishes tokens j = split (mod
  // splits), reading every CTA's partial over DSMEM in split order. Every
  // thread of every CTA of the cluster passes the same cluster barriers.
  __syncthreads();  // all roles done: loads landed, MMAs committed or abandoned
  const bool run = *abort_flag == 0;
  tc_fence_after();
  float* red = reinterpret_cast<float*>(smem);
  const size_t ring = size_t(S) * (kABytes + b_bytes);
  int chunk = static_cast<int>(ring / (512u * R)) / 16 * 16;  // tokens per round
  if (chunk > p.NB) chunk = p.NB;
  const int rstride = 128 * R;
#pragma unroll 1
  for (int j0 = 0; j0 < p.B; j0 += chunk) {
    const int nj = p.B - j0 < chunk ? p.B - j0 : chunk;
    if (warp >= 2 && run) {
      const int q = warp & 3;
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(32 * q) << 16);
#pragma unroll 1
      for (int r = 0; r < R; ++r)
#pragma unroll 1
        for (int c0 = 0; c0 < nj; c0 += 16) {
          uint32_t u[16];
          tmem_ld16(tb + r * p.NB + j0 + c0, u);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 16; ++c)
            if (c0 + c < nj) red[(c0 + c) * rstride + r * 128 + 32 * q + lane] = __uint_as_float(u[c]);
        }
    }
    cluster_sync();  // every CTA's partials of this round are in its shared memory
    if (warp >= 2 && run) {
      const int e = warp - 2;
#pragma unroll 1
      for (int jj = split + e * p.splits; jj < nj; jj += 4 * p.splits) {
        float v[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        const uint32_t own = smem_u32(red + jj * rstride + lane);
        // every split's values requested before any is added: one DSMEM
        // round trip, then the sum in split order
        float w[kDecMaxSplits][R][4];
#pragma unroll
        for (int sp = 0; sp < kDecMaxSplits; ++sp) {
          const uint32_t ra = map_to_cta(own, static_cast<uint32_t>(sp < p.splits ? sp : 0));
#pragma unroll
          for (int r = 0; r < R; ++r)
#pragma unroll
            for (int i = 0; i < 4; ++i)
              w[sp][r][i] = sp < p.splits ? ld_dsmem_f32(ra + 4u * (r * 128 + 32 * i)) : 0.f;
        }
#pragma unroll
        for (int sp = 0; sp < kDecMaxSplits; ++sp)
#pragma unroll
          for (int r = 0; r < R; ++r)
#pragma unroll
            for (int i = 0; i < 4; ++i) v[r][i] += w[sp][r][i];
        if (j0 + jj == pre_j) {
          dec_epilogue_token<EPI>(p, tile, j0 + jj, lane, v, pre);
        } else {
          DecEpiIn in;
          dec_epilogue_load<EPI>(p, tile, j0 + jj, lane, in);
          dec_epilogue_token<EPI>(p, tile, j0 + jj, lane, v, in);
        }
      }
    }
    cluster_sync();  // no CTA overwrites or leaves its buffer while another may read it
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, tcols);
  }
}

// ---------------------------------------------------------------------------
// Attention of one new row per sequence over its cache (cortiq-engine
// qwen3te.rs `Qwen3Encoder::attention_gemm`, the last row of the causal
// softmax: every cached row and the new row itself, row maximum subtracted).
//
// The two contractions run on tcgen05 with the cache rows as the MMA's M
// operand, so the G <= 8 query heads of KV head g only pad N to 16:
//   S^T [128 rows x 16] = K_chunk [128 x 128] . Q^T        (K-major A and B)
//   O^T [128 dims x 16] = V_chunk^T [128 x 128] . P^T      (V as an MN-major A)
// K and V arrive by TMA (128-byte swizzle); thread t owns TMEM lane t (cache
// row t for the softmax, dimension t for the output).
//
// A work item is a contiguous range of 128-row chunks of one (token b, KV
// head g). The chunks of an item merge on the fly in registers (running max
// m, sum l and o per head, base-2 exponents with log2(e)/sqrt(128) applied to
// S in fp32). The cached rows below len[b] do not change during a decode
// call, so each CTA requests its first chunks before waiting for the QKV
// projection and patches the new row in after the wait. Two forms:
//   - small batches: the cs splits of a (b, g) are one cluster, one CTA per
//     SM with a ring of kAttnMaxBuf chunk stages; the chunks in the ring go
//     through one S / softmax / O pass together, and the cs partials merge
//     over DSMEM;
//   - otherwise three CTAs share an SM with one stage each, about one item
//     per SM; a (b, g) with one item writes o / l, else the last item of the
//     group to finish (a ticket counter) merges the partials from global
//     memory.
// Either merge computes
//   o = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s,  M = max_s m_s.
// ---------------------------------------------------------------------------
constexpr int kAttnCH = 128;    // cache rows per chunk (the MMA's M)
constexpr int kAttnRows = 130;  // per (b, g, h): o[128], m, l, each over the split slots
constexpr int kTcThreads = 128;
constexpr int kAttnBlk = 128 * 64 * 2;     // one [128 rows x 64] bf16 swizzle block (16 KB)
constexpr int kAttnKV = 4 * kAttnBlk;      // K (2 blocks) + V (2 blocks) of one item
constexpr int kAttnSmall = 16 * 64 * 2;    // one [16 rows x 64] bf16 swizzle block (2 KB)

struct DecAttnTcParams {
  const __nv_bfloat16* q;        // [B][nh*128]
  const __nv_bfloat16* kc;       // the caches [n_seq][cap][nkv*128]
  const __nv_bfloat16* vc;
  int64_t cap;
  int n_seq;
  const int32_t* seq;
  const int32_t* len;
  int B, nkv;
  int nc_pad;                    // chunk slots per (b, g): ceil(cap / kAttnCH), rounded up to 4
  float scale_log2;
  __nv_bfloat16* o;              // [B][nh*128]
  float* part;                   // [B][nkv][G][kAttnRows][nc_pad]
  uint32_t* tickets;             // [B][nkv], zero between launches
  int32_t* err;
  int nsplit;                    // most splits of one (b, g); nc_pad = nsplit rounded up to 4
  int nbuf;                      // K/V stages in shared memory (1 .. kAttnMaxBuf)
  int cs;                        // > 0: the nsplit = cs splits of a (b, g) form one cluster
};

constexpr int kAttnMaxBuf = 3;
constexpr int kAttnMaxCs = 16;  // most splits of a (b, g) in one cluster

// Byte offset of element (row r, column c) in a 128-byte-swizzled tile of
// 64-column blocks with `block_bytes` per block (rows of 128 bytes).
__device__ __forceinline__ uint32_t sw128_off(int r, int c, uint32_t block_bytes) {
  return static_cast<uint32_t>(c >> 6) * block_bytes + static_cast<uint32_t>(r) * 128u +
         ((static_cast<uint32_t>((c & 63) >> 3) ^ static_cast<uint32_t>(r & 7)) << 4) +
         static_cast<uint32_t>(c & 7) * 2u;
}

template <int G>
__host__ __device__ constexpr size_t attn_tc_smem_bytes(int nc_pad, int nbuf) {
  return 1024 + size_t(nbuf) * kAttnKV + 2 * kAttnSmall +        // K/V stages, Q
         (nbuf > 1 ? size_t(nbuf) * 2 * kAttnSmall : 0) +         // P (aliases Q if nbuf = 1)
         size_t(2) * G * nc_pad * 4 + size_t(4) * 8 * 4 * 2 +   // merge weights; warp partials
         size_t(G) * 4 + (4 * kDecMaxB + 2) * 4 +               // den; items, slots, lengths
         size_t(G) * kAttnRows * 4 + 128;                        // cluster partial; barriers
}

// NBUF (= p.nbuf) K/V stages: 1 for three CTAs per SM, kAttnMaxBuf for one.
template <int G, int NBUF>
__global__ void __launch_bounds__(kTcThreads, 3)
decode_attn_tc_kernel(const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, DecAttnTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* s_kv = sm;                                      // [nbuf] x (K0 K1 V0 V1)
  uint8_t* s_q = s_kv + size_t(NBUF) * kAttnKV;            // [16 x 128] as 2 blocks
  // P^T [16 x 128] per chunk of a batch. With one stage it reuses Q's tile
  // (Q's reader, the S MMA, completed before P is written, and P's reader,
  // the O MMA, before the next chunk rewrites Q).
  constexpr bool alias_q = NBUF == 1;
  uint8_t* s_pt = alias_q ? s_q : s_q + 2 * kAttnSmall;   // [nbuf] tiles
  float* s_w = reinterpret_cast<float*>(s_q + 2 * kAttnSmall * (alias_q ? 1 : 1 + NBUF));  // [G][nc_pad]
  float* s_cl = s_w + G * p.nc_pad;                        // [G][nc_pad]
  float* s_wm = s_cl + G * p.nc_pad;                       // [4 warps][8]
  float* s_wl = s_wm + 32;                                 // [4 warps][8]
  float* s_den = s_wl + 32;                                // [G]
  int* s_nc = reinterpret_cast<int*>(s_den + G);           // [kDecMaxB] splits per token
  int* s_pref = s_nc + kDecMaxB;                           // [kDecMaxB + 1]
  int* s_last = s_pref + kDecMaxB + 1;
  int* s_slot = s_last + 1;                                // [kDecMaxB] seq[b], or -1 if invalid
  int* s_len = s_slot + kDecMaxB;                          // [kDecMaxB] len[b]
  float* s_part = reinterpret_cast<float*>(s_len + kDecMaxB);  // [G][kAttnRows]: o[128], m, l
  uint64_t* bars = reinterpret_cast<uint64_t*>(
      (reinterpret_cast<uintptr_t>(s_part + G * kAttnRows) + 7) & ~uintptr_t(7));
  uint64_t* kv_full = bars;                                // [kAttnMaxBuf]
  uint64_t* s_full = bars + kAttnMaxBuf;
  uint64_t* o_full = s_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_full + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int nh = G * p.nkv;
  constexpr int nbuf = NBUF;
  constexpr uint32_t kOcol = 16 * NBUF, kTmemCols = NBUF == 1 ? 32 : 64;
  if (t == 0) {
    for (int i = 0; i < kAttnMaxBuf; ++i) mbar_init(kv_full + i, 1);
    mbar_init(s_full, 1);
    mbar_init(o_full, 1);
    *s_abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);  // S^T of batch chunk i in columns 16 i .., O^T at kOcol
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_field = static_cast<uint32_t>(warp * 32) << 16;

  griddep_launch_dependents();
  // items: (token b, KV head g, split s of b's chunks); each split walks a
  // contiguous range of 128-row chunks. Lengths and slots are inputs of the
  // decode call, not outputs of the kernel before this one. In cluster mode
  // every token has cs splits (some may get no chunk) and CTA i is item i.
  for (int b = t; b < p.B; b += kTcThreads) {
    const int slot = p.seq[b], L = p.len[b];
    const bool ok = slot >= 0 && slot < p.n_seq && L >= 0 && static_cast<int64_t>(L) < p.cap;
    const int nc = ok ? (L + kAttnCH) / kAttnCH : 0;  // chunks of rows 0..L
    s_nc[b] = p.cs > 0 ? p.cs : (nc < p.nsplit ? nc : p.nsplit);
    s_slot[b] = ok ? slot : -1;
    s_len[b] = ok ? L : 0;
  }
  __syncthreads();
  if (warp == 0) {
    // exclusive prefix of items per token: lane l owns tokens 8l .. 8l+7
    int loc[8], sum = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int b = 8 * lane + i;
      loc[i] = sum;
      sum += b < p.B ? p.nkv * s_nc[b] : 0;
    }
    int inc = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    const int excl = inc - sum;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int b = 8 * lane + i;
      if (b < p.B) s_pref[b] = excl + loc[i];
    }
    if (lane == 31) s_pref[p.B] = inc;
  }
  __syncthreads();
  const int total = s_pref[p.B];
  // the item `it`: token, KV head, split and its chunk range (empty for a
  // token whose slot or length is out of range)
  auto item = [&](int it, int& b, int& g, int& c0, int& c1, int& splits, int& sidx) {
    int lo = 0, hi = p.B - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_pref[mid] <= it) lo = mid;
      else hi = mid - 1;
    }
    b = lo;
    splits = s_nc[b];
    const int loc = it - s_pref[b];
    g = loc / splits;
    sidx = loc % splits;
    const int nc = s_slot[b] >= 0 ? (s_len[b] + kAttnCH) / kAttnCH : 0;
    c0 = static_cast<int>(int64_t(sidx) * nc / splits);
    c1 = static_cast<int>(int64_t(sidx + 1) * nc / splits);
  };
  // Loads run ahead of the chunk being computed by up to nbuf chunks, along
  // this CTA's sequence of (item, chunk); only thread 0 walks it.
  int l_it = blockIdx.x, l_b = 0, l_g = 0, l_c = 0, l_c1 = 0, n_issued = 0;
  auto loader_seek = [&]() {  // from (l_it, l_c) to the next chunk that exists
    while (l_it < total && l_c >= l_c1) {
      int sp, si, c0;
      item(l_it, l_b, l_g, c0, l_c1, sp, si);
      l_c = c0;
      if (l_c >= l_c1) l_it += gridDim.x;
    }
  };
  auto load_next = [&]() {
    if (l_it >= total) return;
    const int st = n_issued % nbuf;
    uint8_t* dst = s_kv + size_t(st) * kAttnKV;
    const int32_t y = static_cast<int32_t>(int64_t(s_slot[l_b]) * p.cap + int64_t(l_c) * kAttnCH);
    mbar_arrive_expect_tx(kv_full + st, kAttnKV);
    tma_load_2d(dst, &tmK, kv_full + st, l_g * 128, y);
    tma_load_2d(dst + kAttnBlk, &tmK, kv_full + st, l_g * 128 + 64, y);
    tma_load_2d(dst + 2 * kAttnBlk, &tmV, kv_full + st, l_g * 128, y);
    tma_load_2d(dst + 3 * kAttnBlk, &tmV, kv_full + st, l_g * 128 + 64, y);
    ++n_issued;
    ++l_c;
    if (l_c >= l_c1) {
      l_it += gridDim.x;
      loader_seek();
    }
  };
  // The cached rows below len[b] were written before this decode call and
  // do not change during it, so the first nbuf chunks are loaded before
  // waiting for the QKV projection; row len[b] (this token's K/V, written
  // by that projection) is patched in after the wait.
  if (t == 0) {
    loader_seek();
    for (int i = 0; i < nbuf; ++i) load_next();
  }
  griddep_wait();

  constexpr uint32_t idesc_s = idesc_bf16_f32(128, 16, false, false);
  constexpr uint32_t idesc_o = idesc_bf16_f32(128, 16, true, false);
  int k = 0;   // chunks this CTA has processed: the phase of the stage barriers
  int bi = 0;  // batches this CTA has processed: the phase of s_full and o_full
  for (int it = blockIdx.x; it < total; it += gridDim.x) {
    // a wait that timed out anywhere in the block ends the walk for all
    // threads (read after the previous chunk's last barrier, written before
    // it); in cluster mode the one item still reaches both cluster barriers
    if (*s_abort && p.cs == 0) break;
    int b, g, c0, c1, splits, s;
    item(it, b, g, c0, c1, splits, s);
    const int L1 = s_len[b] + 1;
    float m_run[G], l_run[G], o_run[G];
#pragma unroll
    for (int h = 0; h < G; ++h) { m_run[h] = -INFINITY; l_run[h] = 0.f; o_run[h] = 0.f; }

    auto build_q = [&]() {
      // Q^T operand: rows h < G are the query heads of KV head g, rows G..15 zero
      for (int ch = t; ch < 16 * 16; ch += kTcThreads) {
        const int h = ch >> 4, cc = ch & 15;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (h < G)
          v = *reinterpret_cast<const uint4*>(p.q + int64_t(b) * nh * 128 +
                                              int64_t(g * G + h) * 128 + cc * 8);
        *reinterpret_cast<uint4*>(s_q + sw128_off(h, cc * 8, kAttnSmall)) = v;
      }
    };
    if (!alias_q) build_q();
    // Chunks go through in batches of up to nbuf (the stages holding them):
    // one S MMA per chunk, one softmax over all the batch's rows, one O MMA
    // per chunk accumulating into O^T, so the batch pays the chain's latency
    // once.
    for (int c = c0; c < c1;) {
      if (*s_abort) break;
      const int nb = min(nbuf, c1 - c);
      // row len[b]: this token's K and V, from the cache row the QKV
      // projection wrote (read after the wait); it lies in chunk cn
      const int cn = (L1 - 1) / kAttnCH, r_new = L1 - 1 - cn * kAttnCH;
      const bool has_new = cn >= c && cn < c + nb;
      uint4 kv_new = make_uint4(0, 0, 0, 0);
      if (has_new && t < 32) {
        const int64_t row = int64_t(s_slot[b]) * p.cap + (L1 - 1);
        const __nv_bfloat16* src = (t < 16 ? p.kc : p.vc) + row * (int64_t(p.nkv) * 128) + g * 128;
        kv_new = *reinterpret_cast<const uint4*>(src + (t & 15) * 8);
      }
      if (alias_q) build_q();
      for (int i = 0; i < nb; ++i)
        if (!mbar_wait(kv_full + (k + i) % nbuf, ((k + i) / nbuf) & 1, p.err, kWhereDecodeAttn,
                       s_abort))
          *s_abort = 1;
      if (has_new && t < 32)
        *reinterpret_cast<uint4*>(s_kv + size_t((k + cn - c) % nbuf) * kAttnKV +
                                  (t < 16 ? 0 : 2 * kAttnBlk) +
                                  sw128_off(r_new, (t & 15) * 8, kAttnBlk)) = kv_new;
      // rows past the sequence hold whatever the cache had: zero V there (P is
      // zero there, but 0 * NaN would not be); only chunk cn can be partial
      if (has_new) {
        uint8_t* kvn = s_kv + size_t((k + cn - c) % nbuf) * kAttnKV;
        for (int ch = t; ch < (kAttnCH - 1 - r_new) * 16; ch += kTcThreads) {
          const int r = r_new + 1 + (ch >> 4), cc = ch & 15;
          *reinterpret_cast<uint4*>(kvn + 2 * kAttnBlk + (cc >> 3) * kAttnBlk + r * 128 +
                                    (cc & 7) * 16) = make_uint4(0, 0, 0, 0);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();
      if (t == 0 && *s_abort == 0) {
        tc_fence_after();
        const uint32_t q0 = smem_u32(s_q);
        for (int i = 0; i < nb; ++i) {
          const uint32_t k0 = smem_u32(s_kv + size_t((k + i) % nbuf) * kAttnKV);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_bf16_ss(tmem + 16 * i,
                         sdesc_sw128(k0 + (kk >> 2) * kAttnBlk + (kk & 3) * 32, 16, 1024),
                         sdesc_sw128(q0 + (kk >> 2) * kAttnSmall + (kk & 3) * 32, 16, 1024),
                         idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(s_full);
      }
      // softmax over the batch's rows: thread t holds row t of every chunk,
      // the scores of every head
      float sc[NBUF][16];
      {
        bool w_ok = true;
        if (lane == 0) w_ok = mbar_wait(s_full, bi & 1, p.err, kWhereDecodeAttn, s_abort);
        w_ok = __shfl_sync(0xffffffffu, w_ok ? 1 : 0, 0) != 0;
        if (!w_ok) *s_abort = 1;
        tc_fence_after();
#pragma unroll
        for (int i = 0; i < NBUF; ++i) {
          if (i < nb) {
            uint32_t u[16];
            tmem_ld16(tmem + lane_field + 16 * i, u);
            tmem_ld_wait();
            const bool valid = (c + i) * kAttnCH + t < L1;
#pragma unroll
            for (int h = 0; h < 16; ++h)
              sc[i][h] = valid ? __uint_as_float(u[h]) * p.scale_log2 : -INFINITY;
          } else {
#pragma unroll
            for (int h = 0; h < 16; ++h) sc[i][h] = -INFINITY;
          }
        }
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float v = sc[0][h];
#pragma unroll
        for (int i = 1; i < NBUF; ++i) v = fmaxf(v, sc[i][h]);
        const float wm = warp_max(v);
        if (lane == 0) s_wm[warp * 8 + h] = wm;
      }
      __syncthreads();
      float mh[G];
#pragma unroll
      for (int h = 0; h < G; ++h)
        mh[h] = fmaxf(fmaxf(s_wm[h], s_wm[8 + h]), fmaxf(s_wm[16 + h], s_wm[24 + h]));
#pragma unroll
      for (int i = 0; i < NBUF; ++i) {
        if (i < nb) {
          float pr[G];
#pragma unroll
          for (int h = 0; h < G; ++h)
            pr[h] = sc[i][h] == -INFINITY ? 0.f : ex2_approx(sc[i][h] - mh[h]);
          // P^T operand of chunk i: row h, column t (zero for h >= G)
          uint8_t* pt = s_pt + size_t(alias_q ? 0 : i) * 2 * kAttnSmall;
#pragma unroll
          for (int h = 0; h < 16; ++h) {
            const __nv_bfloat16 v = __float2bfloat16_rn(h < G ? pr[h < G ? h : 0] : 0.f);
            *reinterpret_cast<__nv_bfloat16*>(pt + sw128_off(h, t, kAttnSmall)) = v;
          }
#pragma unroll
          for (int h = 0; h < G; ++h) sc[i][h] = pr[h];
        }
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float v = 0.f;
#pragma unroll
        for (int i = 0; i < NBUF; ++i)
          if (i < nb) v += sc[i][h];
        const float ws = warp_sum(v);
        if (lane == 0) s_wl[warp * 8 + h] = ws;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();
      if (t == 0 && *s_abort == 0) {
        tc_fence_after();
        for (int i = 0; i < nb; ++i) {
          const uint32_t v0 = smem_u32(s_kv + size_t((k + i) % nbuf) * kAttnKV + 2 * kAttnBlk);
          const uint32_t p0 = smem_u32(s_pt + size_t(alias_q ? 0 : i) * 2 * kAttnSmall);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_bf16_ss(tmem + kOcol, sdesc_sw128(v0 + kk * 2048, kAttnBlk, 1024),
                         sdesc_sw128(p0 + (kk >> 2) * kAttnSmall + (kk & 3) * 32, 16, 1024),
                         idesc_o, (i | kk) > 0 ? 1u : 0u);
        }
        umma_commit(o_full);
      }
      float acc[G];
      {
        bool w_ok = true;
        if (lane == 0) w_ok = mbar_wait(o_full, bi & 1, p.err, kWhereDecodeAttn, s_abort);
        w_ok = __shfl_sync(0xffffffffu, w_ok ? 1 : 0, 0) != 0;
        if (!w_ok) *s_abort = 1;
        tc_fence_after();
        uint32_t u[16];
        tmem_ld16(tmem + lane_field + kOcol, u);
        tmem_ld_wait();
#pragma unroll
        for (int h = 0; h < G; ++h) acc[h] = __uint_as_float(u[h]);
      }
      tc_fence_before();
      __syncthreads();  // TMEM and the batch's stages are free
      // the stages go to the chunks nbuf ahead
      if (t == 0 && *s_abort == 0)
        for (int i = 0; i < nb; ++i) load_next();
      // merge the batch into the split's running (m, l, o)
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float lj = s_wl[h] + s_wl[8 + h] + s_wl[16 + h] + s_wl[24 + h];
        const float M = fmaxf(m_run[h], mh[h]);
        const float wa = ex2_approx(m_run[h] - M), wb = ex2_approx(mh[h] - M);
        o_run[h] = o_run[h] * wa + acc[h] * wb;
        l_run[h] = l_run[h] * wa + lj * wb;
        m_run[h] = M;
      }
      c += nb;
      k += nb;
      ++bi;
    }
    if (*s_abort && p.cs == 0) break;
    __nv_bfloat16* ob = p.o + int64_t(b) * nh * 128 + int64_t(g) * G * 128;
    if (p.cs > 0) {
      // Cluster merge: the cs CTAs of the cluster are the cs splits of
      // (b, g). Each leaves (o, m, l) of every head in its shared memory;
      // after a cluster barrier CTA r finishes outputs r*128 + t, r*128 +
      // t + 128 cs, ... of the G*128, reading the cs partials over DSMEM in
      // split order; a second barrier keeps every CTA's partial alive until
      // all reads are done. Every CTA passes both barriers.
#pragma unroll
      for (int h = 0; h < G; ++h) {
        s_part[h * kAttnRows + t] = o_run[h];
        if (t == 0) {
          s_part[h * kAttnRows + 128] = m_run[h];
          s_part[h * kAttnRows + 129] = l_run[h];
        }
      }
      cluster_sync();
      const bool tok_ok = s_slot[b] >= 0;
      if (tok_ok && *s_abort == 0) {
        const uint32_t r = cluster_ctarank();
        for (int idx = static_cast<int>(r) * 128 + t; idx < G * 128; idx += p.cs * 128) {
          const int h = idx >> 7, d = idx & 127;
          const uint32_t base = smem_u32(s_part + h * kAttnRows);
          // every split's (m, l, o) requested before any is used: one DSMEM
          // round trip, then the merge in split order
          float ms[kAttnMaxCs], ls[kAttnMaxCs], os[kAttnMaxCs];
#pragma unroll
          for (int sp = 0; sp < kAttnMaxCs; ++sp) {
            const uint32_t ra = map_to_cta(base, static_cast<uint32_t>(sp < p.cs ? sp : 0));
            ms[sp] = sp < p.cs ? ld_dsmem_f32(ra + 128 * 4) : -INFINITY;
            ls[sp] = sp < p.cs ? ld_dsmem_f32(ra + 129 * 4) : 0.f;
            os[sp] = sp < p.cs ? ld_dsmem_f32(ra + 4u * d) : 0.f;
          }
          float M = -INFINITY;
#pragma unroll
          for (int sp = 0; sp < kAttnMaxCs; ++sp) M = fmaxf(M, ms[sp]);
          float num = 0.f, den = 0.f;
#pragma unroll
          for (int sp = 0; sp < kAttnMaxCs; ++sp) {
            if (ms[sp] == -INFINITY) continue;  // a split without chunks, or past cs
            const float w = ex2_approx(ms[sp] - M);
            num = fmaf(w, os[sp], num);
            den = fmaf(w, ls[sp], den);
          }
          if (dcheck(int64_t(b) < p.B, p.err, kWhereDbgDecodeStore))
            ob[h * 128 + d] = __float2bfloat16_rn(num / den);
        }
      }
      cluster_sync();
      if (*s_abort) break;
      continue;
    }
    float* pb = p.part + (size_t(b) * p.nkv + g) * G * kAttnRows * size_t(p.nc_pad);
    if (splits == 1) {
#pragma unroll
      for (int h = 0; h < G; ++h) ob[h * 128 + t] = __float2bfloat16_rn(o_run[h] / l_run[h]);
    } else {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float* ph = pb + size_t(h) * kAttnRows * p.nc_pad;
        ph[size_t(t) * p.nc_pad + s] = o_run[h];
        if (t == 0) {
          ph[size_t(128) * p.nc_pad + s] = m_run[h];
          ph[size_t(129) * p.nc_pad + s] = l_run[h];
        }
      }
      __threadfence();
      __syncthreads();
      if (t == 0) {
        const uint32_t kt = atomicAdd(p.tickets + b * p.nkv + g, 1u);
        *s_last = kt == static_cast<uint32_t>(splits - 1);
        if (*s_last) p.tickets[b * p.nkv + g] = 0;
      }
      __syncthreads();
      if (*s_last) {
        __threadfence();
        // split maxima and sums in shared memory, then every thread merges
        // one dimension of every head with independent 16-byte loads
        for (int idx = t; idx < G * splits; idx += kTcThreads) {
          const int h = idx / splits, cc = idx % splits;
          s_w[h * p.nc_pad + cc] = __ldcg(pb + (size_t(h) * kAttnRows + 128) * p.nc_pad + cc);
          s_cl[h * p.nc_pad + cc] = __ldcg(pb + (size_t(h) * kAttnRows + 129) * p.nc_pad + cc);
        }
        __syncthreads();
        if (t < G) {
          float M = -INFINITY;
          for (int cc = 0; cc < splits; ++cc) M = fmaxf(M, s_w[t * p.nc_pad + cc]);
          float den = 0.f;
          for (int cc = 0; cc < splits; ++cc) {
            const float w = ex2_approx(s_w[t * p.nc_pad + cc] - M);
            s_w[t * p.nc_pad + cc] = w;
            den = fmaf(w, s_cl[t * p.nc_pad + cc], den);
          }
          s_den[t] = den;
        }
        __syncthreads();
        float num[G];
#pragma unroll
        for (int h = 0; h < G; ++h) num[h] = 0.f;
#pragma unroll 4
        for (int c4 = 0; c4 < splits; c4 += 4) {
          float4 v[G];
#pragma unroll
          for (int h = 0; h < G; ++h)
            v[h] = __ldcg(reinterpret_cast<const float4*>(
                pb + (size_t(h) * kAttnRows + t) * p.nc_pad + c4));
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const float* wv = s_w + h * p.nc_pad + c4;
            const float vv[4] = {v[h].x, v[h].y, v[h].z, v[h].w};
#pragma unroll
            for (int u = 0; u < 4; ++u)
              if (c4 + u < splits) num[h] = fmaf(wv[u], vv[u], num[h]);
          }
        }
#pragma unroll
        for (int h = 0; h < G; ++h) ob[h * 128 + t] = __float2bfloat16_rn(num[h] / s_den[h]);
      }
    }
    __syncthreads();  // shared buffers are reused by the next item
  }
  // every issued K/V load lands before the block exits: the loads not yet
  // waited for are those of the last min(nbuf, n_issued) stages
  if (t == 0)
    for (int i = n_issued - nbuf; i < n_issued; ++i)
      if (i >= 0) mbar_wait(kv_full + i % nbuf, (i / nbuf) & 1, p.err, kWhereDecodeAttn, nullptr);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// K/V rows of a prefill (the k and v column ranges of the [S, Ntot] QKV
// buffer) into rows row0 .. row0+S-1 of a cache, 16 bytes per thread.
__global__ void kv_store_kernel(const uint4* __restrict__ qkv, int64_t S, int64_t ntot8,
                                int64_t dq8, int64_t dkv8, uint4* __restrict__ k,
                                uint4* __restrict__ v, int64_t row0) {
  const int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= S * 2 * dkv8) return;
  const int64_t r = idx / (2 * dkv8), c = idx % (2 * dkv8);
  const uint4 val = qkv[r * ntot8 + dq8 + c];
  if (c < dkv8) k[(row0 + r) * dkv8 + c] = val;
  else v[(row0 + r) * dkv8 + (c - dkv8)] = val;
}

// Next text token: len[b] + 1, and every position axis + 1.
__global__ void decode_advance_kernel(int B, int32_t* __restrict__ pos, int32_t* __restrict__ len) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  len[b] += 1;
  pos[b] += 1;
  pos[B + b] += 1;
  pos[2 * B + b] += 1;
}

}  // namespace

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
DecSched dec_gemm_sched(int64_t rows, int64_t K, int B, int R) {
  DecSched s{};
  s.R = R;
  s.NB = (B + 15) / 16 * 16;
  s.tiles = static_cast<int>((rows + 128 * R - 1) / (128 * R));  // TMA zero-fills past `rows`
  s.n_k = static_cast<int>((K + kBK - 1) / kBK);
  const size_t stage = size_t(16384) * R + size_t(s.NB) * 128;
  // up to ~110 KB of stages, so that two CTAs share an SM
  int st = static_cast<int>(size_t(110 * 1024) / stage);
  s.stages = st < 2 ? 2 : (st > 8 ? 8 : st);
  s.smem = 1024 + size_t(s.stages) * stage + size_t(2 * s.stages + 1) * 8 + 16;
  uint32_t tcols = 32;
  while (tcols < static_cast<uint32_t>(s.NB * R)) tcols <<= 1;
  const int resident = (s.smem <= 113 * 1024 && 2 * tcols <= 512) ? 2 : 1;
  // about `resident` CTAs per SM, one wave (measured faster than one CTA per
  // SM with room for the next kernel's CTA); the splits of a tile form one
  // cluster, at most the portable cluster size
  int splits = resident * sm_count() / (s.tiles > 0 ? s.tiles : 1);
  if (splits > kDecMaxSplits) splits = kDecMaxSplits;
  if (splits > s.n_k) splits = s.n_k;
  // A cluster must fit inside one GPC. Counting each GPC as 16 SMs (a
  // B200 has 8 GPCs of 148 SMs in all), lower the split count until every
  // row tile's cluster is resident in the first wave.
  const int gpcs = sm_count() / 18 > 1 ? sm_count() / 18 : 1;
  while (splits > 1 && (16 * resident / splits) * gpcs < s.tiles) --splits;
  s.splits = splits < 1 ? 1 : splits;
  return s;
}

DecLayout dec_layout(const q3vl_config& c, int B, int64_t cap) {
  DecLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  const int64_t H = c.hidden, I = c.intermediate, Dq = q_dim(c);
  L.cos_sin = take(size_t(B) * kHalf * 2 * sizeof(float));
  L.inv = take(size_t(B) * sizeof(float));
  L.rowsq_h = take(size_t(B) * (H / 128) * sizeof(float));
  L.rowsq_x = take(size_t(B) * (H / 128) * sizeof(float));
  L.q = take(size_t(B) * Dq * 2);
  L.o = take(size_t(B) * Dq * 2);
  L.h = take(size_t(B) * H * 2);
  L.act = take(size_t(B) * I * 2);
  const int G = c.n_heads / c.n_kv_heads;
  // partial slots per (b, g): at most one per 128-row chunk of a slot
  const int64_t nc_pad = ((cap + kAttnCH - 1) / kAttnCH + 3) / 4 * 4;
  L.att_part = take(size_t(B) * c.n_kv_heads * G * kAttnRows * nc_pad * sizeof(float));
  // the ticket region comes last; each decode call clears it once
  L.att_tickets = take(size_t(B) * c.n_kv_heads * sizeof(uint32_t));
  L.total = off;
  return L;
}

namespace {

// Launch as a programmatic dependent of the previous kernel in the stream,
// optionally in clusters of `cluster_x` CTAs along x.
template <typename K, typename... Args>
cudaError_t launch_pdl(K kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       int cluster_x, Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  int n = 1;
  if (cluster_x > 1) {
    at[1].id = cudaLaunchAttributeClusterDimension;
    at[1].val.clusterDim.x = static_cast<unsigned>(cluster_x);
    at[1].val.clusterDim.y = 1;
    at[1].val.clusterDim.z = 1;
    n = 2;
  }
  cfg.attrs = at;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

template <int EPI>
cudaError_t launch_dec_epi(const DecGemmArgs& a, int R, cudaStream_t st) {
  const DecSched s = dec_gemm_sched(a.rows, a.K, a.B, R);
  {
    const cudaError_t e =
        smem_attr_at_least(reinterpret_cast<const void*>(decode_gemm_kernel<EPI>), s.smem);
    if (e != cudaSuccess) return e;
  }
  CUtensorMap tmW, tmX;
  if (!make_tmap_bf16(&tmW, a.W, a.rows, a.K, a.K, kBK, 128 * R) ||
      !make_tmap_bf16(&tmX, a.X, a.B, a.K, a.K, kBK, s.NB))
    return cudaErrorInvalidValue;
  DecGemmParams p{};
  p.B = a.B; p.NB = s.NB; p.R = R;
  p.n_k = s.n_k; p.splits = s.splits; p.stages = s.stages;
  p.err = device_error_ptr();
  p.N = a.N; p.out = static_cast<__nv_bfloat16*>(a.out);
  p.out_f32 = static_cast<float*>(a.out);
  p.resid = static_cast<const __nv_bfloat16*>(a.resid);
  p.rowsq_out = a.rowsq_out; p.rowsq_in = a.rowsq_in; p.rowsq_n = a.rowsq_n;
  p.rowsq_width = a.rowsq_width; p.inv = a.inv; p.eps = a.eps;
  p.bias = a.bias; p.q_norm = a.q_norm; p.k_norm = a.k_norm;
  p.cs = reinterpret_cast<const float2*>(a.cos_sin);
  p.n_heads = a.n_heads; p.n_kv = a.n_kv;
  p.k_cache = static_cast<__nv_bfloat16*>(a.k_cache);
  p.v_cache = static_cast<__nv_bfloat16*>(a.v_cache);
  p.cap = a.cap; p.n_seq = a.n_seq; p.seq = a.seq; p.len = a.len;
  const cudaError_t e = launch_pdl(decode_gemm_kernel<EPI>, dim3(s.tiles * s.splits),
                                   dim3(kDecThreads), s.smem, st, s.splits, tmW, tmX, p);
  if (e != cudaSuccess) return e;
  return counted_launch(1);
}

template <int G>
cudaError_t launch_attn_tc_g(const CUtensorMap& tmK, const CUtensorMap& tmV, DecAttnTcParams p,
                             int64_t groups, int64_t max_nc, cudaStream_t st) {
  const void* fn = reinterpret_cast<const void*>(decode_attn_tc_kernel<G, kAttnMaxBuf>);
  // With at least two SMs per (b, g) (small batches) the splits of a (b, g)
  // form one cluster of cs <= 16 CTAs, one CTA per SM with kAttnMaxBuf K/V
  // stages, and merge over DSMEM; cs is the largest size whose clusters are
  // all resident at once. Otherwise three CTAs share an SM with one stage
  // each, items fill the CTA slots, and the last split of a (b, g) to finish
  // merges the partials from global memory; there, about one item per SM
  // (measured faster than filling all three slots: fewer partials to merge,
  // none at all from 148 (b, g) on). Never more splits than the chunks of
  // the longest sequence.
  {
    const cudaError_t e = allow_nonportable_clusters(fn);
    if (e != cudaSuccess) return e;
  }
  int64_t cs = sm_count() / groups;
  if (cs > kAttnMaxCs) cs = kAttnMaxCs;
  if (cs > max_nc) cs = max_nc;
  p.cs = 0;
  for (; cs >= 2; --cs) {
    const int nc_pad = static_cast<int>((cs + 3) / 4 * 4);
    const size_t smem = attn_tc_smem_bytes<G>(nc_pad, kAttnMaxBuf);
    cudaError_t e = smem_attr_at_least(fn, smem);
    if (e != cudaSuccess) return e;
    int clusters = 0;
    e = max_active_clusters(fn, kTcThreads, smem, static_cast<int>(cs), &clusters);
    if (e != cudaSuccess) return e;
    if (clusters >= groups) {
      p.cs = static_cast<int>(cs);
      break;
    }
  }
  int64_t nsplit;
  if (p.cs > 0) {
    nsplit = p.cs;
    p.nbuf = kAttnMaxBuf;
  } else {
    nsplit = (int64_t(sm_count()) + groups - 1) / groups;
    if (nsplit > max_nc) nsplit = max_nc;
    if (nsplit < 1) nsplit = 1;
    p.nbuf = 1;
  }
  p.nsplit = static_cast<int>(nsplit);
  p.nc_pad = static_cast<int>((nsplit + 3) / 4 * 4);
  const int64_t items = groups * nsplit;
  const int64_t cap_grid = 3 * int64_t(sm_count());
  const int grid = static_cast<int>(p.cs > 0 || items < cap_grid ? items : cap_grid);
  const size_t smem = attn_tc_smem_bytes<G>(p.nc_pad, p.nbuf);
  auto kern = p.nbuf == 1 ? decode_attn_tc_kernel<G, 1> : decode_attn_tc_kernel<G, kAttnMaxBuf>;
  {
    const cudaError_t e = smem_attr_at_least(reinterpret_cast<const void*>(kern), smem);
    if (e != cudaSuccess) return e;
  }
  const cudaError_t e = launch_pdl(kern, dim3(grid), dim3(kTcThreads), smem, st,
                                   p.cs > 1 ? p.cs : 1, tmK, tmV, p);
  if (e != cudaSuccess) return e;
  return counted_launch(1);
}

}  // namespace

cudaError_t launch_decode_gemm(Epi epi, const DecGemmArgs& a, cudaStream_t st) {
  switch (epi) {
    case Epi::kQkv: return launch_dec_epi<static_cast<int>(Epi::kQkv)>(a, 1, st);
    case Epi::kResidual: return launch_dec_epi<static_cast<int>(Epi::kResidual)>(a, 1, st);
    case Epi::kSwiGLU: return launch_dec_epi<static_cast<int>(Epi::kSwiGLU)>(a, 2, st);
    case Epi::kPlain: return launch_dec_epi<static_cast<int>(Epi::kPlain)>(a, 1, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_decode_attention(const q3vl_config& c, const void* q, const q3vl_kv_cache& kv,
                                    const int32_t* seq, const int32_t* len, int B, void* o,
                                    float* part, uint32_t* tickets, cudaStream_t st) {
  const int G = c.n_heads / c.n_kv_heads;
  const uint64_t rows = uint64_t(kv.n_seq) * uint64_t(kv.cap), dkv = uint64_t(kv_dim(c));
  CUtensorMap tmK, tmV;
  if (!make_tmap_bf16(&tmK, kv.k, rows, dkv, dkv, 64, kAttnCH) ||
      !make_tmap_bf16(&tmV, kv.v, rows, dkv, dkv, 64, kAttnCH))
    return cudaErrorInvalidValue;
  DecAttnTcParams t{};
  t.q = static_cast<const __nv_bfloat16*>(q);
  t.kc = static_cast<const __nv_bfloat16*>(kv.k);
  t.vc = static_cast<const __nv_bfloat16*>(kv.v);
  t.cap = kv.cap; t.n_seq = kv.n_seq; t.seq = seq; t.len = len;
  t.B = B; t.nkv = c.n_kv_heads;
  const int64_t groups = int64_t(B) * c.n_kv_heads;
  const int64_t max_nc = (kv.cap + kAttnCH - 1) / kAttnCH;
  t.scale_log2 = static_cast<float>(1.4426950408889634 / 11.313708498984761);  // log2(e)/sqrt(128)
  t.o = static_cast<__nv_bfloat16*>(o);
  t.part = part; t.tickets = tickets; t.err = device_error_ptr();
  switch (G) {
    case 1: return launch_attn_tc_g<1>(tmK, tmV, t, groups, max_nc, st);
    case 2: return launch_attn_tc_g<2>(tmK, tmV, t, groups, max_nc, st);
    case 4: return launch_attn_tc_g<4>(tmK, tmV, t, groups, max_nc, st);
    case 8: return launch_attn_tc_g<8>(tmK, tmV, t, groups, max_nc, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_kv_store(const q3vl_config& c, const void* qkv, int64_t S,
                            const q3vl_kv_cache& kv, int32_t seq, cudaStream_t st) {
  const int64_t dkv8 = kv_dim(c) / 8, n = S * 2 * dkv8;
  kv_store_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(
      static_cast<const uint4*>(qkv), S, qkv_dim(c) / 8, q_dim(c) / 8, dkv8,
      static_cast<uint4*>(kv.k), static_cast<uint4*>(kv.v), int64_t(seq) * kv.cap);
  return counted_launch(1);
}

cudaError_t launch_decode_advance(int B, int32_t* pos, int32_t* len, cudaStream_t st) {
  decode_advance_kernel<<<(B + 127) / 128, 128, 0, st>>>(B, pos, len);
  return counted_launch(1);
}

}  // namespace q3vl
