// Host-side internals of libq3vl: workspace layout, kernel launchers and
// shared helpers. Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <string>
#include <utility>

#include "q3vl.h"

namespace q3vl {

constexpr int kHeadDim = 128;
constexpr int kHalf = kHeadDim / 2;
constexpr size_t kSkSlotBytes = size_t(128) * 256 * sizeof(float);

inline size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

inline int64_t q_dim(const q3vl_config& c) { return int64_t(c.n_heads) * c.head_dim; }
inline int64_t kv_dim(const q3vl_config& c) { return int64_t(c.n_kv_heads) * c.head_dim; }
inline int64_t qkv_dim(const q3vl_config& c) { return q_dim(c) + 2 * kv_dim(c); }
inline size_t elem_bytes(const q3vl_config& c) { return c.dtype == Q3VL_DTYPE_BF16 ? 2 : 4; }

// Offsets (bytes) of every region of the layer workspace.
struct WsLayout {
  size_t cos_sin = 0;  // fp32 cos/sin table: [S][64][2] (fp32 layers), slot-major (bf16)
  size_t inv1 = 0;     // fp32 [S] input-norm inv_rms
  size_t inv2 = 0;     // fp32 [S] post-attention-norm inv_rms
  size_t ds_map = 0;   // int32 [S]
  size_t qkv = 0;      // dtype [S][Ntot]
  size_t o = 0;        // dtype [S][Dq]
  size_t h = 0;        // dtype [S][H]
  size_t act = 0;      // dtype [S][I]
  size_t rowsq = 0;    // fp32 [S][H/128] sums of squares of h per N tile (bf16 path)
  size_t rowsq_x = 0;  // fp32 [S][H/128] the same for x' (read by the next layer of a stack)
  size_t sk_part = 0;  // fp32 [sk_slots][128 x 256] stream-K partial tiles
  size_t sk_flags = 0; // int32 [sk_slots], zero between GEMM launches
  int sk_slots = 0;
  size_t total = 0;
};
WsLayout ws_layout(const q3vl_config& c, int64_t S);

// Offsets of the packed-layer regions.
struct PackLayout {
  size_t w_qkv = 0, b_qkv = 0, q_norm = 0, k_norm = 0, w_o = 0, w_gu = 0, w_down = 0, total = 0;
};
PackLayout pack_layout(const q3vl_config& c);

// Per-device error record [code, where] (a __device__ array of 2 int32).
int32_t* device_error_ptr();

// Thread-local last-error message.
int set_error(int code, const std::string& msg);
int cuda_check(cudaError_t e, const char* what);

// Tensor map over a row-major [rows, cols] bf16 matrix with row stride
// `ld` elements, box (box_cols x box_rows), 128-byte swizzle, zero fill.
bool make_tmap_bf16(CUtensorMap* tm, const void* base, uint64_t rows, uint64_t cols,
                    uint64_t ld, uint32_t box_cols, uint32_t box_rows);

// ---------------------------------------------------------------------------
// Launchers (all enqueue on `st`, return the launch status).
// ---------------------------------------------------------------------------
cudaError_t launch_positions(const uint8_t* tt, int64_t S, const int32_t* grids, int n_grids,
                             int32_t* pos, int32_t* info, cudaStream_t st);
cudaError_t launch_rope_table(const q3vl_config& c, const int32_t* pos, int64_t S, float* cs,
                              cudaStream_t st);
// Converts a position-major cos/sin table ([S][64][2], the q3vl_rope_table
// layout) into the slot-major one the bf16 QKV epilogue reads: float4
// t * S + p = (cos, sin) of slots 2t, 2t + 1 at position p.
cudaError_t launch_rope_slot_major(const float* cs, int64_t S, float* out, cudaStream_t st);
// bf16 layer prologue in one launch: the cos/sin table (slot-major), the
// input row statistic of x (skipped when x is NULL) and n_flags zeroed
// stream-K flags.
cudaError_t launch_layer_prologue(const q3vl_config& c, const int32_t* pos, int64_t S, float* cs,
                                  const void* x, float* inv, int32_t* flags, int n_flags,
                                  cudaStream_t st);
cudaError_t launch_rowstat(const q3vl_config& c, const void* x, int64_t S, int64_t width,
                           float* inv, cudaStream_t st);
cudaError_t launch_final_norm(const q3vl_config& c, void* x, int64_t S, const void* gain,
                              cudaStream_t st);
cudaError_t launch_deepstack_map(const int32_t* rows, int n_img, int64_t S, int32_t* map,
                                 cudaStream_t st);
cudaError_t launch_pack(const q3vl_config& c, const q3vl_raw_weights& raw, void* packed,
                        cudaStream_t st);
cudaError_t launch_embed(const q3vl_config& c, const void* table, int64_t vocab,
                         const int32_t* tokens, int64_t S, const void* soft, const int32_t* map,
                         void* x, cudaStream_t st);
cudaError_t launch_selftest_timeout(uint32_t timeout_us, cudaStream_t st);

// bf16 tensor-core path (tcgen05 + TMA).
enum class Epi : int { kQkv = 0, kResidual = 1, kSwiGLU = 2, kPlain = 3 };
struct GemmArgs {
  const void* A;        // [M, K] bf16
  const void* B;        // [N, K] bf16
  int64_t M, N, K;
  void* out;            // bf16; row stride ldo
  int64_t ldo;
  const float* row_scale;  // [M] or null (kQkv, kSwiGLU)
  const float* bias;       // [N] or null (kQkv)
  const float* q_norm;     // [128] (kQkv)
  const float* k_norm;     // [128] (kQkv)
  const float* cos_sin;    // (kQkv, bf16 path) slot-major: float4 t * M + r = (cos, sin) of
                           // slots 2t, 2t + 1 at row r; (fp32 path) [M][64][2]
  int64_t q_cols, k_cols;  // column ranges [0,q_cols) = q heads, [q_cols, q_cols+k_cols) = k
  float eps;
  const void* resid;       // bf16 [M, ldo] (kResidual)
  const void* ds_slab;     // bf16 [n_img, N] (kResidual) or null
  const int32_t* ds_map;   // [M] (kResidual) or null
  // stream-K scratch (bf16 tensor-core path): sk_slots fp32 partial tiles
  // of sk_slot_bytes each, and sk_slots int32 flags that start at zero
  float* sk_partials;
  int32_t* sk_flags;
  int sk_slots;
  size_t sk_slot_bytes;
  // row statistics carried between GEMMs (bf16 tensor-core path):
  // kResidual may write, per row and per 256-column tile, the sum of squares
  // of its bf16 output to rowsq_out[row * rowsq_n + tile]; kSwiGLU and kQkv
  // may read those rowsq_n partials instead of row_scale, as
  // 1 / sqrt(sum / rowsq_width + eps).
  float* rowsq_out;
  const float* rowsq_in;
  int rowsq_n;
  float rowsq_width;
};
cudaError_t launch_gemm_tc(Epi epi, const GemmArgs& a, cudaStream_t st);
cudaError_t launch_attention_tc(const q3vl_config& c, const void* qkv, int64_t S, void* o,
                                cudaStream_t st);

// fp32 CUDA-core path.
cudaError_t launch_gemm_f32(Epi epi, const GemmArgs& a, cudaStream_t st);
cudaError_t launch_qk_norm_rope_f32(const q3vl_config& c, float* qkv, int64_t S,
                                    const float* q_norm, const float* k_norm, const float* cs,
                                    cudaStream_t st);
cudaError_t launch_gemm_swiglu_f32(const float* A, const float* B, int64_t M, int64_t I, int64_t K,
                                   const float* row_scale, float* act, cudaStream_t st);
cudaError_t launch_attention_f32(const q3vl_config& c, const float* qkv, int64_t S, float* o,
                                 cudaStream_t st);

// One-token decode (bf16, tcgen05). Schedule of a skinny projection: row
// tiles of 128 R weight rows, each split over `splits` CTAs along K.
struct DecSched {
  int R = 1, NB = 16, tiles = 0, n_k = 0, stages = 2, splits = 1;
  size_t smem = 0;
};
DecSched dec_gemm_sched(int64_t rows, int64_t K, int B, int R);

// Offsets (bytes) of the decode workspace regions.
struct DecLayout {
  size_t cos_sin = 0;   // fp32 [B][64][2]
  size_t inv = 0;       // fp32 [B] input-norm 1/rms of the first layer
  size_t rowsq_h = 0;   // fp32 [B][H/128] sums of squares of h per 128 columns
  size_t rowsq_x = 0;   // fp32 [B][H/128] the same of x' (read by the next layer)
  size_t q = 0;         // bf16 [B][Dq]
  size_t o = 0;         // bf16 [B][Dq]
  size_t h = 0;         // bf16 [B][H]
  size_t act = 0;       // bf16 [B][I]
  size_t att_part = 0;  // fp32 [B][nkv][G][130][splits] attention split partials
  size_t att_tickets = 0;  // uint32 [B][nkv], zero between launches
  size_t total = 0;
};
DecLayout dec_layout(const q3vl_config& c, int B, int64_t cap);

struct DecGemmArgs {
  const void* W;        // bf16 [rows, K] weights (row tiles of 128 R)
  int64_t rows, K;
  const void* X;        // bf16 [B, K] tokens
  int B;
  int64_t N;            // output row stride / columns
  void* out;            // bf16, or fp32 for kPlain (the LM head's logits)
  const void* resid;
  float* rowsq_out;
  const float* rowsq_in;
  int rowsq_n;
  float rowsq_width;
  const float* inv;
  float eps;
  const float* bias;
  const float* q_norm;
  const float* k_norm;
  const float* cos_sin;
  int n_heads, n_kv;
  void* k_cache;
  void* v_cache;
  int64_t cap;
  int n_seq;
  const int32_t* seq;
  const int32_t* len;
};
cudaError_t launch_decode_gemm(Epi epi, const DecGemmArgs& a, cudaStream_t st);
cudaError_t launch_decode_attention(const q3vl_config& c, const void* q, const q3vl_kv_cache& kv,
                                    const int32_t* seq, const int32_t* len, int B, void* o,
                                    float* part, uint32_t* tickets, cudaStream_t st);
cudaError_t launch_kv_store(const q3vl_config& c, const void* qkv, int64_t S,
                            const q3vl_kv_cache& kv, int32_t seq, cudaStream_t st);
cudaError_t launch_decode_advance(int B, int32_t* pos, int32_t* len, cudaStream_t st);

// Launches `kernel` on `st` as a programmatic dependent of the kernel before
// it in the stream (PDL): it may start while that kernel finishes, and must
// call griddepcontrol.wait before it touches memory that kernel, or any
// earlier one, reads or writes. Compile-time cluster dimensions of the kernel
// apply as usual.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_plain(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Device count of SMs (cached per device).
int sm_count();

// Raises `kernel`'s dynamic shared-memory limit to at least `bytes` on the
// current device. The attribute is set once per (kernel, device, size
// increase), under a lock, so concurrent host threads never lower it under
// one another.
cudaError_t smem_attr_at_least(const void* kernel, size_t bytes);

// Lets `kernel` launch with clusters of more than 8 CTAs on the current
// device; set once per (kernel, device), under a lock.
cudaError_t allow_nonportable_clusters(const void* kernel);

// Most clusters of `cluster` CTAs of `kernel` (with `threads` threads and
// `smem` bytes of dynamic shared memory each) that the current device holds
// at once; cached per (kernel, device) under a lock.
cudaError_t max_active_clusters(const void* kernel, int threads, size_t smem, int cluster,
                                int* out);

// Adds n to the process-wide count of kernels this library enqueued and
// returns the launch status of the last one.
cudaError_t counted_launch(int n);

}  // namespace q3vl
