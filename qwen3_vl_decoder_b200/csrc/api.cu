// C ABI of libq3vl: validation, workspace/packing layouts, tensor-map
// creation and the per-layer launch sequence. All device work is enqueued
// on the caller's stream; nothing here synchronises except
// q3vl_device_status().
#include <atomic>
#include <map>
#include <mutex>
#include <string>
#include <tuple>

#include "q3vl_internal.h"

namespace q3vl {

namespace {
thread_local std::string g_last_error;
std::atomic<uint64_t> g_launches{0};
constexpr int kStageEvents = 9;
thread_local cudaEvent_t g_stage_events[kStageEvents];
thread_local bool g_stage_events_on = false;

void stage_event(int i, cudaStream_t st) {
  if (g_stage_events_on) cudaEventRecord(g_stage_events[i], st);
}
}  // namespace

cudaError_t counted_launch(int n) {
  g_launches.fetch_add(static_cast<uint64_t>(n), std::memory_order_relaxed);
  return cudaGetLastError();
}

int set_error(int code, const std::string& msg) {
  g_last_error = msg;
  return code;
}

int cuda_check(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return Q3VL_OK;
  return set_error(Q3VL_ECUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

int sm_count() {
  static std::atomic<int> cache[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    v = n > 0 ? n : 148;
    cache[dev].store(v, std::memory_order_relaxed);
  }
  return v;
}

cudaError_t smem_attr_at_least(const void* kernel, size_t bytes) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, size_t> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(mu);
  size_t& d = done[{kernel, dev}];
  if (d >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(bytes));
  if (e == cudaSuccess) d = bytes;
  return e;
}

cudaError_t allow_nonportable_clusters(const void* kernel) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, bool> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(mu);
  bool& d = done[{kernel, dev}];
  if (d) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e == cudaSuccess) d = true;
  return e;
}

cudaError_t max_active_clusters(const void* kernel, int threads, size_t smem, int cluster,
                                int* out) {
  static std::mutex mu;
  static std::map<std::tuple<const void*, int, size_t, int>, int> cache;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(mu);
  const auto key = std::make_tuple(kernel, dev, smem, cluster);
  auto it = cache.find(key);
  if (it != cache.end()) {
    *out = it->second;
    return cudaSuccess;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cluster * (sm_count() / cluster));
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = static_cast<unsigned>(cluster);
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int n = 0;
  e = cudaOccupancyMaxActiveClusters(&n, kernel, &cfg);
  if (e != cudaSuccess) return e;
  cache[key] = n;
  *out = n;
  return cudaSuccess;
}

WsLayout ws_layout(const q3vl_config& c, int64_t S) {
  WsLayout L;
  const size_t e = elem_bytes(c);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  L.cos_sin = take(size_t(S) * kHalf * 2 * sizeof(float));
  L.inv1 = take(size_t(S) * sizeof(float));
  L.inv2 = take(size_t(S) * sizeof(float));
  L.ds_map = take(size_t(S) * sizeof(int32_t));
  L.qkv = take(size_t(S) * qkv_dim(c) * e);
  L.o = take(size_t(S) * q_dim(c) * e);
  L.h = take(size_t(S) * c.hidden * e);
  L.act = take(size_t(S) * c.intermediate * e);
  if (c.dtype == Q3VL_DTYPE_BF16) {
    L.rowsq = take(size_t(S) * (c.hidden / 128) * sizeof(float));
    L.rowsq_x = take(size_t(S) * (c.hidden / 128) * sizeof(float));
    L.sk_slots = sm_count();
    L.sk_part = take(size_t(L.sk_slots) * kSkSlotBytes);
    L.sk_flags = take(size_t(L.sk_slots) * sizeof(int32_t));
  }
  L.total = off;
  return L;
}

PackLayout pack_layout(const q3vl_config& c) {
  PackLayout L;
  const size_t e = elem_bytes(c);
  const size_t H = c.hidden, I = c.intermediate;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  L.w_qkv = take(size_t(qkv_dim(c)) * H * e);
  L.b_qkv = take(c.has_qkv_bias ? size_t(qkv_dim(c)) * sizeof(float) : 0);
  L.q_norm = take(kHeadDim * sizeof(float));
  L.k_norm = take(kHeadDim * sizeof(float));
  L.w_o = take(H * size_t(q_dim(c)) * e);
  L.w_gu = take(2 * I * H * e);
  L.w_down = take(H * I * e);
  L.total = off;
  return L;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point, so the
// library needs no link-time libcuda.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool make_tmap_bf16(CUtensorMap* tm, const void* base, uint64_t rows, uint64_t cols, uint64_t ld,
                    uint32_t box_cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  if ((reinterpret_cast<uintptr_t>(base) & 15) != 0 || (ld * 2) % 16 != 0) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {ld * 2};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------------------------
// Validation helpers
// ---------------------------------------------------------------------------
static int check_cfg(const q3vl_config* c) {
  if (c == nullptr) return set_error(Q3VL_EINVAL, "config is NULL");
  if (c->head_dim != kHeadDim)
    return set_error(Q3VL_EUNSUPPORTED, "head_dim must be 128 (got " + std::to_string(c->head_dim) + ")");
  if (c->dtype != Q3VL_DTYPE_FP32 && c->dtype != Q3VL_DTYPE_BF16)
    return set_error(Q3VL_EUNSUPPORTED, "dtype must be Q3VL_DTYPE_FP32 or Q3VL_DTYPE_BF16");
  if (c->hidden <= 0 || c->hidden % 64 != 0)
    return set_error(Q3VL_EINVAL, "hidden must be a positive multiple of 64");
  if (c->n_heads <= 0 || c->n_kv_heads <= 0 || c->n_heads % c->n_kv_heads != 0)
    return set_error(Q3VL_EINVAL, "n_heads must be a positive multiple of n_kv_heads");
  if (c->intermediate <= 0 || c->intermediate % 128 != 0)
    return set_error(Q3VL_EINVAL, "intermediate must be a positive multiple of 128");
  {
    // The interleaved slot rule must give each axis exactly its section.
    int cnt[3] = {0, 0, 0};
    for (int i = 0; i < kHalf; ++i) {
      int axis = 0;
      if (i % 3 == 1 && i < 3 * c->mrope_section[1]) axis = 1;
      else if (i % 3 == 2 && i < 3 * c->mrope_section[2]) axis = 2;
      ++cnt[axis];
    }
    if (cnt[0] != c->mrope_section[0] || cnt[1] != c->mrope_section[1] ||
        cnt[2] != c->mrope_section[2])
      return set_error(Q3VL_EUNSUPPORTED,
                       "mrope_section does not match the interleaved slot rule over 64 slots");
  }
  if (!(c->rope_theta > 0.0) || !(c->rms_eps >= 0.0))
    return set_error(Q3VL_EINVAL, "rope_theta must be > 0 and rms_eps >= 0");
  return Q3VL_OK;
}

static int check_seq(int64_t S) {
  if (S <= 0) return set_error(Q3VL_EINVAL, "sequence length must be >= 1 (empty input)");
  if (S > (int64_t(1) << 30)) return set_error(Q3VL_EINVAL, "sequence length above 2^30");
  return Q3VL_OK;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

static int check_layer(const q3vl_config* c, const q3vl_layer* w) {
  if (w == nullptr || w->w_qkv == nullptr || w->q_norm == nullptr || w->k_norm == nullptr ||
      w->w_o == nullptr || w->w_gu == nullptr || w->w_down == nullptr)
    return set_error(Q3VL_EINVAL, "packed layer has a NULL weight");
  if (c->has_qkv_bias && w->b_qkv == nullptr)
    return set_error(Q3VL_EINVAL, "has_qkv_bias set but b_qkv is NULL");
  if (!aligned16(w->w_qkv) || !aligned16(w->w_o) || !aligned16(w->w_gu) || !aligned16(w->w_down) ||
      !aligned16(w->q_norm) || !aligned16(w->k_norm) || (w->b_qkv && !aligned16(w->b_qkv)))
    return set_error(Q3VL_EINVAL, "packed weights must be 16-byte aligned");
  return Q3VL_OK;
}

}  // namespace q3vl

using namespace q3vl;

#define Q3VL_TRY(expr)            \
  do {                            \
    const int _rc = (expr);       \
    if (_rc != Q3VL_OK) return _rc; \
  } while (0)

#define Q3VL_CUDA(expr, what) Q3VL_TRY(cuda_check((expr), (what)))

// ---------------------------------------------------------------------------
// Step runners shared by the step-level calls and the layer / stack calls
// (validated by the caller).
// ---------------------------------------------------------------------------
namespace q3vl {
namespace {

bool is_bf16(const q3vl_config& c) { return c.dtype == Q3VL_DTYPE_BF16; }

// Stream-K scratch of a layer workspace.
struct Sk {
  float* part = nullptr;
  int32_t* flags = nullptr;
  int slots = 0;
};

Sk sk_of(const WsLayout& L, char* ws) {
  Sk k;
  if (L.sk_slots > 0) {
    k.part = reinterpret_cast<float*>(ws + L.sk_part);
    k.flags = reinterpret_cast<int32_t*>(ws + L.sk_flags);
    k.slots = L.sk_slots;
  }
  return k;
}

void set_sk(GemmArgs& a, const Sk& k) {
  a.sk_partials = k.part;
  a.sk_flags = k.flags;
  a.sk_slots = k.slots;
  a.sk_slot_bytes = kSkSlotBytes;
}

int clear_sk_flags(const Sk& k, cudaStream_t st) {
  if (k.flags == nullptr) return Q3VL_OK;
  return cuda_check(cudaMemsetAsync(k.flags, 0, size_t(k.slots) * sizeof(int32_t), st),
                    "clear stream-K flags");
}

int rowsq_parts(const q3vl_config& c);

int run_qkv(const q3vl_config& c, const q3vl_layer& w, const void* x, int64_t S, const float* inv,
            const float* cs, void* qkv, const Sk& sk, cudaStream_t st,
            const float* rowsq_in = nullptr) {
  GemmArgs a{};
  a.A = x; a.B = w.w_qkv; a.M = S; a.N = qkv_dim(c); a.K = c.hidden;
  a.out = qkv; a.ldo = a.N; a.row_scale = inv; a.bias = w.b_qkv;
  a.q_norm = w.q_norm; a.k_norm = w.k_norm; a.cos_sin = cs;
  a.q_cols = q_dim(c); a.k_cols = kv_dim(c); a.eps = static_cast<float>(c.rms_eps);
  a.rowsq_in = rowsq_in;
  a.rowsq_n = rowsq_parts(c);
  a.rowsq_width = static_cast<float>(c.hidden);
  set_sk(a, sk);
  if (is_bf16(c)) return cuda_check(launch_gemm_tc(Epi::kQkv, a, st), "qkv projection");
  Q3VL_CUDA(launch_gemm_f32(Epi::kPlain, a, st), "qkv projection");
  return cuda_check(launch_qk_norm_rope_f32(c, static_cast<float*>(qkv), S, w.q_norm, w.k_norm,
                                            cs, st),
                    "q/k norm + rope");
}

int run_attention(const q3vl_config& c, const void* qkv, int64_t S, void* o, cudaStream_t st) {
  if (is_bf16(c)) return cuda_check(launch_attention_tc(c, qkv, S, o, st), "attention");
  return cuda_check(launch_attention_f32(c, static_cast<const float*>(qkv), S,
                                         static_cast<float*>(o), st),
                    "attention");
}

// Number of per-row sum-of-squares partials the o-projection leaves for the
// gate/up epilogue: one per N tile of the residual GEMM.
int rowsq_parts(const q3vl_config& c) { return c.hidden % 256 == 0 ? c.hidden / 256 : c.hidden / 128; }

int run_oproj(const q3vl_config& c, const q3vl_layer& w, const void* o, const void* x, int64_t S,
              void* h, const Sk& sk, cudaStream_t st, float* rowsq = nullptr) {
  GemmArgs a{};
  a.A = o; a.B = w.w_o; a.M = S; a.N = c.hidden; a.K = q_dim(c);
  a.out = h; a.ldo = c.hidden; a.resid = x;
  a.rowsq_out = rowsq;
  a.rowsq_n = rowsq_parts(c);
  set_sk(a, sk);
  if (is_bf16(c)) return cuda_check(launch_gemm_tc(Epi::kResidual, a, st), "o projection");
  return cuda_check(launch_gemm_f32(Epi::kResidual, a, st), "o projection");
}

int run_gateup(const q3vl_config& c, const q3vl_layer& w, const void* h, int64_t S,
               const float* inv2, void* act, const Sk& sk, cudaStream_t st,
               const float* rowsq = nullptr) {
  if (is_bf16(c)) {
    GemmArgs a{};
    a.A = h; a.B = w.w_gu; a.M = S; a.N = 2 * int64_t(c.intermediate); a.K = c.hidden;
    a.out = act; a.ldo = c.intermediate; a.row_scale = inv2;
    a.rowsq_in = rowsq;
    a.rowsq_n = rowsq_parts(c);
    a.rowsq_width = static_cast<float>(c.hidden);
    a.eps = static_cast<float>(c.rms_eps);
    set_sk(a, sk);
    return cuda_check(launch_gemm_tc(Epi::kSwiGLU, a, st), "gate/up projection");
  }
  return cuda_check(launch_gemm_swiglu_f32(static_cast<const float*>(h),
                                           static_cast<const float*>(w.w_gu), S, c.intermediate,
                                           c.hidden, inv2, static_cast<float*>(act), st),
                    "gate/up projection");
}

int run_down(const q3vl_config& c, const q3vl_layer& w, const void* act, const void* h, int64_t S,
             const void* ds_slab, const int32_t* ds_map, void* out, const Sk& sk, cudaStream_t st,
             float* rowsq_out = nullptr) {
  GemmArgs a{};
  a.A = act; a.B = w.w_down; a.M = S; a.N = c.hidden; a.K = c.intermediate;
  a.out = out; a.ldo = c.hidden; a.resid = h;
  a.rowsq_out = rowsq_out;
  a.rowsq_n = rowsq_parts(c);
  a.ds_slab = ds_map ? ds_slab : nullptr;
  a.ds_map = ds_slab ? ds_map : nullptr;
  set_sk(a, sk);
  if (is_bf16(c)) return cuda_check(launch_gemm_tc(Epi::kResidual, a, st), "down projection");
  return cuda_check(launch_gemm_f32(Epi::kResidual, a, st), "down projection");
}

// The layer body on a prepared workspace (cos/sin table and DeepStack map
// already written).
// `x_stats_ready`: the previous layer of a stack left the row statistics of
// x in the workspace, so P2 is skipped; `leave_x_stats`: this layer's down
// epilogue leaves them for the next layer (bf16 path only). `inv1_ready`:
// the layer prologue already wrote P2's inv_rms.
// `kv` (optional): the K/V rows of this layer are also written into rows
// 0..S-1 of slot `kv_seq` of that cache.
int run_layer(const q3vl_config& c, const q3vl_layer& w, void* x, int64_t S, char* ws,
              const WsLayout& L, const void* ds_slab, cudaStream_t st, bool x_stats_ready = false,
              bool leave_x_stats = false, const q3vl_kv_cache* kv = nullptr,
              int32_t kv_seq = 0, bool inv1_ready = false) {
  float* cs = reinterpret_cast<float*>(ws + L.cos_sin);
  float* inv1 = reinterpret_cast<float*>(ws + L.inv1);
  float* inv2 = reinterpret_cast<float*>(ws + L.inv2);
  const int32_t* map = reinterpret_cast<const int32_t*>(ws + L.ds_map);
  void* qkv = ws + L.qkv;
  void* o = ws + L.o;
  void* h = ws + L.h;
  void* act = ws + L.act;
  const Sk sk = sk_of(L, ws);
  float* rowsq_x = is_bf16(c) ? reinterpret_cast<float*>(ws + L.rowsq_x) : nullptr;
  const bool use_x_stats = is_bf16(c) && x_stats_ready;
  if (!use_x_stats && !inv1_ready)
    Q3VL_CUDA(launch_rowstat(c, x, S, c.hidden, inv1, st), "input rms");
  stage_event(2, st);
  Q3VL_TRY(run_qkv(c, w, x, S, inv1, cs, qkv, sk, st, use_x_stats ? rowsq_x : nullptr));
  if (kv != nullptr) Q3VL_CUDA(launch_kv_store(c, qkv, S, *kv, kv_seq, st), "kv cache store");
  stage_event(3, st);
  Q3VL_TRY(run_attention(c, qkv, S, o, st));
  stage_event(4, st);
  if (is_bf16(c)) {
    // P7 fused: the o-projection epilogue leaves per-row sums of squares of
    // h, which the gate/up epilogue turns into 1/rms
    float* rowsq = reinterpret_cast<float*>(ws + L.rowsq);
    Q3VL_TRY(run_oproj(c, w, o, x, S, h, sk, st, rowsq));
    stage_event(5, st);
    stage_event(6, st);
    Q3VL_TRY(run_gateup(c, w, h, S, nullptr, act, sk, st, rowsq));
  } else {
    Q3VL_TRY(run_oproj(c, w, o, x, S, h, sk, st));
    stage_event(5, st);
    Q3VL_CUDA(launch_rowstat(c, h, S, c.hidden, inv2, st), "post-attention rms");
    stage_event(6, st);
    Q3VL_TRY(run_gateup(c, w, h, S, inv2, act, sk, st));
  }
  stage_event(7, st);
  Q3VL_TRY(run_down(c, w, act, h, S, ds_slab, ds_slab ? map : nullptr, x, sk, st,
                    is_bf16(c) && leave_x_stats ? rowsq_x : nullptr));
  stage_event(8, st);
  return Q3VL_OK;
}

// The per-call prologue of a layer or stack: the cos/sin table, the input
// row statistic of x (bf16: in the same launch) and cleared stream-K flags.
int run_prologue(const q3vl_config& c, const WsLayout& L, char* ws, const int32_t* pos, int64_t S,
                 const void* x, cudaStream_t st) {
  float* cs = reinterpret_cast<float*>(ws + L.cos_sin);
  if (is_bf16(c)) {
    const Sk sk = sk_of(L, ws);
    return cuda_check(launch_layer_prologue(c, pos, S, cs, x, reinterpret_cast<float*>(ws + L.inv1),
                                            sk.flags, sk.slots, st),
                      "layer prologue");
  }
  Q3VL_TRY(clear_sk_flags(sk_of(L, ws), st));
  return cuda_check(launch_rope_table(c, pos, S, cs, st), "rope table");
}

int check_ws(const q3vl_config& c, int64_t S, const void* ws, size_t ws_bytes) {
  const size_t need = ws_layout(c, S).total;
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255) != 0)
    return set_error(Q3VL_EWORKSPACE, "workspace must be non-NULL and 256-byte aligned");
  if (ws_bytes < need)
    return set_error(Q3VL_EWORKSPACE, "workspace too small: need " + std::to_string(need) +
                                          " bytes, got " + std::to_string(ws_bytes));
  return Q3VL_OK;
}

int check_ptr(const void* p, const char* name, bool need16 = true) {
  if (p == nullptr) return set_error(Q3VL_EINVAL, std::string(name) + " is NULL");
  if (need16 && (reinterpret_cast<uintptr_t>(p) & 15) != 0)
    return set_error(Q3VL_EINVAL, std::string(name) + " must be 16-byte aligned");
  return Q3VL_OK;
}

// Stream-K scratch of a step-level GEMM call: the workspace's stream-K
// region, flags cleared on the stream first.
int step_sk(const q3vl_config& c, int64_t S, void* ws, size_t ws_bytes, cudaStream_t st, Sk* out) {
  Q3VL_TRY(check_ws(c, S, ws, ws_bytes));
  *out = sk_of(ws_layout(c, S), static_cast<char*>(ws));
  return clear_sk_flags(*out, st);
}

int check_kv(const q3vl_config& c, const q3vl_kv_cache* kv, const char* what) {
  if (kv == nullptr) return set_error(Q3VL_EINVAL, std::string(what) + " is NULL");
  Q3VL_TRY(check_ptr(kv->k, "kv cache k"));
  Q3VL_TRY(check_ptr(kv->v, "kv cache v"));
  if (kv->cap < 1 || kv->n_seq < 1)
    return set_error(Q3VL_EINVAL, "kv cache needs cap >= 1 and n_seq >= 1");
  if (kv->cap > 131072)
    return set_error(Q3VL_EUNSUPPORTED, "kv cache cap above 131072 rows per slot");
  if (int64_t(kv->n_seq) * kv->cap > int64_t(0x7fffffff))
    return set_error(Q3VL_EINVAL, "kv cache n_seq * cap must stay below 2^31 rows");
  (void)c;
  return Q3VL_OK;
}

// The decode path covers bf16 layers whose query-group size is 1, 2, 4 or 8
// and whose hidden size is a multiple of 128 (its projection row tiles).
int check_decode_cfg(const q3vl_config& c) {
  if (c.dtype != Q3VL_DTYPE_BF16)
    return set_error(Q3VL_EUNSUPPORTED, "the KV cache and decode calls are bf16 only");
  const int G = c.n_heads / c.n_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8)
    return set_error(Q3VL_EUNSUPPORTED, "decode needs n_heads / n_kv_heads in {1, 2, 4, 8}");
  if (c.hidden % 128 != 0)
    return set_error(Q3VL_EUNSUPPORTED, "decode needs hidden to be a multiple of 128");
  return Q3VL_OK;
}

int check_batch(int32_t B) {
  if (B < 1 || B > 256) return set_error(Q3VL_EINVAL, "decode batch B must be in [1, 256]");
  return Q3VL_OK;
}

int check_dec_ws(const q3vl_config& c, int32_t B, int64_t cap, const void* ws, size_t ws_bytes) {
  const size_t need = dec_layout(c, B, cap).total;
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255) != 0)
    return set_error(Q3VL_EWORKSPACE, "workspace must be non-NULL and 256-byte aligned");
  if (ws_bytes < need)
    return set_error(Q3VL_EWORKSPACE, "decode workspace too small: need " + std::to_string(need) +
                                          " bytes, got " + std::to_string(ws_bytes));
  return Q3VL_OK;
}

// One layer of the decode on a prepared workspace (cos/sin of the B new
// positions written, tickets zero). `x_stats_ready`: the previous layer's
// down epilogue left the row sums of squares of x.
int run_decode_layer(const q3vl_config& c, const q3vl_layer& w, void* x, int32_t B,
                     const q3vl_kv_cache& kv, const int32_t* seq, const int32_t* len, char* ws,
                     const DecLayout& L, cudaStream_t st, bool x_stats_ready, bool leave_x_stats) {
  const int64_t H = c.hidden, I = c.intermediate, Dq = q_dim(c);
  float* inv = reinterpret_cast<float*>(ws + L.inv);
  float* rowsq_h = reinterpret_cast<float*>(ws + L.rowsq_h);
  float* rowsq_x = reinterpret_cast<float*>(ws + L.rowsq_x);
  void* q = ws + L.q;
  void* o = ws + L.o;
  void* h = ws + L.h;
  void* act = ws + L.act;
  if (!x_stats_ready) Q3VL_CUDA(launch_rowstat(c, x, B, H, inv, st), "decode input rms");

  DecGemmArgs a{};
  a.B = B; a.eps = static_cast<float>(c.rms_eps);
  a.n_heads = c.n_heads; a.n_kv = c.n_kv_heads;
  // P3+P4, with this token's K/V row written into the cache
  a.W = w.w_qkv; a.rows = qkv_dim(c); a.K = H; a.X = x;
  a.N = Dq; a.out = q; a.inv = inv;
  a.rowsq_in = x_stats_ready ? rowsq_x : nullptr;
  a.rowsq_n = static_cast<int>(H / 128); a.rowsq_width = static_cast<float>(H);
  a.bias = w.b_qkv; a.q_norm = w.q_norm; a.k_norm = w.k_norm;
  a.cos_sin = reinterpret_cast<const float*>(ws + L.cos_sin);
  a.k_cache = kv.k; a.v_cache = kv.v; a.cap = kv.cap; a.n_seq = kv.n_seq; a.seq = seq; a.len = len;
  Q3VL_CUDA(launch_decode_gemm(Epi::kQkv, a, st), "decode qkv projection");
  // P5 over the cache
  Q3VL_CUDA(launch_decode_attention(c, q, kv, seq, len, B, o,
                                    reinterpret_cast<float*>(ws + L.att_part),
                                    reinterpret_cast<uint32_t*>(ws + L.att_tickets), st),
            "decode attention");
  // P6 (+ the row sums of squares of h for P7)
  DecGemmArgs r{};
  r.B = B; r.eps = a.eps;
  r.W = w.w_o; r.rows = H; r.K = Dq; r.X = o;
  r.N = H; r.out = h; r.resid = x; r.rowsq_out = rowsq_h;
  Q3VL_CUDA(launch_decode_gemm(Epi::kResidual, r, st), "decode o projection");
  // P7+P8
  DecGemmArgs g{};
  g.B = B; g.eps = a.eps;
  g.W = w.w_gu; g.rows = 2 * I; g.K = H; g.X = h;
  g.N = I; g.out = act; g.rowsq_in = rowsq_h;
  g.rowsq_n = static_cast<int>(H / 128); g.rowsq_width = static_cast<float>(H);
  Q3VL_CUDA(launch_decode_gemm(Epi::kSwiGLU, g, st), "decode gate/up projection");
  // P9 (+ the row sums of squares of x' for the next layer)
  DecGemmArgs d{};
  d.B = B; d.eps = a.eps;
  d.W = w.w_down; d.rows = H; d.K = I; d.X = act;
  d.N = H; d.out = x; d.resid = h; d.rowsq_out = leave_x_stats ? rowsq_x : nullptr;
  Q3VL_CUDA(launch_decode_gemm(Epi::kResidual, d, st), "decode down projection");
  return Q3VL_OK;
}

// Positions' cos/sin and zero tickets: once per decode call.
int prepare_decode(const q3vl_config& c, const int32_t* pos, int32_t B, char* ws,
                   const DecLayout& L, cudaStream_t st) {
  Q3VL_CUDA(cudaMemsetAsync(ws + L.att_tickets, 0, L.total - L.att_tickets, st),
            "clear decode tickets");
  return cuda_check(launch_rope_table(c, pos, B, reinterpret_cast<float*>(ws + L.cos_sin), st),
                    "decode rope table");
}

}  // namespace
}  // namespace q3vl

#define ST(s) reinterpret_cast<cudaStream_t>(s)

extern "C" {

const char* q3vl_version(void) { return "q3vl 0.1.0 (sm_100a)"; }

const char* q3vl_last_error(void) { return g_last_error.c_str(); }

size_t q3vl_packed_layer_bytes(const q3vl_config* cfg) {
  if (check_cfg(cfg) != Q3VL_OK) return 0;
  return pack_layout(*cfg).total;
}

int q3vl_layer_views(const q3vl_config* cfg, const void* packed, q3vl_layer* out) {
  Q3VL_TRY(check_cfg(cfg));
  if (packed == nullptr || out == nullptr || (reinterpret_cast<uintptr_t>(packed) & 255) != 0)
    return set_error(Q3VL_EINVAL, "packed buffer must be non-NULL and 256-byte aligned");
  const PackLayout L = pack_layout(*cfg);
  const char* b = static_cast<const char*>(packed);
  out->w_qkv = b + L.w_qkv;
  out->b_qkv = cfg->has_qkv_bias ? reinterpret_cast<const float*>(b + L.b_qkv) : nullptr;
  out->q_norm = reinterpret_cast<const float*>(b + L.q_norm);
  out->k_norm = reinterpret_cast<const float*>(b + L.k_norm);
  out->w_o = b + L.w_o;
  out->w_gu = b + L.w_gu;
  out->w_down = b + L.w_down;
  return Q3VL_OK;
}

int q3vl_pack_layer(const q3vl_config* cfg, const q3vl_raw_weights* raw, void* packed,
                    size_t packed_bytes, q3vl_layer* out, q3vl_stream stream) {
  Q3VL_TRY(check_cfg(cfg));
  if (raw == nullptr) return set_error(Q3VL_EINVAL, "raw weights are NULL");
  const void* need[] = {raw->attn_norm, raw->wq, raw->wk, raw->wv, raw->q_norm, raw->k_norm,
                        raw->wo, raw->ffn_norm, raw->wg, raw->wu, raw->wd};
  for (const void* p : need)
    if (p == nullptr) return set_error(Q3VL_EINVAL, "a raw weight is NULL");
  if (cfg->has_qkv_bias && (raw->bq == nullptr || raw->bk == nullptr || raw->bv == nullptr))
    return set_error(Q3VL_EINVAL, "has_qkv_bias set but a bias is NULL");
  if (packed_bytes < pack_layout(*cfg).total)
    return set_error(Q3VL_EWORKSPACE, "packed buffer too small");
  Q3VL_TRY(q3vl_layer_views(cfg, packed, out));
  return cuda_check(launch_pack(*cfg, *raw, packed, ST(stream)), "pack layer");
}

int q3vl_mrope_positions(const uint8_t* token_types, int64_t S, const int32_t* grids,
                         int32_t n_grids, int32_t* pos, int32_t* info, q3vl_stream stream) {
  Q3VL_TRY(check_seq(S));
  if (token_types == nullptr || pos == nullptr || info == nullptr)
    return set_error(Q3VL_EINVAL, "token_types, pos and info must be non-NULL");
  if (n_grids < 0 || n_grids > 4096) return set_error(Q3VL_EINVAL, "n_grids must be in [0, 4096]");
  if (n_grids > 0 && grids == nullptr) return set_error(Q3VL_EINVAL, "grids is NULL");
  return cuda_check(launch_positions(token_types, S, grids, n_grids, pos, info, ST(stream)),
                    "positions");
}

size_t q3vl_workspace_bytes(const q3vl_config* cfg, int64_t S) {
  if (check_cfg(cfg) != Q3VL_OK || check_seq(S) != Q3VL_OK) return 0;
  return ws_layout(*cfg, S).total;
}

int q3vl_rope_table(const q3vl_config* cfg, const int32_t* pos, int64_t S, float* cos_sin,
                    q3vl_stream stream) {
  Q3VL_TRY(check_cfg(cfg));
  Q3VL_TRY(check_seq(S));
  Q3VL_TRY(check_ptr(pos, "pos", false));
  Q3VL_TRY(check_ptr(cos_sin, "cos_sin"));
  return cuda_check(launch_rope_table(*cfg, pos, S, cos_sin, ST(stream)), "rope table");
}

int q3vl_rms_rowstat(const q3vl_config* cfg, const void* x, int64_t S, int64_t width,
                     float* inv_rms, q3vl_stream stream) {
  Q3VL_TRY(check_cfg(cfg));
  Q3VL_TRY(check_seq(S));
  Q3VL_TRY(check_ptr(x, "x"));
  Q3VL_TRY(check_ptr(inv_rms, "inv_rms", false));
  if (width <= 0 || (width * int64_t(elem_bytes(*cfg))) % 16 != 0)
    return set_error(Q3VL_EINVAL, "width must be positive with 16-byte rows");
  return cuda_check(launch_rowstat(*cfg, x, S, width, inv_rms, ST(stream)), "rowstat");
}

int q3vl_qkv_proj(const q3vl_config* cfg, const q3vl_layer* layer, const void* x, int64_t S,
                  const float* inv_rms, const float* cos_sin, void* qkv, void* ws,
                  size_t ws_bytes, q3vl_stream stream) {
  Q3VL_TRY(check_cfg(cfg));
  Q3VL_TRY(check_seq(S));
  Q3VL_TRY(check_layer(cfg, layer));
  Q3VL_TRY(check_ptr(x, "x"));
  Q3VL_TRY(check_ptr(inv_rms, "inv_rms", false));
  Q3VL_TRY(check_ptr(cos_sin, "cos_sin"));
  Q3VL_TRY(check_ptr(qkv, "qkv"));
  Sk sk;
  Q3VL_TRY(step_sk(*cfg, S, ws, ws_bytes, ST(stream), &sk));
  if (is_bf16(*cfg)) {
    // the bf16 epilogue reads the table slot-major: convert into the workspace
    float* cs_t = reinterpret_cast<float*>(static_cast<char*>(ws) + ws_layout(*cfg, S).cos_sin);
    const size_t tb = size_t(S) * kHalf * 2 * sizeof(float);
    const char* a0 = reinterpret_cast<const char*>(cos_sin);
    const char* b0 = reinterpret_cast<const char*>(cs_t);
    if (a0 < b0 + tb && b0 < a0 + tb)
      return set_error(Q3VL_EINVAL, "cos_sin must not overlap the workspace's table region");
    Q3VL_CUDA(launch_rope_slot_major(cos_sin, S, cs_t, ST(stream)), "cos/sin slot-major");
    return run_qkv(*cfg, *layer, x, S, inv_rms, cs_t, qkv, sk, ST(stream));
  }
  return run_qkv(*cfg, *layer, x, S, inv_rms, cos_sin, qkv, sk, ST(stream));
}

int q3vl_attention(const q3vl_config* cfg, const void* qkv, int64_t S, void* o,
                   q3vl_stream stream) {
  Q3VL_TRY(check_cfg(cfg));
  Q3VL_TRY(check_seq(S));
  Q3VL_TRY(check_ptr(qkv, "qkv"));
  Q3VL_TRY(check_ptr(o, "o"));
  return run_attention(*cfg, qkv, S, o, ST(stream));
}

int q3vl_o_proj(const q3vl_config* cfg, const q3vl_layer* layer, const void* o, const void* x,
                int64_t S, void* h, void* ws, size_t ws_bytes, q3vl_stream stream) {
  Q3VL_TRY(check_cfg(cfg));
  Q3VL_TRY(check_seq(S));
  Q3VL_TRY(check_layer(cfg, layer));
  Q3VL_TRY(check_ptr(o, "o"));
  Q3VL_TRY(check_ptr(x, "x"));
  Q3VL_TRY(check_ptr(h, "h"));
  Sk sk;
  Q3VL_TRY(step_sk(*cfg, S, ws, ws_bytes, ST(stream), &sk));
  return run_oproj(*cfg, *layer, o, x, S, h, sk, ST(stream));
}

int q3vl_gate_up(const q3vl_config* cfg, const q3vl_layer* layer, const void* h, int64_t S,
                 const float* inv_rms2, void* act, void* ws, size_t ws_bytes,
                 q3vl_stream stream) {
  Q3VL_TRY(check_cfg(cfg));
  Q3VL_TRY(check_seq(S));
  Q3VL_TRY(check_layer(cfg, layer));
  Q3VL_TRY(check_ptr(h, "h"));
  Q3VL_TRY(check_ptr(inv_rms2, "inv_rms2", false));
  Q3VL_TRY(check_ptr(act, "act"));
  Sk sk;
  Q3VL_TRY(step_sk(*cfg, S, ws, ws_bytes, ST(stream), &sk));
  return run_gateup(*cfg, *layer, h, S, inv_rms2, act, sk, ST(stream));
}

int q3vl_down(const q3vl_config* cfg, const q3vl_layer* layer, const void* act, const void* h,
              int64_t S, const void* ds_slab, const int32_t* ds_map, void* out, void* ws,
              size_t ws_bytes, q3vl_stream stream) {
  Q3VL_TRY(check_cfg(cfg));
  Q3VL_TRY(check_seq(S));
  Q3VL_TRY(check_layer(cfg, layer));
  Q3VL_TRY(check_ptr(act, "act"));
  Q3VL_TRY(check_ptr(h, "h"));
  Q3VL_TRY(check_ptr(out, "out"));
  if ((ds_slab == nullptr) != (ds_map == nullptr))
    return set_error(Q3VL_EDEEPSTACK, "ds_slab and ds_map must both be given or both be NULL");
  if (ds_slab) Q3VL_TRY(check_ptr(ds_slab, "ds_slab"));
  if (out == h || out == act) return set_error(Q3VL_EINVAL, "out must not alias h or act");
  Sk sk;
  Q3VL_TRY(step_sk(*cfg, S, ws, ws_bytes, ST(stream), &sk));
  return run_down(*cfg, *layer, act, h, S, ds_slab, ds_map, out, sk, ST(stream));
}

int q3vl_deepstack_map(const int32_t* ds_rows, int32_t n_img, int64_t S, int32_t* ds_map,
                       q3vl_stream stream) {
  Q3VL_TRY(check_seq(S));
  Q3VL_TRY(check_ptr(ds_map, "ds_map", false));
  if (n_img < 0 || n_img > S) return set_error(Q3VL_ERANGE, "n_img must be in [0, S]");
  if (n_img > 0 && ds_rows == nullptr) return set_error(Q3VL_EINVAL, "ds_rows is NULL");
  return cuda_check(launch_deepstack_map(ds_rows, n_img, S, ds_map, ST(stream)), "deepstack map");
}

int q3vl_final_norm(const q3vl_config* cfg, void* x, int64_t S, const void* gain,
                    q3vl_stream stream) {
  Q3VL_TRY(check_cfg(cfg));
  Q3VL_TRY(check_seq(S));
  Q3VL_TRY(check_ptr(x, "x"));
  Q3VL_TRY(check_ptr(gain, "gain"));
  return cuda_check(launch_final_norm(*cfg, x, S, gain, ST(stream)), "final norm");
}

static int layer_prefill_impl(const q3vl_config* cfg, const q3vl_layer* layer, void* x, int64_t S,
                              const int32_t* pos, const void* ds_slab, const int32_t* ds_rows,
                              int32_t n_img, const q3vl_kv_cache* kv, int32_t kv_seq, void* ws,
                              size_t ws_bytes, q3vl_stream stream) {
  Q3VL_TRY(check_cfg(cfg));
  Q3VL_TRY(check_seq(S));
  Q3VL_TRY(check_layer(cfg, layer));
  Q3VL_TRY(check_ptr(x, "x"));
  Q3VL_TRY(check_ptr(pos, "pos", false));
  Q3VL_TRY(check_ws(*cfg, S, ws, ws_bytes));
  if (ds_slab != nullptr) {
    if (ds_rows == nullptr || n_img <= 0)
      return set_error(Q3VL_EDEEPSTACK, "DeepStack slab given without image rows");
    if (n_img > S) return set_error(Q3VL_ERANGE, "more image rows than tokens");
    Q3VL_TRY(check_ptr(ds_slab, "ds_slab"));
  }
  const cudaStream_t st = ST(stream);
  const WsLayout L = ws_layout(*cfg, S);
  char* w = static_cast<char*>(ws);
  stage_event(0, st);
  Q3VL_TRY(run_prologue(*cfg, L, w, pos, S, x, st));
  if (ds_slab != nullptr)
    Q3VL_CUDA(launch_deepstack_map(ds_rows, n_img, S, reinterpret_cast<int32_t*>(w + L.ds_map), st),
              "deepstack map");
  stage_event(1, st);
  return run_layer(*cfg, *layer, x, S, w, L, ds_slab, st, false, false, kv, kv_seq,
                   is_bf16(*cfg));
}

// Cache checks of the *_kv prefill calls: bf16, rows 0..S-1 of one slot.
static int check_prefill_kv(const q3vl_config* cfg, int64_t S, const q3vl_kv_cache* kv,
                            int32_t n, int32_t seq) {
  Q3VL_TRY(check_cfg(cfg));
  if (cfg->dtype != Q3VL_DTYPE_BF16)
    return set_error(Q3VL_EUNSUPPORTED, "the KV cache and decode calls are bf16 only");
  if (kv == nullptr) return set_error(Q3VL_EINVAL, "kv is NULL");
  for (int32_t l = 0; l < n; ++l) {
    Q3VL_TRY(check_kv(*cfg, kv + l, "kv"));
    if (S > kv[l].cap) return set_error(Q3VL_ERANGE, "S exceeds the cache capacity");
    if (seq < 0 || seq >= kv[l].n_seq) return set_error(Q3VL_ERANGE, "seq outside [0, n_seq)");
  }
  return Q3VL_OK;
}

int q3vl_layer_prefill(const q3vl_config* cfg, const q3vl_layer* layer, void* x, int64_t S,
                       const int32_t* pos, const void* ds_slab, const int32_t* ds_rows,
                       int32_t n_img, void* ws, size_t ws_bytes, q3vl_stream stream) {
  return layer_prefill_impl(cfg, layer, x, S, pos, ds_slab, ds_rows, n_img, nullptr, 0, ws,
                            ws_bytes, stream);
}

int q3vl_layer_prefill_kv(const q3vl_config* cfg, const q3vl_layer* layer, void* x, int64_t S,
                          const int32_t* pos, const void* ds_slab, const int32_t* ds_rows,
                          int32_t n_img, const q3vl_kv_cache* kv, int32_t seq, void* ws,
                          size_t ws_bytes, q3vl_stream stream) {
  Q3VL_TRY(check_prefill_kv(cfg, S, kv, 1, seq));
  return layer_prefill_impl(cfg, layer, x, S, pos, ds_slab, ds_rows, n_img, kv, seq, ws,
                            ws_bytes, stream);
}

static int stack_prefill_impl(const q3vl_config* cfg, int32_t n_layers, const q3vl_layer* layers,
                              const void* final_norm, void* x, int64_t S, const int32_t* pos,
                              const void* const* ds_slabs, int32_t n_ds, const int32_t* ds_rows,
                              int32_t n_img, const q3vl_kv_cache* kv, int32_t kv_seq, void* ws,
                              size_t ws_bytes, q3vl_stream stream) {
  Q3VL_TRY(check_cfg(cfg));
  Q3VL_TRY(check_seq(S));
  if (n_layers <= 0 || layers == nullptr)
    return set_error(Q3VL_EINVAL, "n_layers must be >= 1 with a non-NULL layer array");
  for (int32_t l = 0; l < n_layers; ++l) {
    const int rc = check_layer(cfg, layers + l);
    if (rc != Q3VL_OK) return set_error(rc, "layer " + std::to_string(l) + ": " + g_last_error);
  }
  Q3VL_TRY(check_ptr(x, "x"));
  Q3VL_TRY(check_ptr(pos, "pos", false));
  Q3VL_TRY(check_ws(*cfg, S, ws, ws_bytes));
  if (final_norm != nullptr) Q3VL_TRY(check_ptr(final_norm, "final_norm"));
  if (n_ds < 0) return set_error(Q3VL_EDEEPSTACK, "n_ds must be >= 0");
  if (n_ds > 0) {
    if (ds_slabs == nullptr) return set_error(Q3VL_EDEEPSTACK, "ds_slabs is NULL");
    if (n_ds < 3)
      return set_error(Q3VL_EDEEPSTACK, "fewer DeepStack slabs (" + std::to_string(n_ds) +
                                            ") than DeepStack layers (3)");
    if (n_img <= 0 || ds_rows == nullptr)
      return set_error(Q3VL_EDEEPSTACK, "DeepStack slabs given without image rows");
    if (n_img > S) return set_error(Q3VL_ERANGE, "more image rows than tokens");
    for (int32_t l = 0; l < n_ds; ++l) Q3VL_TRY(check_ptr(ds_slabs[l], "ds_slabs[l]"));
  }
  const cudaStream_t st = ST(stream);
  const WsLayout L = ws_layout(*cfg, S);
  char* w = static_cast<char*>(ws);
  Q3VL_TRY(run_prologue(*cfg, L, w, pos, S, x, st));
  if (n_ds > 0)
    Q3VL_CUDA(launch_deepstack_map(ds_rows, n_img, S, reinterpret_cast<int32_t*>(w + L.ds_map), st),
              "deepstack map");
  const bool events = g_stage_events_on;
  g_stage_events_on = false;  // stage events describe single-layer calls only
  for (int32_t l = 0; l < n_layers; ++l) {
    const void* slab = l < n_ds ? ds_slabs[l] : nullptr;
    // P2 of layer l > 0 comes from layer l-1's down epilogue
    const int rc = run_layer(*cfg, layers[l], x, S, w, L, slab, st, l > 0, l + 1 < n_layers,
                             kv != nullptr ? kv + l : nullptr, kv_seq, l == 0 && is_bf16(*cfg));
    if (rc != Q3VL_OK) g_stage_events_on = events;
    if (rc != Q3VL_OK) return set_error(rc, "layer " + std::to_string(l) + ": " + g_last_error);
  }
  g_stage_events_on = events;
  if (final_norm != nullptr)
    Q3VL_CUDA(launch_final_norm(*cfg, x, S, final_norm, st), "final norm");
  return Q3VL_OK;
}

int q3vl_stack_prefill(const q3vl_config* cfg, int32_t n_layers, const q3vl_layer* layers,
                       const void* final_norm, void* x, int64_t S, const int32_t* pos,
                       const void* const* ds_slabs, int32_t n_ds, const int32_t* ds_rows,
                       int32_t n_img, void* ws, size_t ws_bytes, q3vl_stream stream) {
  return stack_prefill_impl(cfg, n_layers, layers, final_norm, x, S, pos, ds_slabs, n_ds,
                            ds_rows, n_img, nullptr, 0, ws, ws_bytes, stream);
}

int q3vl_stack_prefill_kv(const q3vl_config* cfg, int32_t n_layers, const q3vl_layer* layers,
                          const void* final_norm, void* x, int64_t S, const int32_t* pos,
                          const void* const* ds_slabs, int32_t n_ds, const int32_t* ds_rows,
                          int32_t n_img, const q3vl_kv_cache* kv, int32_t seq, void* ws,
                          size_t ws_bytes, q3vl_stream stream) {
  if (n_layers <= 0) return set_error(Q3VL_EINVAL, "n_layers must be >= 1");
  Q3VL_TRY(check_prefill_kv(cfg, S, kv, n_layers, seq));
  return stack_prefill_impl(cfg, n_layers, layers, final_norm, x, S, pos, ds_slabs, n_ds,
                            ds_rows, n_img, kv, seq, ws, ws_bytes, stream);
}

size_t q3vl_decode_workspace_bytes(const q3vl_config* cfg, int32_t B, int64_t cap) {
  if (check_cfg(cfg) != Q3VL_OK || check_decode_cfg(*cfg) != Q3VL_OK || check_batch(B) != Q3VL_OK ||
      cap < 1)
    return 0;
  return dec_layout(*cfg, B, cap).total;
}

static int decode_checks(const q3vl_config* cfg, int32_t n_layers, const q3vl_layer* layers,
                         void* x, int32_t B, const int32_t* pos, const q3vl_kv_cache* kv,
                         const int32_t* seq, const int32_t* len, void* ws, size_t ws_bytes) {
  Q3VL_TRY(check_cfg(cfg));
  Q3VL_TRY(check_decode_cfg(*cfg));
  Q3VL_TRY(check_batch(B));
  if (layers == nullptr || kv == nullptr) return set_error(Q3VL_EINVAL, "layers / kv are NULL");
  int64_t cap = 0;
  for (int32_t l = 0; l < n_layers; ++l) {
    const int rc = check_layer(cfg, layers + l);
    if (rc != Q3VL_OK) return set_error(rc, "layer " + std::to_string(l) + ": " + g_last_error);
    Q3VL_TRY(check_kv(*cfg, kv + l, "kv"));
    if (kv[l].cap > cap) cap = kv[l].cap;
  }
  Q3VL_TRY(check_ptr(x, "x"));
  Q3VL_TRY(check_ptr(pos, "pos", false));
  Q3VL_TRY(check_ptr(seq, "seq", false));
  Q3VL_TRY(check_ptr(len, "len", false));
  return check_dec_ws(*cfg, B, cap, ws, ws_bytes);
}

int q3vl_layer_decode(const q3vl_config* cfg, const q3vl_layer* layer, void* x, int32_t B,
                      const int32_t* pos, const q3vl_kv_cache* kv, const int32_t* seq,
                      const int32_t* len, void* ws, size_t ws_bytes, q3vl_stream stream) {
  Q3VL_TRY(decode_checks(cfg, 1, layer, x, B, pos, kv, seq, len, ws, ws_bytes));
  const cudaStream_t st = ST(stream);
  const DecLayout L = dec_layout(*cfg, B, kv->cap);
  char* w = static_cast<char*>(ws);
  Q3VL_TRY(prepare_decode(*cfg, pos, B, w, L, st));
  return run_decode_layer(*cfg, *layer, x, B, *kv, seq, len, w, L, st, false, false);
}

int q3vl_stack_decode(const q3vl_config* cfg, int32_t n_layers, const q3vl_layer* layers,
                      const void* final_norm, void* x, int32_t B, const int32_t* pos,
                      const q3vl_kv_cache* kv, const int32_t* seq, const int32_t* len, void* ws,
                      size_t ws_bytes, q3vl_stream stream) {
  if (n_layers <= 0) return set_error(Q3VL_EINVAL, "n_layers must be >= 1");
  Q3VL_TRY(decode_checks(cfg, n_layers, layers, x, B, pos, kv, seq, len, ws, ws_bytes));
  if (final_norm != nullptr) Q3VL_TRY(check_ptr(final_norm, "final_norm"));
  int64_t cap = 0;
  for (int32_t l = 0; l < n_layers; ++l) cap = kv[l].cap > cap ? kv[l].cap : cap;
  const cudaStream_t st = ST(stream);
  const DecLayout L = dec_layout(*cfg, B, cap);
  char* w = static_cast<char*>(ws);
  Q3VL_TRY(prepare_decode(*cfg, pos, B, w, L, st));
  for (int32_t l = 0; l < n_layers; ++l) {
    const int rc = run_decode_layer(*cfg, layers[l], x, B, kv[l], seq, len, w, L, st, l > 0,
                                    l + 1 < n_layers);
    if (rc != Q3VL_OK) return set_error(rc, "layer " + std::to_string(l) + ": " + g_last_error);
  }
  if (final_norm != nullptr)
    Q3VL_CUDA(launch_final_norm(*cfg, x, B, final_norm, st), "final norm");
  return Q3VL_OK;
}

int q3vl_embed(const q3vl_config* cfg, const void* table, int64_t vocab, const int32_t* tokens,
               int64_t S, const void* soft, const int32_t* soft_rows, int32_t n_soft, void* x,
               void* ws, size_t ws_bytes, q3vl_stream stream) {
  Q3VL_TRY(check_cfg(cfg));
  Q3VL_TRY(check_seq(S));
  if (vocab < 1) return set_error(Q3VL_EINVAL, "vocab must be >= 1");
  Q3VL_TRY(check_ptr(table, "table"));
  Q3VL_TRY(check_ptr(tokens, "tokens", false));
  Q3VL_TRY(check_ptr(x, "x"));
  if (n_soft < 0) return set_error(Q3VL_EINVAL, "n_soft must be >= 0");
  const cudaStream_t st = ST(stream);
  int32_t* map = nullptr;
  if (n_soft > 0) {
    Q3VL_TRY(check_ptr(soft, "soft"));
    Q3VL_TRY(check_ptr(soft_rows, "soft_rows", false));
    if (n_soft > S) return set_error(Q3VL_ERANGE, "more soft-token rows than tokens");
    if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255) != 0 ||
        ws_bytes < size_t(S) * sizeof(int32_t))
      return set_error(Q3VL_EWORKSPACE, "embed with soft tokens needs >= 4*S bytes of workspace");
    map = static_cast<int32_t*>(ws);
    Q3VL_CUDA(launch_deepstack_map(soft_rows, n_soft, S, map, st), "soft-token row map");
  }
  return cuda_check(launch_embed(*cfg, table, vocab, tokens, S, soft, map, x, st), "embed");
}

size_t q3vl_lm_head_workspace_bytes(const q3vl_config* cfg, int32_t B) {
  if (check_cfg(cfg) != Q3VL_OK || cfg->dtype != Q3VL_DTYPE_BF16 || check_batch(B) != Q3VL_OK)
    return 0;
  return align256(size_t(B) * cfg->hidden * 2);
}

int q3vl_lm_head(const q3vl_config* cfg, const void* x, int32_t B, const void* final_norm,
                 const void* weight, int64_t vocab, float* logits, void* ws, size_t ws_bytes,
                 q3vl_stream stream) {
  Q3VL_TRY(check_cfg(cfg));
  if (cfg->dtype != Q3VL_DTYPE_BF16)
    return set_error(Q3VL_EUNSUPPORTED, "the LM head is bf16 only");
  Q3VL_TRY(check_batch(B));
  if (vocab < 1 || vocab > (int64_t(1) << 30)) return set_error(Q3VL_EINVAL, "vocab out of range");
  Q3VL_TRY(check_ptr(x, "x"));
  Q3VL_TRY(check_ptr(weight, "weight"));
  Q3VL_TRY(check_ptr(logits, "logits", false));
  if (final_norm != nullptr) Q3VL_TRY(check_ptr(final_norm, "final_norm"));
  const size_t need = align256(size_t(B) * cfg->hidden * 2);
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255) != 0 || ws_bytes < need)
    return set_error(Q3VL_EWORKSPACE, "lm head workspace too small: need " +
                                          std::to_string(need) + " bytes");
  const cudaStream_t st = ST(stream);
  // the rows, normalised in the workspace (x itself is left as it is)
  Q3VL_CUDA(cudaMemcpyAsync(ws, x, size_t(B) * cfg->hidden * 2, cudaMemcpyDeviceToDevice, st),
            "lm head rows");
  if (final_norm != nullptr)
    Q3VL_CUDA(launch_final_norm(*cfg, ws, B, final_norm, st), "lm head final norm");
  DecGemmArgs a{};
  a.W = weight; a.rows = vocab; a.K = cfg->hidden; a.X = ws; a.B = B;
  a.N = vocab; a.out = logits;
  return cuda_check(launch_decode_gemm(Epi::kPlain, a, st), "lm head");
}

int q3vl_decode_advance(int32_t B, int32_t* pos, int32_t* len, q3vl_stream stream) {
  Q3VL_TRY(check_batch(B));
  Q3VL_TRY(check_ptr(pos, "pos", false));
  Q3VL_TRY(check_ptr(len, "len", false));
  return cuda_check(launch_decode_advance(B, pos, len, ST(stream)), "decode advance");
}

int q3vl_set_stage_events(void* const* events, int32_t n_events) {
  if (n_events == 0) {
    g_stage_events_on = false;
    return Q3VL_OK;
  }
  if (events == nullptr || n_events != kStageEvents)
    return set_error(Q3VL_EINVAL, "stage events: pass 9 events, or 0 to stop");
  for (int i = 0; i < kStageEvents; ++i) {
    if (events[i] == nullptr) return set_error(Q3VL_EINVAL, "stage event is NULL");
    g_stage_events[i] = static_cast<cudaEvent_t>(events[i]);
  }
  g_stage_events_on = true;
  return Q3VL_OK;
}

uint64_t q3vl_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int q3vl_device_status(q3vl_stream stream, int32_t* code, int32_t* where) {
  if (code == nullptr || where == nullptr) return set_error(Q3VL_EINVAL, "code/where are NULL");
  Q3VL_CUDA(cudaStreamSynchronize(ST(stream)), "stream synchronize");
  int32_t* rec = device_error_ptr();
  if (rec == nullptr) return set_error(Q3VL_ECUDA, "device error record unavailable");
  int32_t h[2] = {0, 0};
  Q3VL_CUDA(cudaMemcpy(h, rec, sizeof(h), cudaMemcpyDeviceToHost), "read error record");
  Q3VL_CUDA(cudaMemset(rec, 0, sizeof(h)), "clear error record");
  Q3VL_CUDA(cudaDeviceSynchronize(), "clear error record");
  *code = h[0];
  *where = h[1];
  return Q3VL_OK;
}

int q3vl_selftest_wait_timeout(uint32_t timeout_us, q3vl_stream stream) {
  if (timeout_us == 0 || timeout_us > 10u * 1000u * 1000u)
    return set_error(Q3VL_EINVAL, "timeout_us must be in [1, 10^7]");
  return cuda_check(launch_selftest_timeout(timeout_us, ST(stream)), "selftest");
}

}  // extern "C"
