// q3vl_layer_prefill_noalloc: one decoder layer with the library's own,
// statically sized scratch memory instead of a caller workspace.
//
// Who needs it: callers that cannot allocate device memory at all, such as
// a plug-in hosted by a framework whose memory manager has already reserved
// the GPU's memory for its own pool, a C caller with no device allocator of
// its own, or a latency-critical path where the implicit device-wide
// synchronisation of cudaMalloc is not allowed. They still pass x, the
// positions and the packed weights; only the scratch space is built in.
//
// The scratch is one file-scope device array of kNoAllocScratchBytes
// (64 MiB). Every GPU that loads this library keeps that array for the life
// of the process. Its device address is looked up once per device, on the
// first call made with that device current (cudaGetSymbolAddress), so make
// that first call before any stream capture. The looked-up address is kept
// for the life of the process, so the entry point must not be used on a
// device after cudaDeviceReset (or another teardown of its primary context):
// that reloads this module's device code, and the array, at a new address.
// All calls share the one array:
// calls that overlap on the GPU (different streams, or different host
// threads) race on it and must be serialised by the caller. Nothing in the
// scratch needs to start at zero: each call writes every scratch region it
// reads (including the DeepStack row map) before reading it, so the
// contents left by the previous call are never used.
#include <mutex>
#include <string>

#include "q3vl_internal.h"

namespace q3vl {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch on the current device (set up once per
// device); nullptr with the CUDA error in *err on failure.
void* scratch_address(cudaError_t* err) {
  static std::mutex mu;
  static void* addr[64] = {nullptr};
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= 64) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    *err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (*err != cudaSuccess) return nullptr;
    addr[dev] = p;
  }
  return addr[dev];
}

}  // namespace
}  // namespace q3vl

extern "C" {

int q3vl_layer_prefill_noalloc(const q3vl_config* cfg, const q3vl_layer* layer, void* x,
                               int64_t S, const int32_t* pos, const void* ds_slab,
                               const int32_t* ds_rows, int32_t n_img, q3vl_stream stream) {
  const size_t need = q3vl_workspace_bytes(cfg, S);
  if (need == 0)  // invalid config or length: let the full validation report it
    return q3vl_layer_prefill(cfg, layer, x, S, pos, ds_slab, ds_rows, n_img, nullptr, 0, stream);
  if (need > q3vl::kNoAllocScratchBytes)
    return q3vl::set_error(
        Q3VL_EWORKSPACE,
        "q3vl_layer_prefill_noalloc: this layer at S=" + std::to_string(S) + " needs " +
            std::to_string(need) + " bytes of scratch, above the built-in " +
            std::to_string(q3vl::kNoAllocScratchBytes) +
            " bytes; use q3vl_layer_prefill with a caller workspace");
  cudaError_t e = cudaSuccess;
  void* scratch = q3vl::scratch_address(&e);
  if (scratch == nullptr) return q3vl::cuda_check(e, "q3vl_layer_prefill_noalloc: scratch address");
  return q3vl_layer_prefill(cfg, layer, x, S, pos, ds_slab, ds_rows, n_img, scratch,
                            q3vl::kNoAllocScratchBytes, stream);
}

}  // extern "C"
