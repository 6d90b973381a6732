// fp_noalloc.cu -- fp_sparse_prefill_noalloc: the one-call sparse prefill without a caller workspace.
//
// Some callers cannot call cudaMalloc: serving loops that plan all device memory up front and may not
// grow it in the middle of a step, plugin hosts that hand an operator no workspace, and code where the
// implicit device synchronisation of cudaMalloc is not acceptable. For them this entry point runs the
// same pool -> search -> sparse-attention kernels as fp_sparse_prefill, with the intermediate tensors
// (pooled Q/K, counts, index lists) in a fixed-size array compiled into the library's device image.
// It allocates nothing itself: no cudaMalloc, cudaFree or allocating library routine is called.
//
// Costs and rules of the shared array:
//   - every GPU that loads libfp holds FP_NOALLOC_MAX_BYTES of device memory for it until the process
//     exits;
//   - all calls on a device share the one array and it keeps the previous call's contents; nothing in
//     it has to start at zero (each call writes every count and list entry before reading it), but
//     calls that overlap on the GPU (another stream, another host thread) race on it;
//   - the first call on a device looks up the array's device address (cudaGetSymbolAddress, with that
//     device current); make that first call before any stream capture. The address is cached per
//     device under the id of the device's context; a context destroyed and created again (e.g. by
//     cudaDeviceReset) gets a new id, so the first call after it looks the address up again (make
//     that call, too, outside stream capture);
//   - problems whose intermediates exceed FP_NOALLOC_MAX_BYTES are rejected with FP_ERR_INVALID_ARG.
#include <mutex>

#include "fp_internal.h"

namespace {

// The scratch array. Host code must not use this name as a device address: on the host it is only a
// stand-in, and the kernels receive the address from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[FP_NOALLOC_MAX_BYTES];

constexpr int kMaxDevices = fp::kMaxCachedDevices;
std::mutex g_mu;
struct CachedAddr {
  unsigned long long ctx;  // id of the context the address belongs to (0: none cached)
  void* ptr;
};
CachedAddr g_scratch_addr[kMaxDevices] = {};

// Device address of the array in the current device's context. Looked up once per context with
// cudaGetSymbolAddress and cached under the context's unique id: after the context is destroyed and
// created again (cudaDeviceReset), the module is loaded anew, its array may sit elsewhere, and the
// changed id makes the next call look the address up again.
fp_status scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0)
    return fp::set_error(FP_ERR_CUDA, "no current CUDA device: %s", cudaGetErrorString(e));
  if (dev >= kMaxDevices) return fp::set_error(FP_ERR_UNSUPPORTED, "device ordinal %d >= %d", dev, kMaxDevices);
  std::lock_guard<std::mutex> lock(g_mu);
  const unsigned long long id = fp::context_id();
  if (id == 0 || g_scratch_addr[dev].ctx != id || !g_scratch_addr[dev].ptr) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess || !ptr)
      return fp::set_error(FP_ERR_CUDA, "cudaGetSymbolAddress of the static scratch failed: %s",
                           cudaGetErrorString(e));
    g_scratch_addr[dev].ctx = fp::context_id();  // the lookup made the context current
    g_scratch_addr[dev].ptr = ptr;
  }
  *out = g_scratch_addr[dev].ptr;
  return FP_OK;
}

}  // namespace

extern "C" fp_status fp_sparse_prefill_noalloc(const fp_problem* p, const void* q, const void* k, const void* v,
                                               float tau, float softmax_scale, void* out, float* lse,
                                               int32_t* dev_status, void* stream) {
  int64_t need = 0;
  fp_status st = fp_sparse_prefill_workspace(p, &need);
  if (st != FP_OK) return st;
  if (need > (int64_t)FP_NOALLOC_MAX_BYTES)
    return fp::set_error(FP_ERR_INVALID_ARG,
                         "this problem needs %lld bytes of intermediates, more than the %lld-byte static array of "
                         "fp_sparse_prefill_noalloc; call fp_sparse_prefill with a workspace instead",
                         (long long)need, (long long)FP_NOALLOC_MAX_BYTES);
  void* scratch = nullptr;
  if ((st = scratch_address(&scratch)) != FP_OK) return st;
  return fp_sparse_prefill(p, q, k, v, tau, softmax_scale, scratch, (int64_t)FP_NOALLOC_MAX_BYTES, out, lse,
                           dev_status, stream);
}
