// si_indexer_materialize_noalloc: the materialize path without any device
// allocation.
//
// Some callers cannot allocate device memory when they call this library: a
// host application that has already handed nearly all of the GPU's memory to
// its own pool (a serving engine's cache, for instance) and forbids anything
// else from calling cudaMalloc; a plugin interface whose execute step must
// not allocate; a latency-critical loop in which cudaMalloc / cudaFree would
// synchronise the device.  For them this entry point runs the same three
// materialize kernels with their [B,S,H_I,T] logits and [B,S,T] scores placed
// in a fixed device array of this file instead of memory allocated per call.
//
// The array is SI_NOALLOC_SCRATCH_BYTES (64 MiB) on every GPU where the
// library's module is loaded, held until the process exits.  Under CUDA's
// lazy module loading (the default) that happens at the first call of this
// entry point on the device, which therefore itself needs the 64 MiB free:
// a caller whose pool is about to take nearly all memory makes one call
// first (any small problem) to reserve it.  If the reservation fails the
// call returns SI_ERR_OUT_OF_MEMORY.  Problems whose scratch need,
// 4*B*S*T*(H_I+1) + 256 bytes, exceeds the array are rejected.  All calls
// share the array and it keeps the last call's contents; the kernels
// overwrite every word they read before reading it, so nothing needs
// clearing.  Each device has its own copy; two calls on one device whose
// work overlaps on the GPU (on different streams, say) race on it, so
// serialise them.
#include <cuda_runtime.h>

#include "si_internal.h"

namespace si {
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[SI_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch array in the current context.  Host code
// only sees a host-side stand-in for the array's name, so the address is
// asked for on every call, with the caller's device current: no cached
// pointer can outlive a device reset or belong to another context.  The
// first lookup on a device loads the module and so reserves the array.
si_status scratch_address(void** out) {
  void* ptr = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
  if (e == cudaErrorMemoryAllocation) {
    cudaGetLastError();
    return fail(SI_ERR_OUT_OF_MEMORY,
                "reserving the %zu-byte no-alloc scratch array on this device failed (%s); make the "
                "first call before other allocations fill the device",
                static_cast<size_t>(SI_NOALLOC_SCRATCH_BYTES), cudaGetErrorString(e));
  }
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-alloc scratch)");
  *out = ptr;
  return SI_OK;
}

}  // namespace
}  // namespace si

extern "C" si_status si_indexer_materialize_noalloc(const void* q, const void* kc, const float* w,
                                                    int B, int S, int T, int H_I, int D, int m,
                                                    int k, int32_t* out_idx, float* out_score,
                                                    void* stream) {
  using namespace si;
  si_status st = check_common(q, kc, w, B, S, T, H_I, D, m, k, out_idx, out_score);
  if (st != SI_OK) return st;
  if (T > 16384) return fail(SI_ERR_UNSUPPORTED, "materialize path sorts rows of T <= 16384 (got %d)", T);
  const size_t need = materialize_workspace_bytes(B, S, T, H_I);
  if (need > static_cast<size_t>(SI_NOALLOC_SCRATCH_BYTES))
    return fail(SI_ERR_UNSUPPORTED,
                "no-alloc materialize needs %zu bytes of scratch (4*B*S*T*(H_I+1) + 256); its fixed "
                "array holds %zu",
                need, static_cast<size_t>(SI_NOALLOC_SCRATCH_BYTES));
  void* scratch = nullptr;
  st = scratch_address(&scratch);
  if (st != SI_OK) return st;
  return launch_materialize(q, kc, w, B, S, T, H_I, D, m, k, out_idx, out_score,
                            static_cast<cudaStream_t>(stream), scratch,
                            static_cast<size_t>(SI_NOALLOC_SCRATCH_BYTES));
}
