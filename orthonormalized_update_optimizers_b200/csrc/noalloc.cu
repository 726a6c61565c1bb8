// gram_ns_orthogonalize_noalloc: Gram Newton-Schulz for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc: for example a plugin running inside a
// host framework whose own pool owns all device memory, or a latency-critical
// path that must not pay cudaMalloc's implicit device synchronization.  They
// cannot provide the workspace gram_ns_orthogonalize needs, so this entry
// point uses a fixed scratch array that lives in the library's device image
// instead.  The caller still passes its inputs and outputs.
//
// The scratch array is a file-scope __device__ array of
// OUO_NOALLOC_SCRATCH_BYTES bytes; a GPU holds it from the moment this part
// of the library is loaded on it until the process exits.  Host code cannot
// use the array's name as a device address (in host code the name is only a
// stand-in), so every call, with the device current, looks the address up
// with cudaGetSymbolAddress and checks the result.  The first call on a
// device also loads the library's device image there (the set-up); make
// that first call before any stream capture.  The address is not cached:
// after cudaDeviceReset, or any new primary context, the image is loaded
// again and the array may sit elsewhere, and a stale address would send the
// kernels' writes into memory the library does not own.
//
// Every call uses the same array, and a call overwrites every part of it it
// reads, so nothing carries over from one call to the next.  Calls whose
// kernels overlap on the GPU (for example, issued on two different streams
// without ordering between them) race on the array.
#include "internal.h"

namespace ouo {
namespace {

static __device__ __align__(256) unsigned char
    g_noalloc_scratch[OUO_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch array on the current device.
int scratch_address(void** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess || !p)
    return set_error(OUO_ERR_CUDA, "cudaGetSymbolAddress(scratch) failed: %s",
                     cudaGetErrorString(e));
  *out = p;
  return OUO_OK;
}

}  // namespace
}  // namespace ouo

extern "C" int gram_ns_orthogonalize_noalloc(const ouo_mat* X, int x_dtype,
                                             const ouo_mat* O, int o_dtype,
                                             int nmat, const ouo_ns_params* p,
                                             int* dev_status, void* stream) {
  using namespace ouo;
  clear_error();
  // the same argument checks as gram_ns_orthogonalize, before the size is
  // computed from those arguments
  OUO_TRY(ns_check_call(X, x_dtype, O, o_dtype, nmat, p, dev_status));
  if (nmat == 0) return OUO_OK;
  const size_t need = gram_ns_workspace_bytes(X, nmat, p);
  if (need > (size_t)OUO_NOALLOC_SCRATCH_BYTES)
    return set_error(OUO_ERR_WORKSPACE,
                     "gram_ns_orthogonalize_noalloc: this batch needs %zu bytes "
                     "of scratch, the fixed array holds %zu; split the batch or "
                     "use gram_ns_orthogonalize with a caller workspace",
                     need, (size_t)OUO_NOALLOC_SCRATCH_BYTES);
  OUO_TRY(require_sm100());
  void* ws = nullptr;
  OUO_TRY(scratch_address(&ws));
  return gram_ns_orthogonalize(X, x_dtype, O, o_dtype, nmat, p, ws,
                               (size_t)OUO_NOALLOC_SCRATCH_BYTES, dev_status,
                               stream);
}
