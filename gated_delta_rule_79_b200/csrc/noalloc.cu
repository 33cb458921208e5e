// gdn_prefill_noalloc: gdn_prefill with a library-owned, statically allocated
// scratch instead of a caller-provided workspace.
//
// Some callers cannot allocate device memory on the call path: serving loops that
// must never stall the device (cudaMalloc and cudaFree can synchronize it), and
// embedders whose device memory belongs to another allocator under a fixed
// budget.  For them this entry point uses a file-scope __device__ array as the
// prefill workspace.  It holds kNoAllocScratchBytes bytes on every GPU that
// loads the library, until the process exits; requests that would need more
// scratch than that are rejected.
//
// The array's host-side name is only a stand-in for the device symbol (handing it
// to a kernel would fault, or silently touch host memory where the GPU can reach
// it), so its device address is looked up with cudaGetSymbolAddress, once per
// device, the first time the entry point runs with that device current.  That
// first call therefore performs a CUDA runtime query and should happen before any
// stream capture on that device.
//
// Every call shares the one array.  The kernels only ever set bits of the status
// word at its start; the entry point clears the word after each launch, so it is
// zero when the next call starts.  Calls that overlap on the GPU (different
// streams without ordering between them) race on the array.

#include <stdio.h>

#include <mutex>

#include "gdr.h"
#include "launch.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 4096;
constexpr size_t kStatusBytes = 256;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

void* g_scratch_ptr[kMaxDevices];
cudaError_t g_scratch_err[kMaxDevices];
std::once_flag g_scratch_once[kMaxDevices];

gdr_status fail(gdr_status s, const char* fmt, size_t a = 0, size_t b = 0) {
  char msg[256];
  snprintf(msg, sizeof msg, fmt, a, b);
  return (gdr_status)gdr::report_error(s, msg);
}

}  // namespace

extern "C" gdr_status gdn_prefill_noalloc(const void* q, const void* k, const void* v,
                                          const float* alpha, const float* beta, const float* s0,
                                          void* o, float* s_final, int B, int T, int H, int dk,
                                          int dv, int in_dtype, int out_dtype, int chunk,
                                          void* stream) {
  // The static scratch serves the single-kernel prefill, which needs the status word
  // only; the faster two-kernel path would need gdr_prefill_workspace_bytes(...).
  const size_t need = gdr_prefill_workspace_bytes(B, T, H, dk, dv, 0) ? kStatusBytes : 0;
  if (need > kNoAllocScratchBytes)
    return fail(GDR_ERR_INVALID_ARG,
                "gdn_prefill_noalloc: these sizes need %zu bytes of scratch; the static "
                "scratch holds %zu",
                need, kNoAllocScratchBytes);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess)
    return fail(GDR_ERR_CUDA, "gdn_prefill_noalloc: cudaGetDevice failed");
  if (dev < 0 || dev >= kMaxDevices)
    return fail(GDR_ERR_UNSUPPORTED, "gdn_prefill_noalloc: device ordinal %zu beyond %zu",
                (size_t)dev, (size_t)kMaxDevices);
  std::call_once(g_scratch_once[dev], [dev] {
    g_scratch_err[dev] = cudaGetSymbolAddress(&g_scratch_ptr[dev], g_noalloc_scratch);
  });
  if (g_scratch_err[dev] != cudaSuccess || g_scratch_ptr[dev] == nullptr)
    return fail(GDR_ERR_CUDA, "gdn_prefill_noalloc: cudaGetSymbolAddress of the scratch failed");
  const gdr_status s = gdn_prefill(q, k, v, alpha, beta, s0, o, s_final, B, T, H, dk, dv,
                                   in_dtype, out_dtype, chunk, g_scratch_ptr[dev],
                                   kNoAllocScratchBytes, stream);
  if (s != GDR_OK) return s;
  // leave the status word at zero for the next call on this device
  if (cudaMemsetAsync(g_scratch_ptr[dev], 0, kStatusBytes, (cudaStream_t)stream) != cudaSuccess)
    return fail(GDR_ERR_CUDA, "gdn_prefill_noalloc: clearing the scratch status word failed");
  return GDR_OK;
}
