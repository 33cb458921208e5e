// gdn_prefill_noalloc: gdn_prefill with a library-owned, statically allocated
// scratch instead of a caller-provided workspace, and gdr_noalloc_status, which
// reports what that scratch recorded.
//
// Some callers cannot allocate device memory on the call path: serving loops that
// must never stall the device (cudaMalloc and cudaFree can synchronize it), and
// embedders whose device memory belongs to another allocator under a fixed
// budget.  For them this entry point uses a file-scope __device__ array as the
// prefill workspace.  It holds kNoAllocScratchBytes bytes on every GPU that
// loads the library, until the process exits.  The prefill it runs (the
// single-kernel tensor-core kernel, or the CUDA-core kernel) needs only the
// status word at the start of its workspace, whatever the sizes, so no size
// needs more scratch than the array holds; sizes the library cannot index are
// rejected here, under this function's name.
//
// The array's host-side name is only a stand-in for the device symbol (handing it
// to a kernel would fault, or silently touch host memory where the GPU can reach
// it), so its device address is looked up with cudaGetSymbolAddress, per device,
// the first time the entry point runs with that device current; only a successful
// lookup is kept, so a failed one is tried again on the next call.  That first call
// therefore performs a CUDA runtime query and should happen before any stream
// capture on that device.
//
// Every call shares the one array.  The kernels only ever set bits of the status
// word at its start.  After each prefill the entry point launches a one-warp kernel
// that ORs that word into a second, sticky device word and clears it, so the word
// is zero when the next call starts and a bounded wait that gave up stays on record
// until gdr_noalloc_status reads (and clears) it.  Calls that overlap on the GPU
// (different streams without ordering between them) race on the array.

#include <stdarg.h>
#include <stdio.h>

#include <mutex>

#include "gdr.h"
#include "launch.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 4096;
constexpr size_t kStatusBytes = 256;
constexpr int kMaxDevices = 64;
static_assert(kStatusBytes <= kNoAllocScratchBytes, "the status word must fit the scratch");

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
// Bits of every status word the prefill kernels left in the scratch since the last
// gdr_noalloc_status on this device.
__device__ unsigned int g_noalloc_sticky;

struct DeviceSymbols {
  std::mutex mu;
  bool resolved = false;
  void* scratch = nullptr;
  void* sticky = nullptr;
};
DeviceSymbols g_sym[kMaxDevices];

gdr_status fail(gdr_status s, const char* fmt, ...) {
  char msg[320];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(msg, sizeof msg, fmt, ap);
  va_end(ap);
  return (gdr_status)gdr::report_error(s, msg);
}

// Device addresses of the scratch and of the sticky word on the current device, looked
// up once per device (a failed lookup is not cached).
gdr_status symbols(const char* fn, void** scratch, void** sticky) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(GDR_ERR_CUDA, "%s: cudaGetDevice failed", fn);
  if (dev < 0 || dev >= kMaxDevices)
    return fail(GDR_ERR_UNSUPPORTED, "%s: device ordinal %d beyond %d", fn, dev, kMaxDevices);
  DeviceSymbols& s = g_sym[dev];
  std::lock_guard<std::mutex> lock(s.mu);
  if (!s.resolved) {
    void* a = nullptr;
    void* b = nullptr;
    const cudaError_t e1 = cudaGetSymbolAddress(&a, g_noalloc_scratch);
    const cudaError_t e2 = e1 == cudaSuccess ? cudaGetSymbolAddress(&b, g_noalloc_sticky) : e1;
    if (e2 != cudaSuccess || a == nullptr || b == nullptr)
      return fail(GDR_ERR_CUDA, "%s: cudaGetSymbolAddress of the static scratch failed (%s)", fn,
                  cudaGetErrorString(e2));
    s.scratch = a;
    s.sticky = b;
    s.resolved = true;
  }
  *scratch = s.scratch;
  *sticky = s.sticky;
  return GDR_OK;
}

// One warp: fold the scratch's status word into the sticky word and clear it.
__global__ void noalloc_settle_kernel() {
  if (threadIdx.x == 0) {
    unsigned int* word = reinterpret_cast<unsigned int*>(g_noalloc_scratch);
    const unsigned int w = *word;
    if (w != 0) {
      atomicOr(&g_noalloc_sticky, w);
      *word = 0u;
    }
  }
}

}  // namespace

extern "C" gdr_status gdn_prefill_noalloc(const void* q, const void* k, const void* v,
                                          const float* alpha, const float* beta, const float* s0,
                                          void* o, float* s_final, int B, int T, int H, int dk,
                                          int dv, int in_dtype, int out_dtype, int chunk,
                                          void* stream) {
  // gdr_prefill_workspace_bytes is 0 for negative sizes and for sizes whose workspace
  // arithmetic would overflow: beyond what the library indexes.  The paths this entry
  // point reaches need kStatusBytes of scratch for any size (checked at compile time).
  if (B >= 0 && T >= 0 && H >= 0 && gdr_prefill_workspace_bytes(B, T, H, dk, dv, 0) == 0 &&
      (dk == 32 || dk == 64 || dk == 128) && (dv == 32 || dv == 64 || dv == 128))
    return fail(GDR_ERR_INVALID_ARG,
                "gdn_prefill_noalloc: B=%d T=%d H=%d d_k=%d d_v=%d exceed the sizes the library "
                "indexes", B, T, H, dk, dv);
  void* scratch = nullptr;
  void* sticky = nullptr;
  const gdr_status r = symbols("gdn_prefill_noalloc", &scratch, &sticky);
  if (r != GDR_OK) return r;
  const gdr_status s = gdn_prefill(q, k, v, alpha, beta, s0, o, s_final, B, T, H, dk, dv,
                                   in_dtype, out_dtype, chunk, scratch, kNoAllocScratchBytes,
                                   stream);
  if (s != GDR_OK) return s;
  noalloc_settle_kernel<<<1, 32, 0, (cudaStream_t)stream>>>();
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return fail(GDR_ERR_CUDA,
                "gdn_prefill_noalloc: the prefill was enqueued, but the launch that records its "
                "status failed (%s)", cudaGetErrorString(e));
  return GDR_OK;
}

extern "C" gdr_status gdr_noalloc_status(void* stream) {
  void* scratch = nullptr;
  void* sticky = nullptr;
  const gdr_status r = symbols("gdr_noalloc_status", &scratch, &sticky);
  if (r != GDR_OK) return r;
  cudaStream_t st = (cudaStream_t)stream;
  unsigned int word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, sticky, sizeof word, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess && word != 0) e = cudaMemsetAsync(sticky, 0, sizeof word, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return fail(GDR_ERR_CUDA, "gdr_noalloc_status: %s", cudaGetErrorString(e));
  if (word & 3u)
    return fail(GDR_ERR_TIMEOUT,
                "a bounded device wait of gdn_prefill_noalloc gave up (status bits 0x%08x); the "
                "outputs of the calls since the last query are undefined", word);
  if (word != 0) return fail(GDR_ERR_CUDA, "gdn_prefill_noalloc recorded status bits 0x%08x", word);
  return (gdr_status)gdr::report_error(GDR_OK, "");
}
