// C ABI of libgdr (declared in include/gdr.h): argument validation, kernel
// selection and error reporting.  Every entry point validates all of its
// arguments on the host before anything is enqueued, so a rejected call leaves
// the device untouched.

#include <stdarg.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include <mutex>
#include <string>

#include "gdr.h"
#include "launch.h"

namespace gdr {

static thread_local std::string g_last_error;

static gdr_status fail(gdr_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

int report_error(int s, const char* msg) { return fail((gdr_status)s, "%s", msg); }

#ifdef GDR_CHECKS
static std::mutex g_checks_mu;
static unsigned int* g_checks[64];

unsigned int* checks_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(g_checks_mu);
  if (!g_checks[dev]) {
    void* p = nullptr;
    if (cudaMalloc(&p, sizeof(unsigned int)) != cudaSuccess) return nullptr;
    if (cudaMemset(p, 0, sizeof(unsigned int)) != cudaSuccess ||
        cudaDeviceSynchronize() != cudaSuccess) {
      cudaFree(p);
      return nullptr;
    }
    g_checks[dev] = static_cast<unsigned int*>(p);
  }
  return g_checks[dev];
}
#else
unsigned int* checks_word() { return nullptr; }
#endif

static gdr_status ok() {
  g_last_error.clear();
  return GDR_OK;
}

static bool head_ok(int d) { return d == 32 || d == 64 || d == 128; }
static bool dtype_ok(int t) { return t == GDR_F32 || t == GDR_BF16; }
static bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// Bytes of the status word area at the start of a prefill workspace.
constexpr size_t kStatusBytes = 256;
constexpr unsigned kPrologueFlags = GDR_PROLOGUE_L2NORM_QK | GDR_PROLOGUE_GATE_LOGIT;

bool tc_prefill_supported(const PrefillArgs& a);   // prefill_tc.cu
size_t tc_prefill_workspace(int B, int T, int H, int dk, int dv, bool kda);
cudaError_t launch_prefill_tc(const PrefillArgs& a, cudaStream_t stream);

static gdr_status prefill(bool kda, const void* q, const void* k, const void* v,
                          const float* alpha, const float* beta, const float* s0, void* o,
                          float* s_final, int B, int T, int H, int dk, int dv, int in_dtype,
                          int out_dtype, int chunk, void* workspace, size_t ws_bytes,
                          void* stream, unsigned pro) {
  const char* fn = kda ? "kda_prefill" : "gdn_prefill";
  if (pro & ~kPrologueFlags) return fail(GDR_ERR_INVALID_ARG, "%s: unknown prologue flags 0x%x", fn, pro);
  if (B < 0 || T < 0 || H < 0)
    return fail(GDR_ERR_INVALID_ARG, "%s: negative size B=%d T=%d H=%d", fn, B, T, H);
  if (!head_ok(dk) || !head_ok(dv))
    return fail(GDR_ERR_UNSUPPORTED, "%s: d_k=%d d_v=%d (supported: 32, 64, 128)", fn, dk, dv);
  if (!dtype_ok(in_dtype) || !dtype_ok(out_dtype))
    return fail(GDR_ERR_INVALID_ARG, "%s: bad dtype in=%d out=%d", fn, in_dtype, out_dtype);
  if (chunk != GDR_CHUNK)
    return fail(GDR_ERR_UNSUPPORTED, "%s: chunk=%d (only %d is supported)", fn, chunk, GDR_CHUNK);
  const size_t need = gdr_prefill_workspace_bytes(B, T, H, dk, dv, kda);
  if (need == 0) return fail(GDR_ERR_INVALID_ARG, "%s: sizes overflow", fn);
  if (!workspace || ws_bytes < kStatusBytes)
    return fail(GDR_ERR_INVALID_ARG, "%s: workspace %p of %zu bytes, need at least %zu", fn,
                workspace, ws_bytes, kStatusBytes);
  if (((uintptr_t)workspace & 255u) != 0)
    return fail(GDR_ERR_INVALID_ARG, "%s: workspace must be 256-byte aligned", fn);
  cudaStream_t st = (cudaStream_t)stream;
  const size_t state_bytes = (size_t)B * H * dv * dk * sizeof(float);
  if (B == 0 || H == 0) return ok();
  if (T == 0) {
    if (!s_final) return ok();
    if (!aligned16(s_final)) return fail(GDR_ERR_INVALID_ARG, "%s: s_final misaligned", fn);
    cudaError_t e = s0 ? (s0 == s_final ? cudaSuccess
                                        : cudaMemcpyAsync(s_final, s0, state_bytes,
                                                          cudaMemcpyDeviceToDevice, st))
                       : cudaMemsetAsync(s_final, 0, state_bytes, st);
    if (e != cudaSuccess) return fail(GDR_ERR_CUDA, "%s: %s", fn, cudaGetErrorString(e));
    return ok();
  }
  const void* need_ptrs[] = {q, k, v, alpha, beta, o};
  const char* names[] = {"q", "k", "v", "alpha", "beta", "o"};
  for (int i = 0; i < 6; ++i) {
    if (!need_ptrs[i]) return fail(GDR_ERR_INVALID_ARG, "%s: %s is NULL", fn, names[i]);
    if (!aligned16(need_ptrs[i]))
      return fail(GDR_ERR_INVALID_ARG, "%s: %s is not 16-byte aligned", fn, names[i]);
  }
  if ((s0 && !aligned16(s0)) || (s_final && !aligned16(s_final)))
    return fail(GDR_ERR_INVALID_ARG, "%s: s0/s_final not 16-byte aligned", fn);
  PrefillArgs a{q, k, v, alpha, beta, s0, o, s_final, B, T, H, dk, dv,
                in_dtype, out_dtype, kda, workspace, ws_bytes, pro};
  timing_mark(st, -1);
  // the fused prologue runs in the two-kernel tensor-core prefill or in the CUDA-core
  // kernel, not in the single-kernel tensor-core fallbacks (used with a small workspace)
  const bool tc = tc_prefill_supported(a) && (pro == 0 || ws_bytes >= need);
  cudaError_t e = tc ? launch_prefill_tc(a, st) : launch_prefill_simt(a, st);
  if (e != cudaSuccess) return fail(GDR_ERR_CUDA, "%s: launch failed: %s", fn, cudaGetErrorString(e));
  return ok();
}

static gdr_status decode(bool kda, const void* q, const void* k, const void* v,
                         const float* alpha, const float* beta, float* state, void* o, int N,
                         int H, int dk, int dv, int in_dtype, int out_dtype, void* stream,
                         unsigned pro) {
  const char* fn = kda ? "kda_decode" : "gdn_decode";
  if (pro & ~kPrologueFlags) return fail(GDR_ERR_INVALID_ARG, "%s: unknown prologue flags 0x%x", fn, pro);
  if (N < 0 || H < 0) return fail(GDR_ERR_INVALID_ARG, "%s: negative size N=%d H=%d", fn, N, H);
  if (!head_ok(dk) || !head_ok(dv))
    return fail(GDR_ERR_UNSUPPORTED, "%s: d_k=%d d_v=%d (supported: 32, 64, 128)", fn, dk, dv);
  if (!dtype_ok(in_dtype) || !dtype_ok(out_dtype))
    return fail(GDR_ERR_INVALID_ARG, "%s: bad dtype in=%d out=%d", fn, in_dtype, out_dtype);
  if ((long long)N * H > (1LL << 31) / 4)
    return fail(GDR_ERR_INVALID_ARG, "%s: N*H too large", fn);
  if (N == 0 || H == 0) return ok();
  const void* need_ptrs[] = {q, k, v, alpha, beta, state, o};
  const char* names[] = {"q", "k", "v", "alpha", "beta", "state", "o"};
  for (int i = 0; i < 7; ++i) {
    if (!need_ptrs[i]) return fail(GDR_ERR_INVALID_ARG, "%s: %s is NULL", fn, names[i]);
    if (!aligned16(need_ptrs[i]))
      return fail(GDR_ERR_INVALID_ARG, "%s: %s is not 16-byte aligned", fn, names[i]);
  }
  DecodeArgs a{q, k, v, alpha, beta, state, o, N, H, dk, dv, in_dtype, out_dtype, kda, pro};
  cudaError_t e = launch_decode(a, (cudaStream_t)stream);
  if (e != cudaSuccess) return fail(GDR_ERR_CUDA, "%s: launch failed: %s", fn, cudaGetErrorString(e));
  return ok();
}

static gdr_status verify(bool kda, const void* q, const void* k, const void* v,
                         const float* alpha, const float* beta, float* state, float* snapshots,
                         void* o, int N, int K, int H, int dk, int dv, int in_dtype,
                         int out_dtype, void* stream, unsigned pro) {
  const char* fn = kda ? "kda_verify" : "gdn_verify";
  if (pro & ~kPrologueFlags) return fail(GDR_ERR_INVALID_ARG, "%s: unknown prologue flags 0x%x", fn, pro);
  if (N < 0 || H < 0) return fail(GDR_ERR_INVALID_ARG, "%s: negative size N=%d H=%d", fn, N, H);
  if (K < 1 || K > GDR_VERIFY_MAX_TOKENS)
    return fail(GDR_ERR_UNSUPPORTED, "%s: K=%d tokens (supported: 1 to %d)", fn, K,
                GDR_VERIFY_MAX_TOKENS);
  if (!head_ok(dk) || !head_ok(dv))
    return fail(GDR_ERR_UNSUPPORTED, "%s: d_k=%d d_v=%d (supported: 32, 64, 128)", fn, dk, dv);
  if (!dtype_ok(in_dtype) || !dtype_ok(out_dtype))
    return fail(GDR_ERR_INVALID_ARG, "%s: bad dtype in=%d out=%d", fn, in_dtype, out_dtype);
  if ((long long)N * H > (1LL << 31) / 4 || (long long)N * H * K * (dk > dv ? dk : dv) > (1LL << 40))
    return fail(GDR_ERR_INVALID_ARG, "%s: N*H too large", fn);
  if (N == 0 || H == 0) return ok();
  const void* need_ptrs[] = {q, k, v, alpha, beta, state, o};
  const char* names[] = {"q", "k", "v", "alpha", "beta", "state", "o"};
  for (int i = 0; i < 7; ++i) {
    if (!need_ptrs[i]) return fail(GDR_ERR_INVALID_ARG, "%s: %s is NULL", fn, names[i]);
    if (!aligned16(need_ptrs[i]))
      return fail(GDR_ERR_INVALID_ARG, "%s: %s is not 16-byte aligned", fn, names[i]);
  }
  if (snapshots && !aligned16(snapshots))
    return fail(GDR_ERR_INVALID_ARG, "%s: snapshots is not 16-byte aligned", fn);
  VerifyArgs a{q, k, v, alpha, beta, state, snapshots, o, N, K, H, dk, dv,
               in_dtype, out_dtype, kda, pro};
  cudaError_t e = launch_verify(a, (cudaStream_t)stream);
  if (e != cudaSuccess) return fail(GDR_ERR_CUDA, "%s: launch failed: %s", fn, cudaGetErrorString(e));
  return ok();
}

static gdr_status backward(bool kda, const void* q, const void* k, const void* v,
                           const float* alpha, const float* beta, const float* s0,
                           const void* dO, const float* ds_final, float* dq, float* dkk,
                           float* dvv, float* dalpha, float* dbeta, float* ds0, int B, int T,
                           int H, int dk, int dv, int in_dtype, int do_dtype, void* workspace,
                           size_t ws_bytes, void* stream) {
  const char* fn = kda ? "kda_backward" : "gdn_backward";
  if (B < 0 || T < 0 || H < 0)
    return fail(GDR_ERR_INVALID_ARG, "%s: negative size B=%d T=%d H=%d", fn, B, T, H);
  if (!head_ok(dk) || !head_ok(dv))
    return fail(GDR_ERR_UNSUPPORTED, "%s: d_k=%d d_v=%d (supported: 32, 64, 128)", fn, dk, dv);
  if (!dtype_ok(in_dtype) || !dtype_ok(do_dtype))
    return fail(GDR_ERR_INVALID_ARG, "%s: bad dtype in=%d do=%d", fn, in_dtype, do_dtype);
  if ((long long)B * H > (1LL << 24) || T > (1 << 28) ||
      (long long)B * T * H * (dk > dv ? dk : dv) > (1LL << 40))
    return fail(GDR_ERR_INVALID_ARG, "%s: sizes too large", fn);
  if (B == 0 || H == 0) return ok();
  const void* need_ptrs[] = {q, k, v, alpha, beta, dO, dq, dkk, dvv, dalpha, dbeta, ds0};
  const char* names[] = {"q", "k", "v", "alpha", "beta", "do", "dq", "dk", "dv", "dalpha",
                         "dbeta", "ds0"};
  for (int i = 0; i < 12; ++i) {
    if (!need_ptrs[i] && (T > 0 || i == 11))
      return fail(GDR_ERR_INVALID_ARG, "%s: %s is NULL", fn, names[i]);
    if (!aligned16(need_ptrs[i]))
      return fail(GDR_ERR_INVALID_ARG, "%s: %s is not 16-byte aligned", fn, names[i]);
  }
  if ((s0 && !aligned16(s0)) || (ds_final && !aligned16(ds_final)))
    return fail(GDR_ERR_INVALID_ARG, "%s: s0/ds_final not 16-byte aligned", fn);
  const size_t need = backward_workspace_bytes(B, T, H, dk, dv);
  if (need > 0 && (!workspace || ws_bytes < need || !aligned16(workspace)))
    return fail(GDR_ERR_INVALID_ARG,
                "%s: workspace of %zu bytes needed (gdr_backward_workspace_bytes), 16-byte "
                "aligned", fn, need);
  BackwardArgs a{q, k, v, alpha, beta, s0, dO, ds_final, dq, dkk, dvv, dalpha, dbeta, ds0,
                 B, T, H, dk, dv, in_dtype, do_dtype, kda, workspace};
  cudaError_t e = launch_backward(a, (cudaStream_t)stream);
  if (e != cudaSuccess) return fail(GDR_ERR_CUDA, "%s: launch failed: %s", fn, cudaGetErrorString(e));
  return ok();
}

}  // namespace gdr

extern "C" {

int gdr_version(void) { return 100; }

const char* gdr_last_error(void) { return gdr::g_last_error.c_str(); }

size_t gdr_prefill_workspace_bytes(int B, int T, int H, int dk, int dv, int kda) {
  if (B < 0 || T < 0 || H < 0) return 0;
  if ((long long)B * H > (1LL << 24) || T > (1 << 28)) return 0;
  return gdr::kStatusBytes + gdr::tc_prefill_workspace(B, T, H, dk, dv, kda != 0);
}

gdr_status gdn_prefill(const void* q, const void* k, const void* v, const float* alpha,
                       const float* beta, const float* s0, void* o, float* s_final, int B,
                       int T, int H, int dk, int dv, int in_dtype, int out_dtype, int chunk,
                       void* workspace, size_t ws_bytes, void* stream) {
  return gdr::prefill(false, q, k, v, alpha, beta, s0, o, s_final, B, T, H, dk, dv, in_dtype,
                      out_dtype, chunk, workspace, ws_bytes, stream, 0u);
}

gdr_status gdn_prefill_ex(const void* q, const void* k, const void* v, const float* alpha,
                          const float* beta, const float* s0, void* o, float* s_final, int B,
                          int T, int H, int dk, int dv, int in_dtype, int out_dtype, int chunk,
                          void* workspace, size_t ws_bytes, void* stream, unsigned prologue) {
  return gdr::prefill(false, q, k, v, alpha, beta, s0, o, s_final, B, T, H, dk, dv, in_dtype,
                      out_dtype, chunk, workspace, ws_bytes, stream, prologue);
}

gdr_status kda_prefill(const void* q, const void* k, const void* v, const float* alpha,
                       const float* beta, const float* s0, void* o, float* s_final, int B,
                       int T, int H, int dk, int dv, int in_dtype, int out_dtype, int chunk,
                       void* workspace, size_t ws_bytes, void* stream) {
  return gdr::prefill(true, q, k, v, alpha, beta, s0, o, s_final, B, T, H, dk, dv, in_dtype,
                      out_dtype, chunk, workspace, ws_bytes, stream, 0u);
}

gdr_status kda_prefill_ex(const void* q, const void* k, const void* v, const float* alpha,
                          const float* beta, const float* s0, void* o, float* s_final, int B,
                          int T, int H, int dk, int dv, int in_dtype, int out_dtype, int chunk,
                          void* workspace, size_t ws_bytes, void* stream, unsigned prologue) {
  return gdr::prefill(true, q, k, v, alpha, beta, s0, o, s_final, B, T, H, dk, dv, in_dtype,
                      out_dtype, chunk, workspace, ws_bytes, stream, prologue);
}

gdr_status gdn_decode(const void* q, const void* k, const void* v, const float* alpha,
                      const float* beta, float* state, void* o, int N, int H, int dk, int dv,
                      int in_dtype, int out_dtype, void* stream) {
  return gdr::decode(false, q, k, v, alpha, beta, state, o, N, H, dk, dv, in_dtype, out_dtype,
                     stream, 0u);
}

gdr_status gdn_decode_ex(const void* q, const void* k, const void* v, const float* alpha,
                         const float* beta, float* state, void* o, int N, int H, int dk, int dv,
                         int in_dtype, int out_dtype, void* stream, unsigned prologue) {
  return gdr::decode(false, q, k, v, alpha, beta, state, o, N, H, dk, dv, in_dtype, out_dtype,
                     stream, prologue);
}

gdr_status kda_decode(const void* q, const void* k, const void* v, const float* alpha,
                      const float* beta, float* state, void* o, int N, int H, int dk, int dv,
                      int in_dtype, int out_dtype, void* stream) {
  return gdr::decode(true, q, k, v, alpha, beta, state, o, N, H, dk, dv, in_dtype, out_dtype,
                     stream, 0u);
}

gdr_status kda_decode_ex(const void* q, const void* k, const void* v, const float* alpha,
                         const float* beta, float* state, void* o, int N, int H, int dk, int dv,
                         int in_dtype, int out_dtype, void* stream, unsigned prologue) {
  return gdr::decode(true, q, k, v, alpha, beta, state, o, N, H, dk, dv, in_dtype, out_dtype,
                     stream, prologue);
}

gdr_status gdn_verify(const void* q, const void* k, const void* v, const float* alpha,
                      const float* beta, float* state, float* snapshots, void* o, int N, int K,
                      int H, int dk, int dv, int in_dtype, int out_dtype, void* stream) {
  return gdr::verify(false, q, k, v, alpha, beta, state, snapshots, o, N, K, H, dk, dv, in_dtype,
                     out_dtype, stream, 0u);
}

gdr_status gdn_verify_ex(const void* q, const void* k, const void* v, const float* alpha,
                         const float* beta, float* state, float* snapshots, void* o, int N,
                         int K, int H, int dk, int dv, int in_dtype, int out_dtype, void* stream,
                         unsigned prologue) {
  return gdr::verify(false, q, k, v, alpha, beta, state, snapshots, o, N, K, H, dk, dv, in_dtype,
                     out_dtype, stream, prologue);
}

gdr_status kda_verify(const void* q, const void* k, const void* v, const float* alpha,
                      const float* beta, float* state, float* snapshots, void* o, int N, int K,
                      int H, int dk, int dv, int in_dtype, int out_dtype, void* stream) {
  return gdr::verify(true, q, k, v, alpha, beta, state, snapshots, o, N, K, H, dk, dv, in_dtype,
                     out_dtype, stream, 0u);
}

gdr_status kda_verify_ex(const void* q, const void* k, const void* v, const float* alpha,
                         const float* beta, float* state, float* snapshots, void* o, int N,
                         int K, int H, int dk, int dv, int in_dtype, int out_dtype, void* stream,
                         unsigned prologue) {
  return gdr::verify(true, q, k, v, alpha, beta, state, snapshots, o, N, K, H, dk, dv, in_dtype,
                     out_dtype, stream, prologue);
}

size_t gdr_backward_workspace_bytes(int B, int T, int H, int dk, int dv, int kda) {
  (void)kda;
  if (B < 0 || T < 0 || H < 0 || !gdr::head_ok(dk) || !gdr::head_ok(dv)) return 0;
  if ((long long)B * H > (1LL << 24) || T > (1 << 28)) return 0;
  return gdr::backward_workspace_bytes(B, T, H, dk, dv);
}

gdr_status gdn_backward(const void* q, const void* k, const void* v, const float* alpha,
                        const float* beta, const float* s0, const void* dO,
                        const float* ds_final, float* dq, float* dk_, float* dv_,
                        float* dalpha, float* dbeta, float* ds0, int B, int T, int H, int dk,
                        int dv, int in_dtype, int do_dtype, void* workspace, size_t ws_bytes,
                        void* stream) {
  return gdr::backward(false, q, k, v, alpha, beta, s0, dO, ds_final, dq, dk_, dv_, dalpha,
                       dbeta, ds0, B, T, H, dk, dv, in_dtype, do_dtype, workspace, ws_bytes,
                       stream);
}

gdr_status kda_backward(const void* q, const void* k, const void* v, const float* alpha,
                        const float* beta, const float* s0, const void* dO,
                        const float* ds_final, float* dq, float* dk_, float* dv_,
                        float* dalpha, float* dbeta, float* ds0, int B, int T, int H, int dk,
                        int dv, int in_dtype, int do_dtype, void* workspace, size_t ws_bytes,
                        void* stream) {
  return gdr::backward(true, q, k, v, alpha, beta, s0, dO, ds_final, dq, dk_, dv_, dalpha,
                       dbeta, ds0, B, T, H, dk, dv, in_dtype, do_dtype, workspace, ws_bytes,
                       stream);
}

int gdr_prefill_path(int dk, int dv, int in_dtype, int kda) {
  if (!gdr::head_ok(dk) || !gdr::head_ok(dv) || !gdr::dtype_ok(in_dtype)) return -1;
  gdr::PrefillArgs a{};
  a.dk = dk;
  a.dv = dv;
  a.in_dtype = in_dtype;
  a.kda = kda != 0;
  return gdr::tc_prefill_supported(a) ? 1 : 0;
}

gdr_status gdr_check_status(void* stream) {
#ifdef GDR_CHECKS
  unsigned int* w = gdr::checks_word();
  if (!w) return gdr::fail(GDR_ERR_CUDA, "gdr_check_status: no device word for the checks");
  cudaStream_t st = (cudaStream_t)stream;
  unsigned int word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, w, sizeof word, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess && word != 0) e = cudaMemsetAsync(w, 0, sizeof word, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return gdr::fail(GDR_ERR_CUDA, "gdr_check_status: %s", cudaGetErrorString(e));
  if (word != 0)
    return gdr::fail(GDR_ERR_INVALID_ARG,
                     "device-side index checks failed (bits 0x%x: 1 chunk location, 2 state "
                     "index, 4 chunk image, 8 decode/verify row layout); the accesses were "
                     "skipped", word);
  return gdr::ok();
#else
  (void)stream;
  return gdr::fail(GDR_ERR_UNSUPPORTED,
                   "gdr_check_status: this library was built without GDR_CHECKS (the checks "
                   "build is libgdr_checks.so)");
#endif
}

gdr_status gdr_workspace_status(void* workspace, size_t ws_bytes, void* stream) {
  if (!workspace || ws_bytes < gdr::kStatusBytes)
    return gdr::fail(GDR_ERR_INVALID_ARG, "gdr_workspace_status: bad workspace");
  cudaStream_t st = (cudaStream_t)stream;
  unsigned int word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, workspace, sizeof word, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess && word != 0) e = cudaMemsetAsync(workspace, 0, sizeof word, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess)
    return gdr::fail(GDR_ERR_CUDA, "gdr_workspace_status: %s", cudaGetErrorString(e));
  if (word & 3u)
    return gdr::fail(GDR_ERR_TIMEOUT, "a bounded device wait gave up (status word 0x%08x)", word);
  if (word != 0)
    return gdr::fail(GDR_ERR_INVALID_ARG,
                     "packed-sequence offsets were not a partition of the tokens (status word "
                     "0x%08x); no chunk was processed", word);
  return gdr::ok();
}

}  // extern "C"
