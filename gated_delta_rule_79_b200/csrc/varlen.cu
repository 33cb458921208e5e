// Packed variable-length prefill: several sequences of different lengths in one
// call, as a serving engine batches prompts, each starting from (and ending in) its
// own slot of a state pool.
//
// "Super Apriel: One Checkpoint, Many Speeds", §2D (inference and serving: the
// supernet is served by an inference engine, vLLM extensions) and §4 (context-length
// scaling): prompts of many lengths are prefilled together and the recurrent state of
// each is kept for its later decode steps.  The tensors are packed along the token
// axis ([total, H, *], sequence i at tokens cu_seqlens[i] .. cu_seqlens[i+1]-1); the
// chunks of 64 tokens never cross a sequence boundary, so a sequence of length L is
// ceil(L / 64) chunks, the last one partial.
//
// varlen_index_kernel numbers the chunks of all sequences (one CTA: a block-wide scan
// of the per-sequence chunk counts) into the workspace, then the two-kernel prefill
// runs with a map that locates each chunk through that index (chunkmap.cuh).  Offsets
// that are not a valid partition of [0, total) (cu_seqlens[0] != 0, a decreasing
// pair, cu_seqlens[nseq] != total) are reported through the workspace status word
// (GDR_ERR_INVALID_ARG from gdr_workspace_status) and no chunk is processed.

#include <stdint.h>
#include <stdio.h>

#include "chunkmap.cuh"
#include "gdr.h"
#include "launch.h"

namespace gdr {
namespace {

constexpr int kIndexThreads = 1024;
constexpr size_t kStatusBytes = 256;

__global__ void __launch_bounds__(kIndexThreads)
varlen_index_kernel(const int* __restrict__ cu, int nseq, int total, int nck,
                    int* __restrict__ cstart, int* __restrict__ cseq,
                    unsigned int* __restrict__ status) {
  __shared__ int wsum[32];
  __shared__ int carry;
  __shared__ int bad;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    carry = 0;
    bad = (cu[0] != 0 || cu[nseq] != total) ? 1 : 0;
  }
  __syncthreads();
  for (int base = 0; base < nseq; base += kIndexThreads) {
    const int i = base + tid;
    int n = 0;
    if (i < nseq) {
      const int len = cu[i + 1] - cu[i];
      if (len < 0) atomicOr(&bad, 1);
      n = len > 0 ? (len + 63) / 64 : 0;
    }
    int x = n;   // inclusive scan inside the warp
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int w = wsum[lane];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, w, off);
        if (lane >= off) w += y;
      }
      wsum[lane] = w;   // inclusive over warps
    }
    __syncthreads();
    const int before = (warp > 0 ? wsum[warp - 1] : 0) + x - n;
    if (i < nseq) cstart[i] = carry + before;
    __syncthreads();
    if (tid == 0) carry += wsum[31];
    __syncthreads();
  }
  if (tid == 0) {
    if (carry > nck) bad = 1;
    cstart[nseq] = carry;
  }
  __syncthreads();
  if (bad) {
    for (int i = tid; i <= nseq; i += kIndexThreads) cstart[i] = 0;
    if (tid == 0) atomicOr(status, 4u);
    return;
  }
  for (int i = tid; i < nseq; i += kIndexThreads)
    for (int c = cstart[i]; c < cstart[i + 1]; ++c) cseq[c] = i;
}

size_t round256(size_t x) { return (x + 255) & ~(size_t)255; }

struct VarlenLayout {
  size_t nck, idx_bytes, total;
};

VarlenLayout varlen_layout(int nseq, int total, int H, bool kda) {
  VarlenLayout l;
  l.nck = (size_t)total / 64 + (size_t)nseq;
  l.idx_bytes = round256(4 * ((size_t)nseq + 1 + l.nck));
  l.total = kStatusBytes + l.idx_bytes +
            (size_t)H * l.nck * (kda ? kda_chunk_image_bytes() : split_chunk_image_bytes());
  return l;
}

gdr_status vfail(gdr_status s, const char* fn, const char* what) {
  char msg[256];
  snprintf(msg, sizeof msg, "%s: %s", fn, what);
  return (gdr_status)report_error(s, msg);
}

bool al16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

gdr_status prefill_varlen(bool kda, const void* q, const void* k, const void* v,
                          const float* alpha, const float* beta, const int* cu_seqlens,
                          const int* slots, float* state, void* o, int nseq, int total, int H,
                          int dk, int dv, int in_dtype, int out_dtype, int chunk,
                          void* workspace, size_t ws_bytes, void* stream, unsigned pro) {
  const char* fn = kda ? "kda_prefill_varlen" : "gdn_prefill_varlen";
  if (pro & ~(GDR_PROLOGUE_L2NORM_QK | GDR_PROLOGUE_GATE_LOGIT))
    return vfail(GDR_ERR_INVALID_ARG, fn, "unknown prologue flags");
  if (nseq < 0 || total < 0 || H < 0) return vfail(GDR_ERR_INVALID_ARG, fn, "negative size");
  if ((long long)total * H > (1LL << 31) || nseq > (1 << 24))
    return vfail(GDR_ERR_INVALID_ARG, fn, "sizes too large");
  if (chunk != GDR_CHUNK) return vfail(GDR_ERR_UNSUPPORTED, fn, "chunk must be 64");
  if (in_dtype != GDR_BF16 || dk != 128 || (dv != 32 && dv != 64 && dv != 128) ||
      (out_dtype != GDR_BF16 && out_dtype != GDR_F32))
    return vfail(GDR_ERR_UNSUPPORTED, fn,
                 "packed sequences run on the bf16 tensor-core path: bf16 inputs, d_k = 128, "
                 "d_v in {32, 64, 128}");
  if (nseq == 0 || H == 0) return (gdr_status)report_error(GDR_OK, "");
  const void* ptrs[] = {q, k, v, alpha, beta, state, o};
  const char* names[] = {"q", "k", "v", "alpha", "beta", "state", "o"};
  for (int i = 0; i < 7; ++i) {
    if (!ptrs[i] && total > 0) {
      char m[64];
      snprintf(m, sizeof m, "%s is NULL", names[i]);
      return vfail(GDR_ERR_INVALID_ARG, fn, m);
    }
    if (!al16(ptrs[i])) {
      char m[64];
      snprintf(m, sizeof m, "%s is not 16-byte aligned", names[i]);
      return vfail(GDR_ERR_INVALID_ARG, fn, m);
    }
  }
  if (!cu_seqlens || ((uintptr_t)cu_seqlens & 3u) || ((uintptr_t)slots & 3u))
    return vfail(GDR_ERR_INVALID_ARG, fn, "cu_seqlens must be a device int32 array (slots too)");
  const VarlenLayout lay = varlen_layout(nseq, total, H, kda);
  if (!workspace || ws_bytes < lay.total || ((uintptr_t)workspace & 255u))
    return vfail(GDR_ERR_INVALID_ARG, fn,
                 "workspace smaller than gdr_prefill_varlen_workspace_bytes(...) or not "
                 "256-byte aligned");
  if (total == 0) return (gdr_status)report_error(GDR_OK, "");   // every state unchanged
  cudaStream_t st = (cudaStream_t)stream;
  unsigned char* ws = (unsigned char*)workspace;
  int* cstart = (int*)(ws + kStatusBytes);
  int* cseq = cstart + nseq + 1;
  timing_mark(st, -1);
  varlen_index_kernel<<<1, kIndexThreads, 0, st>>>(cu_seqlens, nseq, total, (int)lay.nck, cstart,
                                                   cseq, (unsigned int*)workspace);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) {
    ChunkMap m{};
    m.cu = cu_seqlens;
    m.cseq = cseq;
    m.cstart = cstart;
    m.slots = slots;
    m.nseq = nseq;
    m.T = total;
    m.nchunks = 0;
    m.nck = (int)lay.nck;
    m.img_base = kStatusBytes + lay.idx_bytes;
    m.checks = checks_word();
    PrefillArgs a{q, k, v, alpha, beta, state, o, state, 1, total, H, dk, dv,
                  in_dtype, out_dtype, kda, workspace, ws_bytes, pro};
    e = kda ? launch_prefill_kda_split(a, m, st) : launch_prefill_split(a, m, st);
  }
  if (e != cudaSuccess) {
    char m[160];
    snprintf(m, sizeof m, "launch failed: %s", cudaGetErrorString(e));
    return vfail(GDR_ERR_CUDA, fn, m);
  }
  return (gdr_status)report_error(GDR_OK, "");
}

}  // namespace
}  // namespace gdr

extern "C" {

size_t gdr_prefill_varlen_workspace_bytes(int nseq, int total, int H, int dk, int dv, int kda) {
  if (nseq < 0 || total < 0 || H < 0 || dk != 128 || (dv != 32 && dv != 64 && dv != 128))
    return 0;
  return gdr::varlen_layout(nseq, total, H, kda != 0).total;
}

gdr_status gdn_prefill_varlen(const void* q, const void* k, const void* v, const float* alpha,
                              const float* beta, const int* cu_seqlens, const int* slots,
                              float* state, void* o, int nseq, int total, int H, int dk, int dv,
                              int in_dtype, int out_dtype, int chunk, void* workspace,
                              size_t ws_bytes, void* stream) {
  return gdr::prefill_varlen(false, q, k, v, alpha, beta, cu_seqlens, slots, state, o, nseq,
                             total, H, dk, dv, in_dtype, out_dtype, chunk, workspace, ws_bytes,
                             stream, 0u);
}

gdr_status gdn_prefill_varlen_ex(const void* q, const void* k, const void* v,
                                 const float* alpha, const float* beta, const int* cu_seqlens,
                                 const int* slots, float* state, void* o, int nseq, int total,
                                 int H, int dk, int dv, int in_dtype, int out_dtype, int chunk,
                                 void* workspace, size_t ws_bytes, void* stream,
                                 unsigned prologue) {
  return gdr::prefill_varlen(false, q, k, v, alpha, beta, cu_seqlens, slots, state, o, nseq,
                             total, H, dk, dv, in_dtype, out_dtype, chunk, workspace, ws_bytes,
                             stream, prologue);
}

gdr_status kda_prefill_varlen(const void* q, const void* k, const void* v, const float* alpha,
                              const float* beta, const int* cu_seqlens, const int* slots,
                              float* state, void* o, int nseq, int total, int H, int dk, int dv,
                              int in_dtype, int out_dtype, int chunk, void* workspace,
                              size_t ws_bytes, void* stream) {
  return gdr::prefill_varlen(true, q, k, v, alpha, beta, cu_seqlens, slots, state, o, nseq,
                             total, H, dk, dv, in_dtype, out_dtype, chunk, workspace, ws_bytes,
                             stream, 0u);
}

gdr_status kda_prefill_varlen_ex(const void* q, const void* k, const void* v,
                                 const float* alpha, const float* beta, const int* cu_seqlens,
                                 const int* slots, float* state, void* o, int nseq, int total,
                                 int H, int dk, int dv, int in_dtype, int out_dtype, int chunk,
                                 void* workspace, size_t ws_bytes, void* stream,
                                 unsigned prologue) {
  return gdr::prefill_varlen(true, q, k, v, alpha, beta, cu_seqlens, slots, state, o, nseq,
                             total, H, dk, dv, in_dtype, out_dtype, chunk, workspace, ws_bytes,
                             stream, prologue);
}

}  // extern "C"
