// Internal launcher declarations of libgdr (host side).  The C ABI in gdr.h
// validates arguments and then calls these.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace gdr {

struct PrefillArgs {
  const void* q;
  const void* k;
  const void* v;
  const float* alpha;
  const float* beta;
  const float* s0;      // may be null (zeros)
  void* o;
  float* s_final;       // may be null
  int B, T, H, dk, dv;
  int in_dtype, out_dtype;
  bool kda;
  void* workspace;
  size_t ws_bytes;
  unsigned pro;         // GDR_PROLOGUE_* flags (0: q, k normalised and alpha given)
};

struct DecodeArgs {
  const void* q;
  const void* k;
  const void* v;
  const float* alpha;
  const float* beta;
  float* state;
  void* o;
  int N, H, dk, dv;
  int in_dtype, out_dtype;
  bool kda;
  unsigned pro;         // GDR_PROLOGUE_* flags
};

struct VerifyArgs {
  const void* q;        // [N, K, H, dk]
  const void* k;
  const void* v;        // [N, K, H, dv]
  const float* alpha;   // [N, K, H] or [N, K, H, dk]
  const float* beta;    // [N, K, H]
  float* state;         // [N, H, dv, dk]: read; updated in place when snapshots is null
  float* snapshots;     // [K, N, H, dv, dk] or null
  void* o;              // [N, K, H, dv]
  int N, K, H, dk, dv;
  int in_dtype, out_dtype;
  bool kda;
  unsigned pro;         // GDR_PROLOGUE_* flags
};

struct ChunkMap;   // chunkmap.cuh

// The two-kernel tensor-core prefills (prefill_split.cu, prefill_kda_split.cu): bf16,
// d_k = 128, d_v a multiple of 32.  Chunk images per (head, chunk) in the workspace.
size_t split_prefill_workspace(int B, int T, int H);
size_t kda_split_workspace(int B, int T, int H);
size_t split_chunk_image_bytes();
size_t kda_chunk_image_bytes();
cudaError_t launch_prefill_split(const PrefillArgs& a, const ChunkMap& m, cudaStream_t stream);
cudaError_t launch_prefill_kda_split(const PrefillArgs& a, const ChunkMap& m,
                                     cudaStream_t stream);
// The state carry both two-kernel prefills share, run after the prep kernel has written
// the chunk images; chunk_image_bytes() is the size of one image.  launch_chunk_carry
// (carry_dispatch.cu) picks the chained carry (carry_chain.cu), the per-head carry
// (carry_rows.cu) or the value-sliced one (carry_sliced.cu).
cudaError_t launch_chunk_carry(const PrefillArgs& a, const ChunkMap& m, uint32_t spin_limit,
                               cudaStream_t stream);
cudaError_t launch_carry_rows(const PrefillArgs& a, const ChunkMap& m, uint32_t spin_limit,
                              cudaStream_t stream);
cudaError_t launch_carry_sliced(const PrefillArgs& a, const ChunkMap& m, uint32_t spin_limit,
                                cudaStream_t stream);
cudaError_t launch_carry_chain(const PrefillArgs& a, const ChunkMap& m, uint32_t spin_limit,
                               cudaStream_t stream);
size_t chunk_image_bytes();

// Gradients of a dense prefill (backward.cu).
struct BackwardArgs {
  const void* q;
  const void* k;
  const void* v;
  const float* alpha;
  const float* beta;
  const float* s0;        // may be null (zeros)
  const void* dO;
  const float* ds_final;  // may be null (zeros)
  float* dq_out;
  float* dk_out;
  float* dv_out;
  float* dalpha;
  float* dbeta;
  float* ds0;
  int B, T, H, dk, dv;
  int in_dtype, do_dtype;
  bool kda;
  void* workspace;
};
size_t backward_workspace_bytes(int B, int T, int H, int dk, int dv);
cudaError_t launch_backward(const BackwardArgs& a, cudaStream_t stream);

// Records `msg` as the calling thread's gdr_last_error() text and returns `s`.
int report_error(int s, const char* msg);

// GDR_CHECKS build: the current device's word that failed device-side index checks set
// (checks.cuh), allocated and zeroed on first use; nullptr in the product build (and if
// that allocation failed).
unsigned int* checks_word();

// Measurement aid (timing.cu): records an event on `stream` when timing is on.
// slot -1 marks the start of a prefill call, slot i the end of its i-th kernel.
void timing_mark(cudaStream_t stream, int slot);

// Each returns cudaSuccess or the launch error; messages are set by the caller.
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_verify(const VerifyArgs& a, cudaStream_t stream);
cudaError_t launch_prefill_simt(const PrefillArgs& a, cudaStream_t stream);

}  // namespace gdr
