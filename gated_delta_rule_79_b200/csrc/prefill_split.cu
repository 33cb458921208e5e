// Gated DeltaNet chunked prefill in two kernels (sm_100a, tcgen05 + TMA).
//
// "Super Apriel: One Checkpoint, Many Speeds", §2A names the GDN mixer (delta rule,
// one scalar gate per head and token).  The chunk algebra (C = 64 tokens, chunk
// entering with state S0, G[t] = sum_{s<=t} log alpha_s chunk-locally):
//
//   P[t,j] = (q_t.k_j) e^{G_t-G_j} (j<=t),  A[t,j] = beta_t (k_t.k_j) e^{G_t-G_j} (j<t)
//   T = (I + A)^{-1} Diag(beta)
//   Y = K S0^T,  R = V - Diag(e^G) Y,  U = T R
//   O = Diag(e^G) Q S0^T + P U
//   S^T <- e^{G_last} S0^T + K^T Diag(e^{G_last-G}) U
//
// Everything but the state-dependent products is computed by gdn_chunk_prep_kernel
// for every chunk of every head at once (the whole GPU works on them in parallel; the
// per-chunk work is gdn_prep.cuh).  It leaves the chunk's operand images for the carry
// in the workspace (chunk_image.cuh).  The state carry that walks the chunks in order is
// shared with KDA (carry_rows.cu, carry_sliced.cu).
//
// Precision: the Gram is exact (bf16 inputs, fp32 accumulation); the carry's products
// run as kind::tf32 with operands rounded to nearest.  Waits are bounded; a give-up
// records GDR_ERR_TIMEOUT in the workspace status word and ends the CTA.

#include <math.h>
#include <stdlib.h>

#include "gdn_prep.cuh"
#include "launch.h"
#include "tma_host.h"

namespace gdr {
namespace {

using namespace tc;
using namespace gdnprep;

template <unsigned PRO>
__global__ void __launch_bounds__(P_THREADS, 5)
gdn_chunk_prep_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k, const float* __restrict__ alpha,
                      const float* __restrict__ beta, unsigned char* __restrict__ ws,
                      const ChunkMap m, int H, unsigned int* __restrict__ status,
                      uint32_t spin_limit) {
  extern __shared__ unsigned char smem_raw[];
  const uint32_t padb = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  unsigned char* sm = smem_raw + padb;
  PrepSmall& ps = *reinterpret_cast<PrepSmall*>(sm + P_SMALL);
  const int tid = threadIdx.x;
  const int gc = blockIdx.x % m.nck;
  const int h = blockIdx.x / m.nck;
  if (!dcheck(h < H, m.checks, kCheckImage)) return;
  if (!chunk_locate(m, gc).valid) return;   // past the last chunk of the packed sequences
  if (tid == 0) prep_init(ps);
  if (tid < 32) tmem_alloc(&ps.tmem, P_TM_COLS);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tb = ps.tmem;
  prep_chunk<PRO, 0>(&tm_q, &tm_k, alpha, beta, ws, m, H, gc, h, sm, tb, tid, 0u, status,
                     spin_limit);
  fence_before_sync();
  __syncthreads();
  if (tid < 32) tmem_dealloc(tb, P_TM_COLS);
}

uint32_t split_spin_limit() {
  const char* e = getenv("GDR_SPIN_LIMIT");
  if (!e || !*e) return 1u << 24;
  return (uint32_t)strtoul(e, nullptr, 10);
}

cudaError_t launch_split_t(const PrefillArgs& a, const ChunkMap& m, cudaStream_t stream) {
  // packed sequences: the tensors are [1, total, H, *]
  const int TB = m.cu ? 1 : a.B;
  CUtensorMap mq, mk;
  if (!encode_bthd_bf16(&mq, a.q, TB, a.T, a.H, kDK, 64, kC, true) ||
      !encode_bthd_bf16(&mk, a.k, TB, a.T, a.H, kDK, 64, kC, true))
    return cudaErrorInvalidValue;
  const uint32_t lim = split_spin_limit();
  auto prep = a.pro == 3 ? gdn_chunk_prep_kernel<3> : a.pro == 2 ? gdn_chunk_prep_kernel<2>
             : a.pro == 1 ? gdn_chunk_prep_kernel<1> : gdn_chunk_prep_kernel<0>;
  cudaError_t e = cudaFuncSetAttribute(prep, cudaFuncAttributeMaxDynamicSharedMemorySize, P_SMEM);
  if (e != cudaSuccess) return e;
  prep<<<a.H * m.nck, P_THREADS, P_SMEM, stream>>>(
      mq, mk, a.alpha, a.beta, (unsigned char*)a.workspace, m, a.H,
      (unsigned int*)a.workspace, lim);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  timing_mark(stream, 0);
  e = launch_chunk_carry(a, m, lim, stream);
  return e;
}

}  // namespace

size_t split_prefill_workspace(int B, int T, int H) {
  const size_t nchunks = ((size_t)T + kC - 1) / kC;
  return (size_t)B * H * nchunks * img::kChunkWs;
}

size_t split_chunk_image_bytes() { return img::kChunkWs; }

cudaError_t launch_prefill_split(const PrefillArgs& a, const ChunkMap& m, cudaStream_t stream) {
  return launch_split_t(a, m, stream);
}

}  // namespace gdr
