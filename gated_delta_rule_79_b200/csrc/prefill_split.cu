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

#include <mutex>

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
  const int np = prep_slots(m);
  const int gc = prep_slot_chunk(m, blockIdx.x % np);
  const int h = blockIdx.x / np;
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

// The side stream of the pipelined prefill on each device (lowest priority, so that the
// carry's CTAs are scheduled first), created on first use.
cudaStream_t side_stream() {
  static std::mutex mu;
  static cudaStream_t streams[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!streams[dev]) {
    int lo = 0, hi = 0;
    cudaDeviceGetStreamPriorityRange(&lo, &hi);
    cudaStream_t st = nullptr;
    if (cudaStreamCreateWithPriority(&st, cudaStreamNonBlocking, lo) != cudaSuccess) return nullptr;
    streams[dev] = st;
  }
  return streams[dev];
}

// The carry takes the value-sliced form for few long chains (carry_dispatch.cu); this
// mirrors its rule so the pipelined prefill is used exactly when that carry runs.
bool sliced_carry_expected(const PrefillArgs& a, const ChunkMap& m) {
  const char* pick = getenv("GDR_CARRY");
  if (pick && pick[0] == 'r') return false;
  if (pick && pick[0] == 's') return true;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return (long)m.nseq * a.H * (a.dv / 32) <= sms;
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
  auto launch_prep = [&](const ChunkMap& mm, cudaStream_t st) {
    prep<<<a.H * prep_slots(mm), P_THREADS, P_SMEM, st>>>(
        mq, mk, a.alpha, a.beta, (unsigned char*)a.workspace, mm, a.H,
        (unsigned int*)a.workspace, lim);
    return cudaGetLastError();
  };

  // Pipelined form (a dense batch on the value-sliced carry, whose few CTAs leave the SMs
  // mostly idle while they wait on their chains): the chunks of every sequence in kParts
  // consecutive parts; part k's carry runs while the prep of part k + 1, on a side stream,
  // fills the room beside it.  The state passes from part to part through the
  // workspace's state area, which follows the chunk images.
  constexpr int kParts = 4;
  const size_t state_off = m.img_base + (size_t)a.H * m.nck * img::kChunkWs;
  const size_t state_bytes = (size_t)m.nseq * a.H * a.dv * kDK * sizeof(float);
  const char* pe = getenv("GDR_PIPELINE");
  const bool pipe = !m.cu && m.nchunks >= 2 * kParts && a.ws_bytes >= state_off + state_bytes &&
                    !(pe && pe[0] == '0') && sliced_carry_expected(a, m);
  cudaStream_t side = pipe ? side_stream() : nullptr;
  if (!side) {
    e = launch_prep(m, stream);
    if (e != cudaSuccess) return e;
    timing_mark(stream, 0);
    return launch_chunk_carry(a, m, lim, stream);
  }
  float* sbuf = reinterpret_cast<float*>(static_cast<unsigned char*>(a.workspace) + state_off);
  ChunkMap part[kParts];
  for (int k = 0; k < kParts; ++k) {
    part[k] = m;
    part[k].c_begin = (int)((long)m.nchunks * k / kParts);
    part[k].c_count = (int)((long)m.nchunks * (k + 1) / kParts) - part[k].c_begin;
  }
  cudaEvent_t ev[kParts] = {};
  for (int k = 0; k < kParts; ++k) {
    e = cudaEventCreateWithFlags(&ev[k], cudaEventDisableTiming);
    if (e != cudaSuccess) break;
  }
  // the side stream starts behind everything the caller put on `stream` before this call
  if (e == cudaSuccess) e = cudaEventRecord(ev[0], stream);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(side, ev[0], 0);
  if (e == cudaSuccess) e = launch_prep(part[0], stream);
  if (e == cudaSuccess) timing_mark(stream, 0);
  for (int k = 0; k < kParts && e == cudaSuccess; ++k) {
    if (k + 1 < kParts) {
      e = launch_prep(part[k + 1], side);
      if (e == cudaSuccess) e = cudaEventRecord(ev[k + 1], side);
    }
    if (e == cudaSuccess && k > 0) e = cudaStreamWaitEvent(stream, ev[k], 0);
    if (e != cudaSuccess) break;
    PrefillArgs pa = a;
    pa.s0 = k == 0 ? a.s0 : sbuf;
    pa.s_final = k + 1 == kParts ? a.s_final : sbuf;
    e = launch_chunk_carry(pa, part[k], lim, stream);
  }
  for (int k = 0; k < kParts; ++k)
    if (ev[k]) cudaEventDestroy(ev[k]);   // released once the work they mark completes
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
