// Streaming GDN chunked prefill: the per-chunk prep and the value-sliced state carry in
// one persistent kernel (sm_100a, tcgen05 + TMA).
//
// "Super Apriel: One Checkpoint, Many Speeds", §2A names the GDN mixer.  The two-kernel
// prefill (prefill_split.cu, carry_sliced.cu) first preps every chunk and then carries the
// state through them; when there are few (sequence, head) chains, the carry is a serial
// chain per (head, value slice) that leaves each SM's tensor pipe and issue slots mostly
// idle, while the prep is throughput work.  Here every SM runs one CTA of 12 warps:
//
//   warps 0-7   the carry of one (sequence, head, 32-column slice) chain, exactly the
//               stand-alone carry's (sliced::carry_body), on the CTAs that have a chain;
//   warps 8-11  a prep group (gdnprep::prep_chunk) that takes chunks from a global
//               ticket counter, chunk position by chunk position (all heads and sequences
//               of chunk 0, then of chunk 1, ...), and publishes each chunk's image with
//               a release flag once it is complete.
//
// The carry's loader reads chunk c of its head once that chunk's flag is set (acquire),
// so the carry starts after the first chunk position is prepped and then runs alongside
// the prep instead of after it; the images it reads were written moments before and are
// still in L2.  Shared memory: the carry's 159 KB (CarryLayout<32>) and the prep group's
// 67 KB; tensor memory: the carry's 256 columns and the prep's 64.
//
// Every CTA is resident at once (a cooperative launch of one CTA per SM), and no prep
// group ever waits on a carry, so every published flag is eventually set.  Waits are
// bounded; a give-up records GDR_ERR_TIMEOUT in the workspace status word.

#include <stdlib.h>

#include "carry_sliced.cuh"
#include "gdn_prep.cuh"
#include "launch.h"
#include "tma_host.h"

namespace gdr {
namespace {

using namespace tc;

constexpr int S_THREADS = 384;                  // warps 0-7 carry, warps 8-11 prep
using CarryLay = sliced::CarryLayout<32>;
constexpr int S_PREP = CarryLay::SMALL + 1024;  // the prep group's shared memory
constexpr int S_TICKET = CarryLay::SMALL + 512; // two ticket slots (after CarrySmall)
constexpr int S_SMEM = S_PREP + gdnprep::P_SMALL + 1024 + 1024;
constexpr uint32_t S_TM_COLS = 512;             // carry [0, 256), prep [256, 320)
constexpr uint32_t S_TM_PREP = 256;
constexpr int S_PREP_BAR = 3;                   // the carry uses hardware barriers 1 and 2
static_assert(S_PREP % 1024 == 0, "prep tiles need 1024-byte alignment");
static_assert(sizeof(sliced::CarrySmall) <= 512, "ticket slots overlap the carry's barriers");
static_assert(S_SMEM <= 232448, "shared memory");
static_assert(CarryLay::COLS <= S_TM_PREP && S_TM_PREP + gdnprep::P_TM_COLS <= S_TM_COLS,
              "tensor memory");

// Workspace past the images: the ticket counter (its own 256 bytes), then one flag per
// (head, global chunk).  Zeroed before every launch.
constexpr size_t kSyncHead = 256;

template <unsigned PRO, typename Tout>
__global__ void __launch_bounds__(S_THREADS, 1)
gdn_stream_kernel(const __grid_constant__ CUtensorMap tm_q,
                  const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const float* __restrict__ alpha,
                  const float* __restrict__ beta, const float* __restrict__ s0,
                  Tout* __restrict__ o, float* __restrict__ s_final, const ChunkMap m, int H,
                  int dv, unsigned char* __restrict__ ws, unsigned int* __restrict__ tickets,
                  unsigned int* __restrict__ ready, int nchains, unsigned int ntickets,
                  unsigned int* __restrict__ status, uint32_t spin_limit) {
  extern __shared__ unsigned char smem_raw[];
  const uint32_t padb = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  unsigned char* sm = smem_raw + padb;
  sliced::CarrySmall& cs = *reinterpret_cast<sliced::CarrySmall*>(sm + CarryLay::SMALL);
  unsigned char* psm = sm + S_PREP;
  gdnprep::PrepSmall& ps = *reinterpret_cast<gdnprep::PrepSmall*>(psm + gdnprep::P_SMALL);
  volatile unsigned* slot = reinterpret_cast<volatile unsigned*>(sm + S_TICKET);

  const int tid = threadIdx.x;
  if (tid == 0) {
    sliced::carry_init(cs);
    gdnprep::prep_init(ps);
  }
  if (tid < 32) tmem_alloc(&cs.tmem, S_TM_COLS);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tb = cs.tmem;

  if (tid < sliced::C_THREADS) {
    if ((int)blockIdx.x < nchains)
      sliced::carry_body<32, Tout, true>(&tm_v, ws, s0, o, s_final, m, H, dv, status,
                                         spin_limit, (int)blockIdx.x, sm, tb, tid, ready);
  } else {
    const int ptid = tid - sliced::C_THREADS;
    const int per = m.nseq * H;      // tickets per chunk position
    uint32_t par = 0;
    for (int k = 0;; ++k) {
      // ticket k of this group in slot k % 2: thread 0 rewrites a slot only after the
      // barrier of the next round, which every thread reaches after reading it
      if (ptid == 0) slot[k & 1] = atomicAdd(tickets, 1u);
      named_bar(S_PREP_BAR, gdnprep::P_THREADS);
      const unsigned tk = slot[k & 1];
      if (tk >= ntickets) break;
      const int li = (int)(tk / (unsigned)per), r = (int)(tk % (unsigned)per);
      const int seq = r / H, h = r % H;
      int first = 0, count = 0;
      chunk_range(m, seq, first, count);
      const int gc = first + li;     // li < count: every sequence has m.nchunks chunks
      const bool ok = gdnprep::prep_chunk<PRO, S_PREP_BAR>(&tm_q, &tm_k, alpha, beta, ws, m, H,
                                                           gc, h, psm, tb + S_TM_PREP, ptid,
                                                           par, status, spin_limit);
      par ^= 1u;
      if (!ok) break;                // the group agreed on the give-up
      // publish: every thread's image writes are ordered before the flag
      __threadfence();
      fence_global_to_async();
      named_bar(S_PREP_BAR, gdnprep::P_THREADS);
      if (ptid == 0) st_release_gpu(ready + (size_t)h * m.nck + gc, 1u);
    }
  }
  fence_before_sync();
  __syncthreads();
  if (tid < 32) tmem_dealloc(tb, S_TM_COLS);
}

template <unsigned PRO, typename Tout>
cudaError_t launch_t(const PrefillArgs& a, const ChunkMap& m, uint32_t lim, int sms,
                     cudaStream_t stream) {
  const int TB = m.cu ? 1 : a.B;
  CUtensorMap mq, mk, mv;
  if (!encode_bthd_bf16(&mq, a.q, TB, a.T, a.H, 128, 64, GDR_CHUNK, true) ||
      !encode_bthd_bf16(&mk, a.k, TB, a.T, a.H, 128, 64, GDR_CHUNK, true) ||
      !encode_bthd_bf16(&mv, a.v, TB, a.T, a.H, a.dv, 32, GDR_CHUNK, false))
    return cudaErrorInvalidValue;
  unsigned char* ws = (unsigned char*)a.workspace;
  unsigned char* sync = ws + gdn_stream_sync_offset(m, a.H);
  unsigned int* tickets = reinterpret_cast<unsigned int*>(sync);
  unsigned int* ready = reinterpret_cast<unsigned int*>(sync + kSyncHead);
  cudaError_t e = cudaMemsetAsync(sync, 0, gdn_stream_sync_bytes(m.nck, a.H), stream);
  if (e != cudaSuccess) return e;
  auto kern = gdn_stream_kernel<PRO, Tout>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S_SMEM);
  if (e != cudaSuccess) return e;
  const int nchains = m.nseq * a.H * (a.dv / 32);
  const unsigned ntickets = (unsigned)m.nchunks * (unsigned)(m.nseq * a.H);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)sms, 1, 1);
  cfg.blockDim = dim3(S_THREADS, 1, 1);
  cfg.dynamicSmemBytes = (size_t)S_SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;   // every CTA resident at once
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, a.alpha, a.beta, a.s0, (Tout*)a.o,
                            a.s_final, m, a.H, a.dv, ws, tickets, ready, nchains, ntickets,
                            (unsigned int*)a.workspace, lim);
}

template <unsigned PRO>
cudaError_t launch_pro(const PrefillArgs& a, const ChunkMap& m, uint32_t lim, int sms,
                       cudaStream_t stream) {
  return a.out_dtype == GDR_F32 ? launch_t<PRO, float>(a, m, lim, sms, stream)
                                : launch_t<PRO, __nv_bfloat16>(a, m, lim, sms, stream);
}

}  // namespace

size_t gdn_stream_sync_bytes(int nck, int H) {
  return kSyncHead + (((size_t)nck * H * sizeof(unsigned) + 255) & ~(size_t)255);
}

size_t gdn_stream_sync_offset(const ChunkMap& m, int H) {
  return m.img_base + (size_t)H * m.nck * img::kChunkWs;
}

bool gdn_stream_eligible(const PrefillArgs& a, const ChunkMap& m) {
  const char* env = getenv("GDR_STREAM");
  if (!env || env[0] != '1') return false;
  const char* pick = getenv("GDR_CARRY");
  if (pick && *pick) return false;   // a carry was named: the two-kernel prefill
  if (a.kda || m.cu || a.dk != 128 || a.dv % 32 != 0) return false;
  int dev = 0, sms = 0, coop = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess)
    return false;
  if (!coop || (long)m.nseq * a.H * (a.dv / 32) > sms) return false;
  return a.ws_bytes >= gdn_stream_sync_offset(m, a.H) + gdn_stream_sync_bytes(m.nck, a.H);
}

cudaError_t launch_gdn_stream(const PrefillArgs& a, const ChunkMap& m, uint32_t spin_limit,
                              cudaStream_t stream) {
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  switch (a.pro) {
    case 1: return launch_pro<1>(a, m, spin_limit, sms, stream);
    case 2: return launch_pro<2>(a, m, spin_limit, sms, stream);
    case 3: return launch_pro<3>(a, m, spin_limit, sms, stream);
    default: return launch_pro<0>(a, m, spin_limit, sms, stream);
  }
}

}  // namespace gdr
