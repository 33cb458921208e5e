// Kimi Delta Attention chunked prefill in two kernels (sm_100a, tcgen05 + TMA).
//
// "Super Apriel: One Checkpoint, Many Speeds", §2A names the KDA mixer: the delta
// rule with one gate per key channel.  For a chunk of C = 64 tokens entering with
// state S0 and the chunk-local cumulative log gate G[t][c] = sum_{s<=t} log alpha_s[c]:
//
//   A[t,j] = beta_t sum_c k_tc k_jc e^{G_tc - G_jc}  (j < t)
//   P[t,j] =        sum_c q_tc k_jc e^{G_tc - G_jc}  (j <= t)
//   T = (I + A)^{-1} Diag(beta)
//   [O1; Y] = [Q (.) e^G; K (.) e^G] S0^T,  R = V - Y,  U = T R
//   O = O1 + P U
//   S^T <- Diag(e^{G_last}) S0^T + (K (.) e^{G_last - G})^T U
//
// Everything except the last three lines is independent of the state.
// kda_chunk_prep_kernel computes it for every chunk of every head at once, two
// CTAs per SM, and leaves per chunk, in the workspace, the operand tiles of the
// carry as tf32 images in the tensor cores' shared-memory layout:
//   group A: [Q (.) e^G; K (.) e^G] (128 x 128) and e^{G_last} (128 floats)
//   group C: T (64 x 64)
//   group D: (K (.) e^{G_last - G})^T (128 x 64) and P (64 x 64)
// kda_chunk_carry_kernel then walks the chunks of each (head, 32-wide value slice).
// Its loader warpgroup only copies: each group has its own full/empty barrier pair
// and is refilled for the next chunk as soon as the product that reads it has
// completed, so one buffer per group keeps the carry fed.  The loader also forms
// the outputs O = O1 + P U of the previous chunk.
//
// The decayed Gram factors through a per-channel reference Gm_c halfway between
// the chunk's first and last G:  e^{G_tc - G_jc} = e^{G_tc - Gm_c} e^{Gm_c - G_jc},
// one tf32 product of L = [Q; K] (.) e^{G - Gm} and R = K (.) e^{Gm - G}.  Both
// factors stay normal fp32 numbers while the channel's log gate drops by at most
// kMaxSpan over the chunk; wider channels are left out of the product and their
// terms are added exactly on the CUDA cores.
//
// Precision: all products run as kind::tf32 with operands rounded to nearest.  Waits
// are bounded; a give-up records GDR_ERR_TIMEOUT in the workspace status word,
// drains what was issued, frees tensor memory and ends the CTA.

#include <math.h>
#include <stdlib.h>

#include "chunk_image.cuh"
#include "chunkmap.cuh"
#include "common.cuh"
#include "launch.h"
#include "solve64.cuh"
#include "tc.cuh"
#include "tma_host.h"

namespace gdr {
namespace {

using namespace tc;
using namespace img;

constexpr int kC = GDR_CHUNK;
constexpr int kDK = 128;
constexpr float kMaxSpan = 168.f;
constexpr uint32_t kDrainLimit = 1u << 26;
constexpr size_t kStatusBytes = 256;

__device__ __forceinline__ float bf16_lo(uint32_t p) { return __uint_as_float(p << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t p) { return __uint_as_float(p & 0xffff0000u); }

// ========================================================================================
// Kernel 1: per-chunk operand images
// ========================================================================================

constexpr int P_THREADS = 256;
constexpr int P_L = 0;            // L = [Q; K] (.) e^{G - Gm}, tf32 [128][128] SW128      64 KB
                                  //   after the Gram: A | X (solve64.cuh layout)
constexpr int P_AS = 0, P_XS = 16384;
constexpr int P_R = 65536;        // R = K (.) e^{Gm - G}, tf32 [64][128] SW128            32 KB
                                  //   after the Gram: G [64 t][128 c] for wide channels
constexpr int P_SMALL = P_R + 32768;
constexpr int P_SMEM = P_SMALL + 3584 + 1024;   // about 100 KB: two CTAs per SM
constexpr uint32_t P_TM_G = 0;    // Gram, M=128 x 64
constexpr uint32_t P_TM_GS = 64;  // G by channel: lane c, columns t
constexpr uint32_t P_TM_COLS = 128;

struct PrepSmall {
  float beta[kC];
  double tot[2][kDK];   // per channel: sum of the log gates of tokens 0-31 and 32-63
  float g0[kDK];        // per channel: G of token 0
  unsigned wmask[4];    // wide channels
  float rscale[2 * kC]; // fused prologue: the L2 scale of q rows 0-63 and k rows 64-127
  uint32_t tmem;
  unsigned long long mma_bar;
  unsigned long long tma_bar;
};
static_assert(sizeof(PrepSmall) <= 3584, "prep small");

template <unsigned PRO>
__global__ void __launch_bounds__(P_THREADS, 2)
kda_chunk_prep_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_a, const __nv_bfloat16* __restrict__ q,
                      const __nv_bfloat16* __restrict__ k, const float* __restrict__ beta,
                      unsigned char* __restrict__ ws, const ChunkMap m, int H,
                      unsigned int* __restrict__ status, uint32_t spin_limit) {
  extern __shared__ unsigned char smem_raw[];
  const uint32_t padb = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  unsigned char* sm = smem_raw + padb;
  unsigned char* tL = sm + P_L;
  unsigned char* tR = sm + P_R;
  float* As = reinterpret_cast<float*>(sm + P_AS);
  float* Xs = reinterpret_cast<float*>(sm + P_XS);
  float* Gw = reinterpret_cast<float*>(tR);
  PrepSmall& ps = *reinterpret_cast<PrepSmall*>(sm + P_SMALL);
  uint64_t* mma_bar = reinterpret_cast<uint64_t*>(&ps.mma_bar);
  uint64_t* tma_bar = reinterpret_cast<uint64_t*>(&ps.tma_bar);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q4 = warp & 3, hw = warp >> 2;
  const int gc = blockIdx.x % m.nck;
  const int h = blockIdx.x / m.nck;
  if (!dcheck(h < H, m.checks, kCheckImage)) return;
  const ChunkLoc loc = chunk_locate(m, gc);
  if (!loc.valid) return;            // past the last chunk of the packed sequences
  const int b = loc.b, t0 = loc.t0, L = loc.L;
  const long row0 = ((long)b * m.T + t0) * H + h;    // token t of the chunk: row0 + t * H
  unsigned char* img = ws + m.img_base + ((size_t)h * m.nck + gc) * kChunkWs;

  // the chunk's q and k (bf16 [64 t][128 c]) land in the L area and its gates (fp32
  // [64 t][128 c]) in the R area; both are read into registers before L and R are built
  if (tid == 0) {
    mbar_init(mma_bar, 1);
    mbar_init(tma_bar, 1);
    fence_mbar_init();
    mbar_expect_tx(tma_bar, 16384 + 16384 + 32768);
    tma_load_4d(smem_u32(tL), &tm_q, 0, h, t0, b, tma_bar);
    tma_load_4d(smem_u32(tL) + 16384, &tm_k, 0, h, t0, b, tma_bar);
    tma_load_4d(smem_u32(tR), &tm_a, 0, h, t0, b, tma_bar);
  }
  if (warp == 0) tmem_alloc(&ps.tmem, P_TM_COLS);
  if (tid < kC) ps.beta[tid] = tid < L ? beta[row0 + (long)tid * H] : 0.f;
  fence_before_sync();
  __syncthreads();
  // ---- 1. this thread's channel cc, tokens 32 hw .. 32 hw + 31 (rows past T read as 0)
  const int cc = 32 * q4 + lane;
  float g[32];
  uint32_t qp[16], kp[16];   // bf16 pairs: tokens (2i, 2i+1) of the half
  {
    bool failed = false;
    if (!mbar_wait(tma_bar, 0, spin_limit)) {
      mbar_wait(tma_bar, 0, kDrainLimit);
      failed = true;
    }
    if (__syncthreads_or(failed)) {
      if (lane == 0) atomicOr(status, 1u);
      fence_after_sync();
      if (warp == 0) tmem_dealloc(ps.tmem, P_TM_COLS);
      return;
    }
    if constexpr ((PRO & GDR_PROLOGUE_L2NORM_QK) != 0) {
      // row tid < 128 of the staged q (0-63) and k (64-127), [t][c] bf16: divided by its
      // L2 norm in fp32 and rounded back to bf16, in place (threads start at different
      // 16-byte pieces of their rows, so a warp's reads spread over the banks)
      if (tid < 2 * kC) {
        // two passes over the row (sum of squares, then the scaled write-back), so that
        // no row is held in registers
        uint4* row = reinterpret_cast<uint4*>(tL + tid * 256);
        float ss = 0.f;
#pragma unroll 4
        for (int i = 0; i < 16; ++i) {
          const uint4 x = row[(i + tid) & 15];
          const __nv_bfloat162* hh = reinterpret_cast<const __nv_bfloat162*>(&x);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(hh[e]);
            ss = fmaf(f.x, f.x, fmaf(f.y, f.y, ss));
          }
        }
        const float sc = l2_scale(ss);
        ps.rscale[tid] = sc;
#pragma unroll 4
        for (int i = 0; i < 16; ++i) {
          uint4 x = row[(i + tid) & 15];
          __nv_bfloat162* hh = reinterpret_cast<__nv_bfloat162*>(&x);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(hh[e]);
            hh[e] = __floats2bfloat162_rn(f.x * sc, f.y * sc);
          }
          row[(i + tid) & 15] = x;
        }
      }
      __syncthreads();
    }
    const unsigned short* qs = reinterpret_cast<const unsigned short*>(tL);
    const unsigned short* ks = reinterpret_cast<const unsigned short*>(tL + 16384);
    const float* as = reinterpret_cast<const float*>(tR);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int ta = 32 * hw + 2 * i;
      qp[i] = (uint32_t)qs[ta * kDK + cc] | ((uint32_t)qs[(ta + 1) * kDK + cc] << 16);
      kp[i] = (uint32_t)ks[ta * kDK + cc] | ((uint32_t)ks[(ta + 1) * kDK + cc] << 16);
      g[2 * i] = as[ta * kDK + cc];
      g[2 * i + 1] = as[(ta + 1) * kDK + cc];
    }
  }
  constexpr bool kLogit = (PRO & GDR_PROLOGUE_GATE_LOGIT) != 0;
  if constexpr (kLogit) {
    // fused prologue: the staged values are the logits x; log alpha = -softplus(x)
#pragma unroll
    for (int x = 0; x < 32; ++x) g[x] = log_gate_from_logit(g[x]);
  }
  // ---- 2. cumulative log gate: fp64 prefix over each half, halves joined by their sums
  {
    double acc = 0.0;
#pragma unroll
    for (int x = 0; x < 32; ++x) {
      acc += (32 * hw + x < L) ? (double)(kLogit ? g[x] : log_gate(g[x])) : 0.0;
      g[x] = (float)acc;
    }
    ps.tot[hw][cc] = acc;
    if (hw == 0) ps.g0[cc] = g[0];
  }
  fence_before_sync();
  __syncthreads();   // also: every read of the staged q, k and gates is done
  fence_after_sync();
  const uint32_t tb = ps.tmem;
  const uint32_t tlane = (uint32_t)(q4 * 32) << 16;
  const double tot0 = ps.tot[0][cc];
  if (hw == 1) {
#pragma unroll
    for (int x = 0; x < 32; ++x) g[x] = (float)(tot0 + (double)g[x]);
  }
  const float glast = (float)(tot0 + ps.tot[1][cc]);
  const float g0c = ps.g0[cc];
  const float gm = 0.5f * (g0c + glast);
  const bool wc = (g0c - glast) > kMaxSpan;
  if (hw == 0) {
    const unsigned wm = __ballot_sync(0xffffffffu, wc);
    if (lane == 0) ps.wmask[q4] = wm;
  }
  tmem_st32(tb + tlane + P_TM_GS + 32 * hw, g);
  // ---- 3. Gram factors L, R (shared memory) and the carry's images (workspace) ----------
  // Element (row r, channel cc) of a 128-byte-swizzled K-major tile sits at
  //   (cc / 32) * rows * 128 + r * 128 + (((cc % 32) / 4 ^ r % 8) * 16) + (cc % 4) * 4;
  // for this thread's rows r = 32 hw + x only x varies, so the offsets are a per-thread
  // base for each x % 8 plus 128 x.
  {
    const uint32_t ch = (uint32_t)(cc & 31) >> 2;
    uint32_t o8[8];
#pragma unroll
    for (int kx = 0; kx < 8; ++kx)
      o8[kx] = (uint32_t)(cc >> 5) * 16384u + (uint32_t)(cc & 3) * 4u + 4096u * hw +
               ((ch ^ (uint32_t)kx) << 4);
    unsigned char* rs = tR - (cc >> 5) * 8192;      // R has 64 rows: panel stride 8 KB
    unsigned char* iqk = img + WS_QK;
    unsigned char* ikh = img + WS_KH;
    const float egl = __expf(glast - gm);
#pragma unroll
    for (int x4 = 0; x4 < 8; ++x4) {
      float kh[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int x = 4 * x4 + u, t = 32 * hw + x;
        const uint32_t p2 = qp[x >> 1], k2 = kp[x >> 1];
        const float qv = (x & 1) ? bf16_hi(p2) : bf16_lo(p2);
        const float kv = (x & 1) ? bf16_hi(k2) : bf16_lo(k2);
        const uint32_t off = o8[x & 7] + 128u * (uint32_t)x;
        float e, ei, eg, el;
        if (!wc) {
          e = __expf(g[x] - gm);
          ei = __expf(gm - g[x]);
          el = egl * ei;                     // e^{G_last - G}, at most 1
        } else {
          e = 0.f;
          ei = 0.f;
          el = __expf(fminf(glast - g[x], 0.f));
        }
        eg = __expf(g[x]);
        *reinterpret_cast<float*>(tL + off) = to_tf32(qv * e);
        *reinterpret_cast<float*>(tL + off + 8192) = to_tf32(kv * e);
        *reinterpret_cast<float*>(rs + off) = to_tf32(kv * ei);
        *reinterpret_cast<float*>(iqk + off) = to_tf32(qv * eg);
        *reinterpret_cast<float*>(iqk + off + 8192) = to_tf32(kv * eg);
        kh[u] = t < L ? kv * el : 0.f;
      }
      *reinterpret_cast<float4*>(ikh + swz_off4(cc, 8 * hw + x4, 128)) =
          tf32x4(kh[0], kh[1], kh[2], kh[3]);
    }
    if (hw == 0) reinterpret_cast<float*>(img + WS_EGL)[cc] = __expf(glast);
  }
  tmem_wait_st();
  fence_smem_to_async();
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const bool anywide = (ps.wmask[0] | ps.wmask[1] | ps.wmask[2] | ps.wmask[3]) != 0u;
  // ---- 4. the decayed Gram on the tensor cores ------------------------------------------
  if (warp == 0) {
    const uint64_t dL = sdesc(smem_u32(tL), 16, 1024), dR = sdesc(smem_u32(tR), 16, 1024);
    const uint32_t id = idesc_tf32(128, 64, false, false);
#pragma unroll
    for (int ks = 0; ks < kDK / 8; ++ks)
      mma_tf32_w(tb + P_TM_G, kstep(dL, 128, ks), kstep(dR, 64, ks), id, ks > 0);
    mma_commit_w(mma_bar);
  }
  bool failed = false;
  if (!mbar_wait(mma_bar, 0, spin_limit)) {
    mbar_wait(mma_bar, 0, kDrainLimit);
    failed = true;
  }
  fence_after_sync();
  if (__syncthreads_or(failed)) {
    if (lane == 0) atomicOr(status, 1u);
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tb, P_TM_COLS);
    return;
  }
  if (anywide) {
    // G as [64 t][128 c] in the (now free) R area, for the exact terms
    float gg[32];
    tmem_ld32(tb + tlane + P_TM_GS + 32 * hw, gg);
    tmem_wait_ld();
#pragma unroll
    for (int x = 0; x < 32; ++x) Gw[(32 * hw + x) * kDK + cc] = gg[x];
    __syncthreads();
  }
  // ---- 5. P (lower) to the image; A (beta, strictly lower) to the solve's scratch -----------
  {
    float d[32];
    tmem_ld32(tb + tlane + P_TM_G + 32 * hw, d);
    const int r = 32 * q4 + lane;      // Gram row: q rows 0-63, k rows 64-127
    const int t = r & 63;
    const float bt = ps.beta[t];
    tmem_wait_ld();
    if (anywide) {
      // the exact terms read q, k again from global memory: with the fused prologue they
      // are normalised here exactly as the staged tile was (same scale, same rounding)
      constexpr bool nrm = (PRO & GDR_PROLOGUE_L2NORM_QK) != 0;
      const __nv_bfloat16* xs = r < 64 ? q : k;
      const float xsc = nrm ? ps.rscale[r] : 1.f;
#pragma unroll 1
      for (int w = 0; w < 4; ++w) {
        unsigned m = ps.wmask[w];
        while (m) {
          const int ch = 32 * w + __ffs(m) - 1;
          m &= m - 1;
          float xv = t < L ? __bfloat162float(xs[(row0 + (long)t * H) * kDK + ch]) : 0.f;
          if constexpr (nrm) xv = as_input<__nv_bfloat16>(xv * xsc);
          const float gt = Gw[t * kDK + ch];
#pragma unroll
          for (int x = 0; x < 32; ++x) {
            const int j = 32 * hw + x;
            if (j <= t && j < L) {
              float kv = __bfloat162float(k[(row0 + (long)j * H) * kDK + ch]);
              if constexpr (nrm) kv = as_input<__nv_bfloat16>(kv * ps.rscale[kC + j]);
              d[x] += xv * kv * __expf(gt - Gw[j * kDK + ch]);
            }
          }
        }
      }
    }
    if (r < 64) {
      unsigned char* ip = img + WS_P;
#pragma unroll
      for (int x = 0; x < 8; ++x) {
        float e[4];
#pragma unroll
        for (int y = 0; y < 4; ++y) e[y] = (32 * hw + 4 * x + y) <= t ? d[4 * x + y] : 0.f;
        *reinterpret_cast<float4*>(ip + swz_off4(t, 8 * hw + x, 64)) = tf32x4(e[0], e[1], e[2], e[3]);
      }
    } else {
      // row t of A, columns 32 hw .. 32 hw + 31, in 16-byte pieces
#pragma unroll
      for (int x = 0; x < 8; ++x) {
        float e[4];
#pragma unroll
        for (int y = 0; y < 4; ++y) e[y] = (32 * hw + 4 * x + y) < t ? bt * d[4 * x + y] : 0.f;
        *reinterpret_cast<float4*>(As + solve64::at4(t, 8 * hw + x)) =
            make_float4(e[0], e[1], e[2], e[3]);
      }
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tb, P_TM_COLS);
  // ---- 6. X = (I + A)^{-1}: the diagonal blocks (warps 0-3), then the column blocks -------
  if (warp < 4) solve64::diag(As, Xs, warp, lane);
  __syncthreads();
  if (warp < 4) solve64::offdiag(As, Xs, warp, lane);
  __syncthreads();
  // ---- 7. T = X Diag(beta) to the image (blocks above the diagonal are zero) ------------------
  {
    const int r = tid & 63, qq = tid >> 6;
    unsigned char* it = img + WS_T;
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      float e[4];
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (qq <= (r >> 4)) v = *reinterpret_cast<const float4*>(Xs + solve64::at4(r, 4 * qq + x));
      const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int y = 0; y < 4; ++y) e[y] = vv[y] * ps.beta[16 * qq + 4 * x + y];
      *reinterpret_cast<float4*>(it + swz_off4(r, 4 * qq + x, 64)) = tf32x4(e[0], e[1], e[2], e[3]);
    }
  }
}

uint32_t kda_split_spin_limit() {
  const char* e = getenv("GDR_SPIN_LIMIT");
  if (!e || !*e) return 1u << 24;
  return (uint32_t)strtoul(e, nullptr, 10);
}

cudaError_t launch_kda_split_t(const PrefillArgs& a, const ChunkMap& m, cudaStream_t stream) {
  // packed sequences: the tensors are [1, total, H, *]
  const int TB = m.cu ? 1 : a.B;
  CUtensorMap mq, mk, ma;
  if (!encode_bthd_bf16(&mq, a.q, TB, a.T, a.H, kDK, kDK, kC, false) ||
      !encode_bthd_bf16(&mk, a.k, TB, a.T, a.H, kDK, kDK, kC, false) ||
      !encode_bthd_f32(&ma, a.alpha, TB, a.T, a.H, kDK, kDK, kC))
    return cudaErrorInvalidValue;
  const uint32_t lim = kda_split_spin_limit();
  auto prep = a.pro == 3 ? kda_chunk_prep_kernel<3> : a.pro == 2 ? kda_chunk_prep_kernel<2>
             : a.pro == 1 ? kda_chunk_prep_kernel<1> : kda_chunk_prep_kernel<0>;
  cudaError_t e = cudaFuncSetAttribute(prep, cudaFuncAttributeMaxDynamicSharedMemorySize, P_SMEM);
  if (e != cudaSuccess) return e;
  prep<<<a.H * m.nck, P_THREADS, P_SMEM, stream>>>(
      mq, mk, ma, (const __nv_bfloat16*)a.q, (const __nv_bfloat16*)a.k, a.beta,
      (unsigned char*)a.workspace, m, a.H, (unsigned int*)a.workspace, lim);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  timing_mark(stream, 0);
  return launch_chunk_carry(a, m, lim, stream);
}

}  // namespace

size_t kda_split_workspace(int B, int T, int H) {
  const size_t nchunks = ((size_t)T + kC - 1) / kC;
  return (size_t)B * H * nchunks * kChunkWs;
}

size_t kda_chunk_image_bytes() { return kChunkWs; }

cudaError_t launch_prefill_kda_split(const PrefillArgs& a, const ChunkMap& m,
                                     cudaStream_t stream) {
  return launch_kda_split_t(a, m, stream);
}

}  // namespace gdr
