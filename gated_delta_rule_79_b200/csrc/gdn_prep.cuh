// The per-chunk prep of the GDN chunked prefill (sm_100a, tcgen05 + TMA): for one chunk
// of one head, the state-independent operands of the carry, left in the workspace as
// the chunk's image (chunk_image.cuh).
//
// "Super Apriel: One Checkpoint, Many Speeds", §2A names the GDN mixer (delta rule,
// one scalar gate per head and token).  For a chunk of C = 64 tokens with the
// chunk-local cumulative log gate G[t] = sum_{s<=t} log alpha_s:
//
//   P[t,j] = (q_t.k_j) e^{G_t-G_j} (j<=t),  A[t,j] = beta_t (k_t.k_j) e^{G_t-G_j} (j<t)
//   T = (I + A)^{-1} Diag(beta)
//
// The Gram [Q; K] K^T runs as one exact kind::f16 product on the bf16 q, k tiles (the
// scalar decays e^{G_t - G_j} are applied on read-back); the solve for T runs on the
// CUDA cores by 16 x 16 blocks (solve64.cuh).  The image holds [Q (.) e^G; K (.) e^G], e^{G_last}, T,
// (K (.) e^{G_last - G})^T and P as tf32 tiles.
//
// prep_chunk is the work of one 128-thread group for one chunk (the kernel is
// prefill_split.cu, one chunk per CTA); a group may run it for chunk after chunk.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "chunk_image.cuh"
#include "chunkmap.cuh"
#include "common.cuh"
#include "solve64.cuh"
#include "tc.cuh"

namespace gdr {
namespace gdnprep {

using namespace tc;

constexpr int kC = GDR_CHUNK;
constexpr int kDK = 128;
constexpr uint32_t kDrainLimit = 1u << 26;

__device__ __forceinline__ uint64_t kstep(uint64_t desc0, int rows, int ks) {
  return desc0 + (uint64_t)((((ks >> 2) * rows * 128) + ((ks & 3) * 32)) >> 4);
}

constexpr int P_THREADS = 128;
constexpr int P_QK = 0;                    // bf16 [128][128] SW128 (q rows 0-63, k 64-127)  32 KB
// once the Gram has been read, the solve's tiles (solve64.cuh layout) reuse the q/k tile:
constexpr int P_A = 0;                     //   strictly lower A (and the solve's scratch)   16 KB
constexpr int P_X = 16384;                 //   X = (I + A)^{-1}                               16 KB
constexpr int P_G = 32768;                 // gate factors: e^{G_t}[64], e^{G_last - G_t}[64], e^{G_last}
constexpr int P_SMALL = P_G + 1024;
constexpr int P_SMEM = P_SMALL + 1024 + 1024;   // 36 KB
constexpr uint32_t P_TM_COLS = 64;

struct PrepSmall {
  float g[kC];
  float beta[kC];
  uint32_t tmem;
  unsigned long long tma_bar;
  unsigned long long mma_bar;
};

// Thread 0 of the group, before the barrier that precedes the first prep_chunk.
__device__ __forceinline__ void prep_init(PrepSmall& ps) {
  mbar_init(reinterpret_cast<uint64_t*>(&ps.tma_bar), 1);
  mbar_init(reinterpret_cast<uint64_t*>(&ps.mma_bar), 1);
  fence_mbar_init();
}

// Chunk gc (a valid chunk of the map) of head h, by the group's threads tid = 0..127 (warps 4 w .. 4 w + 3 of the
// CTA for some w, so that warp i of the group reads TMEM lanes 32 i .. 32 i + 31), with
// hardware barrier BAR among them.  sm: the group's shared memory (1024-aligned,
// P_SMALL + 1024 bytes); tb: its P_TM_COLS tensor-memory columns; par: the parity of
// this call's phases of the group's two mbarriers (0 for the group's first chunk, then
// alternating).  The chunk's image is complete when it returns true; false: a wait gave
// up (GDR_ERR_TIMEOUT recorded in *status).
template <unsigned PRO, int BAR>
__device__ __forceinline__ bool prep_chunk(const CUtensorMap* tm_q, const CUtensorMap* tm_k,
                                           const float* __restrict__ alpha,
                                           const float* __restrict__ beta,
                                           unsigned char* __restrict__ ws, const ChunkMap& m,
                                           int H, int gc, int h, unsigned char* sm, uint32_t tb,
                                           int tid, uint32_t par, unsigned int* status,
                                           uint32_t spin_limit) {
  unsigned char* tQK = sm + P_QK;
  float* gates = reinterpret_cast<float*>(sm + P_G);
  float* Xs = reinterpret_cast<float*>(sm + P_X);
  float* As = reinterpret_cast<float*>(sm + P_A);
  PrepSmall& ps = *reinterpret_cast<PrepSmall*>(sm + P_SMALL);
  uint64_t* tma_bar = reinterpret_cast<uint64_t*>(&ps.tma_bar);
  uint64_t* mma_bar = reinterpret_cast<uint64_t*>(&ps.mma_bar);

  const int warp = tid >> 5, lane = tid & 31;
  const ChunkLoc loc = chunk_locate(m, gc);
  const int b = loc.b, t0 = loc.t0, L = loc.L;
  const uint32_t tlane = (uint32_t)((warp & 3) * 32) << 16;
  const uint32_t aQK = smem_u32(tQK);
  if (tid == 0) {
    mbar_expect_tx(tma_bar, 32768);
    tma_load_4d(aQK, tm_q, 0, h, t0, b, tma_bar);
    tma_load_4d(aQK + 16384, tm_q, 64, h, t0, b, tma_bar);
    tma_load_4d(aQK + 8192, tm_k, 0, h, t0, b, tma_bar);
    tma_load_4d(aQK + 16384 + 8192, tm_k, 64, h, t0, b, tma_bar);
  }
  // gates of the chunk (rows past T: alpha 1, beta 0)
  if (tid < kC) {
    float a = 1.f, bt = 0.f;
    if (tid < L) {
      const long row = ((long)b * m.T + t0 + tid) * H + h;
      a = alpha[row];
      bt = beta[row];
    }
    ps.g[tid] = tid >= L ? 0.f
                : (PRO & GDR_PROLOGUE_GATE_LOGIT) ? log_gate_from_logit(a)
                                                  : log_gate_accurate(a);
    ps.beta[tid] = bt;
  }
  named_bar(BAR, P_THREADS);
  if (warp == 0) {
    const double g0 = ps.g[2 * lane], g1 = ps.g[2 * lane + 1];
    double s = g0 + g1;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const double n = __shfl_up_sync(0xffffffffu, s, off);
      if (lane >= off) s += n;
    }
    const double ex = s - (g0 + g1);
    ps.g[2 * lane] = (float)(ex + g0);
    ps.g[2 * lane + 1] = (float)(ex + g0 + g1);
  }
  named_bar(BAR, P_THREADS);
  if (tid < kC) {
    const float glast = ps.g[L - 1];
    gates[tid] = __expf(ps.g[tid]);
    gates[64 + tid] = __expf(fminf(glast - ps.g[tid], 0.f));
    if (tid == 0) gates[128] = __expf(glast);
  }
  bool failed = false;
  // ---- Gram [q; k] k^T (bf16 operands are exact) ------------------------------------
  if (!mbar_wait(tma_bar, par, spin_limit)) {
    mbar_wait(tma_bar, par, kDrainLimit);
    failed = true;
  }
  if (named_bar_or(BAR, P_THREADS, failed)) {
    if (lane == 0) atomicOr(status, 1u);
    return false;
  }
  if constexpr ((PRO & GDR_PROLOGUE_L2NORM_QK) != 0) {
    // row tid of the q/k tile (0-63 q, 64-127 k): divided by its L2 norm in fp32 and
    // rounded back to bf16, in place, before anything reads it (two passes over the
    // row, so that it is not held in registers)
    const int r = tid;
    auto piece = [&](int i) -> uint4* {
      return reinterpret_cast<uint4*>(tQK + (i >> 3) * 16384 + r * 128 + (((i & 7) ^ (r & 7)) << 4));
    };
    float ss = 0.f;
#pragma unroll 4
    for (int i = 0; i < 16; ++i) {
      const uint4 x = *piece(i);
      const __nv_bfloat162* hh = reinterpret_cast<const __nv_bfloat162*>(&x);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(hh[e]);
        ss = fmaf(f.x, f.x, fmaf(f.y, f.y, ss));
      }
    }
    const float sc = l2_scale(ss);
#pragma unroll 4
    for (int i = 0; i < 16; ++i) {
      uint4 x = *piece(i);
      __nv_bfloat162* hh = reinterpret_cast<__nv_bfloat162*>(&x);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(hh[e]);
        hh[e] = __floats2bfloat162_rn(f.x * sc, f.y * sc);
      }
      *piece(i) = x;
    }
    fence_smem_to_async();
    named_bar(BAR, P_THREADS);
  }
  if (warp == 0) {
    const uint64_t dA = sdesc(aQK, 16, 1024), dB = sdesc(aQK + 8192, 16, 1024);
    const uint32_t id = idesc_bf16(128, 64);
#pragma unroll
    for (int ks = 0; ks < kDK / 16; ++ks)
      mma_bf16_w(tb, kstep(dA, 128, ks), kstep(dB, 128, ks), id, ks > 0);
    mma_commit_w(mma_bar);
  }
  // ---- while the Gram runs: the carry's images of this chunk (chunk_image.cuh), from the
  //      q/k tile (which the solve's scratch overwrites later): [Q (.) e^G; K (.) e^G], e^{G_last},
  //      K^ = (K (.) e^{G_last - G})^T (tokens past L: zero)
  unsigned char* img = ws + m.img_base + ((size_t)h * m.nck + gc) * img::kChunkWs;
  {
    // Each warp store writes four whole 128-byte tile rows: lane l takes 16-byte chunk
    // l % 8 of row 4 i + l / 8 of a panel (4 tf32 channels, or 4 tokens for K^).
    const int sub = lane >> 3, cd = lane & 7;
    // [Q~; K~]: 128 rows x 4 panels of 32 channels
#pragma unroll 4
    for (int it = 0; it < 32; ++it) {
      const int unit = it * 4 + warp;                 // 0..127: (row group, panel)
      const int pd = unit & 3, r = 4 * (unit >> 2) + sub;
      const int ch = 32 * pd + 4 * cd;                // first of the 4 channels
      const uint2 x = *reinterpret_cast<const uint2*>(
          tQK + (ch >> 6) * 16384 + r * 128 + ((((ch & 63) >> 3) ^ (r & 7)) << 4) + ((ch & 7) << 1));
      const float eg = gates[r & 63];
      *reinterpret_cast<float4*>(img + img::WS_QK + pd * 16384 + r * 128 + ((cd ^ (r & 7)) << 4)) =
          img::tf32x4(__uint_as_float(x.x << 16) * eg, __uint_as_float(x.x & 0xffff0000u) * eg,
                      __uint_as_float(x.y << 16) * eg, __uint_as_float(x.y & 0xffff0000u) * eg);
    }
    reinterpret_cast<float*>(img + img::WS_EGL)[tid] = gates[128];
    // K^: 128 rows (channels) x 2 panels of 32 tokens; tokens past L are zero
#pragma unroll 4
    for (int it = 0; it < 16; ++it) {
      const int unit = it * 4 + warp;                 // 0..63: (row group, panel)
      const int pd = unit & 1, c = 4 * (unit >> 1) + sub;
      float f[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = 32 * pd + 4 * cd + u;
        const float kv = __bfloat162float(
            *reinterpret_cast<const __nv_bfloat16*>(tQK + swz_off_bf16(64 + j, c, 128)));
        f[u] = j < L ? kv * gates[64 + j] : 0.f;
      }
      *reinterpret_cast<float4*>(img + img::WS_KH + pd * 16384 + c * 128 + ((cd ^ (c & 7)) << 4)) =
          img::tf32x4(f[0], f[1], f[2], f[3]);
    }
  }
  if (!mbar_wait(mma_bar, par, spin_limit)) {
    mbar_wait(mma_bar, par, kDrainLimit);
    failed = true;
  }
  fence_after_sync();
  if (named_bar_or(BAR, P_THREADS, failed)) {
    if (lane == 0) atomicOr(status, 1u);
    return false;
  }
  // ---- P (decayed, lower) to the image; A (decayed, beta, strictly lower) to the solve ----
  {
    float d[64];
    tmem_ld32(tb + tlane, *reinterpret_cast<float(*)[32]>(&d[0]));
    tmem_ld32(tb + tlane + 32, *reinterpret_cast<float(*)[32]>(&d[32]));
    const int t = tid & 63;
    const float gt = ps.g[t];
    tmem_wait_ld();
    if (tid < 64) {
#pragma unroll
      for (int j = 0; j < 64; ++j) d[j] = j <= t ? d[j] * __expf(gt - ps.g[j]) : 0.f;
      unsigned char* ip = img + img::WS_P;
#pragma unroll
      for (int q = 0; q < 16; ++q)
        *reinterpret_cast<float4*>(ip + swz_off4(t, q, 64)) =
            img::tf32x4(d[4 * q], d[4 * q + 1], d[4 * q + 2], d[4 * q + 3]);
    } else {
      // row t of A in 16-byte pieces, up to the end of its diagonal block
      const float bt = ps.beta[t];
      const int a = t >> 4;
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        if ((q >> 2) <= a) {
          float e[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int j = 4 * q + u;
            e[u] = j < t ? bt * d[j] * __expf(gt - ps.g[j]) : 0.f;
          }
          *reinterpret_cast<float4*>(As + solve64::at4(t, q)) = make_float4(e[0], e[1], e[2], e[3]);
        }
      }
    }
  }
  fence_before_sync();
  named_bar(BAR, P_THREADS);
  // ---- X = (I + A)^{-1}: the diagonal blocks (one per warp), then the column blocks -------
  solve64::diag(As, Xs, warp, lane);
  named_bar(BAR, P_THREADS);
  solve64::offdiag(As, Xs, warp, lane);
  named_bar(BAR, P_THREADS);
  // ---- T = X Diag(beta) (blocks above the diagonal are zero) -------------------------------
  {
    const int r = tid & 63, half = tid >> 6;
    float xr[32];
#pragma unroll
    for (int x = 0; x < 8; ++x) {
      const int q = half * 8 + x;                    // 16-byte piece: columns 4 q .. 4 q + 3
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if ((q >> 2) <= (r >> 4)) v = *reinterpret_cast<const float4*>(Xs + solve64::at4(r, q));
      xr[4 * x] = v.x * ps.beta[4 * q];
      xr[4 * x + 1] = v.y * ps.beta[4 * q + 1];
      xr[4 * x + 2] = v.z * ps.beta[4 * q + 2];
      xr[4 * x + 3] = v.w * ps.beta[4 * q + 3];
    }
    unsigned char* it = img + img::WS_T;
#pragma unroll
    for (int x = 0; x < 8; ++x)
      *reinterpret_cast<float4*>(it + swz_off4(r, half * 8 + x, 64)) =
          img::tf32x4(xr[4 * x], xr[4 * x + 1], xr[4 * x + 2], xr[4 * x + 3]);
  }
  // the scratch is the next chunk's q/k tile: its reads precede that copy
  fence_smem_to_async();
  return true;
}

}  // namespace gdnprep
}  // namespace gdr
