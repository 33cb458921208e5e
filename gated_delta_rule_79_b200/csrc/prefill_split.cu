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
// P, T and the gate factors do not depend on the state, so gdn_chunk_prep_kernel
// computes them for every chunk of every head at once (the whole GPU works on
// them in parallel) and leaves them in the workspace as operand tiles ready to be
// copied; gdn_chunk_carry_kernel then walks the chunks of each (head, 32-wide
// value slice) and only runs the state-dependent products.  Its loader warpgroup
// brings chunk c+1 in (TMA for q, k, v; a bulk copy for P, T, gates) and builds
// k^T while the carry warpgroup works on chunk c.
//
// Precision: q, k, v are bf16 and exact; products with them run as kind::f16 with
// the computed partner (the state, Diag(e^{G_last-G}) U) split into bf16 hi + lo
// (about 16 significant bits).  Products of two computed operands (T R, P U) run
// as kind::tf32 with operands rounded to nearest.  Measured by emulation, single
// bf16 roundings cost about 3e-3 normwise error against a 2e-3 budget.
//
// Waits are bounded; a give-up records GDR_ERR_TIMEOUT in the workspace status
// word, drains what was issued, frees tensor memory and ends the CTA.

#include <math.h>
#include <stdlib.h>

#include "chunkmap.cuh"
#include "common.cuh"
#include "launch.h"
#include "tc.cuh"
#include "tma_host.h"

namespace gdr {
namespace {

using namespace tc;

constexpr int kC = GDR_CHUNK;
constexpr int kDK = 128;
constexpr int kDVS = 32;
constexpr uint32_t kDrainLimit = 1u << 26;

// Workspace per chunk: P tile (fp32, 16 KB) | T tile (16 KB) | gates (1 KB:
// e^{G_t}[64], e^{G_last - G_t}[64], e^{G_last}).
constexpr int kChunkWs = 33792;
constexpr int WS_T = 16384, WS_G = 32768;
constexpr size_t kStatusBytes = 256;

// [64][64] fp32 scratch with the column index XOR-ed by the row (conflict-free rows
// and columns), as in the fused kernel.
__device__ __forceinline__ int sx(int r, int c) { return r * 64 + (c ^ (r & 31)); }

__device__ __forceinline__ void ld4_sx(const float* base, int k, int klo, int c4, float (&e)[4]) {
  const float4 f = *reinterpret_cast<const float4*>(base + k * 64 + (c4 ^ (k & 28)));
  const float v[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
  for (int x = 0; x < 4; ++x) e[x] = v[x ^ klo];
}

// Strictly lower part of A, stored by 16x16 blocks (a, m), m <= a: block index
// a(a+1)/2 + m, entry (r, i) at r*16 + (i ^ r).
__device__ __forceinline__ int pa(int a, int m, int r, int i) {
  return ((a * (a + 1)) / 2 + m) * 256 + r * 16 + (i ^ r);
}

__device__ __forceinline__ uint64_t kstep(uint64_t desc0, int rows, int ks) {
  return desc0 + (uint64_t)((((ks >> 2) * rows * 128) + ((ks & 3) * 32)) >> 4);
}

__device__ __forceinline__ void st_tile4(unsigned char* tile, int rows, int r, int q, float4 x) {
  x.x = to_tf32(x.x); x.y = to_tf32(x.y); x.z = to_tf32(x.z); x.w = to_tf32(x.w);
  *reinterpret_cast<float4*>(tile + swz_off4(r, q, rows)) = x;
}

// ========================================================================================
// Kernel 1: per-chunk P, T and gate factors
// ========================================================================================

constexpr int P_THREADS = 128;
constexpr int P_QK = 0;                    // bf16 [128][128] SW128 (q rows 0-63, k 64-127)  32 KB
// once the Gram has been read, the solve's scratch reuses the q/k tile:
constexpr int P_X = 0;                     //   X scratch, sx() layout                        16 KB
constexpr int P_A = 16384;                 //   packed strictly-lower A                       10 KB
constexpr int P_Z = P_A + 10240;           //   level scratch [3][16][16]                      3 KB
constexpr int P_OUT = 32768;               // P | T | gates: the chunk's workspace image      33 KB
constexpr int P_SMALL = P_OUT + 34816;
constexpr int P_SMEM = P_SMALL + 1024 + 1024;   // 68 KB: three CTAs per SM
constexpr uint32_t P_TM_COLS = 64;

struct PrepSmall {
  float g[kC];
  float beta[kC];
  uint32_t tmem;
  unsigned long long tma_bar;
  unsigned long long mma_bar;
};

__global__ void __launch_bounds__(P_THREADS)
gdn_chunk_prep_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k, const float* __restrict__ alpha,
                      const float* __restrict__ beta, unsigned char* __restrict__ ws,
                      const ChunkMap m, int H, unsigned int* __restrict__ status,
                      uint32_t spin_limit) {
  extern __shared__ unsigned char smem_raw[];
  const uint32_t padb = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  unsigned char* sm = smem_raw + padb;
  unsigned char* tQK = sm + P_QK;
  unsigned char* tP = sm + P_OUT;
  unsigned char* tT = sm + P_OUT + WS_T;
  float* gates = reinterpret_cast<float*>(sm + P_OUT + WS_G);
  float* Xs = reinterpret_cast<float*>(sm + P_X);
  float* As = reinterpret_cast<float*>(sm + P_A);
  float* Zs = reinterpret_cast<float*>(sm + P_Z);
  PrepSmall& ps = *reinterpret_cast<PrepSmall*>(sm + P_SMALL);
  uint64_t* tma_bar = reinterpret_cast<uint64_t*>(&ps.tma_bar);
  uint64_t* mma_bar = reinterpret_cast<uint64_t*>(&ps.mma_bar);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gc = blockIdx.x % m.nck;
  const int h = blockIdx.x / m.nck;
  const ChunkLoc loc = chunk_locate(m, gc);
  if (!loc.valid) return;            // past the last chunk of the packed sequences
  const int b = loc.b, t0 = loc.t0, L = loc.L;

  if (tid == 0) {
    mbar_init(tma_bar, 1);
    mbar_init(mma_bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&ps.tmem, P_TM_COLS);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tb = ps.tmem;
  const uint32_t tlane = (uint32_t)(warp * 32) << 16;
  const uint32_t aQK = smem_u32(tQK);
  if (tid == 0) {
    mbar_expect_tx(tma_bar, 32768);
    tma_load_4d(aQK, &tm_q, 0, h, t0, b, tma_bar);
    tma_load_4d(aQK + 16384, &tm_q, 64, h, t0, b, tma_bar);
    tma_load_4d(aQK + 8192, &tm_k, 0, h, t0, b, tma_bar);
    tma_load_4d(aQK + 16384 + 8192, &tm_k, 64, h, t0, b, tma_bar);
  }
  // gates of the chunk (rows past T: alpha 1, beta 0)
  if (tid < kC) {
    float a = 1.f, bt = 0.f;
    if (tid < L) {
      const long row = ((long)b * m.T + t0 + tid) * H + h;
      a = alpha[row];
      bt = beta[row];
    }
    ps.g[tid] = log_gate_accurate(a);
    ps.beta[tid] = bt;
  }
  __syncthreads();
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
  __syncthreads();
  if (tid < kC) {
    const float glast = ps.g[L - 1];
    gates[tid] = __expf(ps.g[tid]);
    gates[64 + tid] = __expf(fminf(glast - ps.g[tid], 0.f));
    if (tid == 0) gates[128] = __expf(glast);
  }
  bool failed = false;
  // ---- Gram [q; k] k^T (bf16 operands are exact) ------------------------------------
  if (!mbar_wait(tma_bar, 0, spin_limit)) {
    mbar_wait(tma_bar, 0, kDrainLimit);
    failed = true;
  }
  if (__syncthreads_or(failed)) {
    if (lane == 0) atomicOr(status, 1u);
    if (warp == 0) tmem_dealloc(tb, P_TM_COLS);
    return;
  }
  if (warp == 0) {
    const uint64_t dA = sdesc(aQK, 16, 1024), dB = sdesc(aQK + 8192, 16, 1024);
    const uint32_t id = idesc_bf16(128, 64);
#pragma unroll
    for (int ks = 0; ks < kDK / 16; ++ks)
      mma_bf16_w(tb, kstep(dA, 128, ks), kstep(dB, 128, ks), id, ks > 0);
    mma_commit_w(mma_bar);
  }
  if (!mbar_wait(mma_bar, 0, spin_limit)) {
    mbar_wait(mma_bar, 0, kDrainLimit);
    failed = true;
  }
  fence_after_sync();
  if (__syncthreads_or(failed)) {
    if (lane == 0) atomicOr(status, 1u);
    fence_before_sync();
    if (warp == 0) tmem_dealloc(tb, P_TM_COLS);
    return;
  }
  // ---- P (decayed, lower) to the output image; A (decayed, beta, strictly lower) ------
  {
    float d[64], gj[64];
    tmem_ld32(tb + tlane, *reinterpret_cast<float(*)[32]>(&d[0]));
    tmem_ld32(tb + tlane + 32, *reinterpret_cast<float(*)[32]>(&d[32]));
#pragma unroll
    for (int x = 0; x < 64; ++x) gj[x] = ps.g[x];
    tmem_wait_ld();
    const int t = tid & 63;
    const float gt = ps.g[t];
    if (tid < 64) {
#pragma unroll
      for (int j = 0; j < 64; ++j) d[j] = j <= t ? d[j] * __expf(gt - gj[j]) : 0.f;
#pragma unroll
      for (int q = 0; q < 16; ++q)
        st_tile4(tP, 64, t, q, make_float4(d[4 * q], d[4 * q + 1], d[4 * q + 2], d[4 * q + 3]));
    } else {
      const float bt = ps.beta[t];
      const int a = t >> 4, r = t & 15;
#pragma unroll
      for (int j = 0; j < 64; ++j) {
        const int m = j >> 4;
        if (m <= a) As[pa(a, m, r, j & 15)] = j < t ? bt * d[j] * __expf(gt - gj[j]) : 0.f;
      }
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tb, P_TM_COLS);
  // ---- X = (I + A)^{-1}: diagonal blocks (one per warp), then three block levels ------------
  if (lane < 16) {
    const int a = warp, jl = lane, base = 16 * a;
    const int bx = base ^ (base & 16);
    const float* Ab = As + pa(a, a, 0, 0);
    float x[16];
#pragma unroll
    for (int tl = 0; tl < 16; ++tl) {
      float a_row[16];
#pragma unroll
      for (int i = 0; i < tl; ++i) a_row[i] = Ab[tl * 16 + (i ^ tl)];
      float acc0 = (tl == jl) ? 1.f : 0.f, acc1 = 0.f;
#pragma unroll
      for (int i = 0; i < tl; i += 2) {
        acc0 = fmaf(-a_row[i], x[i], acc0);
        if (i + 1 < tl) acc1 = fmaf(-a_row[i + 1], x[i + 1], acc1);
      }
      x[tl] = (tl < jl) ? 0.f : acc0 + acc1;
    }
    float* Xb = Xs + base * 64 + bx;
#pragma unroll
    for (int tl = 0; tl < 16; ++tl) Xb[tl * 64 + (jl ^ tl)] = x[tl];
  }
  __syncthreads();
#pragma unroll
  for (int d = 1; d <= 3; ++d) {
    const int nunits = (4 - d) * 64;           // unit = (block bb, row r, column quad cq)
    float z[2][4];
#pragma unroll
    for (int n = 0; n < 2; ++n) {
      const int u = tid + P_THREADS * n;
      if (u < nunits) {
        const int bb = u >> 6, r = (u >> 2) & 15, cq = u & 3, aa = bb + d;
        float z0 = 0.f, z1 = 0.f, z2 = 0.f, z3 = 0.f;
#pragma unroll
        for (int m = 0; m < d; ++m)
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int k = 16 * (bb + m) + i;
            const float av = As[pa(aa, bb + m, r, i)];
            float e[4];
            ld4_sx(Xs, k, i & 3, 16 * bb + 4 * cq, e);
            z0 = fmaf(av, e[0], z0);
            z1 = fmaf(av, e[1], z1);
            z2 = fmaf(av, e[2], z2);
            z3 = fmaf(av, e[3], z3);
          }
        z[n][0] = z0; z[n][1] = z1; z[n][2] = z2; z[n][3] = z3;
      }
    }
#pragma unroll
    for (int n = 0; n < 2; ++n) {
      const int u = tid + P_THREADS * n;
      if (u < nunits) {
        const int bb = u >> 6, r = (u >> 2) & 15, cq = u & 3;
        *reinterpret_cast<float4*>(&Zs[bb * 256 + r * 16 + 4 * cq]) =
            make_float4(z[n][0], z[n][1], z[n][2], z[n][3]);
      }
    }
    __syncthreads();
#pragma unroll
    for (int n = 0; n < 2; ++n) {
      const int u = tid + P_THREADS * n;
      if (u < nunits) {
        const int bb = u >> 6, r = (u >> 2) & 15, cq = u & 3, aa = bb + d;
        float x0 = 0.f, x1 = 0.f, x2 = 0.f, x3 = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float xa = Xs[sx(16 * aa + r, 16 * aa + i)];
          const float4 zz = *reinterpret_cast<const float4*>(&Zs[bb * 256 + i * 16 + 4 * cq]);
          x0 = fmaf(xa, zz.x, x0);
          x1 = fmaf(xa, zz.y, x1);
          x2 = fmaf(xa, zz.z, x2);
          x3 = fmaf(xa, zz.w, x3);
        }
        z[n][0] = -x0; z[n][1] = -x1; z[n][2] = -x2; z[n][3] = -x3;
      }
    }
#pragma unroll
    for (int n = 0; n < 2; ++n) {
      const int u = tid + P_THREADS * n;
      if (u < nunits) {
        const int bb = u >> 6, r = (u >> 2) & 15, cq = u & 3, aa = bb + d;
        const int row = 16 * aa + r, col = 16 * bb + 4 * cq;
#pragma unroll
        for (int e = 0; e < 4; ++e) Xs[sx(row, col + e)] = z[n][e];
      }
    }
    __syncthreads();
  }
  // ---- T = X Diag(beta) (blocks above the diagonal are zero) -------------------------------
  {
    const int r = tid & 63, half = tid >> 6;
    float xr[32];
#pragma unroll
    for (int x = 0; x < 32; ++x) {
      const int j = half * 32 + x;
      xr[x] = ((j >> 4) <= (r >> 4)) ? Xs[sx(r, j)] * ps.beta[j] : 0.f;
    }
#pragma unroll
    for (int x = 0; x < 8; ++x)
      st_tile4(tT, 64, r, half * 8 + x,
               make_float4(xr[4 * x], xr[4 * x + 1], xr[4 * x + 2], xr[4 * x + 3]));
  }
  fence_smem_to_async();
  __syncthreads();
  if (tid == 0) {
    unsigned char* dst = ws + m.img_base + ((size_t)h * m.nck + gc) * kChunkWs;
    bulk_store(dst, smem_u32(tP), kChunkWs);
    bulk_commit();
    bulk_wait_all();
  }
}

// ========================================================================================
// Kernel 2: the state carry, per (batch, head, 32-wide slice of d_v)
// ========================================================================================

constexpr int C_THREADS = 256;             // warps 0-3 carry, warps 4-7 load
constexpr int C_STAGES = 2;
// one stage (bytes from the stage base)
constexpr int S_QK = 0;                    // bf16 [128][128] SW128 (TMA)                  32 KB
constexpr int S_KT = 32768;                // bf16 [128 c][64 j] SW128 k^T                 16 KB
constexpr int S_PT = 49152;                // P | T | gates (bulk copy of the workspace)   33 KB
constexpr int S_V = S_PT + 34816;          // bf16 [64 j][32 v] (TMA)                       4 KB
constexpr int STAGE_BYTES = S_V + 4096;    // 88 KB
constexpr uint32_t STAGE_TX = 32768 + 4096 + kChunkWs;
// carry-side tiles
constexpr int C_SSH = C_STAGES * STAGE_BYTES;   // bf16 [32 v][128 c] state hi           8 KB
constexpr int C_SSL = C_SSH + 8192;             // state lo                               8 KB
constexpr int C_RT = C_SSL + 8192;              // fp32 [32 v][64 j]; P U exchange        8 KB
constexpr int C_UT = C_RT + 8192;               // fp32 [32 v][64 j]                      8 KB
constexpr int C_UPH = C_UT + 8192;              // bf16 [32 v][64 j] (e^{G_last-G} U) hi  4 KB
constexpr int C_UPL = C_UPH + 4096;             //                                  lo    4 KB
constexpr int C_OX = C_UPL + 4096;              // P U exchange [64 t][32 v] (loader)    8 KB
constexpr int C_SMALL = C_OX + 8192;
constexpr int C_SMEM = C_SMALL + 1024 + 1024;
static_assert(C_SMEM <= 232448, "shared memory");

// [q; k] S0^T (M=128 x 32: rows 0-63 O1, rows 64-127 Y) and P U (M=64 x 32) are
// double-buffered by chunk parity: the loader warpgroup reads chunk c's outputs while
// the carry already runs chunk c+1.
constexpr uint32_t TM_OY = 0;    // + 32 * (c & 1)
constexpr uint32_t TM_O2 = 64;   // + 32 * (c & 1)
constexpr uint32_t TM_U = 128;   // U, M=64 x 32
constexpr uint32_t TM_S = 160;   // S^T, M=128 x 32
constexpr uint32_t C_TM_COLS = 256;

struct CarrySmall {
  unsigned long long full[C_STAGES];    // TMA + bulk copy landed
  unsigned long long ready[C_STAGES];   // k^T built, stage ready for the carry
  unsigned long long empty[C_STAGES];   // carry done with the stage
  unsigned long long mma_bar;
  unsigned long long out_full[2];   // chunk's O1 and P U are in TMEM (carry -> loader)
  unsigned long long out_empty[2];  // loader has read them (loader -> carry)
  float eg_out[2][64];              // e^{G_t} of the chunk whose outputs are pending
  uint32_t tmem;
  int abort;
};

__device__ __forceinline__ void split_bf16(float x, __nv_bfloat16& hi, __nv_bfloat16& lo) {
  hi = __float2bfloat16_rn(x);
  lo = __float2bfloat16_rn(x - __bfloat162float(hi));
}

template <typename Tout>
__global__ void __launch_bounds__(C_THREADS, 1)
gdn_chunk_carry_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v,
                       const unsigned char* __restrict__ ws, const float* __restrict__ s0,
                       Tout* __restrict__ o, float* __restrict__ s_final, const ChunkMap m,
                       int H, int dv, unsigned int* __restrict__ status, uint32_t spin_limit) {
  extern __shared__ unsigned char smem_raw[];
  const uint32_t padb = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  unsigned char* sm = smem_raw + padb;
  CarrySmall& cs = *reinterpret_cast<CarrySmall*>(sm + C_SMALL);
  unsigned char* tSSH = sm + C_SSH;
  unsigned char* tSSL = sm + C_SSL;
  unsigned char* tRT = sm + C_RT;
  unsigned char* tUT = sm + C_UT;
  unsigned char* tUPH = sm + C_UPH;
  unsigned char* tUPL = sm + C_UPL;
  float* Ox = reinterpret_cast<float*>(sm + C_OX);   // P U exchange [64 t][32 v], row-XOR

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q4 = warp & 3;
  const int nslice = dv / kDVS;
  const int slice = blockIdx.x % nslice;
  const int sh = blockIdx.x / nslice;
  const int h = sh % H, seq = sh / H;
  int first = 0, nchunks = 0;
  chunk_range(m, seq, first, nchunks);
  const int v0 = slice * kDVS;

  if (tid == 0) {
    for (int s = 0; s < C_STAGES; ++s) {
      mbar_init(reinterpret_cast<uint64_t*>(&cs.full[s]), 1);
      mbar_init(reinterpret_cast<uint64_t*>(&cs.ready[s]), 1);
      mbar_init(reinterpret_cast<uint64_t*>(&cs.empty[s]), 1);
    }
    mbar_init(reinterpret_cast<uint64_t*>(&cs.mma_bar), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(reinterpret_cast<uint64_t*>(&cs.out_full[s]), 1);
      mbar_init(reinterpret_cast<uint64_t*>(&cs.out_empty[s]), 1);
    }
    cs.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&cs.tmem, C_TM_COLS);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tb = cs.tmem;
  const uint32_t tlane = (uint32_t)(q4 * 32) << 16;
  const unsigned char* wsb = ws + m.img_base + ((size_t)h * m.nck + first) * kChunkWs;

  auto stage = [&](int s) { return sm + s * STAGE_BYTES; };
  // A wait gave up: record the timeout and stop both warpgroups.  For barriers fed by
  // the tensor cores or the copy engines, first drain what was issued (drain = true);
  // the barriers between the two warpgroups have nothing to drain.
  auto give_up = [&](uint64_t* bar, uint32_t parity, bool drain) {
    if (drain) mbar_wait(bar, parity, kDrainLimit);
    atomicOr(status, 1u);
    cs.abort = 1;
  };

  if (warp >= 4) {
    // =========================== loader warpgroup =====================================
    const int lt = tid - 128;
    // O = Diag(e^G) O1 + P U for chunk cc, read from the chunk's TMEM buffers once the
    // carry has finished it; returns false on abort.
    auto write_outputs = [&](int cc) -> bool {
      const int ob = cc & 1;
      const uint32_t use = (uint32_t)(cc >> 1);
      uint64_t* ofull = reinterpret_cast<uint64_t*>(&cs.out_full[ob]);
      if (lt == 0 && !mbar_wait(ofull, use & 1u, spin_limit)) give_up(ofull, use & 1u, false);
      named_bar(2, 128);
      if (cs.abort) return false;
      fence_after_sync();
      const ChunkLoc loc = chunk_locate(m, first + cc);
      const int t0 = loc.t0, L = loc.L, b = loc.b;
      {
        float o2[32];
        tmem_ld32(tb + tlane + TM_O2 + 32 * ob, o2);
        tmem_wait_ld();
        if (lane < 16) {
          const int t = 16 * q4 + lane;
#pragma unroll
          for (int x = 0; x < 32; ++x) Ox[t * 32 + (x ^ (t & 31))] = o2[x];
        }
      }
      named_bar(2, 128);
      if (q4 < 2) {
        const int t = 32 * q4 + lane;
        float o1[32], o2[32];
        tmem_ld32(tb + tlane + TM_OY + 32 * ob, o1);
#pragma unroll
        for (int x = 0; x < 32; ++x) o2[x] = Ox[t * 32 + (x ^ (t & 31))];
        const float eg = cs.eg_out[ob][t];
        tmem_wait_ld();
        if (t < L) {
          Tout* dst = o + (((long)b * m.T + t0 + t) * H + h) * (long)dv + v0;
          if constexpr (sizeof(Tout) == 2) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint4 pk;
              __nv_bfloat162* hp = reinterpret_cast<__nv_bfloat162*>(&pk);
#pragma unroll
              for (int x = 0; x < 4; ++x)
                hp[x] = __floats2bfloat162_rn(fmaf(eg, o1[8 * q + 2 * x], o2[8 * q + 2 * x]),
                                              fmaf(eg, o1[8 * q + 2 * x + 1], o2[8 * q + 2 * x + 1]));
              reinterpret_cast<uint4*>(dst)[q] = pk;
            }
          } else {
#pragma unroll
            for (int q = 0; q < 8; ++q)
              reinterpret_cast<float4*>(dst)[q] =
                  make_float4(fmaf(eg, o1[4 * q], o2[4 * q]), fmaf(eg, o1[4 * q + 1], o2[4 * q + 1]),
                              fmaf(eg, o1[4 * q + 2], o2[4 * q + 2]),
                              fmaf(eg, o1[4 * q + 3], o2[4 * q + 3]));
          }
        }
      }
      fence_before_sync();
      named_bar(2, 128);
      if (lt == 0) mbar_arrive(reinterpret_cast<uint64_t*>(&cs.out_empty[ob]));
      return true;
    };
    for (int c = 0; c < nchunks; ++c) {
      const int s = c & 1;
      const uint32_t use = (uint32_t)(c >> 1);
      unsigned char* st = stage(s);
      uint64_t* full = reinterpret_cast<uint64_t*>(&cs.full[s]);
      uint64_t* empty = reinterpret_cast<uint64_t*>(&cs.empty[s]);
      uint64_t* ready = reinterpret_cast<uint64_t*>(&cs.ready[s]);
      // wait until the carry has released this stage (first use passes at once)
      bool ok = true;
      if (lt == 0) {
        if (!mbar_wait(empty, (use & 1u) ^ 1u, spin_limit)) {
          give_up(empty, (use & 1u) ^ 1u, false);
          ok = false;
        }
      }
      named_bar(2, 128);
      if (cs.abort) break;
      if (lt == 0 && ok) {
        const uint32_t a = smem_u32(st);
        const ChunkLoc loc = chunk_locate(m, first + c);
        const int t0 = loc.t0, b = loc.b;
        mbar_expect_tx(full, STAGE_TX);
        tma_load_4d(a + S_QK, &tm_q, 0, h, t0, b, full);
        tma_load_4d(a + S_QK + 16384, &tm_q, 64, h, t0, b, full);
        tma_load_4d(a + S_QK + 8192, &tm_k, 0, h, t0, b, full);
        tma_load_4d(a + S_QK + 16384 + 8192, &tm_k, 64, h, t0, b, full);
        tma_load_4d(a + S_V, &tm_v, v0, h, t0, b, full);
        bulk_load(a + S_PT, wsb + (size_t)c * kChunkWs, kChunkWs, full);
      }
      if (!mbar_wait(full, use & 1u, spin_limit)) give_up(full, use & 1u, true);
      named_bar(2, 128);
      if (cs.abort) break;
      // the loader forms this chunk's outputs later: keep its e^{G_t}
      if (lt < 64) cs.eg_out[s][lt] = reinterpret_cast<const float*>(st + S_PT + WS_G)[lt];
      // k^T: thread lt takes channel lt of every token of the chunk
      {
        const unsigned char* qk = st + S_QK;
        unsigned char* kt = st + S_KT;
        __nv_bfloat16 col[64];
#pragma unroll
        for (int j = 0; j < 64; ++j)
          col[j] = *reinterpret_cast<const __nv_bfloat16*>(qk + swz_off_bf16(64 + j, lt, 128));
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          uint4 pk;
          __nv_bfloat16* e = reinterpret_cast<__nv_bfloat16*>(&pk);
#pragma unroll
          for (int x = 0; x < 8; ++x) e[x] = col[8 * q + x];
          *reinterpret_cast<uint4*>(kt + lt * 128 + ((q ^ (lt & 7)) << 4)) = pk;
        }
      }
      fence_smem_to_async();
      named_bar(2, 128);
      if (lt == 0) mbar_arrive(ready);
      if (c > 0 && !write_outputs(c - 1)) break;
    }
    if (!cs.abort && nchunks > 0) write_outputs(nchunks - 1);
  } else {
    // =========================== carry warpgroup ======================================
    // state: thread c < 128 owns row c of S^T (S[v0 + v][c], v < 32)
    const long sbase = ((long)chunk_state_index(m, seq) * H + h) * (long)dv * kDK;
    float st[kDVS];
#pragma unroll
    for (int vv = 0; vv < kDVS; ++vv) st[vv] = s0 ? s0[sbase + (long)(v0 + vv) * kDK + tid] : 0.f;
    auto write_state_operand = [&]() {
#pragma unroll
      for (int vv = 0; vv < kDVS; ++vv) {
        __nv_bfloat16 hi, lo;
        split_bf16(st[vv], hi, lo);
        const uint32_t off = swz_off_bf16(vv, tid, kDVS);
        *reinterpret_cast<__nv_bfloat16*>(tSSH + off) = hi;
        *reinterpret_cast<__nv_bfloat16*>(tSSL + off) = lo;
      }
    };
    write_state_operand();
    fence_smem_to_async();
    uint64_t* mma_bar = reinterpret_cast<uint64_t*>(&cs.mma_bar);
    uint32_t mphase = 0;
    const uint32_t aSSH = smem_u32(tSSH), aSSL = smem_u32(tSSL), aRT = smem_u32(tRT);
    const uint32_t aUT = smem_u32(tUT), aUPH = smem_u32(tUPH), aUPL = smem_u32(tUPL);
    const uint64_t dSSH = sdesc(aSSH, 16, 1024), dSSL = sdesc(aSSL, 16, 1024);
    const uint64_t dRT = sdesc(aRT, 16, 1024), dUT = sdesc(aUT, 16, 1024);
    const uint64_t dUPH = sdesc(aUPH, 16, 1024), dUPL = sdesc(aUPL, 16, 1024);
    // bounded wait on the carry's MMA barrier; the result is the same in all 128 threads
    auto wait_mma = [&]() -> bool {
      if (!mbar_wait(mma_bar, mphase, spin_limit)) give_up(mma_bar, mphase, true);
      mphase ^= 1u;
      fence_after_sync();
      named_bar(1, 128);
      return cs.abort != 0;
    };
    bool aborted = false;
    for (int c = 0; c < nchunks; ++c) {
      const int s = c & 1;
      const uint32_t use = (uint32_t)(c >> 1);
      unsigned char* stg = stage(s);
      const uint32_t a = smem_u32(stg);
      const float* gates = reinterpret_cast<const float*>(stg + S_PT + WS_G);
      uint64_t* ready = reinterpret_cast<uint64_t*>(&cs.ready[s]);
      if (tid == 0 && !mbar_wait(ready, use & 1u, spin_limit)) give_up(ready, use & 1u, false);
      named_bar(1, 128);
      if ((aborted = cs.abort != 0)) break;
      fence_after_sync();
      // ---- decay the state in TMEM, then [O1; Y] = [Q; K] (S_hi + S_lo)^T ----------------
      const int ob = c & 1;
      if (c >= 2 && tid == 0) {
        uint64_t* oe = reinterpret_cast<uint64_t*>(&cs.out_empty[ob]);
        const uint32_t par = (uint32_t)((c >> 1) - 1) & 1u;
        if (!mbar_wait(oe, par, spin_limit)) give_up(oe, par, false);
      }
      {
        float sd[kDVS];
        const float egc = gates[128];
#pragma unroll
        for (int vv = 0; vv < kDVS; ++vv) sd[vv] = st[vv] * egc;
        tmem_st32(tb + tlane + TM_S, sd);
        tmem_wait_st();
      }
      fence_before_sync();
      named_bar(1, 128);
      if (warp == 0) {
        fence_after_sync();
        const uint64_t dQK = sdesc(a + S_QK, 16, 1024);
        const uint32_t id = idesc_bf16(128, 32);
#pragma unroll
        for (int ks = 0; ks < kDK / 16; ++ks)
          mma_bf16_w(tb + TM_OY + 32 * ob, kstep(dQK, 128, ks), kstep(dSSH, kDVS, ks), id, ks > 0);
#pragma unroll
        for (int ks = 0; ks < kDK / 16; ++ks)
          mma_bf16_w(tb + TM_OY + 32 * ob, kstep(dQK, 128, ks), kstep(dSSL, kDVS, ks), id, true);
        mma_commit_w(mma_bar);
      }
      if ((aborted = wait_mma())) break;
      // ---- R = V - Diag(e^G) Y as the operand [v][j] (Y rows: TMEM lanes 64-127) ----------
      if (q4 >= 2) {
        const int j = 32 * (q4 - 2) + lane;
        float y[32], vv[32];
        const uint4* vrow = reinterpret_cast<const uint4*>(stg + S_V + j * 64);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 raw = vrow[q];
          const __nv_bfloat162* hh = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            const float2 f = __bfloat1622float2(hh[x]);
            vv[8 * q + 2 * x] = f.x;
            vv[8 * q + 2 * x + 1] = f.y;
          }
        }
        const float eg = gates[j];
        tmem_ld32(tb + tlane + TM_OY + 32 * ob, y);
        tmem_wait_ld();
#pragma unroll
        for (int v = 0; v < kDVS; ++v)
          *reinterpret_cast<float*>(tRT + swz_off(v, j, kDVS)) = to_tf32(fmaf(-eg, y[v], vv[v]));
      }
      fence_smem_to_async();
      fence_before_sync();
      named_bar(1, 128);
      // ---- U = T R (tf32) ----------------------------------------------------------------------
      if (warp == 0) {
        fence_after_sync();
        const uint64_t dT = sdesc(a + S_PT + WS_T, 16, 1024);
        const uint32_t id = idesc_tf32(64, 32, false, false);
#pragma unroll
        for (int ks = 0; ks < kC / 8; ++ks)
          mma_tf32_w(tb + TM_U, kstep(dT, 64, ks), kstep(dRT, kDVS, ks), id, ks > 0);
        mma_commit_w(mma_bar);
      }
      if ((aborted = wait_mma())) break;
      // ---- U (tf32 [v][j]) and U' = Diag(e^{G_last-G}) U (bf16 hi+lo [v][j]) ------------------
      {
        float u[32];
        tmem_ld32(tb + tlane + TM_U, u);
        tmem_wait_ld();
        if (lane < 16) {
          const int j = 16 * q4 + lane;
          const float el = gates[64 + j];
#pragma unroll
          for (int v = 0; v < kDVS; ++v) {
            *reinterpret_cast<float*>(tUT + swz_off(v, j, kDVS)) = to_tf32(u[v]);
            __nv_bfloat16 hi, lo;
            split_bf16(u[v] * el, hi, lo);
            const uint32_t off = swz_off_bf16(v, j, kDVS);
            *reinterpret_cast<__nv_bfloat16*>(tUPH + off) = hi;
            *reinterpret_cast<__nv_bfloat16*>(tUPL + off) = lo;
          }
        }
      }
      fence_smem_to_async();
      fence_before_sync();
      named_bar(1, 128);
      // ---- O2 = P U (tf32);  S^T += K^T (U'_hi + U'_lo) (bf16) ----------------------------------
      if (warp == 0) {
        // the state update first: the chain continues as soon as it completes, while
        // P U (needed only for the outputs) runs behind it; the stage is released and
        // the outputs handed to the loader when both have completed
        fence_after_sync();
        const uint64_t dP = sdesc(a + S_PT, 16, 1024);
        const uint64_t dKT = sdesc(a + S_KT, 16, 1024);
        const uint32_t ib = idesc_bf16(128, 32);
#pragma unroll
        for (int ks = 0; ks < kC / 16; ++ks)
          mma_bf16_w(tb + TM_S, kstep(dKT, 128, ks), kstep(dUPH, kDVS, ks), ib, true);
#pragma unroll
        for (int ks = 0; ks < kC / 16; ++ks)
          mma_bf16_w(tb + TM_S, kstep(dKT, 128, ks), kstep(dUPL, kDVS, ks), ib, true);
        mma_commit_w(mma_bar);
        const uint32_t it = idesc_tf32(64, 32, false, false);
#pragma unroll
        for (int ks = 0; ks < kC / 8; ++ks)
          mma_tf32_w(tb + TM_O2 + 32 * ob, kstep(dP, 64, ks), kstep(dUT, kDVS, ks), it, ks > 0);
        mma_commit_w(reinterpret_cast<uint64_t*>(&cs.empty[s]));
        mma_commit_w(reinterpret_cast<uint64_t*>(&cs.out_full[ob]));
      }
      if ((aborted = wait_mma())) break;
      // ---- new state: the chain's only remaining step before chunk c+1 ----------------------
      tmem_ld32(tb + tlane + TM_S, st);
      tmem_wait_ld();
      write_state_operand();
      fence_smem_to_async();
      fence_before_sync();
      named_bar(1, 128);
    }
    if (!aborted && s_final) {
#pragma unroll
      for (int vv = 0; vv < kDVS; ++vv) s_final[sbase + (long)(v0 + vv) * kDK + tid] = st[vv];
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tb, C_TM_COLS);
}

uint32_t split_spin_limit() {
  const char* e = getenv("GDR_SPIN_LIMIT");
  if (!e || !*e) return 1u << 24;
  return (uint32_t)strtoul(e, nullptr, 10);
}

template <typename Tout>
cudaError_t launch_split_t(const PrefillArgs& a, const ChunkMap& m, cudaStream_t stream) {
  // packed sequences: the tensors are [1, total, H, *]
  const int TB = m.cu ? 1 : a.B;
  CUtensorMap mq, mk, mv;
  if (!encode_bthd_bf16(&mq, a.q, TB, a.T, a.H, kDK, 64, kC, true) ||
      !encode_bthd_bf16(&mk, a.k, TB, a.T, a.H, kDK, 64, kC, true) ||
      !encode_bthd_bf16(&mv, a.v, TB, a.T, a.H, a.dv, kDVS, kC, false))
    return cudaErrorInvalidValue;
  const uint32_t lim = split_spin_limit();
  cudaError_t e = cudaFuncSetAttribute(gdn_chunk_prep_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, P_SMEM);
  if (e != cudaSuccess) return e;
  gdn_chunk_prep_kernel<<<a.H * m.nck, P_THREADS, P_SMEM, stream>>>(
      mq, mk, a.alpha, a.beta, (unsigned char*)a.workspace, m, a.H,
      (unsigned int*)a.workspace, lim);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  timing_mark(stream, 0);
  auto carry = gdn_chunk_carry_kernel<Tout>;
  e = cudaFuncSetAttribute(carry, cudaFuncAttributeMaxDynamicSharedMemorySize, C_SMEM);
  if (e != cudaSuccess) return e;
  carry<<<m.nseq * a.H * (a.dv / kDVS), C_THREADS, C_SMEM, stream>>>(
      mq, mk, mv, (const unsigned char*)a.workspace, a.s0, (Tout*)a.o, a.s_final, m, a.H,
      a.dv, (unsigned int*)a.workspace, lim);
  e = cudaGetLastError();
  if (e == cudaSuccess) timing_mark(stream, 1);
  return e;
}

}  // namespace

size_t split_prefill_workspace(int B, int T, int H) {
  const size_t nchunks = ((size_t)T + kC - 1) / kC;
  return (size_t)B * H * nchunks * kChunkWs;
}

size_t split_chunk_image_bytes() { return kChunkWs; }

cudaError_t launch_prefill_split(const PrefillArgs& a, const ChunkMap& m, cudaStream_t stream) {
  if (a.out_dtype == GDR_F32) return launch_split_t<float>(a, m, stream);
  return launch_split_t<__nv_bfloat16>(a, m, stream);
}

}  // namespace gdr
