// Chunked prefill of Gated DeltaNet on the sm_100a tensor cores (tcgen05).
//
// "Super Apriel: One Checkpoint, Many Speeds", §2A names the GDN mixer (delta
// rule, one scalar gate per head and token).  Per chunk of C = 64 tokens that
// enters with state S0 (d_v x d_k) and G[t] = sum_{s<=t} log alpha_s:
//
//   Gram  [Q; K] K^T                                    (tensor cores)
//   P[t,j] = (q_t.k_j) e^{G_t-G_j} (j<=t), A[t,j] = beta_t (k_t.k_j) e^{G_t-G_j} (j<t)
//   X = (I + A)^{-1}                                     (CUDA cores, blocked)
//   T = X Diag(beta),  T' = X Diag(beta e^G)
//   U = T V - T' (K S0^T)                                (tensor cores)
//   O = Diag(e^G) (Q S0^T) + P U                         (tensor cores)
//   S^T <- e^{G_last} S0^T + K^T Diag(e^{G_last-G}) U    (tensor cores, fp32 in TMEM)
//
// Operands: q, k, v arrive in bf16 and are widened exactly; every product runs as
// kind::tf32 with operands rounded to nearest tf32.  A single bf16 rounding of
// the computed operands (T, U, P, the state) costs about 3e-3 normwise error,
// more than the 2e-3 budget; tf32 costs about 4e-4.
//
// Work split: one CTA (128 threads, one warpgroup) per (batch, head, 32-wide
// slice of d_v) walks the chunks in order.  The state slice S^T (128 x 32 fp32)
// lives in tensor memory as an accumulator and in registers (thread c owns row
// c), and a tf32 copy S_s sits in shared memory as the MMA operand.  Shared
// memory tiles use the 128-byte swizzled K-major layout (tc.cuh); products that
// need the other orientation get a transposed copy written by the threads.
//
// Every wait on the tensor cores is bounded; a wait that gives up records
// GDR_ERR_TIMEOUT in the workspace status word, drains the outstanding MMAs,
// frees tensor memory and ends the CTA.

#include <math.h>
#include <stdlib.h>

#include "common.cuh"
#include "launch.h"
#include "tc.cuh"

namespace gdr {
namespace {

using namespace tc;

constexpr int kC = GDR_CHUNK;
constexpr int kDK = 128;
constexpr int kDVS = 32;
constexpr int kThreads = 128;

// shared-memory map (bytes from a 1024-aligned base)
constexpr int OFF_QK = 0;                     // [128][128]: rows 0-63 q, 64-127 k   64 KB
constexpr int OFF_KT = OFF_QK + 65536;        // [128 c][64 j] transposed k          32 KB
constexpr int OFF_VT = OFF_KT + 32768;        // [32 v][64 j] transposed v slice      8 KB
constexpr int OFF_P = OFF_VT + 8192;          // [64 t][64 j]                        16 KB
constexpr int OFF_TM = OFF_P + 16384;         // T  [64][64]                         16 KB
constexpr int OFF_TP = OFF_TM + 16384;        // T' [64][64]; X scratch in the solve 16 KB
constexpr int OFF_YT = OFF_TP + 16384;        // [32 v][64 j]; A scratch (16 KB) in prep
constexpr int OFF_UT = OFF_YT + 8192;         // [32 v][64 j]
constexpr int OFF_UPT = OFF_UT + 8192;        // [32 v][64 j]; Z scratch in the solve
constexpr int OFF_SS = OFF_UPT + 8192;        // [32 v][128 c] state operand          16 KB
constexpr int OFF_SMALL = OFF_SS + 16384;
constexpr int SMEM_USED = OFF_SMALL + 2048;
constexpr int SMEM_BYTES = SMEM_USED + 1024;  // slack for aligning the base

// tensor-memory columns
constexpr uint32_t TM_G = 0;     // Gram, M=128 x 64
constexpr uint32_t TM_U = 64;    // U~ then U, M=64 x 32
constexpr uint32_t TM_Y = 96;    // K S0^T, M=64 x 32
constexpr uint32_t TM_O1 = 128;  // Q S0^T, M=64 x 32
constexpr uint32_t TM_O2 = 160;  // P U, M=64 x 32
constexpr uint32_t TM_S = 192;   // S^T, M=128 x 32
constexpr uint32_t TM_COLS = 256;

constexpr uint32_t kDrainLimit = 1u << 26;

// K-major descriptor of k-step `ks` (8 tf32 = 32 bytes of K) for a tile with
// `rows` rows, operand starting at row `row0`.
__device__ __forceinline__ uint64_t kdesc(uint32_t tile, int rows, int row0, int ks) {
  return sdesc(tile + (uint32_t)((ks >> 2) * rows * 128 + row0 * 128 + (ks & 3) * 32), 16, 1024);
}

__device__ __forceinline__ void mma_chain(uint32_t tmem_d, uint32_t a_tile, int a_rows,
                                          int a_row0, uint32_t b_tile, int b_rows, int b_row0,
                                          int ksteps, uint32_t idesc, bool accumulate) {
  for (int ks = 0; ks < ksteps; ++ks)
    mma_tf32(tmem_d, kdesc(a_tile, a_rows, a_row0, ks), kdesc(b_tile, b_rows, b_row0, ks), idesc,
             accumulate || ks > 0);
}

struct SmallSmem {
  float g[kC];       // log gates, then cumulative G
  float eg[kC];      // e^{G_t}
  float egl[kC];     // e^{G_last - G_t}
  float beta[kC];
  float egc;         // e^{G_last}
  uint32_t tmem;
  int pad[2];
  unsigned long long bar;
};
static_assert(sizeof(SmallSmem) <= 2048, "small smem");

// store one fp32 (rounded to tf32) at (r, c) of a swizzled tile
__device__ __forceinline__ void st_tile(unsigned char* tile, int rows, int r, int c, float x) {
  *reinterpret_cast<float*>(tile + swz_off(r, c, rows)) = to_tf32(x);
}
__device__ __forceinline__ void st_tile4(unsigned char* tile, int rows, int r, int q, float4 x) {
  x.x = to_tf32(x.x); x.y = to_tf32(x.y); x.z = to_tf32(x.z); x.w = to_tf32(x.w);
  *reinterpret_cast<float4*>(tile + swz_off4(r, q, rows)) = x;
}

template <typename Tout>
__global__ void __launch_bounds__(kThreads, 1)
gdn_prefill_tc_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                      const __nv_bfloat16* __restrict__ v, const float* __restrict__ alpha,
                      const float* __restrict__ beta, const float* __restrict__ s0,
                      Tout* __restrict__ o, float* __restrict__ s_final, int T, int H, int dv,
                      unsigned int* __restrict__ status, uint32_t spin_limit) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* tQK = sm + OFF_QK;
  unsigned char* tKT = sm + OFF_KT;
  unsigned char* tVT = sm + OFF_VT;
  unsigned char* tP = sm + OFF_P;
  unsigned char* tTM = sm + OFF_TM;
  unsigned char* tTP = sm + OFF_TP;
  unsigned char* tYT = sm + OFF_YT;
  unsigned char* tUT = sm + OFF_UT;
  unsigned char* tUPT = sm + OFF_UPT;
  unsigned char* tSS = sm + OFF_SS;
  float* Xs = reinterpret_cast<float*>(tTP);     // [64][64] plain, during the solve
  float* As = reinterpret_cast<float*>(tYT);     // [64][64] plain, during prep
  float* Zs = reinterpret_cast<float*>(tUPT);    // [3][16][16] plain, during the solve
  SmallSmem& ss = *reinterpret_cast<SmallSmem*>(sm + OFF_SMALL);
  uint64_t* bar = reinterpret_cast<uint64_t*>(&ss.bar);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nslice = dv / kDVS;
  const int slice = blockIdx.x % nslice;
  const int bh = blockIdx.x / nslice;
  const int h = bh % H;
  const long b = bh / H;
  const int v0 = slice * kDVS;

  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&ss.tmem, TM_COLS);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tb = ss.tmem;
  const uint32_t tlane = (uint32_t)(warp * 32) << 16;   // this warp's TMEM lane quarter
  uint32_t phase = 0;

  // Wait for the last commit.  A wait that gives up records the timeout and then
  // drains the outstanding MMAs; the return value (the same in every thread, via
  // the barrier reduction) tells the CTA to stop.
  auto wait_mma = [&]() -> bool {
    int failed = 0;
    if (!mbar_wait(bar, phase, spin_limit)) {
      mbar_wait(bar, phase, kDrainLimit);
      if (lane == 0) atomicOr(status, 1u);
      failed = 1;
    }
    phase ^= 1u;
    fence_after_sync();
    return __syncthreads_or(failed) != 0;
  };
  bool aborted = false;

  const uint32_t aQK = smem_u32(tQK), aKT = smem_u32(tKT), aVT = smem_u32(tVT), aP = smem_u32(tP);
  const uint32_t aTM = smem_u32(tTM), aTP = smem_u32(tTP), aYT = smem_u32(tYT);
  const uint32_t aUT = smem_u32(tUT), aUPT = smem_u32(tUPT), aSS = smem_u32(tSS);

  // ---- initial state: thread c holds S0[v0 + v][c] for v < 32, and S_s gets a copy ----
  const long sbase = (b * H + h) * (long)dv * kDK;
  float st[kDVS];
#pragma unroll
  for (int vv = 0; vv < kDVS; ++vv) {
    st[vv] = s0 ? s0[sbase + (long)(v0 + vv) * kDK + tid] : 0.f;
    st_tile(tSS, kDVS, vv, tid, st[vv]);
  }

  for (int t0 = 0; t0 < T; t0 += kC) {
    const int L = min(kC, T - t0);
    // ---- 1. load q, k (rows t < L) into the [q; k] tile, v slice transposed -----------
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      const int i = tid + kThreads * n;        // 1024 vectors of 8 bf16 per tensor
      const int t = i >> 4, q8 = i & 15;
      float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0, c0 = a0, c1 = a0;
      if (t < L) {
        const long row = ((b * T + t0 + t) * H + h) * (long)kDK + q8 * 8;
        a0 = Elem<__nv_bfloat16>::load4(q + row);
        a1 = Elem<__nv_bfloat16>::load4(q + row + 4);
        c0 = Elem<__nv_bfloat16>::load4(k + row);
        c1 = Elem<__nv_bfloat16>::load4(k + row + 4);
      }
      st_tile4(tQK, 128, t, 2 * q8, a0);
      st_tile4(tQK, 128, t, 2 * q8 + 1, a1);
      st_tile4(tQK, 128, 64 + t, 2 * q8, c0);
      st_tile4(tQK, 128, 64 + t, 2 * q8 + 1, c1);
    }
    {
      const int vv = tid & 31, jg = tid >> 5;  // 16 tokens per thread
      float xv[16];
#pragma unroll
      for (int x = 0; x < 16; ++x) {
        const int j = jg * 16 + x;
        xv[x] = j < L ? __bfloat162float(v[((b * T + t0 + j) * H + h) * (long)dv + v0 + vv]) : 0.f;
      }
#pragma unroll
      for (int x = 0; x < 4; ++x)
        st_tile4(tVT, kDVS, vv, jg * 4 + x,
                 make_float4(xv[4 * x], xv[4 * x + 1], xv[4 * x + 2], xv[4 * x + 3]));
    }
    if (tid < kC) {
      const long row = (b * T + t0 + tid) * H + h;
      ss.beta[tid] = tid < L ? beta[row] : 0.f;
      ss.g[tid] = tid < L ? log_gate_accurate(alpha[row]) : 0.f;
    }
    __syncthreads();
    // ---- 2. gates: inclusive cumulative sum (fp64), exponentials; k^T copy ----------
    if (warp == 0) {
      const double g0 = ss.g[2 * lane], g1 = ss.g[2 * lane + 1];
      double s = g0 + g1;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const double n = __shfl_up_sync(0xffffffffu, s, off);
        if (lane >= off) s += n;
      }
      const double ex = s - (g0 + g1);
      __syncwarp();
      ss.g[2 * lane] = (float)(ex + g0);
      ss.g[2 * lane + 1] = (float)(ex + g0 + g1);
    }
    {
      // k^T: thread c reads column c of k from the [q; k] tile, writes row c of KT
      const int c = tid;
#pragma unroll
      for (int jq = 0; jq < 16; ++jq) {
        float4 x;
        x.x = *reinterpret_cast<const float*>(tQK + swz_off(64 + 4 * jq + 0, c, 128));
        x.y = *reinterpret_cast<const float*>(tQK + swz_off(64 + 4 * jq + 1, c, 128));
        x.z = *reinterpret_cast<const float*>(tQK + swz_off(64 + 4 * jq + 2, c, 128));
        x.w = *reinterpret_cast<const float*>(tQK + swz_off(64 + 4 * jq + 3, c, 128));
        *reinterpret_cast<float4*>(tKT + swz_off4(c, jq, 128)) = x;
      }
    }
    __syncthreads();
    if (tid < kC) {
      const float glast = ss.g[L - 1];
      ss.eg[tid] = expf(ss.g[tid]);
      ss.egl[tid] = expf(fminf(glast - ss.g[tid], 0.f));
      if (tid == 0) ss.egc = expf(glast);
    }
    fence_smem_to_async();
    fence_before_sync();
    __syncthreads();
    // ---- 3. Gram [q; k] k^T -----------------------------------------------------------
    if (tid == 0) {
      fence_after_sync();
      mma_chain(tb + TM_G, aQK, 128, 0, aQK, 128, 64, kDK / 8, idesc_tf32(128, 64, false, false),
                false);
      mma_commit(bar);
    }
    // state decay for this chunk (S^T <- e^{G_last} S^T) while the Gram runs
    {
      float sd[kDVS];
      const float egc = ss.egc;
#pragma unroll
      for (int vv = 0; vv < kDVS; ++vv) sd[vv] = st[vv] * egc;
      tmem_st32(tb + tlane + TM_S, sd);
      tmem_wait_st();
    }
    if ((aborted = wait_mma())) break;
    // ---- 4. P and A from the Gram -------------------------------------------------------
    {
      float d0[32], d1[32];
      tmem_ld32(tb + tlane + TM_G, d0);
      tmem_ld32(tb + tlane + TM_G + 32, d1);
      tmem_wait_ld();
      const int r = tid & 63;
      const bool isq = tid < 64;
      const float gt = ss.g[r];
      const float bt = ss.beta[r];
#pragma unroll
      for (int jq = 0; jq < 16; ++jq) {
        float e[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const int j = 4 * jq + x;
          const float d = j < 32 ? d0[j] : d1[j - 32];
          const float dec = __expf(fminf(gt - ss.g[j], 0.f));
          e[x] = isq ? (j <= r ? d * dec : 0.f) : (j < r ? bt * d * dec : 0.f);
        }
        if (isq)
          st_tile4(tP, 64, r, jq, make_float4(e[0], e[1], e[2], e[3]));
        else
          *reinterpret_cast<float4*>(As + r * 64 + 4 * jq) = make_float4(e[0], e[1], e[2], e[3]);
      }
    }
    __syncthreads();
    // ---- 5. X = (I + A)^{-1}: 16x16 diagonal blocks, then block substitution --------------
    for (int i = tid; i < 64 * 64; i += kThreads) Xs[i] = 0.f;
    __syncthreads();
    if (tid < 64) {
      const int a = tid >> 4, jl = tid & 15, base = 16 * a;
      float x[16];
#pragma unroll
      for (int tl = 0; tl < 16; ++tl) {
        float acc = (tl == jl) ? 1.f : 0.f;
#pragma unroll
        for (int i = 0; i < tl; ++i) acc = fmaf(-As[(base + tl) * 64 + base + i], x[i], acc);
        x[tl] = (tl < jl) ? 0.f : acc;
      }
#pragma unroll
      for (int tl = 0; tl < 16; ++tl) Xs[(base + tl) * 64 + base + jl] = x[tl];
    }
    __syncthreads();
    // off-diagonal blocks X[a][b], a - b = d: Z = sum_{m=b}^{a-1} A[a][m] X[m][b];
    // X[a][b] = -X[a][a] Z
    for (int d = 1; d <= 3; ++d) {
      const int nblk = 4 - d;
      for (int e = tid; e < nblk * 256; e += kThreads) {
        const int bb = e >> 8, r = (e >> 4) & 15, c = e & 15, aa = bb + d;
        float z = 0.f;
        for (int m = bb; m < aa; ++m)
#pragma unroll
          for (int i = 0; i < 16; ++i)
            z = fmaf(As[(16 * aa + r) * 64 + 16 * m + i], Xs[(16 * m + i) * 64 + 16 * bb + c], z);
        Zs[bb * 256 + r * 16 + c] = z;
      }
      __syncthreads();
      for (int e = tid; e < nblk * 256; e += kThreads) {
        const int bb = e >> 8, r = (e >> 4) & 15, c = e & 15, aa = bb + d;
        float x = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i)
          x = fmaf(Xs[(16 * aa + r) * 64 + 16 * aa + i], Zs[bb * 256 + i * 16 + c], x);
        Xs[(16 * aa + r) * 64 + 16 * bb + c] = -x;
      }
      __syncthreads();
    }
    // ---- 6. T = X Diag(beta), T' = X Diag(beta e^G) as tf32 operands ---------------------
    {
      const int r = tid & 63, half = tid >> 6;
      float xr[32];
#pragma unroll
      for (int x = 0; x < 32; ++x) xr[x] = Xs[r * 64 + half * 32 + x];
#pragma unroll
      for (int x = 0; x < 8; ++x) {
        const int j = half * 32 + 4 * x;
        st_tile4(tTM, 64, r, j / 4,
                 make_float4(xr[4 * x] * ss.beta[j], xr[4 * x + 1] * ss.beta[j + 1],
                             xr[4 * x + 2] * ss.beta[j + 2], xr[4 * x + 3] * ss.beta[j + 3]));
      }
      __syncthreads();   // X (aliasing T') fully read
#pragma unroll
      for (int x = 0; x < 8; ++x) {
        const int j = half * 32 + 4 * x;
        st_tile4(tTP, 64, r, j / 4,
                 make_float4(xr[4 * x] * ss.beta[j] * ss.eg[j],
                             xr[4 * x + 1] * ss.beta[j + 1] * ss.eg[j + 1],
                             xr[4 * x + 2] * ss.beta[j + 2] * ss.eg[j + 2],
                             xr[4 * x + 3] * ss.beta[j + 3] * ss.eg[j + 3]));
      }
    }
    fence_smem_to_async();
    fence_before_sync();
    __syncthreads();
    // ---- 7. U~ = T V, Y = K S0^T, O1 = Q S0^T ----------------------------------------------
    if (tid == 0) {
      fence_after_sync();
      const uint32_t i64x32 = idesc_tf32(64, 32, false, false);
      mma_chain(tb + TM_U, aTM, 64, 0, aVT, kDVS, 0, kC / 8, i64x32, false);
      mma_chain(tb + TM_Y, aQK, 128, 64, aSS, kDVS, 0, kDK / 8, i64x32, false);
      mma_chain(tb + TM_O1, aQK, 128, 0, aSS, kDVS, 0, kDK / 8, i64x32, false);
      mma_commit(bar);
    }
    if ((aborted = wait_mma())) break;
    // ---- 8. Y -> smem operand (transposed: [v][j]) ------------------------------------------
    {
      float y[32];
      tmem_ld32(tb + tlane + TM_Y, y);
      tmem_wait_ld();
      if (lane < 16) {
        const int j = warp * 16 + lane;
#pragma unroll
        for (int vv = 0; vv < kDVS; ++vv) st_tile(tYT, kDVS, vv, j, y[vv]);
      }
    }
    fence_smem_to_async();
    fence_before_sync();
    __syncthreads();
    // ---- 9. U = U~ - T' Y -------------------------------------------------------------------
    if (tid == 0) {
      fence_after_sync();
      mma_chain(tb + TM_U, aTP, 64, 0, aYT, kDVS, 0, kC / 8, idesc_tf32(64, 32, false, false, true),
                true);
      mma_commit(bar);
    }
    if ((aborted = wait_mma())) break;
    // ---- 10. U, U' = Diag(e^{G_last - G}) U -> smem operands ---------------------------------
    {
      float u[32];
      tmem_ld32(tb + tlane + TM_U, u);
      tmem_wait_ld();
      if (lane < 16) {
        const int j = warp * 16 + lane;
        const float el = ss.egl[j];
#pragma unroll
        for (int vv = 0; vv < kDVS; ++vv) {
          st_tile(tUT, kDVS, vv, j, u[vv]);
          st_tile(tUPT, kDVS, vv, j, u[vv] * el);
        }
      }
    }
    fence_smem_to_async();
    fence_before_sync();
    __syncthreads();
    // ---- 11. O2 = P U;  S^T += K^T U' -------------------------------------------------------
    if (tid == 0) {
      fence_after_sync();
      mma_chain(tb + TM_O2, aP, 64, 0, aUT, kDVS, 0, kC / 8, idesc_tf32(64, 32, false, false),
                false);
      mma_chain(tb + TM_S, aKT, 128, 0, aUPT, kDVS, 0, kC / 8, idesc_tf32(128, 32, false, false),
                true);
      mma_commit(bar);
    }
    if ((aborted = wait_mma())) break;
    // ---- 12. outputs and the new state --------------------------------------------------------
    {
      float o1[32], o2[32];
      tmem_ld32(tb + tlane + TM_O1, o1);
      tmem_ld32(tb + tlane + TM_O2, o2);
      tmem_ld32(tb + tlane + TM_S, st);
      tmem_wait_ld();
      if (lane < 16) {
        const int t = warp * 16 + lane;
        if (t < L) {
          const float eg = ss.eg[t];
          Tout* dst = o + ((b * T + t0 + t) * H + h) * (long)dv + v0;
#pragma unroll
          for (int vv = 0; vv < kDVS; ++vv) Elem<Tout>::store(dst + vv, fmaf(eg, o1[vv], o2[vv]));
        }
      }
#pragma unroll
      for (int vv = 0; vv < kDVS; ++vv) st_tile(tSS, kDVS, vv, tid, st[vv]);
    }
    fence_smem_to_async();
    fence_before_sync();
    __syncthreads();
  }
  if (!aborted && s_final) {
#pragma unroll
    for (int vv = 0; vv < kDVS; ++vv) s_final[sbase + (long)(v0 + vv) * kDK + tid] = st[vv];
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tb, TM_COLS);
}

uint32_t spin_limit_from_env() {
  const char* s = getenv("GDR_SPIN_LIMIT");
  if (!s || !*s) return 1u << 24;
  return (uint32_t)strtoul(s, nullptr, 10);
}

template <typename Tout>
cudaError_t launch_t(const PrefillArgs& a, cudaStream_t st) {
  auto kern = gdn_prefill_tc_kernel<Tout>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int grid = a.B * a.H * (a.dv / kDVS);
  kern<<<grid, kThreads, SMEM_BYTES, st>>>(
      (const __nv_bfloat16*)a.q, (const __nv_bfloat16*)a.k, (const __nv_bfloat16*)a.v, a.alpha,
      a.beta, a.s0, (Tout*)a.o, a.s_final, a.T, a.H, a.dv, (unsigned int*)a.workspace,
      spin_limit_from_env());
  return cudaGetLastError();
}

}  // namespace

bool tc_prefill_supported(const PrefillArgs& a) {
  return a.in_dtype == GDR_BF16 && a.dk == kDK && !a.kda && a.dv % kDVS == 0;
}

size_t tc_prefill_workspace(int, int, int, int, int, bool) { return 0; }

cudaError_t launch_prefill_tc(const PrefillArgs& a, cudaStream_t st) {
  if (a.out_dtype == GDR_F32) return launch_t<float>(a, st);
  return launch_t<__nv_bfloat16>(a, st);
}

}  // namespace gdr
