// Chunked prefill of Gated DeltaNet on the sm_100a tensor cores (tcgen05 + TMA).
//
// "Super Apriel: One Checkpoint, Many Speeds", §2A names the GDN mixer (delta
// rule, one scalar gate per head and token).  For a chunk of C = 64 tokens that
// enters with state S0 (d_v x d_k), G[t] = sum_{s<=t} log alpha_s (chunk-local):
//
//   Gram   [Q; K] K^T                                        (tensor cores)
//   P[t,j] = (q_t.k_j) e^{G_t-G_j} (j<=t),  A[t,j] = beta_t (k_t.k_j) e^{G_t-G_j} (j<t)
//   X = (I + A)^{-1}  (unit lower triangular; CUDA cores, 16x16 blocks)
//   T = X Diag(beta)
//   Y = K S0^T,  R = V - Diag(e^G) Y,  U = T R                (tensor cores)
//   O = Diag(e^G) (Q S0^T) + P U                              (tensor cores)
//   S^T <- e^{G_last} S0^T + K^T Diag(e^{G_last-G}) U         (tensor cores, fp32 in TMEM)
//
// (U = T R is the WY form T V - T Diag(e^G) K S0^T with the two products merged.)
//
// Operands: q, k, v arrive in bf16 by TMA and are widened exactly; every product
// runs as kind::tf32 with operands rounded to nearest tf32.  A single bf16
// rounding of the computed operands (T, U, P, the state) costs about 3e-3
// normwise error, more than the 2e-3 budget; tf32 costs about 4e-4.
//
// Work split: one CTA (256 threads) per (batch, head, 32-wide slice of d_v) walks
// the chunks in order; the TMA load of chunk c+1 overlaps the work on chunk c.
// The state slice S^T (128 x 32 fp32) lives in tensor memory as an accumulator
// and in registers (thread c owns row c); a tf32 copy S_s in shared memory is
// the MMA operand.  Operand tiles use the 128-byte swizzled K-major layout
// (tc.cuh); products that want the other orientation get transposed copies.
//
// Every wait is bounded.  A wait that gives up records GDR_ERR_TIMEOUT in the
// workspace status word, drains the outstanding tensor-core and TMA operations,
// frees tensor memory and ends the CTA.

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
constexpr int kThreads = 256;

// shared-memory map (bytes from a 1024-aligned base)
constexpr int OFF_QK = 0;                  // fp32 [128][128]: rows 0-63 q, 64-127 k    64 KB
constexpr int OFF_KT = OFF_QK + 65536;     // fp32 [128 c][64 j]  k transposed          32 KB
constexpr int OFF_P = OFF_KT + 32768;      // fp32 [64 t][64 j]                         16 KB
constexpr int OFF_TM = OFF_P + 16384;      // fp32 T [64][64]; X scratch in the solve   16 KB
constexpr int OFF_RT = OFF_TM + 16384;     // fp32 [32 v][64 j]; A scratch (16 KB over RT+UT)
constexpr int OFF_UT = OFF_RT + 8192;      //   in prep; P U exchange [64][32] at the end
constexpr int OFF_UPT = OFF_UT + 8192;     // fp32 [32 v][64 j]; Z scratch in the solve
constexpr int OFF_SS = OFF_UPT + 8192;     // fp32 [32 v][128 c]  state operand          16 KB
constexpr int OFF_VF = OFF_SS + 16384;     // fp32 [64 j][32 v]   v slice                 8 KB
constexpr int OFF_STG = OFF_VF + 8192;     // bf16 TMA staging: q, k [64][128], v [64][32]
constexpr int STG_Q = 0, STG_K = 16384, STG_V = 32768, STG_BYTES = 36864;
constexpr int OFF_SMALL = OFF_STG + STG_BYTES;
constexpr int SMEM_USED = OFF_SMALL + 2048;
constexpr int SMEM_BYTES = SMEM_USED + 1024;  // slack for aligning the base
static_assert(SMEM_BYTES <= 232448, "shared memory");

// tensor-memory columns
constexpr uint32_t TM_G = 0;     // Gram [q; k] k^T, M=128 x 64
constexpr uint32_t TM_OY = 64;   // [q; k] S0^T, M=128 x 32: rows 0-63 O1, rows 64-127 Y
constexpr uint32_t TM_U = 96;    // U, M=64 x 32
constexpr uint32_t TM_O2 = 128;  // P U, M=64 x 32
constexpr uint32_t TM_S = 160;   // S^T, M=128 x 32
constexpr uint32_t TM_COLS = 256;

constexpr uint32_t kDrainLimit = 1u << 26;

struct SmallSmem {
  float g[kC];       // log gates, then cumulative G
  float eg[kC];      // e^{G_t}
  float egl[kC];     // e^{G_last - G_t}
  float beta[kC];
  float egc;         // e^{G_last}
  uint32_t tmem;
  unsigned long long mma_bar;
  unsigned long long tma_bar;
};
static_assert(sizeof(SmallSmem) <= 2048, "small smem");

// K-major operand: k-step ks advances 8 tf32 (32 bytes) along a 128-byte panel
// row, then to the next panel (rows * 128 bytes).
__device__ __forceinline__ uint64_t kstep(uint64_t desc0, int rows, int ks) {
  return desc0 + (uint64_t)((((ks >> 2) * rows * 128) + ((ks & 3) * 32)) >> 4);
}

__device__ __forceinline__ void mma_chain(uint32_t tmem_d, uint64_t a0, int a_rows, uint64_t b0,
                                          int b_rows, int ksteps, uint32_t idesc,
                                          bool accumulate) {
#pragma unroll 4
  for (int ks = 0; ks < ksteps; ++ks)
    mma_tf32(tmem_d, kstep(a0, a_rows, ks), kstep(b0, b_rows, ks), idesc, accumulate || ks > 0);
}

__device__ __forceinline__ void st_tile(unsigned char* tile, int rows, int r, int c, float x) {
  *reinterpret_cast<float*>(tile + swz_off(r, c, rows)) = to_tf32(x);
}
__device__ __forceinline__ void st_tile4(unsigned char* tile, int rows, int r, int q, float4 x) {
  x.x = to_tf32(x.x); x.y = to_tf32(x.y); x.z = to_tf32(x.z); x.w = to_tf32(x.w);
  *reinterpret_cast<float4*>(tile + swz_off4(r, q, rows)) = x;
}
// 8 bf16 (16 bytes) -> two float4
__device__ __forceinline__ void bf16x8(const unsigned char* p, float4& a, float4& b) {
  const uint4 raw = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* hh = reinterpret_cast<const __nv_bfloat162*>(&raw);
  const float2 f0 = __bfloat1622float2(hh[0]), f1 = __bfloat1622float2(hh[1]);
  const float2 f2 = __bfloat1622float2(hh[2]), f3 = __bfloat1622float2(hh[3]);
  a = make_float4(f0.x, f0.y, f1.x, f1.y);
  b = make_float4(f2.x, f2.y, f3.x, f3.y);
}

// [64][64] fp32 scratch with the column index XOR-ed by the row, so that both a
// row and a column of 32 consecutive entries fall in distinct banks.
__device__ __forceinline__ int sx(int r, int c) { return r * 64 + (c ^ (r & 31)); }

// Four consecutive entries (row k, columns c4 .. c4+3, c4 a multiple of 4) of an sx()
// tile with one 16-byte load: the XOR by the row keeps aligned groups of four
// together and permutes inside a group by (k & 3), which klo must equal (callers pass
// an unrolled loop index, so the selection folds away at compile time).
__device__ __forceinline__ void ld4_sx(const float* base, int k, int klo, int c4, float (&e)[4]) {
  const float4 f = *reinterpret_cast<const float4*>(base + k * 64 + (c4 ^ (k & 28)));
  const float v[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
  for (int x = 0; x < 4; ++x) e[x] = v[x ^ klo];
}

template <typename Tout>
__global__ void __launch_bounds__(kThreads, 1)
gdn_prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const float* __restrict__ alpha,
                      const float* __restrict__ beta, const float* __restrict__ s0,
                      Tout* __restrict__ o, float* __restrict__ s_final, int T, int H, int dv,
                      unsigned int* __restrict__ status, uint32_t spin_limit) {
  extern __shared__ unsigned char smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  unsigned char* sm = smem_raw + pad;
  unsigned char* tQK = sm + OFF_QK;
  unsigned char* tKT = sm + OFF_KT;
  unsigned char* tP = sm + OFF_P;
  unsigned char* tTM = sm + OFF_TM;
  unsigned char* tRT = sm + OFF_RT;
  unsigned char* tUT = sm + OFF_UT;
  unsigned char* tUPT = sm + OFF_UPT;
  unsigned char* tSS = sm + OFF_SS;
  unsigned char* tVF = sm + OFF_VF;
  unsigned char* stg = sm + OFF_STG;
  float* Xs = reinterpret_cast<float*>(tTM);     // solve scratch, sx() layout
  float* As = reinterpret_cast<float*>(tRT);     // 16 KB over RT + UT, sx() layout
  float* Zs = reinterpret_cast<float*>(tUPT);    // [3][16][16]
  float* Ox = reinterpret_cast<float*>(tRT);     // P U exchange [64 t][32 v], row-XOR layout
  SmallSmem& ss = *reinterpret_cast<SmallSmem*>(sm + OFF_SMALL);
  uint64_t* mma_bar = reinterpret_cast<uint64_t*>(&ss.mma_bar);
  uint64_t* tma_bar = reinterpret_cast<uint64_t*>(&ss.tma_bar);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q4 = warp & 3;          // TMEM lane quarter this warp may access
  const int hw = warp >> 2;         // which half of the CTA (splits columns)
  const int nslice = dv / kDVS;
  const int slice = blockIdx.x % nslice;
  const int bh = blockIdx.x / nslice;
  const int h = bh % H;
  const int b = bh / H;
  const int v0 = slice * kDVS;
  const int nchunks = (T + kC - 1) / kC;

  if (tid == 0) {
    mbar_init(mma_bar, 1);
    mbar_init(tma_bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&ss.tmem, TM_COLS);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tb = ss.tmem;
  const uint32_t tlane = (uint32_t)(q4 * 32) << 16;
  uint32_t mphase = 0, tphase = 0;
  bool tma_inflight = false;

  auto issue_tma = [&](int t0) {
    mbar_expect_tx(tma_bar, STG_BYTES);
    const uint32_t s = smem_u32(stg);
    tma_load_4d(s + STG_Q, &tm_q, 0, h, t0, b, tma_bar);
    tma_load_4d(s + STG_K, &tm_k, 0, h, t0, b, tma_bar);
    tma_load_4d(s + STG_V, &tm_v, v0, h, t0, b, tma_bar);
  };
  // A bounded wait; on give-up record the timeout, drain, and have every thread
  // of the CTA (barrier reduction) agree to stop.
  auto wait_bar = [&](uint64_t* bar, uint32_t& ph) -> bool {
    int failed = 0;
    if (!mbar_wait(bar, ph, spin_limit)) {
      mbar_wait(bar, ph, kDrainLimit);
      if (lane == 0) atomicOr(status, 1u);
      failed = 1;
    }
    ph ^= 1u;
    fence_after_sync();
    return __syncthreads_or(failed) != 0;
  };

  if (tid == 0) issue_tma(0);
  tma_inflight = true;
  // gates of the next chunk, prefetched into registers (rows past T: alpha 1, beta 0)
  float a_next = 1.f, b_next = 0.f;
  if (tid < kC && tid < T) {
    const long row = ((long)b * T + tid) * H + h;
    a_next = alpha[row];
    b_next = beta[row];
  }

  const uint32_t aQK = smem_u32(tQK), aKT = smem_u32(tKT), aP = smem_u32(tP), aTM = smem_u32(tTM);
  const uint32_t aRT = smem_u32(tRT), aUT = smem_u32(tUT), aUPT = smem_u32(tUPT);
  const uint32_t aSS = smem_u32(tSS);
  const uint64_t dQK = sdesc(aQK, 16, 1024), dK = sdesc(aQK + 64 * 128, 16, 1024);
  const uint64_t dKT = sdesc(aKT, 16, 1024), dP = sdesc(aP, 16, 1024), dTM = sdesc(aTM, 16, 1024);
  const uint64_t dRT = sdesc(aRT, 16, 1024), dUT = sdesc(aUT, 16, 1024);
  const uint64_t dUPT = sdesc(aUPT, 16, 1024), dSS = sdesc(aSS, 16, 1024);

  // ---- initial state: thread c < 128 holds S0[v0 + v][c]; S_s gets a tf32 copy ---------
  const long sbase = ((long)b * H + h) * (long)dv * kDK;
  float st[kDVS];
  if (tid < kDK) {
#pragma unroll
    for (int vv = 0; vv < kDVS; ++vv) st[vv] = s0 ? s0[sbase + (long)(v0 + vv) * kDK + tid] : 0.f;
#pragma unroll
    for (int vv = 0; vv < kDVS; ++vv) st_tile(tSS, kDVS, vv, tid, st[vv]);
  }

  bool aborted = false;
  for (int c = 0; c < nchunks; ++c) {
    const int t0 = c * kC;
    const int L = min(kC, T - t0);
    // ---- 1. chunk c has landed: widen it into the operand tiles -----------------------
    aborted = wait_bar(tma_bar, tphase);
    tma_inflight = false;
    if (aborted) break;
    if (tid < kC) {
      ss.g[tid] = log_gate_accurate(a_next);
      ss.beta[tid] = b_next;
    }
    {
      // q and k: 2048 groups of 8 bf16; all loads are issued before any store
      uint4 raw[8];
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        const int i = tid + kThreads * n;
        const int t = (i >> 4) & 63, q8 = i & 15;
        raw[n] = *reinterpret_cast<const uint4*>(stg + ((i >> 10) ? STG_K : STG_Q) + t * 256 + q8 * 16);
      }
      const __nv_bfloat16* kst = reinterpret_cast<const __nv_bfloat16*>(stg + STG_K);
      const int kc = tid & 127, jh = tid >> 7;
      __nv_bfloat16 kcol[32];
#pragma unroll
      for (int x = 0; x < 32; ++x) kcol[x] = kst[(jh * 32 + x) * kDK + kc];
      const uint4 vraw = *reinterpret_cast<const uint4*>(stg + STG_V + (tid >> 2) * 64 + (tid & 3) * 16);
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        const int i = tid + kThreads * n;
        const int t = (i >> 4) & 63, q8 = i & 15, row = (i >> 10) * 64 + t;
        float4 x0, x1;
        bf16x8(reinterpret_cast<const unsigned char*>(&raw[n]), x0, x1);
        *reinterpret_cast<float4*>(tQK + swz_off4(row, 2 * q8, 128)) = x0;
        *reinterpret_cast<float4*>(tQK + swz_off4(row, 2 * q8 + 1, 128)) = x1;
      }
#pragma unroll
      for (int x = 0; x < 8; ++x)
        *reinterpret_cast<float4*>(tKT + swz_off4(kc, jh * 8 + x, 128)) =
            make_float4(__bfloat162float(kcol[4 * x]), __bfloat162float(kcol[4 * x + 1]),
                        __bfloat162float(kcol[4 * x + 2]), __bfloat162float(kcol[4 * x + 3]));
      float4 x0, x1;
      bf16x8(reinterpret_cast<const unsigned char*>(&vraw), x0, x1);
      *reinterpret_cast<float4*>(tVF + swz_off4(tid >> 2, 2 * (tid & 3), 64)) = x0;
      *reinterpret_cast<float4*>(tVF + swz_off4(tid >> 2, 2 * (tid & 3) + 1, 64)) = x1;
    }
    fence_smem_to_async();
    __syncthreads();
    if (c + 1 < nchunks) {
      if (tid == 0) issue_tma(t0 + kC);
      tma_inflight = true;
      a_next = 1.f;
      b_next = 0.f;
      if (tid < kC && t0 + kC + tid < T) {
        const long row = ((long)b * T + t0 + kC + tid) * H + h;
        a_next = alpha[row];
        b_next = beta[row];
      }
    }
    // ---- 2. gates: inclusive cumulative sum in fp64, exponentials -----------------------
    if (warp == 0) {
      const double g0 = ss.g[2 * lane], g1 = ss.g[2 * lane + 1];
      double s = g0 + g1;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const double n = __shfl_up_sync(0xffffffffu, s, off);
        if (lane >= off) s += n;
      }
      const double ex = s - (g0 + g1);
      ss.g[2 * lane] = (float)(ex + g0);
      ss.g[2 * lane + 1] = (float)(ex + g0 + g1);
    }
    __syncthreads();
    if (tid < kC) {
      const float glast = ss.g[L - 1];
      ss.eg[tid] = __expf(ss.g[tid]);
      ss.egl[tid] = __expf(fminf(glast - ss.g[tid], 0.f));
      if (tid == 0) ss.egc = __expf(glast);
    }
    fence_before_sync();
    __syncthreads();
    // ---- 3. Gram [q; k] k^T on the tensor cores; meanwhile decay the state -----------------
    if (tid == 0) {
      fence_after_sync();
      mma_chain(tb + TM_G, dQK, 128, dK, 128, kDK / 8, idesc_tf32(128, 64, false, false), false);
      mma_commit(mma_bar);
    }
    if (tid < kDK) {
      float sd[kDVS];
      const float egc = ss.egc;
#pragma unroll
      for (int vv = 0; vv < kDVS; ++vv) sd[vv] = st[vv] * egc;
      tmem_st32(tb + tlane + TM_S, sd);
      tmem_wait_st();
    }
    if ((aborted = wait_bar(mma_bar, mphase))) break;
    // ---- 4. P (decayed, lower) and A (decayed, beta, strictly lower) --------------------------
    {
      // thread: Gram row r = 32 q4 + lane, columns 32 hw .. 32 hw + 31
      float d[32], gj[32];
      tmem_ld32(tb + tlane + TM_G + 32 * hw, d);
#pragma unroll
      for (int x = 0; x < 32; ++x) gj[x] = ss.g[32 * hw + x];
      const int r = 32 * q4 + lane;
      const int t = r & 63;
      const float gt = ss.g[t];
      const float bt = ss.beta[t];
      tmem_wait_ld();
      if (r < 64) {
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          const int j = 32 * hw + x;
          d[x] = j <= t ? d[x] * __expf(gt - gj[x]) : 0.f;
        }
#pragma unroll
        for (int x = 0; x < 8; ++x)
          st_tile4(tP, 64, t, 8 * hw + x, make_float4(d[4 * x], d[4 * x + 1], d[4 * x + 2], d[4 * x + 3]));
      } else {
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          const int j = 32 * hw + x;
          d[x] = j < t ? bt * d[x] * __expf(gt - gj[x]) : 0.f;
        }
#pragma unroll
        for (int x = 0; x < 32; ++x) As[sx(t, 32 * hw + x)] = d[x];
      }
    }
    __syncthreads();
    // ---- 5. X = (I + A)^{-1}: diagonal 16x16 blocks, then three block levels --------------------
    // Diagonal 16x16 blocks: warp a (a < 4) inverts block a, lane jl < 16 owning column
    // jl.  In the sx() layout, entry (16a + tl, 16a + i) sits at
    // (16a + tl) * 64 + (16a ^ (16a & 16)) + (i ^ tl): a compile-time offset from the
    // block's base once tl and i are unrolled.
    if (warp < 4 && lane < 16) {
      const int base = 16 * warp, jl = lane;
      const int bx = base ^ (base & 16);
      const float* Ab = As + base * 64 + bx;
      float x[16];
#pragma unroll
      for (int tl = 0; tl < 16; ++tl) {
        float a_row[16];
#pragma unroll
        for (int i = 0; i < tl; ++i) a_row[i] = Ab[tl * 64 + (i ^ tl)];
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
    // Off-diagonal blocks, level d = a - b: Z[b] = sum_{m=b}^{a-1} A[a][m] X[m][b], then
    // X[a][b] = -X[a][a] Z[b].  Thread layout per 16x16 block: row r, columns 4cq..4cq+3;
    // 64 threads per block, up to 3 blocks per level.
    {
      const int bb = tid >> 6, r = (tid >> 2) & 15, cq = tid & 3;
#pragma unroll
      for (int d = 1; d <= 3; ++d) {
        const bool act = bb < 4 - d;
        const int aa = bb + d;
        if (act) {
          float z0 = 0.f, z1 = 0.f, z2 = 0.f, z3 = 0.f;
#pragma unroll
          for (int m = 0; m < d; ++m) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int k = 16 * (bb + m) + i;
              const float a = As[sx(16 * aa + r, k)];
              float e[4];
              ld4_sx(Xs, k, i & 3, 16 * bb + 4 * cq, e);
              z0 = fmaf(a, e[0], z0);
              z1 = fmaf(a, e[1], z1);
              z2 = fmaf(a, e[2], z2);
              z3 = fmaf(a, e[3], z3);
            }
          }
          *reinterpret_cast<float4*>(&Zs[bb * 256 + r * 16 + 4 * cq]) = make_float4(z0, z1, z2, z3);
        }
        __syncthreads();
        if (act) {
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
          const int row = 16 * aa + r, col = 16 * bb + 4 * cq;
          Xs[sx(row, col + 0)] = -x0;
          Xs[sx(row, col + 1)] = -x1;
          Xs[sx(row, col + 2)] = -x2;
          Xs[sx(row, col + 3)] = -x3;
        }
        __syncthreads();
      }
    }
    // ---- 6. T = X Diag(beta) as a tf32 operand (blocks above the diagonal are zero) -----------
    {
      const int r = tid & 63, qq = tid >> 6;      // 16 columns per thread
      float xr[16];
#pragma unroll
      for (int x = 0; x < 16; ++x) {
        const int j = qq * 16 + x;
        xr[x] = (qq <= (r >> 4)) ? Xs[sx(r, j)] * ss.beta[j] : 0.f;
      }
      __syncthreads();   // X (which aliases T) fully read
#pragma unroll
      for (int x = 0; x < 4; ++x)
        st_tile4(tTM, 64, r, qq * 4 + x,
                 make_float4(xr[4 * x], xr[4 * x + 1], xr[4 * x + 2], xr[4 * x + 3]));
    }
    fence_smem_to_async();
    fence_before_sync();
    __syncthreads();
    // ---- 7. [O1; Y] = [Q; K] S0^T  (one M=128 product) ------------------------------------------
    if (tid == 0) {
      fence_after_sync();
      mma_chain(tb + TM_OY, dQK, 128, dSS, kDVS, kDK / 8, idesc_tf32(128, 32, false, false), false);
      mma_commit(mma_bar);
    }
    if ((aborted = wait_bar(mma_bar, mphase))) break;
    // ---- 8. R = V - Diag(e^G) Y as the operand [v][j] (Y rows live in lanes 64-127) -------------
    if (hw == 0 && q4 >= 2) {
      const int j = 32 * (q4 - 2) + lane;
      float y[32];
      float4 vx[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) vx[q] = *reinterpret_cast<const float4*>(tVF + swz_off4(j, q, 64));
      const float eg = ss.eg[j];
      tmem_ld32(tb + tlane + TM_OY, y);
      tmem_wait_ld();
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        st_tile(tRT, kDVS, 4 * q + 0, j, fmaf(-eg, y[4 * q + 0], vx[q].x));
        st_tile(tRT, kDVS, 4 * q + 1, j, fmaf(-eg, y[4 * q + 1], vx[q].y));
        st_tile(tRT, kDVS, 4 * q + 2, j, fmaf(-eg, y[4 * q + 2], vx[q].z));
        st_tile(tRT, kDVS, 4 * q + 3, j, fmaf(-eg, y[4 * q + 3], vx[q].w));
      }
    }
    fence_smem_to_async();
    fence_before_sync();
    __syncthreads();
    // ---- 9. U = T R -------------------------------------------------------------------------------
    if (tid == 0) {
      fence_after_sync();
      mma_chain(tb + TM_U, dTM, 64, dRT, kDVS, kC / 8, idesc_tf32(64, 32, false, false), false);
      mma_commit(mma_bar);
    }
    if ((aborted = wait_bar(mma_bar, mphase))) break;
    // ---- 10. U and U' = Diag(e^{G_last - G}) U as operands [v][j] (M=64 rows: lanes 0-15) ---------
    {
      float u[16];
      tmem_ld16(tb + tlane + TM_U + 16 * hw, u);
      tmem_wait_ld();
      if (lane < 16) {
        const int j = 16 * q4 + lane;
        const float el = ss.egl[j];
#pragma unroll
        for (int x = 0; x < 16; ++x) {
          st_tile(tUT, kDVS, 16 * hw + x, j, u[x]);
          st_tile(tUPT, kDVS, 16 * hw + x, j, u[x] * el);
        }
      }
    }
    fence_smem_to_async();
    fence_before_sync();
    __syncthreads();
    // ---- 11. O2 = P U;  S^T += K^T U' ----------------------------------------------------------------
    if (tid == 0) {
      fence_after_sync();
      mma_chain(tb + TM_O2, dP, 64, dUT, kDVS, kC / 8, idesc_tf32(64, 32, false, false), false);
      mma_chain(tb + TM_S, dKT, 128, dUPT, kDVS, kC / 8, idesc_tf32(128, 32, false, false), true);
      mma_commit(mma_bar);
    }
    if ((aborted = wait_bar(mma_bar, mphase))) break;
    // ---- 12. new state (warps 0-3) and outputs O = Diag(e^G) O1 + O2 (warps 4-5) --------------------
    {
      float o2[16];
      tmem_ld16(tb + tlane + TM_O2 + 16 * hw, o2);
      tmem_wait_ld();
      if (lane < 16) {
        const int t = 16 * q4 + lane;
#pragma unroll
        for (int x = 0; x < 16; ++x) Ox[t * 32 + ((16 * hw + x) ^ (t & 31))] = o2[x];
      }
      if (tid < kDK) {
        tmem_ld32(tb + tlane + TM_S, st);
        tmem_wait_ld();
#pragma unroll
        for (int vv = 0; vv < kDVS; ++vv) st_tile(tSS, kDVS, vv, tid, st[vv]);
      }
    }
    __syncthreads();
    if (hw == 1 && q4 < 2) {
      const int t = 32 * q4 + lane;
      float o1[32];
      tmem_ld32(tb + tlane + TM_OY, o1);
      float o2[32];
#pragma unroll
      for (int x = 0; x < 32; ++x) o2[x] = Ox[t * 32 + (x ^ (t & 31))];
      tmem_wait_ld();
      if (t < L) {
        const float eg = ss.eg[t];
        Tout* dst = o + (((long)b * T + t0 + t) * H + h) * (long)dv + v0;
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
    fence_smem_to_async();
    fence_before_sync();
    __syncthreads();
  }
  if (!aborted && s_final && tid < kDK) {
#pragma unroll
    for (int vv = 0; vv < kDVS; ++vv) s_final[sbase + (long)(v0 + vv) * kDK + tid] = st[vv];
  }
  if (tma_inflight) {
    // only after an abort: let the prefetch land before the CTA's memory goes away
    const bool ok = mbar_wait(tma_bar, tphase, kDrainLimit);
    if (!ok && lane == 0) atomicOr(status, 2u);
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
  CUtensorMap mq, mk, mv;
  if (!encode_bthd_bf16(&mq, a.q, a.B, a.T, a.H, kDK, kDK, kC) ||
      !encode_bthd_bf16(&mk, a.k, a.B, a.T, a.H, kDK, kDK, kC) ||
      !encode_bthd_bf16(&mv, a.v, a.B, a.T, a.H, a.dv, kDVS, kC))
    return cudaErrorInvalidValue;
  auto kern = gdn_prefill_tc_kernel<Tout>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int grid = a.B * a.H * (a.dv / kDVS);
  kern<<<grid, kThreads, SMEM_BYTES, st>>>(mq, mk, mv, a.alpha, a.beta, a.s0, (Tout*)a.o,
                                           a.s_final, a.T, a.H, a.dv, (unsigned int*)a.workspace,
                                           spin_limit_from_env());
  e = cudaGetLastError();
  if (e == cudaSuccess) timing_mark(st, 0);
  return e;
}

}  // namespace

// Both mixers take the tensor-core path for bf16 inputs with d_k = 128 and d_v a
// multiple of 32; the rest runs on the CUDA cores.
bool tc_prefill_supported(const PrefillArgs& a) {
  return a.in_dtype == GDR_BF16 && a.dk == kDK && a.dv % kDVS == 0;
}

cudaError_t launch_prefill_kda_tc(const PrefillArgs& a, cudaStream_t stream);  // prefill_kda_tc.cu

// The two-kernel paths (per-chunk prep over the whole GPU, then the carry) need a
// workspace of 128.5 KB per chunk; with a smaller workspace the single-kernel kernels
// run.
size_t tc_prefill_workspace(int B, int T, int H, int dk, int dv, bool kda) {
  PrefillArgs a{};
  a.in_dtype = GDR_BF16;
  a.dk = dk;
  a.dv = dv;
  a.kda = kda;
  if (!tc_prefill_supported(a)) return 0;
  return kda ? kda_split_workspace(B, T, H) : split_prefill_workspace(B, T, H);
}

cudaError_t launch_prefill_tc(const PrefillArgs& a, cudaStream_t st) {
  const bool split = a.ws_bytes >= 256 + (a.kda ? kda_split_workspace(a.B, a.T, a.H)
                                                : split_prefill_workspace(a.B, a.T, a.H));
  if (split) {
    // dense batch: chunk gc of head h is chunk gc % nchunks of sequence gc / nchunks
    ChunkMap m{};
    m.nseq = a.B;
    m.T = a.T;
    m.nchunks = (a.T + GDR_CHUNK - 1) / GDR_CHUNK;
    m.nck = a.B * m.nchunks;
    m.img_base = 256;
    m.checks = checks_word();
    return a.kda ? launch_prefill_kda_split(a, m, st) : launch_prefill_split(a, m, st);
  }
  if (a.kda) return launch_prefill_kda_tc(a, st);
  if (a.out_dtype == GDR_F32) return launch_t<float>(a, st);
  return launch_t<__nv_bfloat16>(a, st);
}

}  // namespace gdr
