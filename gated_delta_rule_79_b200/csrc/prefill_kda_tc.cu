// Chunked prefill of Kimi Delta Attention on the sm_100a tensor cores (tcgen05 + TMA).
//
// "Super Apriel: One Checkpoint, Many Speeds", §2A names the KDA mixer: the delta
// rule with a channel-wise gate.  For a chunk of C = 64 tokens entering with state
// S0 and the chunk-local cumulative log gate G[t][c] = sum_{s<=t} log alpha_s[c]:
//
//   A[t,j] = beta_t sum_c k_tc k_jc e^{G_tc - G_jc}  (j < t)
//   P[t,j] =        sum_c q_tc k_jc e^{G_tc - G_jc}  (j <= t)
//   T = (I + A)^{-1} Diag(beta)
//   Y~ = (K (.) e^G) S0^T,  R = V - Y~,  U = T R
//   O = (Q (.) e^G) S0^T + P U
//   S^T <- Diag(e^{G_last}) S0^T + (K (.) e^{G_last - G})^T U
//
// The per-channel decay sits inside the Gram's contraction.  With a per-channel
// reference Gm_c halfway between the chunk's first and last G, it factors as
//   e^{G_tc - G_jc} = e^{G_tc - Gm_c} e^{Gm_c - G_jc},
// so the decayed Gram is one tensor-core product of L = [Q; K] (.) e^{G - Gm} and
// R = K (.) e^{Gm - G}: every factor lies in [e^{-span/2}, e^{span/2}] with span the
// channel's log-gate drop over the chunk.  While span <= 168 the factors stay normal
// fp32 numbers (|exponent| <= 84) and every product needed (t >= j) is at most 1;
// the masked products (t < j) may overflow, and are never read.  A channel whose
// span exceeds that (gates near zero) is left out of the product, and its terms are
// summed exactly on the CUDA cores.
//
// Everything else follows the GDN tensor-core kernel: one CTA (256 threads) per
// (batch, head, 32-wide slice of d_v) walks the chunks in order; products run as
// kind::tf32 with operands rounded to nearest; the state slice S^T lives in tensor
// memory and in registers; the next chunk's q, k, v and gates arrive by TMA while
// the current one is worked on.  Waits are bounded as in the GDN kernel.

#include <math.h>
#include <stdlib.h>

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
constexpr float kMaxSpan = 168.f;

// shared-memory map (bytes from a 1024-aligned base)
constexpr int OFF_QK = 0;                  // gates alpha [64 t][128 c] (TMA) -> L -> [Q~; K~]  64 KB
constexpr int OFF_KT = OFF_QK + 65536;     // R [64 j][128 c] -> K^ transposed [128 c][64 j]    32 KB
constexpr int OFF_P = OFF_KT + 32768;      // fp32 [64 t][64 j]                                 16 KB
constexpr int OFF_TM = OFF_P + 16384;      // T [64][64]; X scratch in the solve                16 KB
constexpr int OFF_RT = OFF_TM + 16384;     // R operand [32 v][64 j]; A scratch (16 KB over RT+UT)
constexpr int OFF_UT = OFF_RT + 8192;      //   in the solve; P U exchange [64][32] at the end
constexpr int OFF_SS = OFF_UT + 8192;      // fp32 [32 v][128 c] state operand                  16 KB
constexpr int OFF_STG = OFF_SS + 16384;    // bf16 TMA staging: q, k [64][128], v [64][32]
constexpr int STG_Q = 0, STG_K = 16384, STG_V = 32768;
constexpr int OFF_Z = OFF_STG + 36864;     // level scratch [3][16][16]                          3 KB
constexpr int OFF_SMALL = OFF_Z + 3072;
constexpr int SMEM_USED = OFF_SMALL + 2048;
constexpr int SMEM_BYTES = SMEM_USED + 1024;
constexpr uint32_t TMA_BYTES = 16384 + 16384 + 4096 + 32768;
static_assert(SMEM_BYTES <= 232448, "shared memory");

// tensor-memory columns
constexpr uint32_t TM_G = 0;     // Gram, M=128 x 64
constexpr uint32_t TM_OY = 64;   // [Q~; K~] S0^T, M=128 x 32
constexpr uint32_t TM_U = 96;    // U, M=64 x 32
constexpr uint32_t TM_O2 = 128;  // P U, M=64 x 32
constexpr uint32_t TM_S = 160;   // S^T, M=128 x 32
constexpr uint32_t TM_GS = 192;  // G kept by channel: lane c, columns t (64)
constexpr uint32_t TM_COLS = 256;

constexpr uint32_t kDrainLimit = 1u << 26;

struct SmallSmem {
  float beta[kC];
  float gm[kDK];      // per-channel Gram reference (midpoint of the chunk's G)
  float glast[kDK];   // per-channel G of the chunk's last token
  unsigned wmask[4];  // channels whose log gate drops by more than kMaxSpan in the chunk
  uint32_t tmem;
  unsigned long long mma_bar;
  unsigned long long tma_bar;
};

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
__device__ __forceinline__ int sx(int r, int c) { return r * 64 + (c ^ (r & 31)); }
__device__ __forceinline__ void ld4_sx(const float* base, int k, int klo, int c4, float (&e)[4]) {
  const float4 f = *reinterpret_cast<const float4*>(base + k * 64 + (c4 ^ (k & 28)));
  const float v[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
  for (int x = 0; x < 4; ++x) e[x] = v[x ^ klo];
}

template <typename Tout>
__global__ void __launch_bounds__(kThreads, 1)
kda_prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_a, const float* __restrict__ beta,
                      const float* __restrict__ s0, Tout* __restrict__ o,
                      float* __restrict__ s_final, int T, int H, int dv,
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
  unsigned char* tSS = sm + OFF_SS;
  unsigned char* stg = sm + OFF_STG;
  const float* agate = reinterpret_cast<const float*>(tQK);   // [64 t][128 c] after TMA
  float* Gw = reinterpret_cast<float*>(tKT);                  // [64 t][128 c] G, wide chunks
  float* Xs = reinterpret_cast<float*>(tTM);
  float* As = reinterpret_cast<float*>(tRT);
  float* Zs = reinterpret_cast<float*>(sm + OFF_Z);
  float* Ox = reinterpret_cast<float*>(tRT);
  SmallSmem& ss = *reinterpret_cast<SmallSmem*>(sm + OFF_SMALL);
  uint64_t* mma_bar = reinterpret_cast<uint64_t*>(&ss.mma_bar);
  uint64_t* tma_bar = reinterpret_cast<uint64_t*>(&ss.tma_bar);
  const __nv_bfloat16* qst = reinterpret_cast<const __nv_bfloat16*>(stg + STG_Q);
  const __nv_bfloat16* kst = reinterpret_cast<const __nv_bfloat16*>(stg + STG_K);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q4 = warp & 3, hw = warp >> 2;
  const int nslice = dv / kDVS;
  const int slice = blockIdx.x % nslice;
  const int bh = blockIdx.x / nslice;
  const int h = bh % H, b = bh / H;
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
    mbar_expect_tx(tma_bar, TMA_BYTES);
    const uint32_t s = smem_u32(stg);
    tma_load_4d(s + STG_Q, &tm_q, 0, h, t0, b, tma_bar);
    tma_load_4d(s + STG_K, &tm_k, 0, h, t0, b, tma_bar);
    tma_load_4d(s + STG_V, &tm_v, v0, h, t0, b, tma_bar);
    tma_load_4d(smem_u32(tQK), &tm_a, 0, h, t0, b, tma_bar);
  };
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
  float b_next = 0.f;
  if (tid < kC && tid < T) b_next = beta[((long)b * T + tid) * H + h];

  const uint32_t aQK = smem_u32(tQK), aKT = smem_u32(tKT), aP = smem_u32(tP), aTM = smem_u32(tTM);
  const uint32_t aRT = smem_u32(tRT), aUT = smem_u32(tUT), aSS = smem_u32(tSS);
  const uint64_t dQK = sdesc(aQK, 16, 1024), dKT = sdesc(aKT, 16, 1024);
  const uint64_t dP = sdesc(aP, 16, 1024), dTM = sdesc(aTM, 16, 1024);
  const uint64_t dRT = sdesc(aRT, 16, 1024), dUT = sdesc(aUT, 16, 1024), dSS = sdesc(aSS, 16, 1024);

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
    // ---- 1. chunk c has landed ----------------------------------------------------------
    aborted = wait_bar(tma_bar, tphase);
    tma_inflight = false;
    if (aborted) break;
    if (tid < kC) ss.beta[tid] = b_next;
    // ---- 2. per-channel cumulative log gate (thread c owns channel c) ----------------------
    float egc = 1.f;
    if (tid < kDK) {
      float g0[32], g1[32];
#pragma unroll
      for (int t = 0; t < 32; ++t) g0[t] = agate[t * kDK + tid];
#pragma unroll
      for (int t = 0; t < 32; ++t) g1[t] = agate[(32 + t) * kDK + tid];
      double acc = 0.0;
#pragma unroll
      for (int t = 0; t < 32; ++t) {
        acc += (t < L) ? (double)log_gate_accurate(g0[t]) : 0.0;
        g0[t] = (float)acc;
      }
#pragma unroll
      for (int t = 0; t < 32; ++t) {
        acc += (32 + t < L) ? (double)log_gate_accurate(g1[t]) : 0.0;
        g1[t] = (float)acc;
      }
      const float glast = (float)acc;
      ss.gm[tid] = 0.5f * (g0[0] + glast);
      ss.glast[tid] = glast;
      egc = __expf(glast);
      const unsigned wm = __ballot_sync(0xffffffffu, (g0[0] - glast) > kMaxSpan);
      if (lane == 0) ss.wmask[warp] = wm;
      tmem_st32(tb + tlane + TM_GS, g0);
      tmem_st32(tb + tlane + TM_GS + 32, g1);
      tmem_wait_st();
    }
    fence_before_sync();
    __syncthreads();   // also: every gate read from the staging area is done
    fence_after_sync();
    const bool anywide = (ss.wmask[0] | ss.wmask[1] | ss.wmask[2] | ss.wmask[3]) != 0u;
    // ---- 3. Gram factors L = [Q; K] (.) e^{G - Gm}, R = K (.) e^{Gm - G} ---------------------
    //         (thread: channel 32 q4 + lane, tokens 32 hw .. 32 hw + 31); a wide channel's
    //         columns are zero here and its terms are added exactly in step 5
    {
      float g[32];
      tmem_ld32(tb + tlane + TM_GS + 32 * hw, g);
      tmem_wait_ld();
      const int cc = 32 * q4 + lane;
      const float gm = ss.gm[cc];
      const bool wc = (ss.wmask[q4] >> lane) & 1u;
#pragma unroll
      for (int x = 0; x < 32; ++x) {
        const int t = 32 * hw + x;
        const float e = wc ? 0.f : __expf(g[x] - gm);
        const float ei = wc ? 0.f : __expf(gm - g[x]);
        const float qv = __bfloat162float(qst[t * kDK + cc]);
        const float kv = __bfloat162float(kst[t * kDK + cc]);
        st_tile(tQK, 128, t, cc, qv * e);
        st_tile(tQK, 128, 64 + t, cc, kv * e);
        st_tile(tKT, 64, t, cc, kv * ei);
      }
    }
    fence_smem_to_async();
    fence_before_sync();
    __syncthreads();
    // ---- 4. decayed Gram on the tensor cores; meanwhile decay the state ----------------------
    if (tid == 0) {
      fence_after_sync();
      mma_chain(tb + TM_G, dQK, 128, dKT, 64, kDK / 8, idesc_tf32(128, 64, false, false), false);
      mma_commit(mma_bar);
    }
    if (tid < kDK) {
      float sd[kDVS];
#pragma unroll
      for (int vv = 0; vv < kDVS; ++vv) sd[vv] = st[vv] * egc;
      tmem_st32(tb + tlane + TM_S, sd);
      tmem_wait_st();
    }
    if ((aborted = wait_bar(mma_bar, mphase))) break;
    if (anywide) {
      // G as [64 t][128 c] fp32 in the (now free) R area, for the exact terms
      float g[32];
      tmem_ld32(tb + tlane + TM_GS + 32 * hw, g);
      tmem_wait_ld();
#pragma unroll
      for (int x = 0; x < 32; ++x) Gw[(32 * hw + x) * kDK + 32 * q4 + lane] = g[x];
      __syncthreads();
    }
    // ---- 5. P (lower) and A (beta, strictly lower) --------------------------------------------
    {
      float d[32];
      tmem_ld32(tb + tlane + TM_G + 32 * hw, d);
      const int r = 32 * q4 + lane;
      const int t = r & 63;
      const float bt = ss.beta[t];
      tmem_wait_ld();
      if (anywide) {
        const __nv_bfloat16* xs = r < 64 ? qst : kst;
#pragma unroll 1
        for (int w = 0; w < 4; ++w) {
          unsigned m = ss.wmask[w];
          while (m) {
            const int cc = 32 * w + __ffs(m) - 1;
            m &= m - 1;
            const float xv = __bfloat162float(xs[t * kDK + cc]);
            const float gt = Gw[t * kDK + cc];
#pragma unroll
            for (int x = 0; x < 32; ++x) {
              const int j = 32 * hw + x;
              const float term =
                  xv * __bfloat162float(kst[j * kDK + cc]) * __expf(gt - Gw[j * kDK + cc]);
              d[x] += j <= t ? term : 0.f;
            }
          }
        }
      }
      if (r < 64) {
#pragma unroll
        for (int x = 0; x < 32; ++x) d[x] = (32 * hw + x) <= t ? d[x] : 0.f;
#pragma unroll
        for (int x = 0; x < 8; ++x)
          st_tile4(tP, 64, t, 8 * hw + x, make_float4(d[4 * x], d[4 * x + 1], d[4 * x + 2], d[4 * x + 3]));
      } else {
#pragma unroll
        for (int x = 0; x < 32; ++x) d[x] = (32 * hw + x) < t ? bt * d[x] : 0.f;
#pragma unroll
        for (int x = 0; x < 32; ++x) As[sx(t, 32 * hw + x)] = d[x];
      }
    }
    __syncthreads();
    // ---- 6. X = (I + A)^{-1}, then T = X Diag(beta) ----------------------------------------------
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
    {
      const int r = tid & 63, qq = tid >> 6;
      float xr[16];
#pragma unroll
      for (int x = 0; x < 16; ++x) {
        const int j = qq * 16 + x;
        xr[x] = (qq <= (r >> 4)) ? Xs[sx(r, j)] * ss.beta[j] : 0.f;
      }
      __syncthreads();
#pragma unroll
      for (int x = 0; x < 4; ++x)
        st_tile4(tTM, 64, r, qq * 4 + x,
                 make_float4(xr[4 * x], xr[4 * x + 1], xr[4 * x + 2], xr[4 * x + 3]));
    }
    // ---- 7. carry operands: [Q (.) e^G; K (.) e^G] and (K (.) e^{G_last - G})^T --------------
    {
      float g[32];
      tmem_ld32(tb + tlane + TM_GS + 32 * hw, g);
      const int cc = 32 * q4 + lane;
      const float glast = ss.glast[cc];
      tmem_wait_ld();
      float kh[32];
#pragma unroll
      for (int x = 0; x < 32; ++x) {
        const int t = 32 * hw + x;
        const float e = __expf(g[x]);
        const float qv = __bfloat162float(qst[t * kDK + cc]);
        const float kv = __bfloat162float(kst[t * kDK + cc]);
        st_tile(tQK, 128, t, cc, qv * e);
        st_tile(tQK, 128, 64 + t, cc, kv * e);
        kh[x] = t < L ? kv * __expf(fminf(glast - g[x], 0.f)) : 0.f;
      }
#pragma unroll
      for (int x = 0; x < 8; ++x)
        st_tile4(tKT, 128, cc, 8 * hw + x, make_float4(kh[4 * x], kh[4 * x + 1], kh[4 * x + 2], kh[4 * x + 3]));
    }
    fence_smem_to_async();
    fence_before_sync();
    __syncthreads();
    // ---- 8. [O1; Y~] = [Q~; K~] S0^T -------------------------------------------------------------
    if (tid == 0) {
      fence_after_sync();
      mma_chain(tb + TM_OY, dQK, 128, dSS, kDVS, kDK / 8, idesc_tf32(128, 32, false, false), false);
      mma_commit(mma_bar);
    }
    if ((aborted = wait_bar(mma_bar, mphase))) break;
    // ---- 9. R = V - Y~ as the operand [v][j]; then the next chunk's loads -------------------------
    if (hw == 0 && q4 >= 2) {
      const int j = 32 * (q4 - 2) + lane;
      float y[32], vv[32];
      const uint4* vrow = reinterpret_cast<const uint4*>(stg + STG_V + j * 64);
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
      tmem_ld32(tb + tlane + TM_OY, y);
      tmem_wait_ld();
#pragma unroll
      for (int v = 0; v < kDVS; ++v) st_tile(tRT, kDVS, v, j, vv[v] - y[v]);
    }
    fence_smem_to_async();
    fence_before_sync();
    __syncthreads();
    if (c + 1 < nchunks) {
      // staging and the gate area are free: q/k/v were last read above, the [Q~; K~]
      // tile by the product that has completed
      if (tid == 0) issue_tma(t0 + kC);
      tma_inflight = true;
      b_next = 0.f;
      if (tid < kC && t0 + kC + tid < T) b_next = beta[((long)b * T + t0 + kC + tid) * H + h];
    }
    // ---- 10. U = T R -------------------------------------------------------------------------------
    if (tid == 0) {
      fence_after_sync();
      mma_chain(tb + TM_U, dTM, 64, dRT, kDVS, kC / 8, idesc_tf32(64, 32, false, false), false);
      mma_commit(mma_bar);
    }
    if ((aborted = wait_bar(mma_bar, mphase))) break;
    {
      float u[16];
      tmem_ld16(tb + tlane + TM_U + 16 * hw, u);
      tmem_wait_ld();
      if (lane < 16) {
        const int j = 16 * q4 + lane;
#pragma unroll
        for (int x = 0; x < 16; ++x) st_tile(tUT, kDVS, 16 * hw + x, j, u[x]);
      }
    }
    fence_smem_to_async();
    fence_before_sync();
    __syncthreads();
    // ---- 11. O2 = P U;  S^T += K^T U ------------------------------------------------------------------
    if (tid == 0) {
      fence_after_sync();
      mma_chain(tb + TM_O2, dP, 64, dUT, kDVS, kC / 8, idesc_tf32(64, 32, false, false), false);
      mma_chain(tb + TM_S, dKT, 128, dUT, kDVS, kC / 8, idesc_tf32(128, 32, false, false), true);
      mma_commit(mma_bar);
    }
    if ((aborted = wait_bar(mma_bar, mphase))) break;
    // ---- 12. new state (warps 0-3) and outputs O = O1 + O2 (warps 4-5) ----------------------------------
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
      float o1[32], o2[32];
      tmem_ld32(tb + tlane + TM_OY, o1);
#pragma unroll
      for (int x = 0; x < 32; ++x) o2[x] = Ox[t * 32 + (x ^ (t & 31))];
      tmem_wait_ld();
      if (t < L) {
        Tout* dst = o + (((long)b * T + t0 + t) * H + h) * (long)dv + v0;
        if constexpr (sizeof(Tout) == 2) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 pk;
            __nv_bfloat162* hp = reinterpret_cast<__nv_bfloat162*>(&pk);
#pragma unroll
            for (int x = 0; x < 4; ++x)
              hp[x] = __floats2bfloat162_rn(o1[8 * q + 2 * x] + o2[8 * q + 2 * x],
                                            o1[8 * q + 2 * x + 1] + o2[8 * q + 2 * x + 1]);
            reinterpret_cast<uint4*>(dst)[q] = pk;
          }
        } else {
#pragma unroll
          for (int q = 0; q < 8; ++q)
            reinterpret_cast<float4*>(dst)[q] =
                make_float4(o1[4 * q] + o2[4 * q], o1[4 * q + 1] + o2[4 * q + 1],
                            o1[4 * q + 2] + o2[4 * q + 2], o1[4 * q + 3] + o2[4 * q + 3]);
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
    const bool ok = mbar_wait(tma_bar, tphase, kDrainLimit);
    if (!ok && lane == 0) atomicOr(status, 2u);
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tb, TM_COLS);
}

uint32_t kda_spin_limit() {
  const char* e = getenv("GDR_SPIN_LIMIT");
  if (!e || !*e) return 1u << 24;
  return (uint32_t)strtoul(e, nullptr, 10);
}

template <typename Tout>
cudaError_t launch_kda_t(const PrefillArgs& a, cudaStream_t st) {
  CUtensorMap mq, mk, mv, ma;
  if (!encode_bthd_bf16(&mq, a.q, a.B, a.T, a.H, kDK, kDK, kC) ||
      !encode_bthd_bf16(&mk, a.k, a.B, a.T, a.H, kDK, kDK, kC) ||
      !encode_bthd_bf16(&mv, a.v, a.B, a.T, a.H, a.dv, kDVS, kC) ||
      !encode_bthd_f32(&ma, a.alpha, a.B, a.T, a.H, kDK, kDK, kC))
    return cudaErrorInvalidValue;
  auto kern = kda_prefill_tc_kernel<Tout>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  kern<<<a.B * a.H * (a.dv / kDVS), kThreads, SMEM_BYTES, st>>>(
      mq, mk, mv, ma, a.beta, a.s0, (Tout*)a.o, a.s_final, a.T, a.H, a.dv,
      (unsigned int*)a.workspace, kda_spin_limit());
  e = cudaGetLastError();
  if (e == cudaSuccess) timing_mark(st, 0);
  return e;
}

}  // namespace

cudaError_t launch_prefill_kda_tc(const PrefillArgs& a, cudaStream_t st) {
  if (a.out_dtype == GDR_F32) return launch_kda_t<float>(a, st);
  return launch_kda_t<__nv_bfloat16>(a, st);
}

}  // namespace gdr
