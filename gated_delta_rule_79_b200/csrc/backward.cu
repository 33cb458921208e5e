// Gradients of the GDN / KDA mixers (sm_100a): dq, dk, dv, dalpha, dbeta and ds0 for
// a dense batch, given dL/do and optionally dL/dS_T.
//
// "Super Apriel: One Checkpoint, Many Speeds", §2B (Training Recipe): the mixers are
// trained by stochastic distillation and supervised fine-tuning, which back-propagate
// through the recurrence of §2A,
//
//   S~ = S_{t-1} Diag(alpha_t),  r_t = v_t - S~ k_t,  u_t = beta_t r_t,
//   S_t = S~ + u_t k_t^T,        o_t = S_t q_t.
//
// Its reverse, token t (dS = dL/dS_t from token t + 1):
//
//   dS += do_t q_t^T;  dq_t = S_t^T do_t;  du = dS k_t;  dk_t = dS^T u_t - beta_t S~^T du
//   dv_t = beta_t du;  dbeta_t = du . r_t;  dS~ = dS - beta_t du k_t^T
//   dalpha_t[c] = sum_r S_{t-1}[r, c] dS~[r, c];  dS <- dS~ Diag(alpha_t)
//
// Every row r of S (a value channel) evolves on its own, forward and in reverse; only
// dq, dk, dalpha and dbeta sum over rows.  So one warp owns one value row (each lane
// d_k / 32 key channels), a CTA owns 16 rows, and the d_v / 16 CTAs of one (sequence,
// head) form a thread-block cluster that sums the per-row terms through distributed
// shared memory.
//
// Pass 1 runs the recurrence forward and leaves, in the workspace, the state entering
// every chunk of 64 tokens and u_t, r_t of every token.  Pass 2 walks the chunks in
// reverse: from the chunk's entering state it rebuilds the states (no reductions: u_t is
// known) at every eighth token, then in blocks of eight tokens (their states in
// registers) runs the reverse steps.  The per-row terms of a token are summed over the
// CTA's warps in shared memory, and those of each block of eight tokens over the
// cluster's CTAs, which write the results.  Everything is fp32; there is no wait on
// another CTA other than the cluster barrier, which every CTA of a cluster reaches the
// same number of times.

#include <stdio.h>
#include <stdint.h>

#include "common.cuh"
#include "gdr.h"
#include "launch.h"

namespace gdr {
namespace {

constexpr int kC = GDR_CHUNK;
constexpr int BW_ROWS = 16;            // value rows per CTA, one per warp
constexpr int BW_THREADS = 32 * BW_ROWS;
constexpr int BW_BLOCK = 8;            // tokens per reverse block (states in registers)

template <int DK, bool KDA>
struct BwCfg {
  static constexpr int NC = DK / 32;                    // key channels per lane
  static constexpr int NQ = KDA ? 3 * DK + 1 : 2 * DK + 2;   // per-token sums
  // dq at [0, DK), dk at [DK, 2 DK), dalpha at [2 DK, 2 DK + (KDA ? DK : 1)), dbeta last
  static constexpr int NA = KDA ? DK : 1;
};

template <int DK, bool KDA, typename Tin>
struct BwSmem {
  static constexpr int NQ = BwCfg<DK, KDA>::NQ;
  Tin k[kC][DK];
  Tin q[kC][DK];
  float alpha[kC][BwCfg<DK, KDA>::NA];
  float beta[kC];
  float v[kC][BW_ROWS];
  float dO[kC][BW_ROWS];
  float u[kC][BW_ROWS];
  float res[kC][BW_ROWS];
  float scratch[2][BW_ROWS][NQ];                // per-warp terms, by token parity
  float part[2][BW_BLOCK][NQ];                  // the CTA's terms, by block parity
};

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
               "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// fp32 at the same shared-memory offset in CTA `rank` of the cluster
__device__ __forceinline__ float ld_cluster(const float* local, uint32_t rank) {
  uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(local)), ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
  float x;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(x) : "r"(ra) : "memory");
  return x;
}

template <int DK, bool KDA, typename Tin, typename Tdo>
__global__ void __launch_bounds__(BW_THREADS, 1)
gdr_backward_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                    const Tin* __restrict__ v, const float* __restrict__ alpha,
                    const float* __restrict__ beta, const float* __restrict__ s0,
                    const Tdo* __restrict__ dO, const float* __restrict__ ds_final,
                    float* __restrict__ dq, float* __restrict__ dk, float* __restrict__ dv,
                    float* __restrict__ dalpha, float* __restrict__ dbeta,
                    float* __restrict__ ds0, int T, int H, int DV, float* __restrict__ ws) {
  using Cfg = BwCfg<DK, KDA>;
  constexpr int NC = Cfg::NC, NQ = Cfg::NQ, NA = Cfg::NA;
  using Sm = BwSmem<DK, KDA, Tin>;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Sm& sm = *reinterpret_cast<Sm*>(smem_raw);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ncl = DV / BW_ROWS;                   // CTAs per (sequence, head)
  const int rb = blockIdx.x % ncl;
  const int bh = blockIdx.x / ncl;
  const int h = bh % H, b = bh / H;
  const uint32_t crank = cluster_rank();          // == rb: clusters are ncl consecutive CTAs
  const int r = rb * BW_ROWS + warp;              // this warp's value row
  const int nchunks = (T + kC - 1) / kC;
  // workspace of this CTA: entering states [nchunks][16][DK], then u, r [nchunks][2][64][16]
  float* ckpt = ws + (size_t)blockIdx.x * ((size_t)nchunks * BW_ROWS * (DK + 2 * kC));
  float* ures = ckpt + (size_t)nchunks * BW_ROWS * DK;
  const long row_stride = (long)H;                // tokens: ((b T + t) H + h) * width

  // ---- chunk inputs into shared memory (tokens past T: k = q = 0, alpha = 1, beta = 0) ---
  auto load_chunk = [&](int c, bool reverse_pass) {
    const int t0 = c * kC;
    const int L = min(kC, T - t0);
    constexpr int VEC = 16 / sizeof(Tin);         // elements per 16-byte piece
    constexpr int PR = DK / VEC;                  // pieces per token row
    for (int i = tid; i < kC * PR; i += BW_THREADS) {
      const int t = i / PR, p = i - t * PR;
      uint4 x = make_uint4(0, 0, 0, 0), y = make_uint4(0, 0, 0, 0);
      if (t < L) {
        const long off = (((long)b * T + t0 + t) * row_stride + h) * DK + p * VEC;
        x = *reinterpret_cast<const uint4*>(k + off);
        if (reverse_pass) y = *reinterpret_cast<const uint4*>(q + off);
      }
      *reinterpret_cast<uint4*>(&sm.k[t][p * VEC]) = x;
      if (reverse_pass) *reinterpret_cast<uint4*>(&sm.q[t][p * VEC]) = y;
    }
    for (int i = tid; i < kC * NA; i += BW_THREADS) {
      const int t = i / NA, cc = i - t * NA;
      float a = 1.f;
      if (t < L) a = alpha[(((long)b * T + t0 + t) * row_stride + h) * NA + cc];
      sm.alpha[t][cc] = a;
    }
    for (int i = tid; i < kC * BW_ROWS; i += BW_THREADS) {
      const int t = i / BW_ROWS, rr = i - t * BW_ROWS;
      float x = 0.f, y = 0.f;
      if (t < L) {
        const long off = (((long)b * T + t0 + t) * row_stride + h) * DV + rb * BW_ROWS + rr;
        x = Elem<Tin>::load(v + off);
        if (reverse_pass) y = Elem<Tdo>::load(dO + off);
      }
      sm.v[t][rr] = x;
      if (reverse_pass) {
        sm.dO[t][rr] = y;
        sm.u[t][rr] = t < L ? ures[((size_t)c * 2 + 0) * kC * BW_ROWS + i] : 0.f;
        sm.res[t][rr] = t < L ? ures[((size_t)c * 2 + 1) * kC * BW_ROWS + i] : 0.f;
      }
    }
    if (tid < kC) sm.beta[tid] = tid < L ? beta[((long)b * T + t0 + tid) * row_stride + h] : 0.f;
  };
  auto ld_k = [&](int t, float (&x)[NC]) {
#pragma unroll
    for (int j = 0; j < NC; ++j) x[j] = Elem<Tin>::load(&sm.k[t][lane + 32 * j]);
  };
  auto ld_q = [&](int t, float (&x)[NC]) {
#pragma unroll
    for (int j = 0; j < NC; ++j) x[j] = Elem<Tin>::load(&sm.q[t][lane + 32 * j]);
  };
  auto ld_a = [&](int t, float (&x)[NC]) {
#pragma unroll
    for (int j = 0; j < NC; ++j) x[j] = KDA ? sm.alpha[t][(lane + 32 * j) % NA] : sm.alpha[t][0];
  };

  // =============================== pass 1: forward ======================================
  float S[NC];
  {
    const long srow = (((long)b * H + h) * DV + r) * DK;
#pragma unroll
    for (int j = 0; j < NC; ++j) S[j] = s0 ? s0[srow + lane + 32 * j] : 0.f;
  }
  for (int c = 0; c < nchunks; ++c) {
    const int L = min(kC, T - c * kC);
#pragma unroll
    for (int j = 0; j < NC; ++j) ckpt[((size_t)c * BW_ROWS + warp) * DK + lane + 32 * j] = S[j];
    __syncthreads();                              // the previous chunk's inputs are read
    load_chunk(c, false);
    __syncthreads();
    for (int t = 0; t < L; ++t) {
      float kk[NC], aa[NC], a = 0.f;
      ld_k(t, kk);
      ld_a(t, aa);
#pragma unroll
      for (int j = 0; j < NC; ++j) {
        S[j] *= aa[j];
        a = fmaf(S[j], kk[j], a);
      }
      a = warp_sum(a);
      const float rr = sm.v[t][warp] - a, uu = sm.beta[t] * rr;
#pragma unroll
      for (int j = 0; j < NC; ++j) S[j] = fmaf(uu, kk[j], S[j]);
      if (lane == 0) {
        ures[((size_t)c * 2 + 0) * kC * BW_ROWS + t * BW_ROWS + warp] = uu;
        ures[((size_t)c * 2 + 1) * kC * BW_ROWS + t * BW_ROWS + warp] = rr;
      }
    }
  }
  __syncthreads();
  __threadfence_block();

  // =============================== pass 2: reverse ======================================
  float dS[NC];
  {
    const long srow = (((long)b * H + h) * DV + r) * DK;
#pragma unroll
    for (int j = 0; j < NC; ++j) dS[j] = ds_final ? ds_final[srow + lane + 32 * j] : 0.f;
  }
  int sp = 0, pb = 0;                             // token parity (scratch), block parity (part)
  float sub[kC / BW_BLOCK][NC];                   // the state before every eighth token
  for (int c = nchunks - 1; c >= 0; --c) {
    const int t0 = c * kC;
    const int L = min(kC, T - t0);
    __syncthreads();
    load_chunk(c, true);
    __syncthreads();
    {
      float Sx[NC];
#pragma unroll
      for (int j = 0; j < NC; ++j) Sx[j] = ckpt[((size_t)c * BW_ROWS + warp) * DK + lane + 32 * j];
      for (int s = 0; s < kC / BW_BLOCK; ++s) {
#pragma unroll
        for (int j = 0; j < NC; ++j) sub[s][j] = Sx[j];
        for (int t = s * BW_BLOCK; t < min(L, (s + 1) * BW_BLOCK); ++t) {
          float kk[NC], aa[NC];
          ld_k(t, kk);
          ld_a(t, aa);
          const float uu = sm.u[t][warp];
#pragma unroll
          for (int j = 0; j < NC; ++j) Sx[j] = fmaf(uu, kk[j], Sx[j] * aa[j]);
        }
      }
    }
    const int nblk = (L + BW_BLOCK - 1) / BW_BLOCK;
    for (int s = nblk - 1; s >= 0; --s) {
      const int tb = s * BW_BLOCK;
      // states before tokens tb .. tb + 7
      float blk[BW_BLOCK][NC];
#pragma unroll
      for (int j = 0; j < NC; ++j) blk[0][j] = sub[s][j];
#pragma unroll
      for (int i = 1; i < BW_BLOCK; ++i) {
        const int t = tb + i - 1;
        float kk[NC], aa[NC];
        ld_k(t, kk);
        ld_a(t, aa);
        const float uu = sm.u[t][warp];
#pragma unroll
        for (int j = 0; j < NC; ++j) blk[i][j] = fmaf(uu, kk[j], blk[i - 1][j] * aa[j]);
      }
#pragma unroll
      for (int ii = 0; ii < BW_BLOCK; ++ii) {
        const int i = BW_BLOCK - 1 - ii;
        const int t = tb + i;
        if (t >= L) continue;                     // uniform over the CTA
        float kk[NC], qq[NC], aa[NC];
        ld_k(t, kk);
        ld_q(t, qq);
        ld_a(t, aa);
        const float uu = sm.u[t][warp], rr = sm.res[t][warp], bt = sm.beta[t];
        const float od = sm.dO[t][warp];
        float Sd[NC], du = 0.f;
#pragma unroll
        for (int j = 0; j < NC; ++j) {
          Sd[j] = blk[i][j] * aa[j];                   // S~
          dS[j] = fmaf(od, qq[j], dS[j]);              // + do q^T
          du = fmaf(dS[j], kk[j], du);
        }
        du = warp_sum(du);
        float* sc = sm.scratch[sp][warp];
        float ga = 0.f;
#pragma unroll
        for (int j = 0; j < NC; ++j) {
          const int cc = lane + 32 * j;
          const float St = fmaf(uu, kk[j], Sd[j]);     // S_t
          const float dSd = fmaf(-bt * du, kk[j], dS[j]);
          sc[cc] = St * od;                                        // dq
          sc[DK + cc] = fmaf(dS[j], uu, -bt * Sd[j] * du);         // dk
          const float g = blk[i][j] * dSd;                         // dalpha
          if constexpr (KDA) sc[2 * DK + cc] = g;
          else ga += g;
          dS[j] = dSd * aa[j];
        }
        if constexpr (!KDA) ga = warp_sum(ga);
        if (lane == 0) {
          if constexpr (!KDA) sc[2 * DK] = ga;
          sc[NQ - 1] = du * rr;                                    // dbeta
          dv[(((long)b * T + t0 + t) * row_stride + h) * DV + r] = bt * du;
        }
        __syncthreads();
        for (int x = tid; x < NQ; x += BW_THREADS) {
          float acc = 0.f;
#pragma unroll
          for (int w = 0; w < BW_ROWS; ++w) acc += sm.scratch[sp][w][x];
          sm.part[pb][i][x] = acc;
        }
        sp ^= 1;
      }
      // ---- the block's sums over the cluster's CTAs, written out -------------------------
      cluster_sync();
      for (int i = crank; i < BW_BLOCK; i += ncl) {
        const int t = tb + i;
        if (t >= L) continue;
        const long tok = ((long)b * T + t0 + t) * row_stride + h;
        for (int x = tid; x < NQ; x += BW_THREADS) {
          float acc = 0.f;
          for (int rk = 0; rk < ncl; ++rk) acc += ld_cluster(&sm.part[pb][i][x], (uint32_t)rk);
          if (x < DK) dq[tok * DK + x] = acc;
          else if (x < 2 * DK) dk[tok * DK + x - DK] = acc;
          else if (x < 2 * DK + NA) dalpha[tok * NA + x - 2 * DK] = acc;
          else if (x == NQ - 1) dbeta[tok] = acc;
        }
      }
      pb ^= 1;
    }
  }
  {
    const long srow = (((long)b * H + h) * DV + r) * DK;
#pragma unroll
    for (int j = 0; j < NC; ++j) ds0[srow + lane + 32 * j] = dS[j];
  }
  cluster_sync();                                 // no CTA leaves while others read its sums
}

template <int DK, bool KDA, typename Tin, typename Tdo>
cudaError_t launch_bw(const BackwardArgs& a, cudaStream_t st) {
  auto kern = gdr_backward_kernel<DK, KDA, Tin, Tdo>;
  const int smem = (int)sizeof(BwSmem<DK, KDA, Tin>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 0);
  if (e != cudaSuccess) return e;
  const int ncl = a.dv / BW_ROWS;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(a.B * a.H * ncl), 1, 1);
  cfg.blockDim = dim3(BW_THREADS, 1, 1);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)ncl;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, (const Tin*)a.q, (const Tin*)a.k, (const Tin*)a.v,
                            a.alpha, a.beta, a.s0, (const Tdo*)a.dO, a.ds_final, a.dq_out,
                            a.dk_out, a.dv_out, a.dalpha, a.dbeta, a.ds0, a.T, a.H, a.dv,
                            (float*)a.workspace);
}

template <bool KDA, typename Tin, typename Tdo>
cudaError_t launch_bw_dk(const BackwardArgs& a, cudaStream_t st) {
  if (a.dk == 32) return launch_bw<32, KDA, Tin, Tdo>(a, st);
  if (a.dk == 64) return launch_bw<64, KDA, Tin, Tdo>(a, st);
  return launch_bw<128, KDA, Tin, Tdo>(a, st);
}

template <bool KDA>
cudaError_t launch_bw_types(const BackwardArgs& a, cudaStream_t st) {
  if (a.in_dtype == GDR_BF16) {
    if (a.do_dtype == GDR_BF16) return launch_bw_dk<KDA, __nv_bfloat16, __nv_bfloat16>(a, st);
    return launch_bw_dk<KDA, __nv_bfloat16, float>(a, st);
  }
  if (a.do_dtype == GDR_BF16) return launch_bw_dk<KDA, float, __nv_bfloat16>(a, st);
  return launch_bw_dk<KDA, float, float>(a, st);
}

}  // namespace

size_t backward_workspace_bytes(int B, int T, int H, int dk, int dv) {
  const size_t nchunks = ((size_t)T + kC - 1) / kC;
  return (size_t)B * H * nchunks * dv * (dk + 2 * kC) * sizeof(float);
}

cudaError_t launch_backward(const BackwardArgs& a, cudaStream_t st) {
  return a.kda ? launch_bw_types<true>(a, st) : launch_bw_types<false>(a, st);
}

}  // namespace gdr
