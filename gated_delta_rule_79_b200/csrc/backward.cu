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
// dq, dk, dalpha and dbeta sum over rows.  So a warp owns two value rows (each lane
// d_k / 32 key channels of both), a CTA of 16 warps owns 32 rows, and the d_v / 32
// CTAs of one (sequence, head) form a thread-block cluster that sums the per-row terms
// through distributed shared memory.
//
// Pass 1 runs the recurrence forward and leaves, in the workspace, the state entering
// every segment of 32 tokens and u_t, r_t of every token.  Pass 2 walks the segments in
// reverse: from the segment's entering state it rebuilds the state at every eighth token
// (no reductions: u_t is known; four states kept), then in blocks of four tokens (their
// states in registers, rebuilt from the nearest of those) runs the reverse steps.  Each
// warp leaves its rows' terms of the block's four tokens in shared memory; one barrier
// later the CTA sums them over its warps, and one cluster barrier later the cluster's
// CTAs sum those and write the results.  Everything is fp32; there is no wait on another
// CTA other than the cluster barrier, which every CTA of a cluster reaches the same
// number of times.

#include <stdio.h>
#include <stdint.h>

#include "common.cuh"
#include "gdr.h"
#include "launch.h"

namespace gdr {
namespace {

constexpr int BW_WARPS = 16;
constexpr int BW_RPW = 2;                       // value rows per warp
constexpr int BW_ROWS = BW_WARPS * BW_RPW;      // value rows per CTA
constexpr int BW_THREADS = 32 * BW_WARPS;
constexpr int BW_SEG = 32;                      // tokens per staged segment (checkpointed)
constexpr int BW_SUB = 8;                       // tokens between rebuilt states
constexpr int BW_BLOCK = 4;                     // tokens per reverse block
constexpr int BW_NSUB = BW_SEG / BW_SUB;

template <int DK, bool KDA>
struct BwCfg {
  static constexpr int NC = DK / 32;                         // key channels per lane
  static constexpr int NA = KDA ? DK : 1;                    // gate floats per token
  // per-token sums: dq at [0, DK), dk at [DK, 2 DK), dalpha at [2 DK, 2 DK + NA), dbeta
  static constexpr int NQ = 2 * DK + NA + 1;
};

template <int DK, bool KDA, typename Tin>
struct BwSmem {
  static constexpr int NQ = BwCfg<DK, KDA>::NQ;
  Tin k[BW_SEG][DK];
  Tin q[BW_SEG][DK];
  float alpha[BW_SEG][BwCfg<DK, KDA>::NA];
  float beta[BW_SEG];
  float vd[BW_SEG][BW_ROWS];                    // v (pass 1), dL/do (pass 2)
  float u[BW_SEG][BW_ROWS];
  float res[BW_SEG][BW_ROWS];
  float scratch[BW_BLOCK][BW_WARPS][NQ];        // each warp's terms of the block's tokens
  float part[2][BW_BLOCK][NQ];                  // the CTA's sums, by block parity
};

__device__ __forceinline__ void warp_sum2(float& a, float& b) {
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, o);
    b += __shfl_xor_sync(0xffffffffu, b, o);
  }
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

// shared-memory address of the same offset in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t cluster_addr(const float* local, uint32_t rank) {
  uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(local)), ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
  return ra;
}
__device__ __forceinline__ float ld_cluster(uint32_t addr) {
  float x;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(x) : "r"(addr));
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
  const int r0 = rb * BW_ROWS + BW_RPW * warp;    // this warp's first value row
  const int rl = BW_RPW * warp;                   // ... within the CTA
  const int nseg = (T + BW_SEG - 1) / BW_SEG;
  // workspace of this CTA: entering states [nseg][32 rows][DK], then u, r [nseg][2][32][32]
  float* ckpt = ws + (size_t)blockIdx.x * ((size_t)nseg * BW_ROWS * (DK + 2 * BW_SEG));
  float* ures = ckpt + (size_t)nseg * BW_ROWS * DK;
  auto tok = [&](int t) -> long { return ((long)b * T + t) * H + h; };   // token row index

  // ---- one segment's inputs into shared memory (tokens past T: zeros, alpha 1, beta 0) ---
  auto load_seg = [&](int sg, bool reverse_pass) {
    const int t0 = sg * BW_SEG;
    const int L = min(BW_SEG, T - t0);
    constexpr int VEC = 16 / sizeof(Tin);
    constexpr int PR = DK / VEC;
    for (int i = tid; i < BW_SEG * PR; i += BW_THREADS) {
      const int t = i / PR, p = i - t * PR;
      uint4 x = make_uint4(0, 0, 0, 0), y = make_uint4(0, 0, 0, 0);
      if (t < L) {
        const long off = tok(t0 + t) * DK + p * VEC;
        x = *reinterpret_cast<const uint4*>(k + off);
        if (reverse_pass) y = *reinterpret_cast<const uint4*>(q + off);
      }
      *reinterpret_cast<uint4*>(&sm.k[t][p * VEC]) = x;
      if (reverse_pass) *reinterpret_cast<uint4*>(&sm.q[t][p * VEC]) = y;
    }
    for (int i = tid; i < BW_SEG * NA; i += BW_THREADS) {
      const int t = i / NA, c = i - t * NA;
      sm.alpha[t][c] = t < L ? alpha[tok(t0 + t) * NA + c] : 1.f;
    }
    for (int i = tid; i < BW_SEG * BW_ROWS; i += BW_THREADS) {
      const int t = i / BW_ROWS, rr = i - t * BW_ROWS;
      float x = 0.f;
      if (t < L) {
        const long off = tok(t0 + t) * DV + rb * BW_ROWS + rr;
        x = reverse_pass ? Elem<Tdo>::load(dO + off) : Elem<Tin>::load(v + off);
      }
      sm.vd[t][rr] = x;
      if (reverse_pass) {
        sm.u[t][rr] = t < L ? ures[((size_t)sg * 2 + 0) * BW_SEG * BW_ROWS + i] : 0.f;
        sm.res[t][rr] = t < L ? ures[((size_t)sg * 2 + 1) * BW_SEG * BW_ROWS + i] : 0.f;
      }
    }
    if (tid < BW_SEG) sm.beta[tid] = tid < L ? beta[tok(t0 + tid)] : 0.f;
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
  // S <- S Diag(alpha_t) + u_t k_t^T for this warp's two rows (u_t known)
  auto step_known = [&](int t, float (&S)[BW_RPW][NC]) {
    float kk[NC], aa[NC];
    ld_k(t, kk);
    ld_a(t, aa);
#pragma unroll
    for (int p = 0; p < BW_RPW; ++p) {
      const float uu = sm.u[t][rl + p];
#pragma unroll
      for (int j = 0; j < NC; ++j) S[p][j] = fmaf(uu, kk[j], S[p][j] * aa[j]);
    }
  };

  // =============================== pass 1: forward ======================================
  float S[BW_RPW][NC];
#pragma unroll
  for (int p = 0; p < BW_RPW; ++p) {
    const long srow = (((long)b * H + h) * DV + r0 + p) * DK;
#pragma unroll
    for (int j = 0; j < NC; ++j) S[p][j] = s0 ? s0[srow + lane + 32 * j] : 0.f;
  }
  for (int sg = 0; sg < nseg; ++sg) {
    const int L = min(BW_SEG, T - sg * BW_SEG);
#pragma unroll
    for (int p = 0; p < BW_RPW; ++p)
#pragma unroll
      for (int j = 0; j < NC; ++j)
        ckpt[((size_t)sg * BW_ROWS + rl + p) * DK + lane + 32 * j] = S[p][j];
    __syncthreads();                              // the previous segment's inputs are read
    load_seg(sg, false);
    __syncthreads();
    for (int t = 0; t < L; ++t) {
      float kk[NC], aa[NC], a0 = 0.f, a1 = 0.f;
      ld_k(t, kk);
      ld_a(t, aa);
#pragma unroll
      for (int j = 0; j < NC; ++j) {
        S[0][j] *= aa[j];
        S[1][j] *= aa[j];
        a0 = fmaf(S[0][j], kk[j], a0);
        a1 = fmaf(S[1][j], kk[j], a1);
      }
      warp_sum2(a0, a1);
      const float bt = sm.beta[t];
      const float q0 = sm.vd[t][rl] - a0, q1 = sm.vd[t][rl + 1] - a1;
      const float u0 = bt * q0, u1 = bt * q1;
#pragma unroll
      for (int j = 0; j < NC; ++j) {
        S[0][j] = fmaf(u0, kk[j], S[0][j]);
        S[1][j] = fmaf(u1, kk[j], S[1][j]);
      }
      if (lane < 2) {
        sm.u[t][rl + lane] = lane ? u1 : u0;
        sm.res[t][rl + lane] = lane ? q1 : q0;
      }
    }
    __syncthreads();
    for (int i = tid; i < L * BW_ROWS; i += BW_THREADS) {
      const int t = i / BW_ROWS, rr = i - t * BW_ROWS;
      ures[((size_t)sg * 2 + 0) * BW_SEG * BW_ROWS + i] = sm.u[t][rr];
      ures[((size_t)sg * 2 + 1) * BW_SEG * BW_ROWS + i] = sm.res[t][rr];
    }
  }
  __syncthreads();

  // =============================== pass 2: reverse ======================================
  float dS[BW_RPW][NC];
#pragma unroll
  for (int p = 0; p < BW_RPW; ++p) {
    const long srow = (((long)b * H + h) * DV + r0 + p) * DK;
#pragma unroll
    for (int j = 0; j < NC; ++j) dS[p][j] = ds_final ? ds_final[srow + lane + 32 * j] : 0.f;
  }
  int pb = 0;                                     // block parity (part)
  for (int sg = nseg - 1; sg >= 0; --sg) {
    const int t0 = sg * BW_SEG;
    const int L = min(BW_SEG, T - t0);
    __syncthreads();
    load_seg(sg, true);
    __syncthreads();
    // the state before tokens 0, 8, 16, 24 of the segment
    float sub[BW_NSUB][BW_RPW][NC];
    {
      float Sx[BW_RPW][NC];
#pragma unroll
      for (int p = 0; p < BW_RPW; ++p)
#pragma unroll
        for (int j = 0; j < NC; ++j)
          Sx[p][j] = ckpt[((size_t)sg * BW_ROWS + rl + p) * DK + lane + 32 * j];
#pragma unroll
      for (int s = 0; s < BW_NSUB; ++s) {
#pragma unroll
        for (int p = 0; p < BW_RPW; ++p)
#pragma unroll
          for (int j = 0; j < NC; ++j) sub[s][p][j] = Sx[p][j];
        if (s + 1 < BW_NSUB)
          for (int t = s * BW_SUB; t < (s + 1) * BW_SUB; ++t) step_known(t, Sx);
      }
    }
    // blocks of four tokens, last first; block n covers tokens 4n .. 4n + 3
#pragma unroll
    for (int nn = 0; nn < BW_SEG / BW_BLOCK; ++nn) {
      const int n = BW_SEG / BW_BLOCK - 1 - nn;
      const int tb = n * BW_BLOCK;
      if (tb >= L) continue;                      // uniform over the cluster
      // states before tokens tb .. tb + 3, rebuilt from the state before token 8 (n / 2)
      float blk[BW_BLOCK][BW_RPW][NC];
      {
        float Sx[BW_RPW][NC];
#pragma unroll
        for (int p = 0; p < BW_RPW; ++p)
#pragma unroll
          for (int j = 0; j < NC; ++j) Sx[p][j] = sub[n / 2][p][j];
        if (n & 1)
#pragma unroll
          for (int t = tb - BW_BLOCK; t < tb; ++t) step_known(t, Sx);
#pragma unroll
        for (int i = 0; i < BW_BLOCK; ++i) {
#pragma unroll
          for (int p = 0; p < BW_RPW; ++p)
#pragma unroll
            for (int j = 0; j < NC; ++j) blk[i][p][j] = Sx[p][j];
          if (i + 1 < BW_BLOCK) step_known(tb + i, Sx);
        }
      }
#pragma unroll
      for (int ii = 0; ii < BW_BLOCK; ++ii) {
        const int i = BW_BLOCK - 1 - ii;
        const int t = tb + i;
        float* sc = sm.scratch[i][warp];
        if (t >= L) {                             // past the end: no terms
          for (int x = lane; x < NQ; x += 32) sc[x] = 0.f;
          continue;
        }
        float kk[NC], qq[NC], aa[NC];
        ld_k(t, kk);
        ld_q(t, qq);
        ld_a(t, aa);
        const float bt = sm.beta[t];
        float uu[BW_RPW], od[BW_RPW], rr[BW_RPW], du[BW_RPW];
#pragma unroll
        for (int p = 0; p < BW_RPW; ++p) {
          uu[p] = sm.u[t][rl + p];
          od[p] = sm.vd[t][rl + p];
          rr[p] = sm.res[t][rl + p];
          du[p] = 0.f;
        }
#pragma unroll
        for (int p = 0; p < BW_RPW; ++p)
#pragma unroll
          for (int j = 0; j < NC; ++j) {
            dS[p][j] = fmaf(od[p], qq[j], dS[p][j]);           // + do q^T
            du[p] = fmaf(dS[p][j], kk[j], du[p]);
          }
        warp_sum2(du[0], du[1]);
        float ga = 0.f;
#pragma unroll
        for (int j = 0; j < NC; ++j) {
          const int cc = lane + 32 * j;
          float pq = 0.f, pk = 0.f, pa = 0.f;
#pragma unroll
          for (int p = 0; p < BW_RPW; ++p) {
            const float Sd = blk[i][p][j] * aa[j];             // S~
            const float St = fmaf(uu[p], kk[j], Sd);           // S_t
            const float dSd = fmaf(-bt * du[p], kk[j], dS[p][j]);
            pq = fmaf(St, od[p], pq);                          // dq
            pk = fmaf(dS[p][j], uu[p], fmaf(-bt * du[p], Sd, pk));   // dk
            pa = fmaf(blk[i][p][j], dSd, pa);                  // dalpha
            dS[p][j] = dSd * aa[j];
          }
          sc[cc] = pq;
          sc[DK + cc] = pk;
          if constexpr (KDA) sc[2 * DK + cc] = pa;
          else ga += pa;
        }
        if constexpr (!KDA) {
#pragma unroll
          for (int o = 16; o; o >>= 1) ga += __shfl_xor_sync(0xffffffffu, ga, o);
        }
        if (lane == 0) {
          if constexpr (!KDA) sc[2 * DK] = ga;
          sc[NQ - 1] = du[0] * rr[0] + du[1] * rr[1];          // dbeta
        }
        if (lane < BW_RPW)
          dv[tok(t0 + t) * DV + r0 + lane] = bt * (lane ? du[1] : du[0]);
      }
      // ---- the block's sums: over the CTA's warps, then over the cluster's CTAs ---------
      __syncthreads();
      for (int x = tid; x < BW_BLOCK * NQ; x += BW_THREADS) {
        const int i = x / NQ, y = x - i * NQ;
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < BW_WARPS; ++w) acc += sm.scratch[i][w][y];
        sm.part[pb][i][y] = acc;
      }
      cluster_sync();
      for (int i = crank; i < BW_BLOCK; i += ncl) {
        const int t = tb + i;
        if (t >= L) continue;
        const long tr = tok(t0 + t);
        for (int x = tid; x < NQ; x += BW_THREADS) {
          float got[4];
#pragma unroll
          for (int rk = 0; rk < 4; ++rk)
            got[rk] = rk < ncl ? ld_cluster(cluster_addr(&sm.part[pb][i][x], (uint32_t)rk)) : 0.f;
          const float acc = (got[0] + got[1]) + (got[2] + got[3]);
          if (x < DK) dq[tr * DK + x] = acc;
          else if (x < 2 * DK) dk[tr * DK + x - DK] = acc;
          else if (x < 2 * DK + NA) dalpha[tr * NA + x - 2 * DK] = acc;
          else dbeta[tr] = acc;
        }
      }
      pb ^= 1;
    }
  }
#pragma unroll
  for (int p = 0; p < BW_RPW; ++p) {
    const long srow = (((long)b * H + h) * DV + r0 + p) * DK;
#pragma unroll
    for (int j = 0; j < NC; ++j) ds0[srow + lane + 32 * j] = dS[p][j];
  }
  cluster_sync();                                 // no CTA leaves while others read its sums
}

template <int DK, bool KDA, typename Tin, typename Tdo>
cudaError_t launch_bw(const BackwardArgs& a, cudaStream_t st) {
  auto kern = gdr_backward_kernel<DK, KDA, Tin, Tdo>;
  const int smem = (int)sizeof(BwSmem<DK, KDA, Tin>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
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
  const size_t nseg = ((size_t)T + BW_SEG - 1) / BW_SEG;
  return (size_t)B * H * nseg * dv * (dk + 2 * BW_SEG) * sizeof(float);
}

cudaError_t launch_backward(const BackwardArgs& a, cudaStream_t st) {
  return a.kda ? launch_bw_types<true>(a, st) : launch_bw_types<false>(a, st);
}

}  // namespace gdr
