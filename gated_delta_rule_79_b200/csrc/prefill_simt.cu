// Chunked prefill of the gated delta rule on CUDA cores, fp32 arithmetic.
//
// This is the path for fp32 inputs (which must match to 1e-5, ruling out TF32
// and bf16 tensor-core operands) and for head sizes without a tensor-core
// kernel.  It follows the same chunk algebra as the tensor-core kernel.
//
// Chunk algebra ("Super Apriel: One Checkpoint, Many Speeds", §2A names the
// mixers; the unrolling below is the standard chunk-wise form of the gated delta
// rule).  For a chunk of L <= 64 tokens entering with state S0 (d_v x d_k),
// G[t] = sum_{s<=t} log alpha_s (inclusive, chunk-local, per key channel for
// KDA), and decay(t, j) = exp(G[t] - G[j]):
//
//   A[t,j] = beta_t sum_c k_tc k_jc decay_c(t,j)    (j < t)
//   P[t,j] =        sum_c q_tc k_jc decay_c(t,j)    (j <= t)
//   [W | U~] = (I + A)^{-1} Diag(beta) [K (.) e^G | V]      (forward substitution)
//   U  = U~ - W S0^T
//   O  = (Q (.) e^G) S0^T + P U
//   S  = S0 Diag(e^{G[L-1]}) + U^T (K (.) e^{G[L-1] - G})
//
// One CTA owns one (batch, head, 32-wide slice of d_v) and walks the chunks in
// order: the rows of S (the d_v axis) are independent given the chunk's W, U~,
// P and gates, so slicing d_v multiplies the parallelism of the serial carry at
// the cost of recomputing the state-independent products per slice.

#include <math.h>

#include "common.cuh"
#include "launch.h"

namespace gdr {
namespace {

constexpr int kC = GDR_CHUNK;          // chunk length
constexpr int kThreads = 256;
constexpr int kDVS = 32;               // d_v slice per CTA

template <int DK, bool KDA>
struct SimtSmem {
  static constexpr int LDK = DK + 1;   // padded row pitch (bank-conflict free)
  static constexpr int LDV = kDVS + 1;
  static constexpr int LDA = kC + 1;
  static constexpr int GSZ = KDA ? kC * LDK : kC;
  // offsets in floats
  static constexpr int K = 0;
  static constexpr int Q = K + kC * LDK;
  static constexpr int G = Q + kC * LDK;
  static constexpr int V = G + GSZ;
  static constexpr int A = V + kC * LDV;
  static constexpr int P = A + kC * LDA;
  static constexpr int W = P + kC * LDA;
  static constexpr int U = W + kC * LDK;
  static constexpr int S = U + kC * LDV;
  static constexpr int BETA = S + kDVS * LDK;
  static constexpr int EGC = BETA + kC;
  static constexpr int TOTAL = EGC + DK;
  static constexpr size_t BYTES = sizeof(float) * TOTAL;
};

template <int DK, bool KDA, typename Tin, typename Tout>
__global__ void __launch_bounds__(kThreads)
prefill_simt_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                    const Tin* __restrict__ v, const float* __restrict__ alpha,
                    const float* __restrict__ beta, const float* __restrict__ s0,
                    Tout* __restrict__ o, float* __restrict__ s_final,
                    int T, int H, int dv, unsigned pro) {
  using L = SimtSmem<DK, KDA>;
  extern __shared__ float sm[];
  float* Ks = sm + L::K;    // k, later K (.) e^{G_last - G}
  float* Qs = sm + L::Q;    // q, later Q (.) e^G
  float* Gs = sm + L::G;    // chunk-local cumulative log gate
  float* Vs = sm + L::V;
  float* As = sm + L::A;
  float* Ps = sm + L::P;
  float* Ws = sm + L::W;
  float* Us = sm + L::U;    // U~, then U
  float* Ss = sm + L::S;    // state slice [kDVS][DK]
  float* Bs = sm + L::BETA;
  float* Egc = sm + L::EGC;

  const int tid = threadIdx.x;
  const int nslice = dv / kDVS;
  const int slice = blockIdx.x % nslice;
  const int bh = blockIdx.x / nslice;
  const int h = bh % H;
  const long b = bh / H;
  const int v0 = slice * kDVS;

  // initial state slice (rows v0 .. v0+31 of S)
  const long sbase = (b * H + h) * (long)dv * DK;
  for (int i = tid; i < kDVS * DK; i += kThreads) {
    const int r = i / DK, c = i % DK;
    Ss[r * L::LDK + c] = s0 ? s0[sbase + (long)(v0 + r) * DK + c] : 0.f;
  }

  for (int t0 = 0; t0 < T; t0 += kC) {
    const int Lc = min(kC, T - t0);
    __syncthreads();
    // ---- 1. load the chunk (rows >= Lc are zero so they drop out) -----------------
    for (int i = tid; i < kC * DK; i += kThreads) {
      const int t = i / DK, c = i % DK;
      float kv = 0.f, qv = 0.f, g = 0.f;
      if (t < Lc) {
        const long row = ((b * T + t0 + t) * H + h);
        kv = Elem<Tin>::load(k + row * DK + c);
        qv = Elem<Tin>::load(q + row * DK + c);
        if (KDA) {
          const float a = alpha[row * DK + c];
          g = (pro & GDR_PROLOGUE_GATE_LOGIT) ? log_gate_from_logit(a) : log_gate_accurate(a);
        }
      }
      Ks[t * L::LDK + c] = kv;
      Qs[t * L::LDK + c] = qv;
      if (KDA) Gs[t * L::LDK + c] = g;
    }
    for (int i = tid; i < kC * kDVS; i += kThreads) {
      const int t = i / kDVS, c = i % kDVS;
      float vv = 0.f;
      if (t < Lc) vv = Elem<Tin>::load(v + ((b * T + t0 + t) * H + h) * (long)dv + v0 + c);
      Vs[t * L::LDV + c] = vv;
    }
    if (tid < kC) {
      const long row = (b * T + t0 + tid) * H + h;
      Bs[tid] = tid < Lc ? beta[row] : 0.f;
      if (!KDA) {
        const float a = tid < Lc ? alpha[row] : 1.f;
        Gs[tid] = tid >= Lc ? 0.f
                  : (pro & GDR_PROLOGUE_GATE_LOGIT) ? log_gate_from_logit(a)
                                                    : log_gate_accurate(a);
      }
    }
    __syncthreads();
    if (pro & GDR_PROLOGUE_L2NORM_QK) {
      // one warp per token row: q and k divided by their L2 norms (fp32), then held as
      // the input type holds them
      const int lane = tid & 31;
      for (int t = tid >> 5; t < Lc; t += kThreads / 32) {
        float nk = 0.f, nq = 0.f;
        for (int c = lane; c < DK; c += 32) {
          nk = fmaf(Ks[t * L::LDK + c], Ks[t * L::LDK + c], nk);
          nq = fmaf(Qs[t * L::LDK + c], Qs[t * L::LDK + c], nq);
        }
#pragma unroll
        for (int off = 16; off; off >>= 1) {
          nk += __shfl_xor_sync(0xffffffffu, nk, off);
          nq += __shfl_xor_sync(0xffffffffu, nq, off);
        }
        const float sk = l2_scale(nk), sq = l2_scale(nq);
        for (int c = lane; c < DK; c += 32) {
          Ks[t * L::LDK + c] = as_input<Tin>(Ks[t * L::LDK + c] * sk);
          Qs[t * L::LDK + c] = as_input<Tin>(Qs[t * L::LDK + c] * sq);
        }
      }
      __syncthreads();
    }
    // ---- 2. inclusive cumulative sum of the log gates (fp64, rounded once) --------
    if (KDA) {
      if (tid < DK) {
        double acc = 0.0;
        for (int t = 0; t < kC; ++t) {
          acc += (double)Gs[t * L::LDK + tid];
          Gs[t * L::LDK + tid] = (float)acc;
        }
        Egc[tid] = expf(Gs[(Lc - 1) * L::LDK + tid]);
      }
    } else if (tid == 0) {
      double acc = 0.0;
      for (int t = 0; t < kC; ++t) {
        acc += (double)Gs[t];
        Gs[t] = (float)acc;
      }
      Egc[0] = expf(Gs[Lc - 1]);
    }
    __syncthreads();
    auto gate = [&](int t, int c) -> float { return KDA ? Gs[t * L::LDK + c] : Gs[t]; };
    // ---- 3. decayed Gram matrices A (strictly lower) and P (lower) ------------------
    {
      const int tb = (tid / 16) * 4, jb = (tid % 16) * 4;   // 4x4 micro-tile
      float accA[4][4] = {}, accP[4][4] = {};
      if (jb <= tb + 3) {
        for (int c = 0; c < DK; ++c) {
          float kt[4], qt[4], kj[4], gt[4], gj[4];
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            kt[x] = Ks[(tb + x) * L::LDK + c];
            qt[x] = Qs[(tb + x) * L::LDK + c];
            kj[x] = Ks[(jb + x) * L::LDK + c];
            if (KDA) { gt[x] = gate(tb + x, c); gj[x] = gate(jb + x, c); }
          }
#pragma unroll
          for (int x = 0; x < 4; ++x)
#pragma unroll
            for (int y = 0; y < 4; ++y) {
              float kjd = kj[y];
              if (KDA) kjd *= expf(fminf(gt[x] - gj[y], 0.f));
              accA[x][y] = fmaf(kt[x], kjd, accA[x][y]);
              accP[x][y] = fmaf(qt[x], kjd, accP[x][y]);
            }
        }
      }
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) {
          const int t = tb + x, jj = jb + y;
          float d = 1.f;
          if (!KDA && jj <= t) d = expf(Gs[t] - Gs[jj]);
          As[t * L::LDA + jj] = jj < t ? Bs[t] * accA[x][y] * d : 0.f;
          Ps[t * L::LDA + jj] = jj <= t ? accP[x][y] * d : 0.f;
        }
    }
    __syncthreads();
    // ---- 4. forward substitution for [W | U~] --------------------------------------
    if (tid < DK + kDVS) {
      const bool isw = tid < DK;
      const int c = isw ? tid : tid - DK;
      float* X = isw ? Ws : Us;
      const int ld = isw ? L::LDK : L::LDV;
      for (int t = 0; t < kC; ++t) {
        float rhs = isw ? Ks[t * L::LDK + c] * expf(gate(t, c)) : Vs[t * L::LDV + c];
        float x = Bs[t] * rhs;
        for (int jj = 0; jj < t; ++jj) x = fmaf(-As[t * L::LDA + jj], X[jj * ld + c], x);
        X[t * ld + c] = x;
      }
    }
    __syncthreads();
    // ---- 5. gate-scaled operands: Q (.) e^G and K (.) e^{G_last - G} ----------------
    for (int i = tid; i < kC * DK; i += kThreads) {
      const int t = i / DK, c = i % DK;
      const float g = gate(t, c);
      const float glast = gate(Lc - 1, c);
      Qs[t * L::LDK + c] *= expf(g);
      Ks[t * L::LDK + c] *= (t < Lc) ? expf(fminf(glast - g, 0.f)) : 0.f;
    }
    // ---- 6. U = U~ - W S0^T ----------------------------------------------------------
    const int vv = tid % kDVS, tr = tid / kDVS;   // 8 row groups x 32 columns
    __syncthreads();
    {
      float acc[kC / 8];
#pragma unroll
      for (int m = 0; m < kC / 8; ++m) acc[m] = Us[(tr + 8 * m) * L::LDV + vv];
      for (int c = 0; c < DK; ++c) {
        const float s = Ss[vv * L::LDK + c];
#pragma unroll
        for (int m = 0; m < kC / 8; ++m) acc[m] = fmaf(-Ws[(tr + 8 * m) * L::LDK + c], s, acc[m]);
      }
      __syncthreads();
#pragma unroll
      for (int m = 0; m < kC / 8; ++m) Us[(tr + 8 * m) * L::LDV + vv] = acc[m];
    }
    __syncthreads();
    // ---- 7. O = (Q e^G) S0^T + P U ---------------------------------------------------
    {
      float acc[kC / 8] = {};
      for (int c = 0; c < DK; ++c) {
        const float s = Ss[vv * L::LDK + c];
#pragma unroll
        for (int m = 0; m < kC / 8; ++m) acc[m] = fmaf(Qs[(tr + 8 * m) * L::LDK + c], s, acc[m]);
      }
      for (int jj = 0; jj < kC; ++jj) {
        const float u = Us[jj * L::LDV + vv];
#pragma unroll
        for (int m = 0; m < kC / 8; ++m) acc[m] = fmaf(Ps[(tr + 8 * m) * L::LDA + jj], u, acc[m]);
      }
#pragma unroll
      for (int m = 0; m < kC / 8; ++m) {
        const int t = tr + 8 * m;
        if (t < Lc)
          Elem<Tout>::store(o + ((b * T + t0 + t) * H + h) * (long)dv + v0 + vv, acc[m]);
      }
    }
    __syncthreads();
    // ---- 8. S = S0 Diag(e^{G_last}) + U^T (K e^{G_last - G}) -------------------------
    for (int c = tr; c < DK; c += kThreads / kDVS) {
      float acc = Ss[vv * L::LDK + c] * Egc[KDA ? c : 0];
      for (int jj = 0; jj < Lc; ++jj) acc = fmaf(Us[jj * L::LDV + vv], Ks[jj * L::LDK + c], acc);
      Ss[vv * L::LDK + c] = acc;
    }
  }
  __syncthreads();
  if (s_final) {
    for (int i = tid; i < kDVS * DK; i += kThreads) {
      const int r = i / DK, c = i % DK;
      s_final[sbase + (long)(v0 + r) * DK + c] = Ss[r * L::LDK + c];
    }
  }
}

template <int DK, bool KDA, typename Tin, typename Tout>
cudaError_t launch_t(const PrefillArgs& a, cudaStream_t st) {
  using L = SimtSmem<DK, KDA>;
  auto kern = prefill_simt_kernel<DK, KDA, Tin, Tout>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)L::BYTES);
  if (e != cudaSuccess) return e;
  const int grid = a.B * a.H * (a.dv / kDVS);
  kern<<<grid, kThreads, L::BYTES, st>>>((const Tin*)a.q, (const Tin*)a.k, (const Tin*)a.v,
                                         a.alpha, a.beta, a.s0, (Tout*)a.o, a.s_final,
                                         a.T, a.H, a.dv, a.pro);
  e = cudaGetLastError();
  if (e == cudaSuccess) timing_mark(st, 0);
  return e;
}

template <int DK, bool KDA>
cudaError_t launch_k(const PrefillArgs& a, cudaStream_t st) {
  const bool of32 = a.out_dtype == GDR_F32;
  if (a.in_dtype == GDR_F32)
    return of32 ? launch_t<DK, KDA, float, float>(a, st)
                : launch_t<DK, KDA, float, __nv_bfloat16>(a, st);
  return of32 ? launch_t<DK, KDA, __nv_bfloat16, float>(a, st)
              : launch_t<DK, KDA, __nv_bfloat16, __nv_bfloat16>(a, st);
}

template <int DK>
cudaError_t launch_dk(const PrefillArgs& a, cudaStream_t st) {
  return a.kda ? launch_k<DK, true>(a, st) : launch_k<DK, false>(a, st);
}

}  // namespace

cudaError_t launch_prefill_simt(const PrefillArgs& a, cudaStream_t stream) {
  switch (a.dk) {
    case 32: return launch_dk<32>(a, stream);
    case 64: return launch_dk<64>(a, stream);
    case 128: return launch_dk<128>(a, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace gdr
