// Multi-token step of the gated delta rule (GDN / KDA) from a carried state, with the
// state after every token kept ("snapshots"), sm_100a.
//
// "Super Apriel: One Checkpoint, Many Speeds", §2D (inference and serving) and §4
// (speculative decoding): the all-GDN placement of the supernet drafts tokens for the
// all-FA placement to verify, with no separate draft model.  A recurrent mixer that
// takes part in drafting or verifying K tokens must be able to continue from the last
// accepted one, so this kernel runs the recurrence over K tokens of each (sequence,
// head) and writes, besides the K outputs, the state after each of the K tokens; the
// caller keeps the snapshot of the last accepted token as the new state (no copy).
// With no snapshot buffer it is a K-token decode that updates the state in place.
//
// The per-token update is the decode step (decode.cu): for row r of S,
//     s~ = S[r,:] (.) alpha_t;  a = s~ . k_t;  b = s~ . q_t;  u = beta_t (v_t[r] - a)
//     S[r,:] = s~ + u k_t;      o_t[r] = b + u (k_t . q_t)
// Layout: two warps per (sequence, head), each over half of the rows (more, shorter
// tasks: the last partial wave of the grid is a smaller share), a state row spread over
// 8 lanes in float4 pieces; each row group is read from HBM once, carried through the K tokens in
// registers, and each snapshot row is written once (evict-first).  The K tokens' q, k
// and gates, and k_t . q_t, are staged in shared memory per warp.  Bound: HBM, with
// (1 + K) d_v d_k 4 bytes per (sequence, head) (2 d_v d_k 4 without snapshots).

#include "checks.cuh"
#include "common.cuh"
#include "launch.h"

namespace gdr {
namespace {

constexpr int kWarps = 4;

template <int DK, bool KDA, typename Tin, typename Tout>
__global__ void __launch_bounds__(kWarps * 32)
verify_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
              const float* __restrict__ alpha, const float* __restrict__ beta,
              float* __restrict__ state, float* __restrict__ snaps, Tout* __restrict__ o,
              int N, int K, int H, int dv, unsigned pro, unsigned int* checks) {
  constexpr int LPR = 8;               // lanes per state row
  constexpr int RPW = 32 / LPR;        // rows per warp instruction
  constexpr int F4 = DK / (4 * LPR);   // float4 pieces per lane per row
  constexpr int ITER = 2;              // row groups in flight per warp
  constexpr int GA = KDA ? DK : 4;     // floats of gate per token in shared memory
  static_assert(F4 >= 1, "d_k must be a multiple of 32");

  extern __shared__ float vsm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // two warps per (sequence, head), each over half of the d_v rows
  const long task = (long)blockIdx.x * kWarps + warp;
  const long NH = (long)N * H;
  if (task >= 2 * NH) return;
  const long head = task >> 1;                          // n * H + h
  const int rows = dv >> 1;
  // the row loop below covers [0, rows) in whole groups of RPW * ITER rows
  if (!dcheck(2 * rows == dv && rows % (RPW * ITER) == 0, checks, kCheckLayout)) return;
  const int rbase = (int)(task & 1) * rows;
  const long n = head / H, h = head % H;
  // per warp: K x (q[DK], k[DK], gate[GA], {beta, k.q, -, -})
  const int per_tok = 2 * DK + GA + 4;
  float* ws = vsm + (size_t)warp * K * per_tok;

  for (int t = 0; t < K; ++t) {
    const long row = (n * K + t) * H + h;             // [N, K, H, ...]
    float* tk = ws + t * per_tok;
    float kq = 0.f, nq = 0.f, nk = 0.f;
    for (int c = lane; c < DK; c += 32) {
      const float qq = Elem<Tin>::load(q + row * DK + c);
      const float kk = Elem<Tin>::load(k + row * DK + c);
      tk[c] = qq;
      tk[DK + c] = kk;
      if (KDA) {
        const float a = alpha[row * DK + c];
        tk[2 * DK + c] = (pro & GDR_PROLOGUE_GATE_LOGIT) ? gate_from_logit(a) : a;
      }
      nq = fmaf(qq, qq, nq);
      nk = fmaf(kk, kk, nk);
    }
    if (pro & GDR_PROLOGUE_L2NORM_QK) {
#pragma unroll
      for (int off = 16; off; off >>= 1) {
        nq += __shfl_xor_sync(0xffffffffu, nq, off);
        nk += __shfl_xor_sync(0xffffffffu, nk, off);
      }
      const float sq = l2_scale(nq), sk = l2_scale(nk);
      for (int c = lane; c < DK; c += 32) {
        tk[c] = as_input<Tin>(tk[c] * sq);
        tk[DK + c] = as_input<Tin>(tk[DK + c] * sk);
      }
    }
    for (int c = lane; c < DK; c += 32) kq = fmaf(tk[c], tk[DK + c], kq);
#pragma unroll
    for (int off = 16; off; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
    if (lane == 0) {
      if (!KDA) tk[2 * DK] = (pro & GDR_PROLOGUE_GATE_LOGIT) ? gate_from_logit(alpha[row]) : alpha[row];
      tk[2 * DK + GA] = beta[row];
      tk[2 * DK + GA + 1] = kq;
    }
  }
  __syncwarp();

  const int sub = lane / LPR;
  const int j = lane % LPR;
  // this warp's rows, as if they were the whole state
  float* Sh = state + (head * (long)dv + rbase) * DK;
  const long snap_stride = NH * (long)dv * DK;       // one snapshot = one full state
  float* Snb = snaps ? snaps + (head * (long)dv + rbase) * DK : nullptr;
  const Tin* vb = v + rbase;
  Tout* obase = o + rbase;

  for (int r0 = 0; r0 < rows; r0 += RPW * ITER) {
    float4 s[ITER][F4];
#pragma unroll
    for (int it = 0; it < ITER; ++it) {
      const int row = r0 + it * RPW + sub;
#pragma unroll
      for (int m = 0; m < F4; ++m)
        s[it][m] = __ldcs(reinterpret_cast<const float4*>(Sh + (long)row * DK + 4 * (j + LPR * m)));
    }
    for (int t = 0; t < K; ++t) {
      const float* tk = ws + t * per_tok;
      const long trow = (n * K + t) * H + h;
      float4 kr[F4], qr[F4], ar[F4];
#pragma unroll
      for (int m = 0; m < F4; ++m) {
        const int c = 4 * (j + LPR * m);
        qr[m] = *reinterpret_cast<const float4*>(tk + c);
        kr[m] = *reinterpret_cast<const float4*>(tk + DK + c);
        if (KDA) ar[m] = *reinterpret_cast<const float4*>(tk + 2 * DK + c);
      }
      const float a_s = KDA ? 1.f : tk[2 * DK];
      const float bt = tk[2 * DK + GA], kq = tk[2 * DK + GA + 1];
      float vr[ITER];
#pragma unroll
      for (int it = 0; it < ITER; ++it) vr[it] = Elem<Tin>::load(vb + trow * dv + r0 + it * RPW + sub);
#pragma unroll
      for (int it = 0; it < ITER; ++it) {
        const int row = r0 + it * RPW + sub;
        float pa = 0.f, pb = 0.f;
#pragma unroll
        for (int m = 0; m < F4; ++m) {
          float* e = reinterpret_cast<float*>(&s[it][m]);
          const float* kk = reinterpret_cast<const float*>(&kr[m]);
          const float* qq = reinterpret_cast<const float*>(&qr[m]);
          const float* aa = reinterpret_cast<const float*>(&ar[m]);
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            e[x] *= KDA ? aa[x] : a_s;
            pa = fmaf(e[x], kk[x], pa);
            pb = fmaf(e[x], qq[x], pb);
          }
        }
#pragma unroll
        for (int off = 1; off < LPR; off <<= 1) {
          pa += __shfl_xor_sync(0xffffffffu, pa, off);
          pb += __shfl_xor_sync(0xffffffffu, pb, off);
        }
        const float u = bt * (vr[it] - pa);
#pragma unroll
        for (int m = 0; m < F4; ++m) {
          float* e = reinterpret_cast<float*>(&s[it][m]);
          const float* kk = reinterpret_cast<const float*>(&kr[m]);
#pragma unroll
          for (int x = 0; x < 4; ++x) e[x] = fmaf(u, kk[x], e[x]);
          if (snaps)
            __stcs(reinterpret_cast<float4*>(Snb + t * snap_stride + (long)row * DK +
                                             4 * (j + LPR * m)),
                   s[it][m]);
        }
        if (j == 0) Elem<Tout>::store(obase + trow * dv + row, fmaf(u, kq, pb));
      }
    }
    if (!snaps) {
#pragma unroll
      for (int it = 0; it < ITER; ++it) {
        const int row = r0 + it * RPW + sub;
#pragma unroll
        for (int m = 0; m < F4; ++m)
          __stcs(reinterpret_cast<float4*>(Sh + (long)row * DK + 4 * (j + LPR * m)), s[it][m]);
      }
    }
  }
}

template <int DK, bool KDA, typename Tin>
cudaError_t launch_t(const VerifyArgs& a, cudaStream_t st) {
  const long NH = (long)a.N * a.H;
  const int grid = (int)((2 * NH + kWarps - 1) / kWarps);
  constexpr int GA = KDA ? DK : 4;
  const size_t smem = (size_t)kWarps * a.K * (2 * DK + GA + 4) * sizeof(float);
  cudaError_t e;
  if (a.out_dtype == GDR_F32) {
    auto kern = verify_kernel<DK, KDA, Tin, float>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kWarps * 32, smem, st>>>((const Tin*)a.q, (const Tin*)a.k, (const Tin*)a.v,
                                          a.alpha, a.beta, a.state, a.snapshots, (float*)a.o,
                                          a.N, a.K, a.H, a.dv, a.pro, checks_word());
  } else {
    auto kern = verify_kernel<DK, KDA, Tin, __nv_bfloat16>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kWarps * 32, smem, st>>>((const Tin*)a.q, (const Tin*)a.k, (const Tin*)a.v,
                                          a.alpha, a.beta, a.state, a.snapshots,
                                          (__nv_bfloat16*)a.o, a.N, a.K, a.H, a.dv, a.pro,
                                          checks_word());
  }
  return cudaGetLastError();
}

template <int DK>
cudaError_t launch_dk(const VerifyArgs& a, cudaStream_t st) {
  if (a.in_dtype == GDR_F32)
    return a.kda ? launch_t<DK, true, float>(a, st) : launch_t<DK, false, float>(a, st);
  return a.kda ? launch_t<DK, true, __nv_bfloat16>(a, st)
               : launch_t<DK, false, __nv_bfloat16>(a, st);
}

}  // namespace

cudaError_t launch_verify(const VerifyArgs& a, cudaStream_t stream) {
  switch (a.dk) {
    case 32: return launch_dk<32>(a, stream);
    case 64: return launch_dk<64>(a, stream);
    case 128: return launch_dk<128>(a, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace gdr
