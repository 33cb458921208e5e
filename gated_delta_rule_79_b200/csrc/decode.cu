// Batched one-token decode of the gated delta rule (GDN / KDA), sm_100a.
//
// "Super Apriel: One Checkpoint, Many Speeds", §1 and §4 (decode throughput,
// context-length scaling): the GDN/KDA mixers carry a fixed-size state instead
// of a KV cache, so one decode step reads and rewrites that state once.  For a
// (sequence, head) with state S (d_v x d_k, fp32) and the token's q, k, v,
// gate alpha (scalar or per key channel) and beta, row r of S becomes
//
//     s~ = S[r,:] * alpha           (S Diag(alpha))
//     a  = s~ . k,   b = s~ . q
//     u  = beta (v_r - a)
//     S[r,:] = s~ + u k             (S~ (I - beta k k^T) + beta v k^T, row r)
//     o_r = S[r,:] . q = b + u (k . q)
//
// The step is bound by HBM: 2 * d_v * d_k * 4 bytes of state per token-head
// against ~4 flops per state element.  Layout: two warps per (sequence, head),
// each over half of the rows; a row is spread over LPR = 8 lanes holding DK/8 consecutive-in-
// float4 pieces each, so each warp instruction moves four whole rows with fully
// coalesced 128-bit loads and stores, and the two row dot products need only a
// 3-step shuffle reduction inside the 8-lane group.  ITER row groups are loaded
// before any is used, to keep enough bytes in flight to cover HBM latency.
// The state is streamed (evict-first) because one step's 0.5 GB of state does
// not fit in L2.

#include "checks.cuh"
#include "common.cuh"
#include "launch.h"

namespace gdr {
namespace {

constexpr int kDecodeWarps = 4;

// Two warps per (sequence, head), each updating half of its d_v rows (and loading q, k
// and the gates itself): 8192 states then make 4.6 waves of 4-warp CTAs instead of 2.3,
// and the last partial wave costs a smaller share of the step (measured on B200 with
// 256 x 32 states of 128 x 128: 185.6 -> 168.5 us per step; four warps per state 169.0).
constexpr int kRowShift = 1;

template <int DK, bool KDA, typename Tin, typename Tout>
__global__ void __launch_bounds__(kDecodeWarps * 32)
decode_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
              const Tin* __restrict__ v, const float* __restrict__ alpha,
              const float* __restrict__ beta, float* __restrict__ state,
              Tout* __restrict__ o, int NH, int dv, unsigned pro, int rshift,
              unsigned int* checks) {
  constexpr int LPR = 8;               // lanes per state row
  constexpr int RPW = 32 / LPR;        // rows per warp instruction
  constexpr int F4 = DK / (4 * LPR);   // float4 pieces per lane per row
  constexpr int ITER = 2;              // row groups in flight per warp
  static_assert(F4 >= 1, "d_k must be a multiple of 32");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // task = (sequence-head, part): the warp updates rows [part, part + 1) * (dv >> rshift)
  const int task = blockIdx.x * kDecodeWarps + warp;
  if (task >= (NH << rshift)) return;
  const long head = task >> rshift;
  const int part = task & ((1 << rshift) - 1);
  const int rows = dv >> rshift;
  // the row loop below covers [0, rows) in whole groups of RPW * ITER rows
  if (!dcheck((rows << rshift) == dv && rows % (RPW * ITER) == 0, checks, kCheckLayout)) return;
  const int sub = lane / LPR;          // which of the 4 rows of an instruction
  const int j = lane % LPR;            // position inside the row group

  // This lane owns channels 4p..4p+3 for p = j + LPR*m, m < F4.
  float kr[F4][4], qr[F4][4], ar[F4][4];
  const Tin* kh = k + head * DK;
  const Tin* qh = q + head * DK;
  float kq = 0.f, nk = 0.f, nq = 0.f;
#pragma unroll
  for (int m = 0; m < F4; ++m) {
    const int c = 4 * (j + LPR * m);
    float4 kk = Elem<Tin>::load4(kh + c);
    float4 qq = Elem<Tin>::load4(qh + c);
    kr[m][0] = kk.x; kr[m][1] = kk.y; kr[m][2] = kk.z; kr[m][3] = kk.w;
    qr[m][0] = qq.x; qr[m][1] = qq.y; qr[m][2] = qq.z; qr[m][3] = qq.w;
    if (KDA) {
      float4 aa = *reinterpret_cast<const float4*>(alpha + head * DK + c);
      ar[m][0] = aa.x; ar[m][1] = aa.y; ar[m][2] = aa.z; ar[m][3] = aa.w;
      if (pro & GDR_PROLOGUE_GATE_LOGIT) {
#pragma unroll
        for (int e = 0; e < 4; ++e) ar[m][e] = gate_from_logit(ar[m][e]);
      }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      nk = fmaf(kr[m][e], kr[m][e], nk);
      nq = fmaf(qr[m][e], qr[m][e], nq);
    }
  }
  if (pro & GDR_PROLOGUE_L2NORM_QK) {
    // the 8 lanes of a row group hold the whole vectors
#pragma unroll
    for (int off = 1; off < LPR; off <<= 1) {
      nk += __shfl_xor_sync(0xffffffffu, nk, off);
      nq += __shfl_xor_sync(0xffffffffu, nq, off);
    }
    const float sk = l2_scale(nk), sq = l2_scale(nq);
#pragma unroll
    for (int m = 0; m < F4; ++m)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        kr[m][e] = as_input<Tin>(kr[m][e] * sk);
        qr[m][e] = as_input<Tin>(qr[m][e] * sq);
      }
  }
#pragma unroll
  for (int m = 0; m < F4; ++m)
#pragma unroll
    for (int e = 0; e < 4; ++e) kq = fmaf(kr[m][e], qr[m][e], kq);
  kq += __shfl_xor_sync(0xffffffffu, kq, 1);
  kq += __shfl_xor_sync(0xffffffffu, kq, 2);
  kq += __shfl_xor_sync(0xffffffffu, kq, 4);
  const float a_s = KDA ? 1.f
                        : ((pro & GDR_PROLOGUE_GATE_LOGIT) ? gate_from_logit(alpha[head])
                                                           : alpha[head]);
  const float bt = beta[head];

  float* Sh = state + head * (long)dv * DK;
  const Tin* vh = v + head * (long)dv;
  Tout* oh = o + head * (long)dv;

  // this part's rows, as if they were the whole state
  Sh += (long)part * rows * DK;
  vh += part * rows;
  oh += part * rows;
  for (int r0 = 0; r0 < rows; r0 += RPW * ITER) {
    float4 s[ITER][F4];
    float vr[ITER];
#pragma unroll
    for (int it = 0; it < ITER; ++it) {
      const int row = r0 + it * RPW + sub;
#pragma unroll
      for (int m = 0; m < F4; ++m)
        s[it][m] = __ldcs(reinterpret_cast<const float4*>(Sh + (long)row * DK +
                                                          4 * (j + LPR * m)));
      vr[it] = Elem<Tin>::load(vh + row);
    }
#pragma unroll
    for (int it = 0; it < ITER; ++it) {
      const int row = r0 + it * RPW + sub;
      float pa = 0.f, pb = 0.f;
#pragma unroll
      for (int m = 0; m < F4; ++m) {
        float* e = reinterpret_cast<float*>(&s[it][m]);
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          e[x] *= KDA ? ar[m][x] : a_s;
          pa = fmaf(e[x], kr[m][x], pa);
          pb = fmaf(e[x], qr[m][x], pb);
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
#pragma unroll
        for (int x = 0; x < 4; ++x) e[x] = fmaf(u, kr[m][x], e[x]);
        __stcs(reinterpret_cast<float4*>(Sh + (long)row * DK + 4 * (j + LPR * m)), s[it][m]);
      }
      if (j == 0) Elem<Tout>::store(oh + row, fmaf(u, kq, pb));
    }
  }
}

template <int DK, bool KDA, typename Tin>
cudaError_t launch_t(const DecodeArgs& a, cudaStream_t st) {
  const int NH = a.N * a.H;
  const int rshift = kRowShift;
  const long tasks = (long)NH << rshift;
  const int grid = (int)((tasks + kDecodeWarps - 1) / kDecodeWarps);
  if (a.out_dtype == GDR_F32)
    decode_kernel<DK, KDA, Tin, float><<<grid, kDecodeWarps * 32, 0, st>>>(
        (const Tin*)a.q, (const Tin*)a.k, (const Tin*)a.v, a.alpha, a.beta, a.state,
        (float*)a.o, NH, a.dv, a.pro, rshift, checks_word());
  else
    decode_kernel<DK, KDA, Tin, __nv_bfloat16><<<grid, kDecodeWarps * 32, 0, st>>>(
        (const Tin*)a.q, (const Tin*)a.k, (const Tin*)a.v, a.alpha, a.beta, a.state,
        (__nv_bfloat16*)a.o, NH, a.dv, a.pro, rshift, checks_word());
  return cudaGetLastError();
}

template <int DK>
cudaError_t launch_dk(const DecodeArgs& a, cudaStream_t st) {
  if (a.in_dtype == GDR_F32)
    return a.kda ? launch_t<DK, true, float>(a, st) : launch_t<DK, false, float>(a, st);
  return a.kda ? launch_t<DK, true, __nv_bfloat16>(a, st)
               : launch_t<DK, false, __nv_bfloat16>(a, st);
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  switch (a.dk) {
    case 32: return launch_dk<32>(a, stream);
    case 64: return launch_dk<64>(a, stream);
    case 128: return launch_dk<128>(a, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace gdr
