// Second step of the two-segment state carry (sm_100a, tcgen05 + TMA): add the entering
// state's share to the second segment's outputs and form the final state.
//
// "Super Apriel: One Checkpoint, Many Speeds", §2A (the GDN / KDA recurrent mixers): the
// gated delta rule is linear in the state, so over a run of chunks S_out = S_in M + B and
// o_t = o_t(zero state) + S_in (M_t q_t), with M the run's transition and M_t the part of
// it up to token t.  The carry (carry_rows.cu, nseg = 2) ran the second half of each
// chain twice, from a zero state (outputs and final state B) and with the identity as its
// state rows and zero values (outputs M_t q_t, final state M, stored transposed), while
// the first half produced S_in.  This kernel finishes each chain:
//
//   o[t][v]       = O0[t][v] + sum_r Sin[v][r] OI[t][r]     (tokens of the second half)
//   S_final[v][c] = B[v][c]  + sum_r Sin[v][r] M[r][c]
//
// as M = 128 products on the tensor cores (kind::tf32; Sin, OI and M were rounded to tf32
// when the carry stored them), fed by TMA in the 128-byte-swizzled K-major layout: one CTA
// per 128 tokens of a chain (A = OI rows, B = Sin) and one per chain for the state
// (A = Sin, B = M^T).  Waits are bounded; a give-up records GDR_ERR_TIMEOUT in the
// workspace status word, drains and frees what the CTA holds.

#include <stdlib.h>

#include "chunk_image.cuh"
#include "chunkmap.cuh"
#include "common.cuh"
#include "launch.h"
#include "tc.cuh"
#include "tma_host.h"

namespace gdr {
namespace {

using namespace tc;
using namespace img;

constexpr int kDK = 128;
constexpr int F_THREADS = 128;
constexpr uint32_t kDrainLimit = 1u << 26;
constexpr int F_A = 0;              // A tile: 128 rows x 128 fp32, four 32-column panels   64 KB
constexpr int F_B = 65536;          // B tile: 128 rows x 128 fp32                         64 KB
constexpr int F_SMALL = 131072;
constexpr int F_SMEM = F_SMALL + 1024 + 1024;

// Tensor map over a row-major fp32 matrix [rows][128] whose boxes are 32 columns x 128 rows,
// 128-byte swizzled (one K panel of a tf32 operand tile); rows past the end read as zero.
bool encode_rows128(CUtensorMap* m, const float* base, long rows) {
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kDK, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kDK * 4};
  cuuint32_t box[2] = {32, 128};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, int c0, int c1,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];"
      :: "r"(dst), "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

struct FixSmall {
  unsigned long long tma_bar;
  unsigned long long mma_bar;
  uint32_t tmem;
};

// CTA (chain, p): p < npairs: tokens [128 p, 128 p + 128) of the chain's second segment;
// p == npairs: the chain's final state (only launched with s_final).
//   tm_out: the two output slabs as rows [2 BH t1p][128] (slab 0: from zero, slab 1: OI)
//   tm_st:  the states as rows [3 BH 128][128] (0: Sin, 1: B, 2: M^T)
template <typename Tout>
__global__ void __launch_bounds__(F_THREADS, 1)
segment_fixup_kernel(const __grid_constant__ CUtensorMap tm_out,
                     const __grid_constant__ CUtensorMap tm_st, const float* __restrict__ outs,
                     const float* __restrict__ states, Tout* __restrict__ o,
                     float* __restrict__ s_final, const ChunkMap m, int H, int dv, int t1p,
                     int npairs, unsigned int* __restrict__ status, uint32_t spin_limit) {
  extern __shared__ unsigned char smem_raw[];
  const uint32_t padb = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  unsigned char* sm = smem_raw + padb;
  FixSmall& fs = *reinterpret_cast<FixSmall*>(sm + F_SMALL);
  uint64_t* tma_bar = reinterpret_cast<uint64_t*>(&fs.tma_bar);
  uint64_t* mma_bar = reinterpret_cast<uint64_t*>(&fs.mma_bar);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int BH = m.nseq * H;
  const int chain = blockIdx.x / (npairs + 1), p = blockIdx.x % (npairs + 1);
  const int h = chain % H, seq = chain / H;
  const bool state_cta = p == npairs;
  int first = 0, nchunks = 0;
  chunk_range(m, seq, first, nchunks);
  const int n0 = (nchunks + 1) >> 1;
  const int sidx = chunk_state_index(m, seq);
  if (state_cta && (!s_final || sidx < 0)) return;
  const uint32_t sa = smem_u32(sm + F_A), sb = smem_u32(sm + F_B);
  if (tid == 0) {
    mbar_init(tma_bar, 1);
    mbar_init(mma_bar, 1);
    fence_mbar_init();
    mbar_expect_tx(tma_bar, 2u * 65536u);
    // A: OI rows (outputs) or Sin (state); B: Sin (outputs) or M^T (state)
    const int arow = state_cta ? chain * kDK : (BH + chain) * t1p + 128 * p;
    const int brow = state_cta ? (2 * BH + chain) * kDK : chain * kDK;
    const CUtensorMap* amap = state_cta ? &tm_st : &tm_out;
    for (int k = 0; k < 4; ++k) {
      tma_load_2d(sa + k * 16384, amap, 32 * k, arow, tma_bar);
      tma_load_2d(sb + k * 16384, &tm_st, 32 * k, brow, tma_bar);
    }
  }
  if (warp == 0) tmem_alloc(&fs.tmem, 128);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tb = fs.tmem;
  bool failed = false;
  if (!mbar_wait(tma_bar, 0, spin_limit)) {
    mbar_wait(tma_bar, 0, kDrainLimit);
    failed = true;
  }
  if (__syncthreads_or(failed)) {
    if (tid == 0) atomicOr(status, 1u);
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tb, 128);
    return;
  }
  const int ncols = state_cta ? kDK : dv;      // N of the product
  if (warp == 0) {
    const uint64_t dA = sdesc(sa, 16, 1024), dB = sdesc(sb, 16, 1024);
    const uint32_t id = idesc_tf32(128, ncols, false, false);
#pragma unroll
    for (int ks = 0; ks < kDK / 8; ++ks)
      mma_tf32_w(tb, kstep(dA, 128, ks), kstep(dB, 128, ks), id, ks > 0);
    mma_commit_w(mma_bar);
  }
  if (!mbar_wait(mma_bar, 0, spin_limit)) {
    mbar_wait(mma_bar, 0, kDrainLimit);
    failed = true;
  }
  fence_after_sync();
  if (__syncthreads_or(failed)) {
    if (tid == 0) atomicOr(status, 1u);
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tb, 128);
    return;
  }
  // row r of D (TMEM lane r) is this thread's: token r of the pair, or value row r
  const int r = 32 * warp + lane;
  const uint32_t tlane = (uint32_t)(32 * warp) << 16;
  if (state_cta) {
    if (r < dv) {
      const float* bsrc = states + ((size_t)BH + chain) * kDK * kDK + (size_t)r * kDK;
      float* dst = s_final + (((size_t)sidx * H + h) * dv + r) * kDK;
#pragma unroll 1
      for (int nb = 0; nb < kDK / 32; ++nb) {
        float d[32];
        tmem_ld32(tb + tlane + 32 * nb, d);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 bb = *reinterpret_cast<const float4*>(bsrc + 32 * nb + 4 * q);
          *reinterpret_cast<float4*>(dst + 32 * nb + 4 * q) =
              make_float4(d[4 * q] + bb.x, d[4 * q + 1] + bb.y, d[4 * q + 2] + bb.z,
                          d[4 * q + 3] + bb.w);
        }
      }
    } else {
#pragma unroll 1
      for (int nb = 0; nb < kDK / 32; ++nb) {
        float d[32];
        tmem_ld32(tb + tlane + 32 * nb, d);   // every warp takes part in the load
        tmem_wait_ld();
      }
    }
  } else {
    const int ts = 128 * p + r;                              // token of the second segment
    ChunkLoc loc{};
    bool live = false;
    if ((ts >> 6) < nchunks - n0) {
      loc = chunk_locate(m, first + n0 + (ts >> 6));
      live = loc.valid && (ts & 63) < loc.L;
    }
    const float* osrc = outs + ((size_t)chain * t1p + ts) * kDK;
    Tout* dst = o + (((long)loc.b * m.T + loc.t0 + (ts & 63)) * H + h) * (long)dv;
#pragma unroll 1
    for (int nb = 0; nb < dv / 32; ++nb) {
      float d[32];
      tmem_ld32(tb + tlane + 32 * nb, d);
      tmem_wait_ld();
      if (live) {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 z = *reinterpret_cast<const float4*>(osrc + 32 * nb + 4 * q);
          d[4 * q] += z.x;
          d[4 * q + 1] += z.y;
          d[4 * q + 2] += z.z;
          d[4 * q + 3] += z.w;
        }
        if constexpr (sizeof(Tout) == 2) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 pk;
            __nv_bfloat162* hp = reinterpret_cast<__nv_bfloat162*>(&pk);
#pragma unroll
            for (int x = 0; x < 4; ++x)
              hp[x] = __floats2bfloat162_rn(d[8 * q + 2 * x], d[8 * q + 2 * x + 1]);
            reinterpret_cast<uint4*>(dst + 32 * nb)[q] = pk;
          }
        } else {
#pragma unroll
          for (int q = 0; q < 8; ++q)
            reinterpret_cast<float4*>(dst + 32 * nb)[q] =
                make_float4(d[4 * q], d[4 * q + 1], d[4 * q + 2], d[4 * q + 3]);
        }
      }
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tb, 128);
}

template <typename Tout>
cudaError_t launch_fix_t(const PrefillArgs& a, const ChunkMap& m, uint32_t lim,
                         cudaStream_t stream, const SegmentBuffers& seg) {
  const int BH = m.nseq * a.H;
  const int nchunks = m.nchunks;
  const int n1 = nchunks - ((nchunks + 1) >> 1);
  const int npairs = (n1 + 1) / 2;
  CUtensorMap mo, ms;
  if (!encode_rows128(&mo, seg.outputs, 2L * BH * seg.t1p) ||
      !encode_rows128(&ms, seg.states, 3L * BH * kDK))
    return cudaErrorInvalidValue;
  auto fix = segment_fixup_kernel<Tout>;
  cudaError_t e = cudaFuncSetAttribute(fix, cudaFuncAttributeMaxDynamicSharedMemorySize, F_SMEM);
  if (e != cudaSuccess) return e;
  fix<<<BH * (npairs + 1), F_THREADS, F_SMEM, stream>>>(
      mo, ms, seg.outputs, seg.states, (Tout*)a.o, a.s_final, m, a.H, a.dv, seg.t1p, npairs,
      (unsigned int*)a.workspace, lim);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_segment_fixup(const PrefillArgs& a, const ChunkMap& m, uint32_t spin_limit,
                                 cudaStream_t stream, const SegmentBuffers& seg) {
  if (a.out_dtype == GDR_F32) return launch_fix_t<float>(a, m, spin_limit, stream, seg);
  return launch_fix_t<__nv_bfloat16>(a, m, spin_limit, stream, seg);
}

size_t segment_workspace_bytes(int B, int T, int H) {
  const long nchunks = ((long)T + GDR_CHUNK - 1) / GDR_CHUNK;
  const long n1 = nchunks - ((nchunks + 1) >> 1);
  const long BH = (long)B * H;
  if (BH > kSegMaxChains || nchunks < 2) return 0;
  return (size_t)(3 * BH * kDK * kDK * 4 + 2 * BH * (n1 * GDR_CHUNK) * kDK * 4);
}

}  // namespace gdr
