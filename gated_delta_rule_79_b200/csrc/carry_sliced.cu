// The value-sliced state carry kernel of the GDN and KDA two-kernel prefills (its body is
// carry_sliced.cuh).  It is taken when there are
// too few (sequence, head) chains to fill the GPU; otherwise the per-head carry
// (carry_rows.cu) reads each chunk's operands once instead of once per slice.  NV = 64
// (two value slices sharing each chunk's operands) is taken when that still gives every
// SM a chain.

#include <stdlib.h>

#include "carry_sliced.cuh"
#include "launch.h"
#include "tma_host.h"

namespace gdr {
namespace {

using namespace tc;
using namespace sliced;

template <int NV, typename Tout>
__global__ void __launch_bounds__(C_THREADS, 1)
sliced_carry_kernel(const __grid_constant__ CUtensorMap tm_v,
                    const unsigned char* __restrict__ ws, const float* __restrict__ s0,
                    Tout* __restrict__ o, float* __restrict__ s_final, const ChunkMap m, int H,
                    int dv, unsigned int* __restrict__ status, uint32_t spin_limit) {
  using Lay = CarryLayout<NV>;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t padb = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  unsigned char* sm = smem_raw + padb;
  CarrySmall& cs = *reinterpret_cast<CarrySmall*>(sm + Lay::SMALL);
  const int tid = threadIdx.x;
  if (tid == 0) carry_init(cs);
  if (tid < 32) tmem_alloc(&cs.tmem, Lay::COLS);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tb = cs.tmem;
  carry_body<NV, Tout>(&tm_v, ws, s0, o, s_final, m, H, dv, status, spin_limit,
                       (int)blockIdx.x, sm, tb, tid);
  fence_before_sync();
  __syncthreads();
  if (tid < 32) tmem_dealloc(tb, Lay::COLS);
}

}  // namespace

template <typename Tout>
cudaError_t launch_sliced_t(const PrefillArgs& a, const ChunkMap& m, uint32_t lim,
                           cudaStream_t stream) {
  // packed sequences: the tensors are [1, total, H, *]
  const int TB = m.cu ? 1 : a.B;
  CUtensorMap mv;
  if (!encode_bthd_bf16(&mv, a.v, TB, a.T, a.H, a.dv, 32, kC, false)) return cudaErrorInvalidValue;
  cudaError_t e;
  // 64 value columns per CTA when that still gives every SM a chain (the chunk operands
  // are then shared by two slices), else 32
  const long ctas64 = (long)m.nseq * a.H * (a.dv / 64);
  int sms = 148;
  {
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess)
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  }
  if (a.dv % 64 == 0 && ctas64 >= sms) {
    auto carry = sliced_carry_kernel<64, Tout>;
    e = cudaFuncSetAttribute(carry, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             CarryLayout<64>::SMEM);
    if (e != cudaSuccess) return e;
    carry<<<m.nseq * a.H * (a.dv / 64), C_THREADS, CarryLayout<64>::SMEM, stream>>>(
        mv, (const unsigned char*)a.workspace, a.s0, (Tout*)a.o, a.s_final, m, a.H, a.dv,
        (unsigned int*)a.workspace, lim);
  } else {
    auto carry = sliced_carry_kernel<32, Tout>;
    e = cudaFuncSetAttribute(carry, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             CarryLayout<32>::SMEM);
    if (e != cudaSuccess) return e;
    carry<<<m.nseq * a.H * (a.dv / 32), C_THREADS, CarryLayout<32>::SMEM, stream>>>(
        mv, (const unsigned char*)a.workspace, a.s0, (Tout*)a.o, a.s_final, m, a.H, a.dv,
        (unsigned int*)a.workspace, lim);
  }
  return cudaGetLastError();
}

cudaError_t launch_carry_sliced(const PrefillArgs& a, const ChunkMap& m, uint32_t spin_limit,
                                cudaStream_t stream) {
  if (a.out_dtype == GDR_F32) return launch_sliced_t<float>(a, m, spin_limit, stream);
  return launch_sliced_t<__nv_bfloat16>(a, m, spin_limit, stream);
}


}  // namespace gdr
