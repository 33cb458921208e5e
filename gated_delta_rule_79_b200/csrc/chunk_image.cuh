// The per-chunk operand images that both two-kernel prefills (GDN and KDA) leave in the
// workspace for the state carry (carry_rows.cu, carry_sliced.cu), and small helpers for the 128-byte-swizzled
// tf32 tiles they are stored as.  For chunk c of a sequence, with G the chunk-local
// cumulative log gate (per token for GDN, per token and key channel for KDA):
//   group A: [Q (.) e^G; K (.) e^G] (128 x 128) and e^{G_last} per key channel
//   group C: T = (I + A)^{-1} Diag(beta) (64 x 64)
//   group D: (K (.) e^{G_last - G})^T (128 x 64) and P (64 x 64)
// All tiles are tf32 (rounded to nearest), K-major, 128-byte swizzled, exactly as the
// tensor cores read them from shared memory, so the carry copies them in unchanged.
#pragma once

#include <stdint.h>

#include "tc.cuh"

namespace gdr {
namespace img {

constexpr int WS_QK = 0;                   // [Q~; K~] tf32 SW128, 128 rows x 128     64 KB
constexpr int WS_EGL = 65536;              // e^{G_last} per channel                 512 B
constexpr int WS_A_BYTES = 66048;
constexpr int WS_T = WS_A_BYTES;           // T tf32 SW128, 64 x 64                   16 KB
constexpr int WS_KH = WS_T + 16384;        // K^ tf32 SW128, 128 rows (c) x 64 (j)    32 KB
constexpr int WS_P = WS_KH + 32768;        // P tf32 SW128, 64 x 64                   16 KB
constexpr int WS_D_BYTES = 32768 + 16384;
constexpr int kChunkWs = WS_P + 16384;     // 131584 bytes per chunk

// Descriptor of k-step ks (8 tf32 or 16 bf16 elements of K) of a K-major SW128 tile.
__device__ __forceinline__ uint64_t kstep(uint64_t desc0, int rows, int ks) {
  return desc0 + (uint64_t)((((ks >> 2) * rows * 128) + ((ks & 3) * 32)) >> 4);
}

__device__ __forceinline__ void st_tile(unsigned char* tile, int rows, int r, int c, float x) {
  *reinterpret_cast<float*>(tile + tc::swz_off(r, c, rows)) = tc::to_tf32(x);
}

__device__ __forceinline__ float4 tf32x4(float a, float b, float c, float d) {
  return make_float4(tc::to_tf32(a), tc::to_tf32(b), tc::to_tf32(c), tc::to_tf32(d));
}

}  // namespace img
}  // namespace gdr
