// X = (I + A)^{-1} for the 64 x 64 strictly lower triangular A of one chunk, on the
// CUDA cores, shared by both preps.
//
// "Super Apriel: One Checkpoint, Many Speeds", §2A (GDN and KDA mixers): the chunked
// delta rule needs T = (I + A)^{-1} Diag(beta), A[t][j] = beta_t k_t . (Gamma_t/Gamma_j) k_j
// for j < t.  With A cut into 16 x 16 blocks A[a][m] (a, m = 0..3) the inverse X is block
// lower triangular, with
//
//   X[a][a] = (I + A[a][a])^{-1}                                 (forward substitution)
//   X[a][b] = -X[a][a] sum_{m=b}^{a-1} A[a][m] X[m][b]           (a > b)
//
// Column block b of X depends only on A and on the diagonal blocks, so after the four
// diagonal inverses (one warp each) warp b walks its own column block down the rows
// a = b+1 .. 3 with no barrier between the steps; each lane keeps a 4 x 2 tile of the
// 16 x 16 block in registers.
//
// Layout of A and X in shared memory: [64][64] fp32 rows of 64, each row's sixteen
// 16-byte pieces permuted by piece ^ (row % 8) (at, at4): a warp storing one row per
// lane in 16-byte pieces, and a quarter-warp reading one row in 16-byte pieces, meet no
// bank conflicts.  Only the strictly lower part of A (with the diagonal blocks' strictly
// lower parts) is read; the blocks (b, 3), b < 3, above the block diagonal hold warp b's
// 16 x 16 scratch.  X's blocks above the block diagonal are not written (they are zero).
#pragma once

namespace gdr {
namespace solve64 {

// Index of element (r, c) of a [64][64] tile in the layout above.
__device__ __forceinline__ int at(int r, int c) {
  return r * 64 + (((c >> 2) ^ (r & 7)) << 2) + (c & 3);
}

// Float offset of the 16-byte piece holding elements (r, 4q .. 4q+3).
__device__ __forceinline__ int at4(int r, int q) {
  return r * 64 + ((q ^ (r & 7)) << 2);
}

// Phase 1, warps 0-3 of the group (warp w inverts diagonal block w; lanes 16-31 idle):
// X[w][w] with its upper triangle set to zero.
__device__ __forceinline__ void diag(const float* __restrict__ As, float* __restrict__ Xs, int w,
                                     int lane) {
  if (lane >= 16) return;
  const int base = 16 * w, jl = lane;
  float x[16];
#pragma unroll
  for (int tl = 0; tl < 16; ++tl) {
    float acc0 = (tl == jl) ? 1.f : 0.f, acc1 = 0.f;
#pragma unroll
    for (int i = 0; i < tl; i += 2) {
      acc0 = fmaf(-As[at(base + tl, base + i)], x[i], acc0);
      if (i + 1 < tl) acc1 = fmaf(-As[at(base + tl, base + i + 1)], x[i + 1], acc1);
    }
    x[tl] = (tl < jl) ? 0.f : acc0 + acc1;
  }
#pragma unroll
  for (int tl = 0; tl < 16; ++tl) Xs[at(base + tl, base + jl)] = x[tl];
}

// Phase 2, after a barrier that follows phase 1; warp w (0..2) fills column block w of X
// below the diagonal.  `As` is written only in warp w's scratch block (w, 3).
__device__ __forceinline__ void offdiag(float* __restrict__ As, float* __restrict__ Xs, int w,
                                        int lane) {
  if (w >= 3) return;
  const int b = w;
  const int rg = lane >> 3, cg = lane & 7;        // rows 4 rg .. 4 rg + 3, columns 2 cg, 2 cg + 1
  const int c0 = 16 * b + 2 * cg;                 // this lane's first column of X
  for (int a = b + 1; a < 4; ++a) {
    // Z = sum_{m=b}^{a-1} A[a][m] X[m][b]  (16 x 16, this lane's 4 x 2)
    float z[4][2];
#pragma unroll
    for (int p = 0; p < 4; ++p) z[p][0] = z[p][1] = 0.f;
    for (int k = 16 * b; k < 16 * a; k += 4) {
      float4 ar[4];
#pragma unroll
      for (int p = 0; p < 4; ++p)
        ar[p] = *reinterpret_cast<const float4*>(As + at4(16 * a + 4 * rg + p, k >> 2));
      float2 xk[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) xk[u] = *reinterpret_cast<const float2*>(Xs + at(k + u, c0));
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const float av[4] = {ar[p].x, ar[p].y, ar[p].z, ar[p].w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          z[p][0] = fmaf(av[u], xk[u].x, z[p][0]);
          z[p][1] = fmaf(av[u], xk[u].y, z[p][1]);
        }
      }
    }
    // Z to the warp's scratch block (rows 16 b + i, columns 48 + j), then X[a][b] = -X[a][a] Z
#pragma unroll
    for (int p = 0; p < 4; ++p)
      *reinterpret_cast<float2*>(As + at(16 * b + 4 * rg + p, 48 + 2 * cg)) =
          make_float2(z[p][0], z[p][1]);
    __syncwarp();
    float x[4][2];
#pragma unroll
    for (int p = 0; p < 4; ++p) x[p][0] = x[p][1] = 0.f;
#pragma unroll
    for (int i = 0; i < 16; i += 4) {
      float4 dr[4];
#pragma unroll
      for (int p = 0; p < 4; ++p)
        dr[p] = *reinterpret_cast<const float4*>(Xs + at4(16 * a + 4 * rg + p, (16 * a + i) >> 2));
      float2 zk[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        zk[u] = *reinterpret_cast<const float2*>(As + at(16 * b + i + u, 48 + 2 * cg));
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const float dv[4] = {dr[p].x, dr[p].y, dr[p].z, dr[p].w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          x[p][0] = fmaf(dv[u], zk[u].x, x[p][0]);
          x[p][1] = fmaf(dv[u], zk[u].y, x[p][1]);
        }
      }
    }
#pragma unroll
    for (int p = 0; p < 4; ++p)
      *reinterpret_cast<float2*>(Xs + at(16 * a + 4 * rg + p, c0)) = make_float2(-x[p][0], -x[p][1]);
    __syncwarp();   // X[a][b] is read by the next step; the scratch is rewritten by it
  }
}

}  // namespace solve64
}  // namespace gdr
