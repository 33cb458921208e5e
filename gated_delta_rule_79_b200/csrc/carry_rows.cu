// The per-head state carry of the GDN and KDA two-kernel prefills (sm_100a, tcgen05):
// one CTA per (sequence, head) with the value rows in tensor-memory lanes.
//
// "Super Apriel: One Checkpoint, Many Speeds", §2A names the two mixers (delta rule with
// a scalar gate, GDN, and with a per-channel gate, KDA).  Once the prep kernel of either
// has left each chunk's state-independent operands in the workspace (chunk_image.cuh),
// what remains is the same for both: for a chunk entering with state S0 [d_v x d_k],
//
//   [O1; Y] = [Q~; K~] S0^T,  R = V - Y,  U = T R
//   O = O1 + P U
//   S <- S0 Diag(e^{G_last}) + U^T K^^T
//
// with Q~ = Q (.) e^G, K~ = K (.) e^G, K^ = (K (.) e^{G_last - G})^T.  This carry runs the
// products transposed, one value row v per TMEM lane:
//
//   D[v][t]       = sum_c S0[v][c] [Q~; K~][t][c]        (t < 64: O1^T, t >= 64: Y^T)
//   U^T[v][j]     = sum_i R^T[v][i] T[j][i]
//   S[v][c]      += sum_j U^T[v][j] K^[c][j]
//   O^T[v][t]    += sum_j U^T[v][j] P[t][j]
//
// so the state-dependent operand (S0, R^T, U^T) is always the A operand, read from tensor
// memory, and every B operand is a chunk image tile exactly as the prep stored it
// (K-major, 128-byte swizzled).  The state never leaves tensor memory between chunks: an
// fp32 copy accumulates and a tf32-rounded copy feeds the next chunk; the decay of the
// next chunk is applied in the same pass that rounds.  All d_v <= 128 value rows share the
// CTA (M = 128; rows past d_v stay zero), so the chunk operands are read once per head.
// A loader warp copies each operand group in as soon as the products that read the
// previous copy have completed.  While a chunk's first product runs, the carry warps
// stage the previous chunk's outputs in shared memory (one value column per thread);
// while its second runs, they store the staged token rows with coalesced 16-byte stores.
//
// The value-sliced carry (carry_sliced.cu) spreads one head over several SMs instead; it
// wins when there are too few (sequence, head) chains to fill the GPU.
//
// Precision: kind::tf32 products with every operand rounded to nearest.  Waits are
// bounded; a give-up records GDR_ERR_TIMEOUT in the workspace status word, drains what
// was issued, frees tensor memory and ends the CTA.

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

constexpr int kC = GDR_CHUNK;
constexpr int kDK = 128;
constexpr uint32_t kDrainLimit = 1u << 26;

constexpr int R_THREADS = 160;       // warps 0-3 carry and write outputs, warp 4 loads

// Shared memory: [Q~; K~] | e^{G_last}, T | v, K^ | P (one buffer each), output staging.
constexpr int L_A = 0;
constexpr int L_C = 66560;           // T (16 KB) | v bf16 [64 j][32 v] blocks
constexpr int L_V = L_C + 16384;
constexpr int L_D = L_C + 32768;     // K^ (32 KB) | P (16 KB)
constexpr int L_O = L_D + WS_D_BYTES;   // outputs [64 t][d_v], fp32 or bf16
constexpr int L_SMALL = L_O + 32768;
constexpr int L_SMEM = L_SMALL + 1024 + 1024;
static_assert(L_C >= WS_A_BYTES && L_C % 1024 == 0 && L_D % 1024 == 0, "tile alignment");
static_assert(L_SMEM <= 232448, "shared memory");

// Tensor memory (512 columns, lane = value row v): the fp32 state, its tf32 operand copy
// (whose first 64 columns hold R^T while a chunk runs), and two D buffers by chunk
// parity (columns 0-63 O^T, 64-127 Y^T and then U^T).
constexpr uint32_t T_S = 0, T_SR = 128, T_D = 256, T_COLS = 512;

constexpr int G_A = 0, G_C = 1, G_D = 2, NG = 3;   // operand groups

struct RowSmall {
  unsigned long long full[NG];      // the group's copy has landed
  unsigned long long empty[NG];     // the products that read the group have completed
  unsigned long long mma_bar;
  unsigned long long out_full[2];   // the chunk's O^T is complete in TMEM
  uint32_t tmem;
  int abort;
};

__device__ __forceinline__ void round32(float (&x)[32]) {
#pragma unroll
  for (int i = 0; i < 32; ++i) x[i] = to_tf32(x[i]);
}


template <typename Tout>
__global__ void __launch_bounds__(R_THREADS, 1)
row_carry_kernel(const __grid_constant__ CUtensorMap tm_v, const unsigned char* __restrict__ ws,
                 const float* __restrict__ s0, Tout* __restrict__ o, float* __restrict__ s_final,
                 const ChunkMap m, int H, int dv, unsigned int* __restrict__ status,
                 uint32_t spin_limit) {
  extern __shared__ unsigned char smem_raw[];
  const uint32_t padb = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  unsigned char* sm = smem_raw + padb;
  RowSmall& cs = *reinterpret_cast<RowSmall*>(sm + L_SMALL);
  uint64_t* full = reinterpret_cast<uint64_t*>(&cs.full[0]);
  uint64_t* empty = reinterpret_cast<uint64_t*>(&cs.empty[0]);
  uint64_t* mma_bar = reinterpret_cast<uint64_t*>(&cs.mma_bar);
  uint64_t* out_full = reinterpret_cast<uint64_t*>(&cs.out_full[0]);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x % H, seq = blockIdx.x / H;
  int first = 0, nchunks = 0;
  chunk_range(m, seq, first, nchunks);
  const int nvb = dv / 32;           // blocks of 32 value columns

  if (tid == 0) {
    for (int g = 0; g < NG; ++g) {
      mbar_init(full + g, 1);
      mbar_init(empty + g, 1);
    }
    mbar_init(mma_bar, 1);
    for (int s = 0; s < 2; ++s) mbar_init(out_full + s, 1);
    cs.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&cs.tmem, T_COLS);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tb = cs.tmem;
  const uint32_t tlane = (uint32_t)((warp & 3) * 32) << 16;
  const unsigned char* wsb = ws + m.img_base + ((size_t)h * m.nck + first) * kChunkWs;
  const uint32_t sbase_u = smem_u32(sm);

  auto give_up = [&](uint64_t* bar, uint32_t parity, bool drain) {
    if (drain) mbar_wait(bar, parity, kDrainLimit);
    atomicOr(status, 1u);
    cs.abort = 1;
  };

  if (warp == 4) {
    // =============================== loader =========================================
    if (lane == 0) {
      bool issued[NG] = {false, false, false};
      uint32_t last_par[NG] = {0, 0, 0};
      volatile int* abort_flag = &cs.abort;
      for (int c = 0; c < nchunks && !*abort_flag; ++c) {
        // each group: wait until the products that read its previous copy have completed
        // (the first use passes at once), then copy chunk c's part in
        const unsigned char* src = wsb + (size_t)c * kChunkWs;
        const uint32_t par = (uint32_t)c & 1u;
        const uint32_t dst[NG] = {sbase_u + L_A, sbase_u + L_C, sbase_u + L_D};
        const uint32_t off[NG] = {WS_QK, WS_T, WS_KH};
        const uint32_t bytes[NG] = {WS_A_BYTES, 16384, WS_D_BYTES};
        for (int g = 0; g < NG; ++g) {
          if (!mbar_wait(empty + g, par ^ 1u, spin_limit)) {
            give_up(empty + g, par ^ 1u, false);
            break;
          }
          mbar_expect_tx(full + g, bytes[g] + (g == G_C ? (uint32_t)(nvb * 4096) : 0u));
          bulk_load(dst[g], src + off[g], bytes[g], full + g);
          if (g == G_C) {
            const ChunkLoc loc = chunk_locate(m, first + c);
            for (int nb = 0; nb < nvb; ++nb)
              tma_load_4d(sbase_u + L_V + nb * 4096, &tm_v, 32 * nb, h, loc.t0, loc.b, full + g);
          }
          issued[g] = true;
          last_par[g] = par;
        }
        if (c + 1 < nchunks) bulk_prefetch_l2(src + kChunkWs, kChunkWs);
      }
      if (*abort_flag) {
        // copies issued here may still be landing in shared memory: let them finish (a
        // group's phases complete in order, so its last copy is the one to wait for)
        for (int g = 0; g < NG; ++g)
          if (issued[g]) mbar_wait(full + g, last_par[g], kDrainLimit);
      }
    }
  } else {
    // =========================== carry warpgroup ======================================
    const int v = tid;               // value row = TMEM lane
    const long srow = (((long)chunk_state_index(m, seq) * H + h) * dv + v) * kDK;
    const float4* egl = reinterpret_cast<const float4*>(sm + L_A + WS_EGL);
    uint32_t mphase = 0;
    const uint64_t dQK = sdesc(sbase_u + L_A, 16, 1024);
    const uint64_t dT = sdesc(sbase_u + L_C, 16, 1024);
    const uint64_t dKH = sdesc(sbase_u + L_D, 16, 1024);
    const uint64_t dP = sdesc(sbase_u + L_D + 32768, 16, 1024);
    const uint32_t i128 = idesc_tf32(128, 128, false, false);
    const uint32_t i64 = idesc_tf32(128, 64, false, false);
    auto wait_mma = [&]() -> bool {
      if (!mbar_wait(mma_bar, mphase, spin_limit)) give_up(mma_bar, mphase, true);
      mphase ^= 1u;
      fence_after_sync();
      named_bar(1, 128);
      return cs.abort != 0;
    };
    // S <- x (.) e^{G_last} (the decay of the chunk whose [Q~; K~] | e^{G_last} copy is in
    // shared memory) and the operand copy <- tf32(x), one block of 32 channels
    auto store_state = [&](int nb, float (&x)[32], bool decay) {
      float d[32];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float4 e = decay ? egl[8 * nb + q] : make_float4(1.f, 1.f, 1.f, 1.f);
        d[4 * q] = x[4 * q] * e.x;
        d[4 * q + 1] = x[4 * q + 1] * e.y;
        d[4 * q + 2] = x[4 * q + 2] * e.z;
        d[4 * q + 3] = x[4 * q + 3] * e.w;
      }
      tmem_st32(tb + tlane + T_S + 32 * nb, d);
      round32(x);
      tmem_st32(tb + tlane + T_SR + 32 * nb, x);
    };
    const unsigned char* vrow = sm + L_V + (v >> 5) * 4096 + (v & 31) * 2;
    const int rowb = dv * (int)sizeof(Tout);
    unsigned char* stage = sm + L_O;
    // O^T of chunk cc (D buffer cc & 1, columns 0-63) into the staging tile, one value
    // column per thread (the tile's previous rows were stored before the last barrier)
    auto stage_outputs = [&](int cc) {
      const uint32_t po = (uint32_t)cc & 1u, pu = (uint32_t)(cc >> 1) & 1u;
      if (!mbar_wait(out_full + po, pu, spin_limit)) give_up(out_full + po, pu, true);
      fence_after_sync();
      float ov[2][32];
      tmem_ld32(tb + tlane + T_D + 128 * po, ov[0]);
      tmem_ld32(tb + tlane + T_D + 128 * po + 32, ov[1]);
      tmem_wait_ld();
      if (v < dv) {
#pragma unroll
        for (int t = 0; t < kC; ++t) {
          if constexpr (sizeof(Tout) == 2)
            *reinterpret_cast<__nv_bfloat16*>(stage + t * rowb + 2 * v) =
                __float2bfloat16_rn(ov[t >> 5][t & 31]);
          else
            *reinterpret_cast<float*>(stage + t * rowb + 4 * v) = ov[t >> 5][t & 31];
        }
      }
    };
    // after a barrier: chunk cc's staged token rows (t < L) to the output, 16 bytes a thread
    auto store_rows = [&](int cc) {
      const ChunkLoc loc = chunk_locate(m, first + cc);
      const int lq = __ffs(rowb >> 4) - 1;       // log2 of the 16-byte pieces per row
      const int n = kC << lq;
      for (int i = tid; i < n; i += 128) {
        const int t = i >> lq, q = i & ((1 << lq) - 1);
        if (t < loc.L) {
          const uint4 x = *reinterpret_cast<const uint4*>(stage + t * rowb + 16 * q);
          *reinterpret_cast<uint4*>(reinterpret_cast<unsigned char*>(
              o + (((long)loc.b * m.T + loc.t0 + t) * H + h) * (long)dv) + 16 * q) = x;
        }
      }
    };
    bool aborted = false;
    // ---- the entering state (rows past d_v zero), decayed by the first chunk's gates -------
    // (a full barrier's copies are the loader's to drain, the products' are this group's)
    if (nchunks > 0 && !mbar_wait(full + G_A, 0, spin_limit)) give_up(full + G_A, 0, false);
    named_bar(1, 128);
    aborted = cs.abort != 0;
    if (!aborted) {
#pragma unroll
      for (int nb = 0; nb < 4; ++nb) {
        float x[32];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
          if (s0 && v < dv) f = *reinterpret_cast<const float4*>(s0 + srow + 32 * nb + 4 * q);
          x[4 * q] = f.x;
          x[4 * q + 1] = f.y;
          x[4 * q + 2] = f.z;
          x[4 * q + 3] = f.w;
        }
        store_state(nb, x, nchunks > 0);
      }
      tmem_wait_st();
    }
    fence_before_sync();
    named_bar(1, 128);
    for (int c = 0; c < nchunks && !aborted; ++c) {
      const uint32_t pc = (uint32_t)c & 1u;
      const uint32_t tD = T_D + 128u * pc;
      // [Q~; K~] has landed (waited for before the decay); this D buffer was read when the
      // outputs of chunk c - 2 were staged
      if ((aborted = cs.abort != 0)) break;
      fence_after_sync();
      // ---- D = S0 [Q~; K~]^T: O1^T and Y^T -------------------------------------------------
      if (warp == 0) {
#pragma unroll
        for (int ks = 0; ks < kDK / 8; ++ks)
          mma_tf32_ta_w(tb + tD, tb + T_SR + 8 * ks, kstep(dQK, 128, ks), i128, ks > 0);
        mma_commit_w(mma_bar);
        mma_commit_w(empty + G_A);
      }
      // ---- meanwhile: the previous chunk's outputs into the staging tile -------------------
      if (c > 0) stage_outputs(c - 1);
      fence_before_sync();
      if ((aborted = wait_mma())) break;
      // ---- R^T = V^T - Y^T, rounded, into the operand copy's first 64 columns ---------------
      if (!mbar_wait(full + G_C, pc, spin_limit)) give_up(full + G_C, pc, false);
      {
        float y[2][32];
        tmem_ld32(tb + tlane + tD + 64, y[0]);
        tmem_ld32(tb + tlane + tD + 96, y[1]);
        tmem_wait_ld();
#pragma unroll
        for (int nb = 0; nb < 2; ++nb) {
#pragma unroll
          for (int x = 0; x < 32; ++x) {
            const float vv = v < dv ? __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(
                                          vrow + (32 * nb + x) * 64))
                                    : 0.f;
            y[nb][x] = to_tf32(vv - y[nb][x]);
          }
          tmem_st32(tb + tlane + T_SR + 32 * nb, y[nb]);
        }
        tmem_wait_st();
      }
      fence_before_sync();
      named_bar(1, 128);
      // ---- U^T = R^T T^T, over Y^T in the D buffer -------------------------------------------
      if (warp == 0) {
        fence_after_sync();
#pragma unroll
        for (int ks = 0; ks < kC / 8; ++ks)
          mma_tf32_ta_w(tb + tD + 64, tb + T_SR + 8 * ks, kstep(dT, 64, ks), i64, ks > 0);
        mma_commit_w(mma_bar);
        mma_commit_w(empty + G_C);
      }
      // ---- meanwhile: the staged rows to the output ----------------------------------------
      if (c > 0) store_rows(c - 1);
      if ((aborted = wait_mma())) break;
      // ---- U^T rounded in place: it is the A operand of the two products below -------------
      {
        float u[2][32];
        tmem_ld32(tb + tlane + tD + 64, u[0]);
        tmem_ld32(tb + tlane + tD + 96, u[1]);
        tmem_wait_ld();
        round32(u[0]);
        round32(u[1]);
        tmem_st32(tb + tlane + tD + 64, u[0]);
        tmem_st32(tb + tlane + tD + 96, u[1]);
        tmem_wait_st();
      }
      fence_before_sync();
      named_bar(1, 128);
      // ---- S += U^T K^^T (the chain continues when it completes); O^T += U^T P^T -------------
      if (warp == 0) {
        if (lane == 0 && !mbar_wait(full + G_D, pc, spin_limit)) give_up(full + G_D, pc, false);
        __syncwarp();
        fence_after_sync();
#pragma unroll
        for (int ks = 0; ks < kC / 8; ++ks)
          mma_tf32_ta_w(tb + T_S, tb + tD + 64 + 8 * ks, kstep(dKH, 128, ks), i128, true);
        mma_commit_w(mma_bar);
#pragma unroll
        for (int ks = 0; ks < kC / 8; ++ks)
          mma_tf32_ta_w(tb + tD, tb + tD + 64 + 8 * ks, kstep(dP, 64, ks), i64, true);
        mma_commit_w(empty + G_D);
        mma_commit_w(out_full + pc);
      }
      // the next chunk's [Q~; K~] | e^{G_last} (its decay is applied below)
      const bool more = c + 1 < nchunks;
      if (more && !mbar_wait(full + G_A, pc ^ 1u, spin_limit)) give_up(full + G_A, pc ^ 1u, false);
      if ((aborted = wait_mma())) break;
      // ---- the new state: decayed for the next chunk, and rounded as its operand ----------
#pragma unroll
      for (int hb = 0; hb < 4; hb += 2) {
        float x[2][32];
        tmem_ld32(tb + tlane + T_S + 32 * hb, x[0]);
        tmem_ld32(tb + tlane + T_S + 32 * hb + 32, x[1]);
        tmem_wait_ld();
        store_state(hb, x[0], more);
        store_state(hb + 1, x[1], more);
      }
      tmem_wait_st();
      fence_before_sync();
      named_bar(1, 128);
    }
    if (!aborted && nchunks > 0) {
      stage_outputs(nchunks - 1);
      fence_before_sync();
      named_bar(1, 128);
      store_rows(nchunks - 1);
    }
    if (!aborted && s_final) {
      // the last pass left the state undecayed in S
#pragma unroll
      for (int nb = 0; nb < 4; ++nb) {
        float x[32];
        tmem_ld32(tb + tlane + T_S + 32 * nb, x);
        tmem_wait_ld();
        if (v < dv) {
#pragma unroll
          for (int q = 0; q < 8; ++q)
            *reinterpret_cast<float4*>(s_final + srow + 32 * nb + 4 * q) =
                make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
        }
      }
    }
    if (aborted) cs.abort = 1;
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tb, T_COLS);
}

}  // namespace

template <typename Tout>
cudaError_t launch_rows_t(const PrefillArgs& a, const ChunkMap& m, uint32_t lim,
                          cudaStream_t stream) {
  // packed sequences: the tensors are [1, total, H, *]
  const int TB = m.cu ? 1 : a.B;
  CUtensorMap mv;
  if (!encode_bthd_bf16(&mv, a.v, TB, a.T, a.H, a.dv, 32, kC, false)) return cudaErrorInvalidValue;
  auto carry = row_carry_kernel<Tout>;
  cudaError_t e = cudaFuncSetAttribute(carry, cudaFuncAttributeMaxDynamicSharedMemorySize, L_SMEM);
  if (e != cudaSuccess) return e;
  carry<<<m.nseq * a.H, R_THREADS, L_SMEM, stream>>>(mv, (const unsigned char*)a.workspace, a.s0,
                                                     (Tout*)a.o, a.s_final, m, a.H, a.dv,
                                                     (unsigned int*)a.workspace, lim);
  return cudaGetLastError();
}

cudaError_t launch_carry_rows(const PrefillArgs& a, const ChunkMap& m, uint32_t spin_limit,
                              cudaStream_t stream) {
  if (a.out_dtype == GDR_F32) return launch_rows_t<float>(a, m, spin_limit, stream);
  return launch_rows_t<__nv_bfloat16>(a, m, spin_limit, stream);
}

// The value-sliced carry while one 32-column slice per CTA still fits a single wave of
// SMs (a few long chains: several SMs share each head), else the per-head carry (it
// spends a quarter of the SM time per chunk).  GDR_CARRY=rows or GDR_CARRY=sliced picks
// one regardless.
cudaError_t launch_chunk_carry(const PrefillArgs& a, const ChunkMap& m, uint32_t spin_limit,
                               cudaStream_t stream) {
  const char* pick = getenv("GDR_CARRY");
  bool rows;
  if (pick && pick[0] == 'r') {
    rows = true;
  } else if (pick && pick[0] == 's') {
    rows = false;
  } else {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    rows = (long)m.nseq * a.H * (a.dv / 32) > sms;
  }
  return rows ? launch_carry_rows(a, m, spin_limit, stream)
              : launch_carry_sliced(a, m, spin_limit, stream);
}

size_t chunk_image_bytes() { return kChunkWs; }

}  // namespace gdr
