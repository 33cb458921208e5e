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
//   Y^T[v][j]     = sum_c S0[v][c] K~[j][c]        O1^T[v][t] = sum_c S0[v][c] Q~[t][c]
//   U^T[v][j]     = sum_i R^T[v][i] T[j][i]
//   S[v][c]      += sum_j U^T[v][j] K^[c][j]       O^T[v][t] += sum_j U^T[v][j] P[t][j]
//
// so the state-dependent operand (S0, R^T, U^T) is always the A operand, read from tensor
// memory, and every B operand is a chunk image tile exactly as the prep stored it
// (K-major, 128-byte swizzled).  The state never leaves tensor memory between chunks: an
// fp32 copy accumulates and a tf32-rounded copy feeds the next chunk; the decay of the
// next chunk is applied in the same pass that rounds.  All d_v <= 128 value rows share the
// CTA (M = 128; rows past d_v stay zero), so the chunk operands are read once per head.
//
// Only Y, U and the state update sit on the chain from one chunk to the next; the two
// output products (O1 and P U) are issued by the loader thread behind them, so that the
// tensor core runs them while the carry warps do the per-element passes.  Handshake
// barriers order those products against the chain's (O1 before U overwrites the operand
// copy's first columns, P U after U is rounded).  Eight carry warps (two per SM
// sub-partition, each pair splitting a value row's columns) run the per-element passes;
// while a chunk's Y product runs they stage the previous chunk's outputs in shared memory
// (one value column per thread) as the [64 token][d_v] tile that one TMA tensor store
// then writes (a packed sequence's partial last chunk, whose rows past its end belong to
// the next sequence, is stored row by row instead).
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

constexpr int R_THREADS = 288;       // warps 0-7 carry and write outputs, warp 8 loads
constexpr int R_CARRY = 256;         // carry threads: value row tid % 128, column half tid / 128
constexpr int R_STORER = 128;        // the carry thread that issues the output stores

// Shared memory: [Q~; K~] | e^{G_last}, T | v, K^ | P (one buffer each), output staging.
constexpr int L_A = 0;
constexpr int L_C = 66560;           // T (16 KB) | v bf16 [64 j][32 v] blocks
constexpr int L_V = L_C + 16384;
constexpr int L_D = L_C + 32768;     // K^ (32 KB) | P (16 KB)
constexpr int L_O = L_D + WS_D_BYTES;   // outputs [64 t][d_v], fp32 or bf16
constexpr int L_SMALL = L_O + 32768;
constexpr int L_SMEM = L_SMALL + 1024 + 1024;
static_assert(L_C >= WS_A_BYTES && L_C % 1024 == 0 && L_D % 1024 == 0, "tile alignment");
static_assert(L_O % 128 == 0, "TMA store source");
static_assert(L_SMEM <= 232448, "shared memory");

// Tensor memory (512 columns, lane = value row v): the fp32 state, its tf32 operand copy,
// and two D buffers by chunk parity.  In D: columns 0-63 O1^T and then O^T; columns
// 64-127 Y^T, then R^T (in place), then the rounded U^T.  U = T R lands in the operand
// copy's first 64 columns (the O1 product has read them by then) and is rounded into
// D, where it stays until the P U product has read it.
constexpr uint32_t T_S = 0, T_SR = 128, T_D = 256, T_COLS = 512;

constexpr int G_A = 0, G_C = 1, G_D = 2, NG = 3;   // operand groups

struct RowSmall {
  unsigned long long full[NG];      // the group's copy has landed
  unsigned long long empty[NG];     // the products that read the group have completed
  unsigned long long mma_bar;       // the chain's products (carry warps)
  unsigned long long out_full[2];   // the chunk's O^T is complete in TMEM
  unsigned long long y_issued;      // the Y product is issued (carry -> loader)
  unsigned long long o1_issued;     // the O1 product is issued (loader -> carry)
  unsigned long long u_ready;       // the rounded U is in D (carry -> loader)
  unsigned long long ld_done;       // the loader's products have completed (teardown)
  uint32_t tmem;
  int abort;
};

__device__ __forceinline__ void round32(float (&x)[32]) {
#pragma unroll
  for (int i = 0; i < 32; ++i) x[i] = to_tf32(x[i]);
}

// tcgen05 product with A in tensor memory, issued by the calling thread alone
__device__ __forceinline__ void mma_tf32_ta_1(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc,
                                              uint32_t idesc, bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}\n"
      :
      : "r"(tmem_d), "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate ? 1 : 0));
}

template <typename Tout>
__global__ void __launch_bounds__(R_THREADS, 1)
row_carry_kernel(const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                 const unsigned char* __restrict__ ws, const float* __restrict__ s0,
                 Tout* __restrict__ o, float* __restrict__ s_final, const ChunkMap m, int H,
                 int dv, unsigned int* __restrict__ status, uint32_t spin_limit) {
  extern __shared__ unsigned char smem_raw[];
  const uint32_t padb = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  unsigned char* sm = smem_raw + padb;
  RowSmall& cs = *reinterpret_cast<RowSmall*>(sm + L_SMALL);
  uint64_t* full = reinterpret_cast<uint64_t*>(&cs.full[0]);
  uint64_t* empty = reinterpret_cast<uint64_t*>(&cs.empty[0]);
  uint64_t* mma_bar = reinterpret_cast<uint64_t*>(&cs.mma_bar);
  uint64_t* out_full = reinterpret_cast<uint64_t*>(&cs.out_full[0]);
  uint64_t* y_issued = reinterpret_cast<uint64_t*>(&cs.y_issued);
  uint64_t* o1_issued = reinterpret_cast<uint64_t*>(&cs.o1_issued);
  uint64_t* u_ready = reinterpret_cast<uint64_t*>(&cs.u_ready);
  uint64_t* ld_done = reinterpret_cast<uint64_t*>(&cs.ld_done);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x % H, seq = blockIdx.x / H;
  int first = 0, nchunks = 0;
  chunk_range(m, seq, first, nchunks);
  if (!dcheck(dv <= 128, m.checks, kCheckImage)) nchunks = 0;
  const int nvb = dv / 32;           // blocks of 32 value columns

  if (tid == 0) {
    for (int g = 0; g < NG; ++g) {
      mbar_init(full + g, 1);
      // [Q~; K~] and K^ | P are each read by one product of the carry warps and one of
      // the loader: their copies are free after two arrivals
      mbar_init(empty + g, g == G_C ? 1 : 2);
    }
    mbar_init(mma_bar, 1);
    for (int s = 0; s < 2; ++s) mbar_init(out_full + s, 1);
    mbar_init(y_issued, 1);
    mbar_init(o1_issued, 1);
    mbar_init(u_ready, 1);
    mbar_init(ld_done, 1);
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
  // B operands: [Q~; K~] rows 0-63 (Q~) and 64-127 (K~) of each 128-row panel, T, K^, P
  const uint64_t dQ = sdesc(sbase_u + L_A, 16, 1024);
  const uint64_t dK = sdesc(sbase_u + L_A + 64 * 128, 16, 1024);
  const uint64_t dT = sdesc(sbase_u + L_C, 16, 1024);
  const uint64_t dKH = sdesc(sbase_u + L_D, 16, 1024);
  const uint64_t dP = sdesc(sbase_u + L_D + 32768, 16, 1024);
  const uint32_t i128 = idesc_tf32(128, 128, false, false);
  const uint32_t i64 = idesc_tf32(128, 64, false, false);

  auto give_up = [&](uint64_t* bar, uint32_t parity, bool drain) {
    if (drain) mbar_wait(bar, parity, kDrainLimit);
    atomicOr(status, 1u);
    cs.abort = 1;
  };

  if (warp == 8) {
    // =============================== loader =========================================
    // Copies each operand group in once what read its previous copy has completed, and
    // issues the two output products of every chunk (O1 behind the carry's Y product, P U
    // once U is rounded).
    if (lane == 0) {
      bool issued[NG] = {false, false, false};
      uint32_t last_par[NG] = {0, 0, 0};
      bool any_mma = false;
      volatile int* abort_flag = &cs.abort;
      // P U of chunk cc (its D buffer accumulates onto O1), then its outputs are complete
      auto issue_pu = [&](int cc) -> bool {
        const uint32_t pu = (uint32_t)cc & 1u;
        if (!mbar_wait(u_ready, pu, spin_limit)) {
          give_up(u_ready, pu, false);
          return false;
        }
        fence_after_sync();
        const uint32_t tD = T_D + 128u * pu;
#pragma unroll
        for (int ks = 0; ks < kC / 8; ++ks)
          mma_tf32_ta_1(tb + tD, tb + tD + 64 + 8 * ks, kstep(dP, 64, ks), i64, true);
        mma_commit(empty + G_D);
        mma_commit(out_full + pu);
        any_mma = true;
        return true;
      };
      for (int c = 0; c < nchunks && !*abort_flag; ++c) {
        const unsigned char* src = wsb + (size_t)c * kChunkWs;
        const uint32_t par = (uint32_t)c & 1u;
        const uint32_t dst[NG] = {sbase_u + L_A, sbase_u + L_C, sbase_u + L_D};
        const uint32_t off[NG] = {WS_QK, WS_T, WS_KH};
        const uint32_t bytes[NG] = {WS_A_BYTES, 16384, WS_D_BYTES};
        bool ok = true;
        for (int g = 0; g < NG && ok; ++g) {
          if (g == G_D && c > 0 && !issue_pu(c - 1)) {
            ok = false;
            break;
          }
          if (!mbar_wait(empty + g, par ^ 1u, spin_limit)) {
            give_up(empty + g, par ^ 1u, false);
            ok = false;
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
        if (!ok) break;
        if (c + 1 < nchunks) bulk_prefetch_l2(src + kChunkWs, kChunkWs);
        // O1 of chunk c, behind the carry's Y product (whose copy of [Q~; K~] it shares)
        if (!mbar_wait(y_issued, par, spin_limit)) {
          give_up(y_issued, par, false);
          break;
        }
        fence_after_sync();
        const uint32_t tD = T_D + 128u * par;
#pragma unroll
        for (int ks = 0; ks < kDK / 8; ++ks)
          mma_tf32_ta_1(tb + tD, tb + T_SR + 8 * ks, kstep(dQ, 128, ks), i64, ks > 0);
        mma_commit(empty + G_A);
        mma_commit(o1_issued);          // completes with O1: U may then overwrite its operand
        any_mma = true;
      }
      if (!*abort_flag && nchunks > 0) issue_pu(nchunks - 1);
      // the products issued here complete before tensor memory is freed
      if (any_mma) {
        mma_commit(ld_done);
        mbar_wait(ld_done, 0, kDrainLimit);
      }
      if (*abort_flag) {
        // copies issued here may still be landing in shared memory: let them finish (a
        // group's phases complete in order, so its last copy is the one to wait for)
        for (int g = 0; g < NG; ++g)
          if (issued[g]) mbar_wait(full + g, last_par[g], kDrainLimit);
      }
    }
  } else {
    // =========================== carry warpgroups =====================================
    const int v = tid & 127;         // value row = TMEM lane
    const int hf = tid >> 7;         // which half of the row's columns this thread owns
    const int sidx = chunk_state_index(m, seq);
    const long srow = (((long)max(sidx, 0) * H + h) * dv + v) * kDK;
    const float4* egl = reinterpret_cast<const float4*>(sm + L_A + WS_EGL);
    uint32_t mphase = 0;
    auto wait_mma = [&]() -> bool {
      if (!mbar_wait(mma_bar, mphase, spin_limit)) give_up(mma_bar, mphase, true);
      mphase ^= 1u;
      fence_after_sync();
      return named_bar_or(1, R_CARRY, cs.abort != 0);
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
    // column per thread (the tile's previous store has read it: see the end of a chunk).
    // Warp 0 is issuing the Y product meanwhile; warp 4 (the same TMEM lanes) does its share.
    auto stage_outputs = [&](int cc) {
      if (warp == 0) return;
      const uint32_t po = (uint32_t)cc & 1u, pu = (uint32_t)(cc >> 1) & 1u;
      if (!mbar_wait(out_full + po, pu, spin_limit)) give_up(out_full + po, pu, false);
      fence_after_sync();
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        if (hh == 1 && warp != 4) break;
        const int half = warp == 4 ? hh : hf;
        float ov[32];
        tmem_ld32(tb + tlane + T_D + 128 * po + 32 * half, ov);
        tmem_wait_ld();
        if (v < dv) {
#pragma unroll
          for (int x = 0; x < 32; ++x) {
            const int t = 32 * half + x;
            if constexpr (sizeof(Tout) == 2)
              *reinterpret_cast<__nv_bfloat16*>(stage + t * rowb + 2 * v) = __float2bfloat16_rn(ov[x]);
            else
              *reinterpret_cast<float*>(stage + t * rowb + 4 * v) = ov[x];
          }
        }
      }
      fence_smem_to_async();
    };
    // after a barrier: chunk cc's staged token rows (t < L) to the output: one TMA tensor
    // store (rows past the tensor's end are not written), or for a packed sequence's
    // partial chunk 16 bytes a thread
    auto store_rows = [&](int cc) {
      const ChunkLoc loc = chunk_locate(m, first + cc);
      if (!loc.valid) return;
      if (!m.cu || loc.L == kC) {
        if (tid == R_STORER) {
          tma_store_4d(&tm_o, smem_u32(stage), 0, h, loc.t0, loc.b);
          bulk_commit();
        }
        return;
      }
      const int lq = __ffs(rowb >> 4) - 1;       // log2 of the 16-byte pieces per row
      const int n = kC << lq;
      for (int i = tid; i < n; i += R_CARRY) {
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
    aborted = named_bar_or(1, R_CARRY, cs.abort != 0);
    if (!aborted) {
#pragma unroll
      for (int nh = 0; nh < 2; ++nh) {
        const int nb = 2 * hf + nh;
        float x[32];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
          if (s0 && v < dv && sidx >= 0)
            f = *reinterpret_cast<const float4*>(s0 + srow + 32 * nb + 4 * q);
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
    aborted = named_bar_or(1, R_CARRY, cs.abort != 0) || aborted;
    for (int c = 0; c < nchunks && !aborted; ++c) {
      const uint32_t pc = (uint32_t)c & 1u;
      const uint32_t tD = T_D + 128u * pc;
      // [Q~; K~] has landed (waited for before the decay); this D buffer was read when the
      // outputs of chunk c - 2 were staged (a give-up anywhere stops the loop at the barrier
      // that ends the previous chunk)
      fence_after_sync();
      // ---- Y^T = S0 K~^T (the loader issues O1^T = S0 Q~^T behind it) -----------------------
      if (warp == 0) {
#pragma unroll
        for (int ks = 0; ks < kDK / 8; ++ks)
          mma_tf32_ta_w(tb + tD + 64, tb + T_SR + 8 * ks, kstep(dK, 128, ks), i64, ks > 0);
        mma_commit_w(mma_bar);
        mma_commit_w(empty + G_A);
        if (lane == 0) mbar_arrive(y_issued);
      }
      // ---- meanwhile: the previous chunk's outputs into the staging tile -------------------
      if (c > 0) stage_outputs(c - 1);
      fence_before_sync();
      if ((aborted = wait_mma())) break;
      // ---- R^T = V^T - Y^T, rounded, in place of Y^T ----------------------------------------
      if (!mbar_wait(full + G_C, pc, spin_limit)) give_up(full + G_C, pc, false);
      {
        float y[32];
        tmem_ld32(tb + tlane + tD + 64 + 32 * hf, y);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          const float vv = v < dv ? __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(
                                        vrow + (32 * hf + x) * 64))
                                  : 0.f;
          y[x] = to_tf32(vv - y[x]);
        }
        tmem_st32(tb + tlane + tD + 64 + 32 * hf, y);
        tmem_wait_st();
      }
      fence_before_sync();
      named_bar(1, R_CARRY);
      // ---- U^T = R^T T^T into the operand copy's first columns, once O1 has read them ---------
      if (warp == 0) {
        if (lane == 0 && !mbar_wait(o1_issued, pc, spin_limit)) give_up(o1_issued, pc, false);
        __syncwarp();
        fence_after_sync();
#pragma unroll
        for (int ks = 0; ks < kC / 8; ++ks)
          mma_tf32_ta_w(tb + T_SR, tb + tD + 64 + 8 * ks, kstep(dT, 64, ks), i64, ks > 0);
        mma_commit_w(mma_bar);
        mma_commit_w(empty + G_C);
      }
      // ---- meanwhile: the staged rows to the output ----------------------------------------
      if (c > 0) store_rows(c - 1);
      if ((aborted = wait_mma())) break;
      // ---- U^T rounded into D (R^T's place): the A operand of S += U^T K^^T and of P U -------
      {
        float u[32];
        tmem_ld32(tb + tlane + T_SR + 32 * hf, u);
        tmem_wait_ld();
        round32(u);
        tmem_st32(tb + tlane + tD + 64 + 32 * hf, u);
        tmem_wait_st();
      }
      fence_before_sync();
      named_bar(1, R_CARRY);
      // ---- S += U^T K^^T (the chain continues when it completes; the loader adds P U) --------
      if (warp == 0) {
        if (lane == 0 && !mbar_wait(full + G_D, pc, spin_limit)) give_up(full + G_D, pc, false);
        __syncwarp();
        fence_after_sync();
#pragma unroll
        for (int ks = 0; ks < kC / 8; ++ks)
          mma_tf32_ta_w(tb + T_S, tb + tD + 64 + 8 * ks, kstep(dKH, 128, ks), i128, true);
        mma_commit_w(mma_bar);
        mma_commit_w(empty + G_D);
        if (lane == 0) mbar_arrive(u_ready);
      }
      // the next chunk's [Q~; K~] | e^{G_last} (its decay is applied below)
      const bool more = c + 1 < nchunks;
      if (more && !mbar_wait(full + G_A, pc ^ 1u, spin_limit)) give_up(full + G_A, pc ^ 1u, false);
      if ((aborted = wait_mma())) break;
      // ---- the new state: decayed for the next chunk, and rounded as its operand ----------
      {
        const int hb = 2 * hf;
        float x[2][32];
        tmem_ld32(tb + tlane + T_S + 32 * hb, x[0]);
        tmem_ld32(tb + tlane + T_S + 32 * hb + 32, x[1]);
        tmem_wait_ld();
        store_state(hb, x[0], more);
        store_state(hb + 1, x[1], more);
      }
      tmem_wait_st();
      if (tid == R_STORER) bulk_wait_read_all();   // the staging tile is free for the next chunk
      fence_before_sync();
      aborted = named_bar_or(1, R_CARRY, cs.abort != 0);
    }
    if (!aborted && nchunks > 0) {
      stage_outputs(nchunks - 1);
      fence_before_sync();
      named_bar(1, R_CARRY);
      store_rows(nchunks - 1);
    }
    if (!aborted && s_final) {
      // the last pass left the state undecayed in S
#pragma unroll
      for (int nh = 0; nh < 2; ++nh) {
        const int nb = 2 * hf + nh;
        float x[32];
        tmem_ld32(tb + tlane + T_S + 32 * nb, x);
        tmem_wait_ld();
        if (v < dv && sidx >= 0) {
#pragma unroll
          for (int q = 0; q < 8; ++q)
            *reinterpret_cast<float4*>(s_final + srow + 32 * nb + 4 * q) =
                make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
        }
      }
    }
    if (aborted) cs.abort = 1;
    if (tid == R_STORER) bulk_wait_all();    // the output stores read shared memory until done
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
  CUtensorMap mv, mo;
  if (!encode_bthd_bf16(&mv, a.v, TB, a.T, a.H, a.dv, 32, kC, false)) return cudaErrorInvalidValue;
  const bool out_ok =
      sizeof(Tout) == 2 ? encode_bthd_bf16(&mo, a.o, TB, a.T, a.H, a.dv, a.dv, kC, false)
                        : encode_bthd_f32(&mo, (const float*)a.o, TB, a.T, a.H, a.dv, a.dv, kC);
  if (!out_ok) return cudaErrorInvalidValue;
  auto carry = row_carry_kernel<Tout>;
  cudaError_t e = cudaFuncSetAttribute(carry, cudaFuncAttributeMaxDynamicSharedMemorySize, L_SMEM);
  if (e != cudaSuccess) return e;
  carry<<<m.nseq * a.H, R_THREADS, L_SMEM, stream>>>(mv, mo, (const unsigned char*)a.workspace, a.s0,
                                                     (Tout*)a.o, a.s_final, m, a.H, a.dv,
                                                     (unsigned int*)a.workspace, lim);
  return cudaGetLastError();
}

cudaError_t launch_carry_rows(const PrefillArgs& a, const ChunkMap& m, uint32_t spin_limit,
                              cudaStream_t stream) {
  if (a.out_dtype == GDR_F32) return launch_rows_t<float>(a, m, spin_limit, stream);
  return launch_rows_t<__nv_bfloat16>(a, m, spin_limit, stream);
}

}  // namespace gdr
