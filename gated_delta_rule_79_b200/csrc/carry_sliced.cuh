// The value-sliced state carry of the GDN and KDA chunked prefills (sm_100a, tcgen05):
// one CTA per (sequence, head, slice of NV value columns), so one head's carry runs on
// several SMs at once.
//
// "Super Apriel: One Checkpoint, Many Speeds", §2A names the two mixers (delta rule with
// a scalar gate, GDN, and with a per-channel gate, KDA).  Once a prep has left each
// chunk's state-independent operands in the workspace (chunk_image.cuh), what remains is
// the same for both: for a chunk entering with state S0,
//
//   [O1; Y] = [Q~; K~] S0^T,  R = V - Y,  U = T R
//   O = O1 + P U
//   S^T <- Diag(e^{G_last}) S0^T + K^ U
//
// with Q~ = Q (.) e^G, K~ = K (.) e^G, K^ = (K (.) e^{G_last - G})^T, each product with the
// chunk image tile as the A operand (M = 128 token or channel rows) and the value slice
// as N.  The loader warpgroup (warps 4-7) only copies: each operand group has its own
// full / empty barrier pair and is refilled for the next chunk as soon as the products
// that read it have completed; the loader also forms the outputs of the previous chunk.
// The carry warpgroup (warps 0-3) keeps the state as an fp32 TMEM accumulator and a tf32
// operand tile.
//
// carry_body is the whole of one carry CTA after its barriers are initialised and its
// tensor memory allocated (the kernel is carry_sliced.cu).
//
// Precision: kind::tf32 products with operands rounded to nearest.  Waits are bounded; a
// give-up records GDR_ERR_TIMEOUT in the workspace status word, drains what was issued
// and ends the carry.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "chunk_image.cuh"
#include "chunkmap.cuh"
#include "common.cuh"
#include "tc.cuh"

namespace gdr {
namespace sliced {

using namespace tc;
using namespace img;

constexpr int kC = GDR_CHUNK;
constexpr int kDK = 128;
constexpr uint32_t kDrainLimit = 1u << 26;

constexpr int C_THREADS = 256;               // warps 0-3 carry, warps 4-7 load

// Layout of one carry CTA over NV value columns (NV = 32 or 64).  Each operand group has
// one buffer and is refilled once the products that read it have completed.  R and U
// share one tile: U = T R has completed before U is written.
template <int NV>
struct CarryLayout {
  static constexpr int A = 0;                       // [Q~; K~] | e^{G_last}              66 KB
  static constexpr int C = 67584;                   // T (16 KB) | v bf16 [64 j][NV v]
  static constexpr int V = C + 16384;
  static constexpr int D = V + NV * 128;            // K^ (32 KB) | P (16 KB)
  static constexpr int SS = D + WS_D_BYTES;         // tf32 [NV v][128 c] state operand
  static constexpr int RU = SS + NV * 512;          // tf32 [NV v][64 j]: R, then U
  static constexpr int SMALL = RU + NV * 256;
  static constexpr int SMEM = SMALL + 1024 + 1024;
  // TMEM: [O1; Y] and P U are M = 128 (P U over P and 64 rows past it, whose results
  // are not read), so output row t is TMEM lane t for both; U is M = 64 (row j in lane
  // 32 (j / 16) + j % 16).  [O1; Y] and P U are double-buffered by chunk parity.
  static constexpr uint32_t OY = 0;                 // + NV * (c & 1)
  static constexpr uint32_t O2 = 2 * NV;            // + NV * (c & 1)
  static constexpr uint32_t U = 4 * NV;
  static constexpr uint32_t S = 5 * NV;             // S^T, M = 128
  static constexpr uint32_t COLS = NV == 32 ? 256 : 512;
  static_assert(C % 1024 == 0 && D % 1024 == 0 && SS % 1024 == 0 && RU % 1024 == 0,
                "tile alignment");
  static_assert(SMEM <= 232448, "shared memory");
  static_assert(6 * NV <= (int)COLS, "tensor memory");
};

constexpr int G_A = 0, G_C = 1, G_D = 2, NG = 3;   // operand groups

struct CarrySmall {
  unsigned long long full[NG];    // the group's copy has landed
  unsigned long long empty[NG];   // the products that read the group have completed
  unsigned long long mma_bar;
  unsigned long long out_full[2];   // chunk's O1 and P U are in TMEM (carry -> loader)
  unsigned long long out_empty[2];  // loader has read them (loader -> carry)
  uint32_t tmem;
  int abort;
};

// Thread 0 of a carry CTA, before the CTA-wide barrier that precedes carry_body.
__device__ __forceinline__ void carry_init(CarrySmall& cs) {
  for (int g = 0; g < NG; ++g) {
    mbar_init(reinterpret_cast<uint64_t*>(&cs.full[g]), 1);
    mbar_init(reinterpret_cast<uint64_t*>(&cs.empty[g]), 1);
  }
  mbar_init(reinterpret_cast<uint64_t*>(&cs.mma_bar), 1);
  for (int s = 0; s < 2; ++s) {
    mbar_init(reinterpret_cast<uint64_t*>(&cs.out_full[s]), 1);
    mbar_init(reinterpret_cast<uint64_t*>(&cs.out_empty[s]), 1);
  }
  cs.abort = 0;
  fence_mbar_init();
}

// One carry CTA: chain `chain` = (sequence, head, slice) in slice-fastest order, threads
// tid = 0..255 of the CTA, shared memory `sm` (1024-aligned, CarryLayout<NV>), tensor
// memory columns [tb, tb + CarryLayout<NV>::COLS).
template <int NV, typename Tout>
__device__ __forceinline__ void carry_body(const CUtensorMap* tm_v, const unsigned char* ws,
                                           const float* s0, Tout* o, float* s_final,
                                           const ChunkMap& m, int H, int dv,
                                           unsigned int* status, uint32_t spin_limit,
                                           int chain, unsigned char* sm, uint32_t tb,
                                           int tid) {
  using Lay = CarryLayout<NV>;
  constexpr int NB = NV / 32;        // blocks of 32 value columns
  CarrySmall& cs = *reinterpret_cast<CarrySmall*>(sm + Lay::SMALL);
  unsigned char* tSS = sm + Lay::SS;
  unsigned char* tRU = sm + Lay::RU;
  uint64_t* full = reinterpret_cast<uint64_t*>(&cs.full[0]);
  uint64_t* empty = reinterpret_cast<uint64_t*>(&cs.empty[0]);

  const int warp = tid >> 5, lane = tid & 31;
  const int q4 = warp & 3;
  const int nslice = dv / NV;
  const int slice = chain % nslice;
  const int sh = chain / nslice;
  const int h = sh % H, seq = sh / H;
  int first = 0, nchunks = 0;
  chunk_range(m, seq, first, nchunks);
  if (!dcheck(h < H && (slice + 1) * NV <= dv, m.checks, kCheckImage)) nchunks = 0;
  const int v0 = slice * NV;
  const uint32_t tlane = (uint32_t)(q4 * 32) << 16;
  const unsigned char* wsb = ws + m.img_base + ((size_t)h * m.nck + first) * kChunkWs;
  const uint32_t sbase_u = smem_u32(sm);

  auto give_up = [&](uint64_t* bar, uint32_t parity, bool drain) {
    if (drain) mbar_wait(bar, parity, kDrainLimit);
    atomicOr(status, 1u);
    cs.abort = 1;
  };

  if (warp >= 4) {
    // =========================== loader warpgroup =====================================
    const int lt = tid - 128;
    // O = O1 + P U of chunk cc: row t of both lies in TMEM lane t (warps 4 and 5)
    auto write_outputs = [&](int cc) -> bool {
      const int ob = cc & 1;
      const uint32_t use = (uint32_t)(cc >> 1);
      uint64_t* ofull = reinterpret_cast<uint64_t*>(&cs.out_full[ob]);
      if (lt == 0 && !mbar_wait(ofull, use & 1u, spin_limit)) give_up(ofull, use & 1u, false);
      if (named_bar_or(2, 128, cs.abort != 0)) return false;
      fence_after_sync();
      const ChunkLoc loc = chunk_locate(m, first + cc);
      const int t = 32 * q4 + lane;
      if (q4 < 2) {
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
          float o1[32], o2[32];
          tmem_ld32(tb + tlane + Lay::OY + NV * ob + 32 * nb, o1);
          tmem_ld32(tb + tlane + Lay::O2 + NV * ob + 32 * nb, o2);
          tmem_wait_ld();
          if (t < loc.L) {
            Tout* dst = o + (((long)loc.b * m.T + loc.t0 + t) * H + h) * (long)dv + v0 + 32 * nb;
            if constexpr (sizeof(Tout) == 2) {
#pragma unroll
              for (int qq = 0; qq < 4; ++qq) {
                uint4 pk;
                __nv_bfloat162* hp = reinterpret_cast<__nv_bfloat162*>(&pk);
#pragma unroll
                for (int x = 0; x < 4; ++x)
                  hp[x] = __floats2bfloat162_rn(o1[8 * qq + 2 * x] + o2[8 * qq + 2 * x],
                                                o1[8 * qq + 2 * x + 1] + o2[8 * qq + 2 * x + 1]);
                reinterpret_cast<uint4*>(dst)[qq] = pk;
              }
            } else {
#pragma unroll
              for (int qq = 0; qq < 8; ++qq)
                reinterpret_cast<float4*>(dst)[qq] =
                    make_float4(o1[4 * qq] + o2[4 * qq], o1[4 * qq + 1] + o2[4 * qq + 1],
                                o1[4 * qq + 2] + o2[4 * qq + 2], o1[4 * qq + 3] + o2[4 * qq + 3]);
            }
          }
        }
      }
      fence_before_sync();
      named_bar(2, 128);
      if (lt == 0) mbar_arrive(reinterpret_cast<uint64_t*>(&cs.out_empty[ob]));
      return true;
    };
    uint32_t pending = 0;      // thread lt == 0: groups with a copy issued, for draining
    uint32_t last_par = 0;
    for (int c = 0; c < nchunks; ++c) {
      if (lt == 0) {
        // each group: wait until the products that read it for chunk c-1 have completed
        // (the first use passes at once), then copy chunk c's part in
        const unsigned char* src = wsb + (size_t)c * kChunkWs;
        const uint32_t par = (uint32_t)c & 1u;
        const uint32_t dst[NG] = {sbase_u + Lay::A, sbase_u + Lay::C, sbase_u + Lay::D};
        const uint32_t off[NG] = {WS_QK, WS_T, WS_KH};
        const uint32_t bytes[NG] = {WS_A_BYTES, 16384, WS_D_BYTES};
        last_par = par;
        pending = 0;
        for (int g = 0; g < NG; ++g) {
          if (!mbar_wait(empty + g, par ^ 1u, spin_limit)) {
            give_up(empty + g, par ^ 1u, false);
            break;
          }
          mbar_expect_tx(full + g, bytes[g] + (g == G_C ? (uint32_t)(NV * 128) : 0u));
          bulk_load(dst[g], src + off[g], bytes[g], full + g);
          if (g == G_C) {
            const ChunkLoc loc = chunk_locate(m, first + c);
#pragma unroll
            for (int nb = 0; nb < NB; ++nb)
              tma_load_4d(sbase_u + Lay::V + nb * 4096, tm_v, v0 + 32 * nb, h, loc.t0, loc.b,
                          full + g);
          }
          pending |= 1u << g;
        }
        if (c + 1 < nchunks) bulk_prefetch_l2(src + kChunkWs, kChunkWs);
      }
      if (named_bar_or(2, 128, cs.abort != 0)) break;
      if (c > 0 && !write_outputs(c - 1)) break;
    }
    // one decision for the whole warpgroup (a give-up elsewhere may land between reads)
    const bool ab = named_bar_or(2, 128, cs.abort != 0);
    if (ab && lt == 0) {
      // copies this thread issued may still be landing in shared memory: let them finish
      for (int g = 0; g < NG; ++g)
        if (pending & (1u << g)) mbar_wait(full + g, last_par, kDrainLimit);
    }
    if (!ab && nchunks > 0) write_outputs(nchunks - 1);
  } else {
    // =========================== carry warpgroup ======================================
    const int sidx = chunk_state_index(m, seq);
    const long sbase = ((long)max(sidx, 0) * H + h) * (long)dv * kDK;
    float st[NV];
#pragma unroll
    for (int vv = 0; vv < NV; ++vv)
      st[vv] = (s0 && sidx >= 0) ? s0[sbase + (long)(v0 + vv) * kDK + tid] : 0.f;
    auto write_state_operand = [&]() {
#pragma unroll
      for (int vv = 0; vv < NV; ++vv) st_tile(tSS, NV, vv, tid, st[vv]);
    };
    write_state_operand();
    fence_smem_to_async();
    uint64_t* mma_bar = reinterpret_cast<uint64_t*>(&cs.mma_bar);
    uint32_t mphase = 0;
    const uint64_t dSS = sdesc(smem_u32(tSS), 16, 1024);
    const uint64_t dRU = sdesc(smem_u32(tRU), 16, 1024);
    const uint64_t dQK = sdesc(sbase_u + Lay::A, 16, 1024), dT = sdesc(sbase_u + Lay::C, 16, 1024);
    const uint64_t dKH = sdesc(sbase_u + Lay::D, 16, 1024);
    const uint64_t dP = sdesc(sbase_u + Lay::D + 32768, 16, 1024);
    const uint32_t i64 = idesc_tf32(64, NV, false, false);
    const uint32_t i128 = idesc_tf32(128, NV, false, false);
    const float* egl = reinterpret_cast<const float*>(sm + Lay::A + WS_EGL);
    auto wait_mma = [&]() -> bool {
      if (!mbar_wait(mma_bar, mphase, spin_limit)) give_up(mma_bar, mphase, true);
      mphase ^= 1u;
      fence_after_sync();
      return named_bar_or(1, 128, cs.abort != 0);
    };
    bool aborted = false;
    for (int c = 0; c < nchunks; ++c) {
      const uint32_t par = (uint32_t)c & 1u;
      const int ob = c & 1;
      // ---- group A has landed; the output buffer is free ----------------------------------
      if (tid == 0) {
        if (!mbar_wait(full + G_A, par, spin_limit)) give_up(full + G_A, par, true);
        if (c >= 2) {
          uint64_t* oe = reinterpret_cast<uint64_t*>(&cs.out_empty[ob]);
          const uint32_t p2 = (uint32_t)((c >> 1) - 1) & 1u;
          if (!mbar_wait(oe, p2, spin_limit)) give_up(oe, p2, false);
        }
      }
      if ((aborted = named_bar_or(1, 128, cs.abort != 0))) break;
      fence_after_sync();
      // ---- decay the state in TMEM, then [O1; Y] = [Q~; K~] S0^T -----------------------------
      {
        const float e = egl[tid];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
          float sd[32];
#pragma unroll
          for (int vv = 0; vv < 32; ++vv) sd[vv] = st[32 * nb + vv] * e;
          tmem_st32(tb + tlane + Lay::S + 32 * nb, sd);
        }
        tmem_wait_st();
      }
      fence_before_sync();
      named_bar(1, 128);
      if (warp == 0) {
        fence_after_sync();
#pragma unroll
        for (int ks = 0; ks < kDK / 8; ++ks)
          mma_tf32_w(tb + Lay::OY + NV * ob, kstep(dQK, 128, ks), kstep(dSS, NV, ks), i128, ks > 0);
        mma_commit_w(mma_bar);
        mma_commit_w(empty + G_A);
      }
      if ((aborted = wait_mma())) break;
      // ---- R = V - Y as the operand [v][j] (Y rows: TMEM lanes 64-127) --------------------
      if (q4 >= 2) {
        if (!mbar_wait(full + G_C, par, spin_limit)) give_up(full + G_C, par, true);
        const int j = 32 * (q4 - 2) + lane;
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
          float y[32], vv[32];
          tmem_ld32(tb + tlane + Lay::OY + NV * ob + 32 * nb, y);
          const uint4* vrow = reinterpret_cast<const uint4*>(sm + Lay::V + nb * 4096 + j * 64);
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) {
            const uint4 raw = vrow[qq];
            const __nv_bfloat162* hh = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
            for (int x = 0; x < 4; ++x) {
              const float2 f = __bfloat1622float2(hh[x]);
              vv[8 * qq + 2 * x] = f.x;
              vv[8 * qq + 2 * x + 1] = f.y;
            }
          }
          tmem_wait_ld();
#pragma unroll
          for (int v = 0; v < 32; ++v) st_tile(tRU, NV, 32 * nb + v, j, vv[v] - y[v]);
        }
      }
      fence_smem_to_async();
      fence_before_sync();
      named_bar(1, 128);
      // ---- U = T R ---------------------------------------------------------------------------
      if (warp == 0) {
        fence_after_sync();
#pragma unroll
        for (int ks = 0; ks < kC / 8; ++ks)
          mma_tf32_w(tb + Lay::U, kstep(dT, 64, ks), kstep(dRU, NV, ks), i64, ks > 0);
        mma_commit_w(mma_bar);
        mma_commit_w(empty + G_C);
      }
      if ((aborted = wait_mma())) break;
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        float u[32];
        tmem_ld32(tb + tlane + Lay::U + 32 * nb, u);
        tmem_wait_ld();
        if (lane < 16) {
          const int j = 16 * q4 + lane;
#pragma unroll
          for (int v = 0; v < 32; ++v) st_tile(tRU, NV, 32 * nb + v, j, u[v]);
        }
      }
      fence_smem_to_async();
      fence_before_sync();
      named_bar(1, 128);
      // ---- S^T += K^ U (the chain continues when it completes); O2 = P U behind it ---------
      if (warp == 0) {
        if (lane == 0 && !mbar_wait(full + G_D, par, spin_limit)) give_up(full + G_D, par, true);
        __syncwarp();
        fence_after_sync();
#pragma unroll
        for (int ks = 0; ks < kC / 8; ++ks)
          mma_tf32_w(tb + Lay::S, kstep(dKH, 128, ks), kstep(dRU, NV, ks), i128, true);
        mma_commit_w(mma_bar);
        // M = 128 over P: rows 64-127 read past P and land in lanes 64-127, never read
#pragma unroll
        for (int ks = 0; ks < kC / 8; ++ks)
          mma_tf32_w(tb + Lay::O2 + NV * ob, kstep(dP, 64, ks), kstep(dRU, NV, ks), i128, ks > 0);
        mma_commit_w(empty + G_D);
        mma_commit_w(reinterpret_cast<uint64_t*>(&cs.out_full[ob]));
      }
      if ((aborted = wait_mma())) break;
      // ---- new state ---------------------------------------------------------------------------
#pragma unroll
      for (int nb = 0; nb < NB; ++nb)
        tmem_ld32(tb + tlane + Lay::S + 32 * nb, *reinterpret_cast<float(*)[32]>(&st[32 * nb]));
      tmem_wait_ld();
      write_state_operand();
      fence_smem_to_async();
      fence_before_sync();
      named_bar(1, 128);
    }
    if (!aborted && s_final && sidx >= 0) {
#pragma unroll
      for (int vv = 0; vv < NV; ++vv) s_final[sbase + (long)(v0 + vv) * kDK + tid] = st[vv];
    }
    if (aborted) cs.abort = 1;
  }
}

}  // namespace sliced
}  // namespace gdr
