// The chained state carry of the GDN and KDA two-kernel prefills (sm_100a, tcgen05): one
// CTA per (sequence, head), the state and every per-chunk intermediate kept in tensor
// memory, and each product of the chunk-to-chunk chain fed straight by the one before it.
//
// "Super Apriel: One Checkpoint, Many Speeds", §2A names the two mixers (delta rule with
// a scalar gate, GDN, and with a per-channel gate, KDA).  Once the prep kernel of either
// has left each chunk's state-independent operands in the workspace (chunk_image.cuh),
// what remains is the same for both.  With one value row v per tensor-memory lane, a
// chunk entering with state S_c [d_v x d_k] takes
//
//   R^T     = V^T - S_c K~^T                 (V^T preloaded, the product's A negated)
//   O^T     = S_c Q~^T
//   U^T     = R^T T^T
//   S_{c+1} = S_c Diag(e^{G_last}) + U^T K^^T
//   O^T    += U^T P^T
//
// with Q~ = Q (.) e^G, K~ = K (.) e^G, K^ = (K (.) e^{G_last - G})^T and T = (I + A)^{-1}
// Diag(beta).  Every state-dependent operand (S_c, R^T, U^T) is the A operand, read from
// the fp32 accumulator that the previous product left in tensor memory, and every B
// operand is a chunk image tile exactly as the prep stored it.  So the chain from one
// chunk to the next is three products (R, U, S) with only a completion wait between
// them; the CUDA cores work beside the chain: they preload V^T for the next chunk, write
// the decayed copy S_c Diag(e^{G_last}) into the second state buffer (which the S product
// then accumulates onto) while the R and O products read S_c, and store the outputs.  The
// two output products fill the tensor pipe while the issuing warp waits for R and U.
//
// Roles: warps 0-3 the chain's per-element passes (V^T preload, decayed state copy; value
// row = lane of the warp's sub-partition), warps 4-7 the outputs, warp 8 the loader (bulk
// copies of the chunk images, the V tiles by TMA, L2 prefetch two chunks ahead), warp 9
// the issuing warp.  [Q~; K~] and e^{G_last} are double-buffered; T, V, and K^ | P have
// one buffer each, refilled as soon as what reads them has completed.  The outputs leave
// through shared memory, one TMA tensor store per chunk (scattered 2-byte stores from every
// thread cost several times more).
//
// Precision: kind::tf32 products.  The B operands were rounded to tf32 by the prep; the A
// operands are fp32 accumulators, of which the tensor cores use the tf32 part (the lower
// 13 mantissa bits are not rounded in first).  The state itself accumulates in fp32.
// Waits are bounded; a give-up records GDR_ERR_TIMEOUT in the workspace status word,
// drains what was issued, frees tensor memory and ends the CTA.

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

#ifndef GDR_CHAIN_PREFETCH
#define GDR_CHAIN_PREFETCH 2
#endif
constexpr int kPrefetch = GDR_CHAIN_PREFETCH;   // chunks the loader prefetches into L2 ahead
constexpr int K_THREADS = 320;       // warps 0-7 per-element passes, 8 loader, 9 issuer
constexpr int K_LANES = 256;

// Shared memory: the [Q~; K~] tiles twice, T, K^ | P, V (bf16 [64 t][32 v] blocks: one
// TMA box per 32 value columns, which lands sooner than a single box of 64 long rows),
// e^{G_last} twice, the barriers, and the 16 KB output staging tile.
constexpr int K_A0 = 0;
constexpr int K_A1 = WS_EGL;                  // 64 KB
constexpr int K_T = 2 * WS_EGL;
constexpr int K_D = K_T + 16384;
constexpr int K_V = K_D + WS_D_BYTES;
constexpr int K_EGL = K_V + 16384;
constexpr int K_SMALL = K_EGL + 1024;
constexpr int K_STAGE = K_SMALL + 256;
constexpr int K_SMEM = K_STAGE + 16384 + 1024;
static_assert(K_A1 % 1024 == 0 && K_T % 1024 == 0 && K_D % 1024 == 0 && K_V % 128 == 0,
              "tile alignment");
static_assert(K_STAGE % 128 == 0, "TMA store source");
static_assert(K_SMEM <= 232448, "shared memory");

// Tensor memory (512 columns, lane = value row v): two state buffers (S_c and the next
// state by chunk parity), two O^T buffers by chunk parity, R^T and U^T.
constexpr uint32_t T_S = 0, T_O = 256, T_R = 384, T_U = 448, T_COLS = 512;

struct ChainSmall {
  unsigned long long full_a[2];   // [Q~; K~] and e^{G_last} buffer has landed
  unsigned long long empty_a[2];  // ... and its readers are done (products + decay pass)
  unsigned long long full_t, empty_t;
  unsigned long long full_v, empty_v;
  unsigned long long full_d, empty_d;
  unsigned long long r_done;      // the R^T product has completed
  unsigned long long u_done;      // the U^T product has completed (R^T is free)
  unsigned long long s_done;      // the state product has completed
  unsigned long long out_full[2]; // the chunk's O^T is complete
  unsigned long long out_free[2]; // ... and has been read
  unsigned long long v_ready;     // V^T is preloaded into R^T's columns
  unsigned long long d_ready;     // the decayed state copy is written
  unsigned long long s0_ready;    // the entering state is in tensor memory
  unsigned long long drained;     // every product of the issuing warp has completed
  uint32_t tmem;
  int abort;
};
static_assert(sizeof(ChainSmall) <= 256, "small area");

template <typename Tout>
__device__ __forceinline__ Tout out_cast(float x);
template <>
__device__ __forceinline__ float out_cast<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 out_cast<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

template <typename Tout>
__global__ void __launch_bounds__(K_THREADS, 1)
chain_carry_kernel(const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                   const unsigned char* __restrict__ ws,
                   const float* __restrict__ s0, Tout* __restrict__ o,
                   float* __restrict__ s_final, const ChunkMap m, int H, int dv,
                   unsigned int* __restrict__ status, uint32_t spin_limit) {
  extern __shared__ unsigned char smem_raw[];
  const uint32_t padb = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  unsigned char* sm = smem_raw + padb;
  ChainSmall& cs = *reinterpret_cast<ChainSmall*>(sm + K_SMALL);
  uint64_t* full_a = reinterpret_cast<uint64_t*>(&cs.full_a[0]);
  uint64_t* empty_a = reinterpret_cast<uint64_t*>(&cs.empty_a[0]);
  uint64_t* full_t = reinterpret_cast<uint64_t*>(&cs.full_t);
  uint64_t* empty_t = reinterpret_cast<uint64_t*>(&cs.empty_t);
  uint64_t* full_v = reinterpret_cast<uint64_t*>(&cs.full_v);
  uint64_t* empty_v = reinterpret_cast<uint64_t*>(&cs.empty_v);
  uint64_t* full_d = reinterpret_cast<uint64_t*>(&cs.full_d);
  uint64_t* empty_d = reinterpret_cast<uint64_t*>(&cs.empty_d);
  uint64_t* r_done = reinterpret_cast<uint64_t*>(&cs.r_done);
  uint64_t* u_done = reinterpret_cast<uint64_t*>(&cs.u_done);
  uint64_t* s_done = reinterpret_cast<uint64_t*>(&cs.s_done);
  uint64_t* out_full = reinterpret_cast<uint64_t*>(&cs.out_full[0]);
  uint64_t* out_free = reinterpret_cast<uint64_t*>(&cs.out_free[0]);
  uint64_t* v_ready = reinterpret_cast<uint64_t*>(&cs.v_ready);
  uint64_t* d_ready = reinterpret_cast<uint64_t*>(&cs.d_ready);
  uint64_t* s0_ready = reinterpret_cast<uint64_t*>(&cs.s0_ready);
  uint64_t* drained = reinterpret_cast<uint64_t*>(&cs.drained);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x % H, seq = blockIdx.x / H;
  int first = 0, nchunks = 0;
  chunk_range(m, seq, first, nchunks);
  if (!dcheck(dv <= 128 && dv % 32 == 0, m.checks, kCheckImage)) nchunks = 0;
  const int nvb = dv / 32;           // TMA boxes of 32 value columns

  if (tid == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(full_a + b, 1);
      mbar_init(empty_a + b, 2);     // the products' commit and the decay pass
      mbar_init(out_full + b, 1);
      mbar_init(out_free + b, 1);
    }
    mbar_init(full_t, 1);
    mbar_init(empty_t, 1);
    mbar_init(full_v, 1);
    mbar_init(empty_v, 1);
    mbar_init(full_d, 1);
    mbar_init(empty_d, 1);
    mbar_init(r_done, 1);
    mbar_init(u_done, 1);
    mbar_init(s_done, 1);
    mbar_init(v_ready, 1);
    mbar_init(d_ready, 1);
    mbar_init(s0_ready, 1);
    mbar_init(drained, 1);
    cs.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&cs.tmem, T_COLS);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tb = cs.tmem;
  const unsigned char* wsb = ws + m.img_base + ((size_t)h * m.nck + first) * kChunkWs;
  const uint32_t sbase_u = smem_u32(sm);
  volatile int* abort_flag = &cs.abort;

  if (warp == 9) {
    // ============================= issuing warp ========================================
    // The whole warp runs this loop with warp-uniform operands and one elected lane issues
    // each product (the warp-collective form keeps the operands in uniform registers: a
    // product issues in about half the time a lone thread takes).
    {
      const uint64_t dT = sdesc(sbase_u + K_T, 16, 1024);
      const uint64_t dKH = sdesc(sbase_u + K_D, 16, 1024);
      const uint64_t dP = sdesc(sbase_u + K_D + 32768, 16, 1024);
      const uint32_t i64 = idesc_tf32(128, 64, false, false);
      const uint32_t i64n = idesc_tf32(128, 64, false, false, true);   // -A
      const uint32_t i128 = idesc_tf32(128, 128, false, false);
      bool any = false;
      auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
        if (__all_sync(0xffffffffu, mbar_wait(bar, parity, spin_limit))) return true;
        if (lane == 0) {
          atomicOr(status, 1u);
          cs.abort = 1;
        }
        return false;
      };
      bool ok = nchunks == 0 || wait(s0_ready, 0);
      for (int c = 0; c < nchunks && ok && !__any_sync(0xffffffffu, *abort_flag != 0); ++c) {
        const int b = c & 1;
        const uint32_t pc = (uint32_t)c & 1u, pb = (uint32_t)(c >> 1) & 1u;
        const uint32_t tS = T_S + 128u * b, tSn = T_S + 128u * (b ^ 1), tO = T_O + 64u * b;
        const uint32_t sa = sbase_u + (b ? K_A1 : K_A0);
        const uint64_t dQ = sdesc(sa, 16, 1024), dK = sdesc(sa + 64 * 128, 16, 1024);
        // S_c complete (the previous state product), V^T preloaded, the chunk's [Q~; K~]
        // landed, and this O^T buffer read out (chunk c - 2)
        ok = (c == 0 || wait(s_done, pc ^ 1u)) && wait(v_ready, pc) && wait(full_a + b, pb) &&
             (c < 2 || wait(out_free + b, pb ^ 1u));
        if (!ok) break;
        fence_after_sync();
        // ---- R^T = V^T - S_c K~^T, then the first half of O^T = S_c Q~^T ----------------------
#pragma unroll
        for (int ks = 0; ks < kDK / 8; ++ks)
          mma_tf32_ta_w(tb + T_R, tb + tS + 8 * ks, kstep(dK, 128, ks), i64n, true);
        mma_commit_w(r_done);
#pragma unroll
        for (int ks = 0; ks < kDK / 16; ++ks)
          mma_tf32_ta_w(tb + tO, tb + tS + 8 * ks, kstep(dQ, 128, ks), i64, ks > 0);
        any = true;
        ok = wait(r_done, pc) && wait(full_t, pc);
        if (!ok) break;
        fence_after_sync();
        // ---- U^T = R^T T^T, then the second half of O^T = S_c Q~^T ------------------------
#pragma unroll
        for (int ks = 0; ks < kC / 8; ++ks)
          mma_tf32_ta_w(tb + T_U, tb + T_R + 8 * ks, kstep(dT, 64, ks), i64, ks > 0);
        mma_commit_w(u_done);
        mma_commit_w(empty_t);
#pragma unroll
        for (int ks = kDK / 16; ks < kDK / 8; ++ks)
          mma_tf32_ta_w(tb + tO, tb + tS + 8 * ks, kstep(dQ, 128, ks), i64, true);
        mma_commit_w(empty_a + b);
        ok = wait(u_done, pc) && wait(full_d, pc) && wait(d_ready, pc);
        if (!ok) break;
        fence_after_sync();
        // ---- S_{c+1} = S_c Diag(e^{G_last}) + U^T K^^T, then O^T += U^T P^T ---------------
#pragma unroll
        for (int ks = 0; ks < kC / 8; ++ks)
          mma_tf32_ta_w(tb + tSn, tb + T_U + 8 * ks, kstep(dKH, 128, ks), i128, true);
        mma_commit_w(s_done);
#pragma unroll
        for (int ks = 0; ks < kC / 8; ++ks)
          mma_tf32_ta_w(tb + tO, tb + T_U + 8 * ks, kstep(dP, 64, ks), i64, true);
        mma_commit_w(empty_d);
        mma_commit_w(out_full + b);
      }
      // the products issued here complete before tensor memory is freed
      if (any) {
        mma_commit_w(drained);
        mbar_wait(drained, 0, kDrainLimit);
      }
    }
  } else if (warp == 8) {
    // ================================ loader ===========================================
    if (lane == 0) {
      bool issued_a[2] = {false, false}, issued_t = false, issued_v = false, issued_d = false;
      uint32_t last_a[2] = {0, 0}, last_t = 0, last_v = 0, last_d = 0;
      auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
        if (mbar_wait(bar, parity, spin_limit)) return true;
        atomicOr(status, 1u);
        cs.abort = 1;
        return false;
      };
      for (int c = 0; c < nchunks && !*abort_flag; ++c) {
        const unsigned char* src = wsb + (size_t)c * kChunkWs;
        const int b = c & 1;
        const uint32_t pc = (uint32_t)c & 1u, pb = (uint32_t)(c >> 1) & 1u;
        const ChunkLoc loc = chunk_locate(m, first + c);
        // in the order their buffers free up: [Q~; K~] (chunk c - 2's), V, T, K^ | P
        if (!wait(empty_a + b, pb ^ 1u)) break;
        mbar_expect_tx(full_a + b, WS_A_BYTES);
        bulk_load(sbase_u + (b ? K_A1 : K_A0), src + WS_QK, WS_EGL, full_a + b);
        bulk_load(sbase_u + K_EGL + 512 * b, src + WS_EGL, WS_A_BYTES - WS_EGL, full_a + b);
        issued_a[b] = true;
        last_a[b] = pb;
        if (!wait(empty_v, pc ^ 1u)) break;
        mbar_expect_tx(full_v, (uint32_t)(nvb * 4096));
        for (int nb = 0; nb < nvb; ++nb)
          tma_load_4d(sbase_u + K_V + nb * 4096, &tm_v, 32 * nb, h, loc.t0, loc.b, full_v);
        issued_v = true;
        last_v = pc;
        if (!wait(empty_t, pc ^ 1u)) break;
        mbar_expect_tx(full_t, 16384);
        bulk_load(sbase_u + K_T, src + WS_T, 16384, full_t);
        issued_t = true;
        last_t = pc;
        if (!wait(empty_d, pc ^ 1u)) break;
        mbar_expect_tx(full_d, WS_D_BYTES);
        bulk_load(sbase_u + K_D, src + WS_KH, WS_D_BYTES, full_d);
        issued_d = true;
        last_d = pc;
        // L2 prefetch kPrefetch chunks ahead (the first ones at the start)
        for (int p = c == 0 ? 1 : kPrefetch; p <= kPrefetch && c + p < nchunks; ++p) {
          bulk_prefetch_l2(src + (size_t)p * kChunkWs, kChunkWs);
          const ChunkLoc l2 = chunk_locate(m, first + c + p);
          for (int nb = 0; nb < nvb; ++nb) tma_prefetch_4d(&tm_v, 32 * nb, h, l2.t0, l2.b);
        }
      }
      {
        // copies issued here may still be landing in shared memory (after a give-up
        // anywhere): let them finish (a barrier's phases complete in order, so its last
        // copy is the one to wait for; after a normal run they all have)
        for (int b = 0; b < 2; ++b)
          if (issued_a[b]) mbar_wait(full_a + b, last_a[b], kDrainLimit);
        if (issued_v) mbar_wait(full_v, last_v, kDrainLimit);
        if (issued_t) mbar_wait(full_t, last_t, kDrainLimit);
        if (issued_d) mbar_wait(full_d, last_d, kDrainLimit);
      }
    }
  } else {
    // ========================== per-element passes =====================================
    // Two groups of four warps, each covering all 128 value rows (warp w % 4 reaches TMEM
    // lanes 32 (w % 4) ..): warps 0-3 keep the chain fed (V^T preload, decayed state copy,
    // entering and final state), warps 4-7 write the outputs, so neither waits for the other.
    const bool outg = warp >= 4;
    const int gid = tid & 127;
    const int v = gid;                      // value row = TMEM lane
    const uint32_t tlane = (uint32_t)((warp & 3) * 32) << 16;
    const int sidx = chunk_state_index(m, seq);
    const long srow = (((long)max(sidx, 0) * H + h) * dv + v) * kDK;
    bool fail = false;
    // a wait every thread makes; the group barrier after the pass tells all of its threads
    // whether anyone gave up (the passes only touch this CTA's shared and tensor memory, so
    // a pass over stale data is harmless)
    auto pass_wait = [&](uint64_t* bar, uint32_t parity) {
      if (!fail && !mbar_wait(bar, parity, spin_limit)) fail = true;
    };
    auto agree = [&]() -> bool {
      return named_bar_or(outg ? 2 : 1, K_LANES / 2, fail || *abort_flag != 0);
    };
    bool stop = false;
    if (!outg) {
      // ---------------------------- chain warps ----------------------------------------
      const unsigned char* vcol = sm + K_V + (v >> 5) * 4096 + (v & 31) * 2;
      // the entering state (rows past d_v zero) into state buffer 0
#pragma unroll
      for (int nb = 0; nb < 4; ++nb) {
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
        tmem_st32(tb + tlane + T_S + 32 * nb, x);
      }
      tmem_wait_st();
      fence_before_sync();
      stop = agree();
      if (!stop && gid == 0) mbar_arrive(s0_ready);
      for (int c = 0; c < nchunks && !stop; ++c) {
        const int b = c & 1;
        const uint32_t pc = (uint32_t)c & 1u, pb = (uint32_t)(c >> 1) & 1u;
        // ---- V^T into R^T's columns, once the previous chunk's U^T product has read R^T --
        pass_wait(full_v, pc);
        if (c > 0) pass_wait(u_done, pc ^ 1u);
        fence_after_sync();
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float x[32];
#pragma unroll
          for (int i = 0; i < 32; ++i)
            x[i] = v < dv ? __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(
                                vcol + (32 * hh + i) * 64))
                          : 0.f;
          tmem_st32(tb + tlane + T_R + 32 * hh, x);
        }
        tmem_wait_st();
        fence_before_sync();
        if ((stop = agree())) break;
        if (gid == 0) {
          mbar_arrive(v_ready);
          mbar_arrive(empty_v);
        }
        // ---- S_c Diag(e^{G_last}) into the other state buffer, once S_c is complete ------
        pass_wait(full_a + b, pb);
        if (c > 0) pass_wait(s_done, pc ^ 1u);
        fence_after_sync();
        {
          const float4* egl = reinterpret_cast<const float4*>(sm + K_EGL + 512 * b);
          const uint32_t tS = T_S + 128u * b, tSn = T_S + 128u * (b ^ 1);
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            float x[2][32];
            tmem_ld32(tb + tlane + tS + 64 * hh, x[0]);
            tmem_ld32(tb + tlane + tS + 64 * hh + 32, x[1]);
            tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 2; ++u) {
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                const float4 e = egl[16 * hh + 8 * u + q];
                x[u][4 * q] *= e.x;
                x[u][4 * q + 1] *= e.y;
                x[u][4 * q + 2] *= e.z;
                x[u][4 * q + 3] *= e.w;
              }
              tmem_st32(tb + tlane + tSn + 64 * hh + 32 * u, x[u]);
            }
          }
        }
        tmem_wait_st();
        fence_before_sync();
        if ((stop = agree())) break;
        if (gid == 0) {
          mbar_arrive(d_ready);
          mbar_arrive(empty_a + b);
        }
      }
      // the final state (the last state product's result, undecayed)
      if (!stop && s_final) {
        if (nchunks > 0) pass_wait(s_done, (uint32_t)(nchunks - 1) & 1u);
        fence_after_sync();
        const uint32_t tS = T_S + 128u * (uint32_t)(nchunks & 1);
#pragma unroll
        for (int nb = 0; nb < 4; ++nb) {
          float x[32];
          tmem_ld32(tb + tlane + tS + 32 * nb, x);
          tmem_wait_ld();
          if (!fail && v < dv && sidx >= 0) {
#pragma unroll
            for (int q = 0; q < 8; ++q)
              *reinterpret_cast<float4*>(s_final + srow + 32 * nb + 4 * q) =
                  make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
          }
        }
        if (fail) stop = true;
      }
    } else {
      // ---------------------------- output warps ---------------------------------------
      // O^T of each chunk: one value column of 64 tokens per thread, staged as [t][d_v] and
      // written by one TMA tensor store per 16 KB tile (rows past the tensor's end are not
      // written).  A packed sequence's partial last chunk, whose rows past its end belong
      // to the next sequence, is stored element by element instead.
      constexpr int kRounds = (int)sizeof(Tout) / 2;     // 16 KB tiles per chunk
      constexpr int kTok = 64 / kRounds;
      unsigned char* stage = sm + K_STAGE;
      const bool storer = gid == 0;
      for (int c = 0; c < nchunks && !stop; ++c) {
        const int b = c & 1;
        pass_wait(out_full + b, (uint32_t)(c >> 1) & 1u);
        fence_after_sync();
        float x[64];
        tmem_ld32(tb + tlane + T_O + 64 * b, *reinterpret_cast<float(*)[32]>(&x[0]));
        tmem_ld32(tb + tlane + T_O + 64 * b + 32, *reinterpret_cast<float(*)[32]>(&x[32]));
        tmem_wait_ld();
        fence_before_sync();
        if ((stop = agree())) break;
        if (storer) mbar_arrive(out_free + b);
        const ChunkLoc loc = chunk_locate(m, first + c);
        if (!loc.valid) continue;
        if (m.cu && loc.L < kC) {
          if (v < dv) {
            const long tstride = (long)H * dv;
            Tout* col = o + (((long)loc.b * m.T + loc.t0) * H + h) * (long)dv + v;
#pragma unroll
            for (int t = 0; t < kC; ++t)
              if (t < loc.L) col[t * tstride] = out_cast<Tout>(x[t]);
          }
          continue;
        }
#pragma unroll
        for (int r = 0; r < kRounds; ++r) {
          if (kTok * r >= loc.L) break;          // the tile starts past the tensor's end
          if (storer) bulk_wait_read_all();      // the tile's previous store has read it
          named_bar(3, K_LANES / 2);
          if (v < dv) {
#pragma unroll
            for (int i = 0; i < kTok; ++i)
              *reinterpret_cast<Tout*>(stage + (i * dv + v) * (int)sizeof(Tout)) =
                  out_cast<Tout>(x[kTok * r + i]);
          }
          fence_smem_to_async();
          named_bar(3, K_LANES / 2);
          if (storer) {
            tma_store_4d(&tm_o, smem_u32(stage), 0, h, loc.t0 + kTok * r, loc.b);
            bulk_commit();
          }
        }
      }
      if (storer) bulk_wait_all();    // the output stores read shared memory until done
    }
    if (stop && gid == 0) {
      atomicOr(status, 1u);
      cs.abort = 1;
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tb, T_COLS);
}

}  // namespace

template <typename Tout>
cudaError_t launch_chain_t(const PrefillArgs& a, const ChunkMap& m, uint32_t lim,
                           cudaStream_t stream) {
  // packed sequences: the tensors are [1, total, H, *]
  const int TB = m.cu ? 1 : a.B;
  CUtensorMap mv, mo;
  if (!encode_bthd_bf16(&mv, a.v, TB, a.T, a.H, a.dv, 32, kC, false)) return cudaErrorInvalidValue;
  // output boxes of 16 KB: 64 tokens of bf16 or 32 of fp32
  const bool out_ok =
      sizeof(Tout) == 2 ? encode_bthd_bf16(&mo, a.o, TB, a.T, a.H, a.dv, a.dv, 64, false)
                        : encode_bthd_f32(&mo, (const float*)a.o, TB, a.T, a.H, a.dv, a.dv, 32);
  if (!out_ok) return cudaErrorInvalidValue;
  auto carry = chain_carry_kernel<Tout>;
  cudaError_t e = cudaFuncSetAttribute(carry, cudaFuncAttributeMaxDynamicSharedMemorySize, K_SMEM);
  if (e != cudaSuccess) return e;
  carry<<<m.nseq * a.H, K_THREADS, K_SMEM, stream>>>(mv, mo, (const unsigned char*)a.workspace,
                                                     a.s0, (Tout*)a.o, a.s_final, m, a.H, a.dv,
                                                     (unsigned int*)a.workspace, lim);
  return cudaGetLastError();
}

cudaError_t launch_carry_chain(const PrefillArgs& a, const ChunkMap& m, uint32_t spin_limit,
                               cudaStream_t stream) {
  if (a.out_dtype == GDR_F32) return launch_chain_t<float>(a, m, spin_limit, stream);
  return launch_chain_t<__nv_bfloat16>(a, m, spin_limit, stream);
}

}  // namespace gdr
