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
// two output products fill the tensor pipe while the issuing warp waits for R and for S.
//
// Roles: warps 0-3 write the decayed state copy and the outputs (value row = lane of the
// warp's sub-partition), warps 4-7 preload V^T (from V columns they read from global
// memory a chunk ahead), warp 8 the loader (bulk copies of the chunk images;
// L2 prefetch of the images and the V tiles a chunk ahead: two or three chunks ahead
// measured slower with many chains), warp 9 the issuing warp.
// [Q~; K~] with e^{G_last}, and T are double-buffered; K^ and P have one buffer each,
// refilled as soon as the product that reads it has completed.  The outputs leave through
// shared memory, one TMA tensor store per chunk (scattered 2-byte stores from every
// thread cost several times more).  The issuing warp tests every barrier a step needs at
// once, with non-blocking tests (one blocking wait after another cost ~150-200 cycles
// each, ten times a chunk, even when the phase had long completed).
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
#define GDR_CHAIN_PREFETCH 1
#endif
constexpr int kPrefetch = GDR_CHAIN_PREFETCH;   // chunks the loader prefetches into L2 ahead
constexpr int K_THREADS = 320;       // warps 0-7 per-element passes, 8 loader, 9 issuer
constexpr int K_LANES = 256;

// Shared memory: the [Q~; K~] tiles twice, T twice, K^, P, e^{G_last} twice, the barriers,
// and the 16 KB output staging tile.  (V never passes through shared memory: warps 4-7
// read it from global memory a chunk ahead.)
constexpr int K_A0 = 0;
constexpr int K_A1 = WS_EGL;                  // 64 KB
constexpr int K_T = 2 * WS_EGL;               // 16 KB each
constexpr int K_KH = K_T + 2 * 16384;         // 32 KB
constexpr int K_P = K_KH + 32768;             // 16 KB
constexpr int K_EGL = K_P + 16384;
constexpr int K_SMALL = K_EGL + 1024;
constexpr int K_STAGE = K_SMALL + 256;
constexpr int K_SMEM = K_STAGE + 16384 + 1024;
static_assert(K_A1 % 1024 == 0 && K_T % 1024 == 0 && K_KH % 1024 == 0 && K_P % 1024 == 0,
              "tile alignment");
static_assert(K_STAGE % 128 == 0, "TMA store source");
static_assert(K_SMEM <= 232448, "shared memory");

// Tensor memory (512 columns, lane = value row v): two state buffers (S_c and the next
// state by chunk parity), two O^T buffers by chunk parity, R^T and U^T.
constexpr uint32_t T_S = 0, T_O = 256, T_R = 384, T_U = 448, T_COLS = 512;

struct ChainSmall {
  unsigned long long full_a[2];   // [Q~; K~] and e^{G_last} buffer has landed
  unsigned long long empty_a[2];  // ... and its readers are done (products + decay pass)
  unsigned long long full_t[2], empty_t[2];
  unsigned long long full_k, empty_k;   // K^
  unsigned long long full_p, empty_p;   // P
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

// V of chunk gc for the lane pair of value column v: the even lane reads columns
// (v & ~1, v | 1) of tokens 2i, the odd lane of tokens 2i + 1, 4 bytes a load, zero past
// the chunk's length or past d_v.  Only the loads are issued here; vcol_pair() swaps the
// halves between the pair once the data is needed, so the loads stay in flight meanwhile.
__device__ __forceinline__ void fetch_v(uint32_t (&raw)[GDR_CHUNK / 2],
                                        const __nv_bfloat16* __restrict__ vin,
                                        const ChunkMap& m, int gc, int H, int h, int dv, int v) {
  const ChunkLoc l = chunk_locate(m, gc);
  const int odd = v & 1, vb = v & ~1;
  const int n = vb < dv ? l.L : 0;      // tokens of the chunk to read
  const __nv_bfloat16* p = vin + (((long)l.b * m.T + l.t0 + odd) * H + h) * (long)dv + vb;
  const long ts2 = 2L * H * dv;
#pragma unroll
  for (int i = 0; i < GDR_CHUNK / 2; ++i) {
    raw[i] = 2 * i + odd < n ? __ldg(reinterpret_cast<const unsigned int*>(p)) : 0u;
    p += ts2;
  }
}
// Word i of column v: bf16 of tokens 2i (low half) and 2i + 1 (high half).  All 32 lanes
// of the warp take part.
__device__ __forceinline__ uint32_t vcol_pair(uint32_t raw, int v) {
  const uint32_t o = __shfl_xor_sync(0xffffffffu, raw, 1);
  return (v & 1) ? __byte_perm(o, raw, 0x7632) : __byte_perm(raw, o, 0x5410);
}

// Non-blocking test of an mbarrier phase (no suspension, so tests of several barriers
// issued back to back overlap their latency).
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

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
chain_carry_kernel(const __grid_constant__ CUtensorMap tm_o, const __grid_constant__ CUtensorMap tm_v,
                   const __nv_bfloat16* __restrict__ vin,
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
  uint64_t* full_t = reinterpret_cast<uint64_t*>(&cs.full_t[0]);
  uint64_t* empty_t = reinterpret_cast<uint64_t*>(&cs.empty_t[0]);
  uint64_t* full_k = reinterpret_cast<uint64_t*>(&cs.full_k);
  uint64_t* empty_k = reinterpret_cast<uint64_t*>(&cs.empty_k);
  uint64_t* full_p = reinterpret_cast<uint64_t*>(&cs.full_p);
  uint64_t* empty_p = reinterpret_cast<uint64_t*>(&cs.empty_p);
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

  if (tid == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(full_a + b, 1);
      mbar_init(empty_a + b, 2);     // the products' commit and the decay pass
      mbar_init(out_full + b, 1);
      mbar_init(out_free + b, 1);
      mbar_init(full_t + b, 1);
      mbar_init(empty_t + b, 1);
    }
    mbar_init(full_k, 1);
    mbar_init(empty_k, 1);
    mbar_init(full_p, 1);
    mbar_init(empty_p, 1);
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
      const uint64_t dKH = sdesc(sbase_u + K_KH, 16, 1024);
      const uint64_t dP = sdesc(sbase_u + K_P, 16, 1024);
      const uint32_t i64 = idesc_tf32(128, 64, false, false);
      const uint32_t i64n = idesc_tf32(128, 64, false, false, true);   // -A
      const uint32_t i128 = idesc_tf32(128, 128, false, false);
      bool any = false;
      // Each wait point tests all the barriers it needs together, warp-uniformly, until
      // all have completed or the limit is reached (then the give-up is recorded).
      auto spin = [&](auto&& ready) -> bool {
        for (uint32_t i = 0; i < spin_limit; ++i)
          if (__all_sync(0xffffffffu, ready())) return true;
        if (lane == 0) {
          atomicOr(status, 1u);
          cs.abort = 1;
        }
        return false;
      };
      auto done = [&](uint64_t* bar, uint32_t parity, bool need) -> bool {
        return !need || mbar_test(bar, parity);
      };
      bool ok = nchunks == 0 || spin([&] { return done(s0_ready, 0, true); });
      for (int c = 0; c < nchunks && ok && !__any_sync(0xffffffffu, *abort_flag != 0); ++c) {
        const int b = c & 1;
        const uint32_t pc = (uint32_t)c & 1u, pb = (uint32_t)(c >> 1) & 1u;
        const uint32_t tS = T_S + 128u * b, tSn = T_S + 128u * (b ^ 1), tO = T_O + 64u * b;
        const uint32_t sa = sbase_u + (b ? K_A1 : K_A0);
        const uint64_t dQ = sdesc(sa, 16, 1024), dK = sdesc(sa + 64 * 128, 16, 1024);
        const uint64_t dT = sdesc(sbase_u + K_T + 16384 * b, 16, 1024);
        // S_c complete (the previous state product), V^T preloaded, the chunk's [Q~; K~]
        // landed, and this O^T buffer read out (chunk c - 2)
        ok = spin([&] {
          return done(s_done, pc ^ 1u, c > 0) & done(v_ready, pc, true) &
                 done(full_a + b, pb, true) & done(out_free + b, pb ^ 1u, c >= 2);
        });
        if (!ok) break;
        fence_after_sync();
        // ---- R^T = V^T - S_c K~^T, then O^T = S_c Q~^T (which the pipe runs while the issuing
        //      warp waits for R: measured faster than splitting it around U) ------------------
#pragma unroll
        for (int ks = 0; ks < kDK / 8; ++ks)
          mma_tf32_ta_w(tb + T_R, tb + tS + 8 * ks, kstep(dK, 128, ks), i64n, true);
        mma_commit_w(r_done);
#pragma unroll
        for (int ks = 0; ks < kDK / 8; ++ks)
          mma_tf32_ta_w(tb + tO, tb + tS + 8 * ks, kstep(dQ, 128, ks), i64, ks > 0);
        mma_commit_w(empty_a + b);
        any = true;
        ok = spin([&] { return done(r_done, pc, true) & done(full_t + b, pb, true); });
        if (!ok) break;
        fence_after_sync();
        // ---- U^T = R^T T^T --------------------------------------------------------------------
#pragma unroll
        for (int ks = 0; ks < kC / 8; ++ks)
          mma_tf32_ta_w(tb + T_U, tb + T_R + 8 * ks, kstep(dT, 64, ks), i64, ks > 0);
        mma_commit_w(u_done);
        mma_commit_w(empty_t + b);
        ok = spin([&] {
          return done(u_done, pc, true) & done(full_k, pc, true) & done(d_ready, pc, true);
        });
        if (!ok) break;
        fence_after_sync();
        // ---- S_{c+1} = S_c Diag(e^{G_last}) + U^T K^^T, then O^T += U^T P^T ---------------
#pragma unroll
        for (int ks = 0; ks < kC / 8; ++ks)
          mma_tf32_ta_w(tb + tSn, tb + T_U + 8 * ks, kstep(dKH, 128, ks), i128, true);
        mma_commit_w(s_done);
        mma_commit_w(empty_k);
        if (!(ok = spin([&] { return done(full_p, pc, true); }))) break;
        fence_after_sync();
#pragma unroll
        for (int ks = 0; ks < kC / 8; ++ks)
          mma_tf32_ta_w(tb + tO, tb + T_U + 8 * ks, kstep(dP, 64, ks), i64, true);
        mma_commit_w(empty_p);
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
      bool issued_a[2] = {false, false}, issued_t[2] = {false, false}, issued_k = false,
           issued_p = false;
      uint32_t last_a[2] = {0, 0}, last_t[2] = {0, 0}, last_k = 0, last_p = 0;
      auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
        if (mbar_wait(bar, parity, spin_limit)) return true;
        atomicOr(status, 1u);
        cs.abort = 1;
        return false;
      };
      // [Q~; K~] and e^{G_last} of chunk cc into buffer cc & 1 once chunk cc - 2 is done with it
      auto load_a = [&](int cc) -> bool {
        const unsigned char* src = wsb + (size_t)cc * kChunkWs;
        const int b = cc & 1;
        const uint32_t pb = (uint32_t)(cc >> 1) & 1u;
        if (!wait(empty_a + b, pb ^ 1u)) return false;
        mbar_expect_tx(full_a + b, WS_A_BYTES);
        bulk_load(sbase_u + (b ? K_A1 : K_A0), src + WS_QK, WS_EGL, full_a + b);
        bulk_load(sbase_u + K_EGL + 512 * b, src + WS_EGL, WS_A_BYTES - WS_EGL, full_a + b);
        issued_a[b] = true;
        last_a[b] = pb;
        return true;
      };
      if (nchunks > 0) load_a(0);
      for (int c = 0; c < nchunks && !*abort_flag; ++c) {
        const unsigned char* src = wsb + (size_t)c * kChunkWs;
        const int b = c & 1;
        const uint32_t pc = (uint32_t)c & 1u, pb = (uint32_t)(c >> 1) & 1u;
        // in the order their buffers free up: [Q~; K~] one chunk further ahead (its buffer
        // frees in the middle of chunk c - 1), T (chunk c - 2's), K^, P
        if (c + 1 < nchunks && !load_a(c + 1)) break;
        if (!wait(empty_t + b, pb ^ 1u)) break;
        mbar_expect_tx(full_t + b, 16384);
        bulk_load(sbase_u + K_T + 16384 * b, src + WS_T, 16384, full_t + b);
        issued_t[b] = true;
        last_t[b] = pb;
        if (!wait(empty_k, pc ^ 1u)) break;
        mbar_expect_tx(full_k, 32768);
        bulk_load(sbase_u + K_KH, src + WS_KH, 32768, full_k);
        issued_k = true;
        last_k = pc;
        if (!wait(empty_p, pc ^ 1u)) break;
        mbar_expect_tx(full_p, 16384);
        bulk_load(sbase_u + K_P, src + WS_P, 16384, full_p);
        issued_p = true;
        last_p = pc;
        // L2 prefetch kPrefetch chunks ahead (the first ones at the start): the chunk image,
        // and the V tile that the V warps read with plain loads a chunk ahead
        for (int p = c == 0 ? 1 : kPrefetch; p <= kPrefetch && c + p < nchunks; ++p) {
          bulk_prefetch_l2(src + (size_t)p * kChunkWs, kChunkWs);
          const ChunkLoc lp = chunk_locate(m, first + c + p);
          tma_prefetch_4d(&tm_v, 0, h, lp.t0, lp.b);
        }
      }
      {
        // copies issued here may still be landing in shared memory (after a give-up
        // anywhere): let them finish (a barrier's phases complete in order, so its last
        // copy is the one to wait for; after a normal run they all have)
        for (int b = 0; b < 2; ++b) {
          if (issued_a[b]) mbar_wait(full_a + b, last_a[b], kDrainLimit);
          if (issued_t[b]) mbar_wait(full_t + b, last_t[b], kDrainLimit);
        }
        if (issued_k) mbar_wait(full_k, last_k, kDrainLimit);
        if (issued_p) mbar_wait(full_p, last_p, kDrainLimit);
      }
    }
  } else {
    // ========================== per-element passes =====================================
    // Two groups of four warps, each covering all 128 value rows (warp w % 4 reaches TMEM
    // lanes 32 (w % 4) ..).  Warps 0-3 write the entering state, each chunk's decayed state
    // copy, the outputs and the final state; warps 4-7 preload V^T and read the next
    // chunk's V from global memory (issuing those loads stalls for a while when many are
    // in flight, so it comes after the preload has been signalled).
    const bool vg = warp >= 4;
    const int gid = tid & 127;
    const int v = gid;                      // value row = TMEM lane
    const uint32_t tlane = (uint32_t)((warp & 3) * 32) << 16;
    bool fail = false;
    // a wait every thread makes; the group barrier after the pass tells all of its threads
    // whether anyone gave up (a pass over stale data touches only this CTA's shared and
    // tensor memory and its own output rows, so it is harmless: the give-up is recorded)
    auto pass_wait = [&](uint64_t* bar, uint32_t parity) {
      if (!fail && !mbar_wait(bar, parity, spin_limit)) fail = true;
    };
    auto agree = [&]() -> bool {
      return named_bar_or(vg ? 2 : 1, K_LANES / 2, fail || *abort_flag != 0);
    };
    bool stop = false;
    if (vg) {
      // ------------------------------- V warps -----------------------------------------
      uint32_t vraw[kC / 2];
      if (nchunks > 0) fetch_v(vraw, vin, m, first, H, h, dv, v);
      for (int c = 0; c < nchunks && !stop; ++c) {
        // V^T of chunk c into R^T's columns, once chunk c - 1's U^T product has read R^T
        if (c > 0) pass_wait(u_done, (uint32_t)(c - 1) & 1u);
        fence_after_sync();
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float x[32];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const uint32_t w = vcol_pair(vraw[16 * hh + i], v);
            x[2 * i] = __uint_as_float(w << 16);
            x[2 * i + 1] = __uint_as_float(w & 0xffff0000u);
          }
          tmem_st32(tb + tlane + T_R + 32 * hh, x);
        }
        tmem_wait_st();
        fence_before_sync();
        if ((stop = agree())) break;
        if (gid == 0) mbar_arrive(v_ready);
        if (c + 1 < nchunks) fetch_v(vraw, vin, m, first + c + 1, H, h, dv, v);
      }
    } else {
      // --------------------------- state and output warps ------------------------------
      const int sidx = chunk_state_index(m, seq);
      const long srow = (((long)max(sidx, 0) * H + h) * dv + v) * kDK;
      // O^T of chunk c: one value column of 64 tokens per thread, staged as [t][d_v] and
      // written by one TMA tensor store per 16 KB tile (rows past the tensor's end are not
      // written).  A packed sequence's partial last chunk, whose rows past its end belong
      // to the next sequence, is stored element by element instead.
      constexpr int kRounds = (int)sizeof(Tout) / 2;     // 16 KB tiles per chunk
      unsigned char* stage = sm + K_STAGE;
      const bool storer = gid == 0;
      auto write_outputs = [&](int c) -> bool {
        const int b = c & 1;
        pass_wait(out_full + b, (uint32_t)(c >> 1) & 1u);
        fence_after_sync();
        const ChunkLoc loc = chunk_locate(m, first + c);
        const bool tma = loc.valid && !(m.cu && loc.L < kC);
        Tout* col = o + (((long)loc.b * m.T + loc.t0) * H + h) * (long)dv + v;
        const long tstride = (long)H * dv;
        if (tma) {
          if (storer) bulk_wait_read_all();      // the tile's previous store has read it
          named_bar(3, K_LANES / 2);
        }
        // 32 tokens at a time: bf16 outputs fill one 64-token tile, fp32 ones two tiles of
        // 32 tokens in turn (the first stored before the second is staged)
#pragma unroll 1
        for (int hh = 0; hh < 2; ++hh) {
          float x[32];
          tmem_ld32(tb + tlane + T_O + 64 * b + 32 * hh, x);
          tmem_wait_ld();
          if (kRounds == 2 && hh == 1 && tma) {
            if (storer) bulk_wait_read_all();
            named_bar(3, K_LANES / 2);
          }
          if (loc.valid && v < dv) {
            if (tma) {
              const int row0 = kRounds == 2 ? 0 : 32 * hh;
#pragma unroll
              for (int i = 0; i < 32; ++i)
                *reinterpret_cast<Tout*>(stage + ((row0 + i) * dv + v) * (int)sizeof(Tout)) =
                    out_cast<Tout>(x[i]);
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (32 * hh + i < loc.L) col[(32 * hh + i) * tstride] = out_cast<Tout>(x[i]);
            }
          }
          if (kRounds == 2 && hh == 0 && tma) {
            fence_smem_to_async();
            named_bar(3, K_LANES / 2);
            if (storer) {
              tma_store_4d(&tm_o, smem_u32(stage), 0, h, loc.t0, loc.b);
              bulk_commit();
            }
          }
        }
        fence_smem_to_async();
        fence_before_sync();
        if (agree()) return false;
        if (storer) {
          mbar_arrive(out_free + b);
          const int r0 = kRounds == 2 ? 32 : 0;       // the tile staged last
          if (tma && r0 < loc.L) {
            tma_store_4d(&tm_o, smem_u32(stage), 0, h, loc.t0 + r0, loc.b);
            bulk_commit();
          }
        }
        return true;
      };
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
      for (int c = 0; c <= nchunks && !stop; ++c) {
        if (c == nchunks) {
          stop = nchunks > 0 && !write_outputs(c - 1);
          break;
        }
        const int b = c & 1;
        const uint32_t pc = (uint32_t)c & 1u, pb = (uint32_t)(c >> 1) & 1u;
        // ---- S_c Diag(e^{G_last}) into the other state buffer, once S_c is complete ------
        pass_wait(full_a + b, pb);
        if (c > 0) pass_wait(s_done, pc ^ 1u);
        fence_after_sync();
        {
          const float4* egl = reinterpret_cast<const float4*>(sm + K_EGL + 512 * b);
          const uint32_t tS = T_S + 128u * b, tSn = T_S + 128u * (b ^ 1);
#pragma unroll
          for (int nb = 0; nb < 4; ++nb) {
            float x[32];
            tmem_ld32(tb + tlane + tS + 32 * nb, x);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float4 e = egl[8 * nb + q];
              x[4 * q] *= e.x;
              x[4 * q + 1] *= e.y;
              x[4 * q + 2] *= e.z;
              x[4 * q + 3] *= e.w;
            }
            tmem_st32(tb + tlane + tSn + 32 * nb, x);
          }
        }
        tmem_wait_st();
        fence_before_sync();
        if ((stop = agree())) break;
        if (gid == 0) {
          mbar_arrive(d_ready);
          mbar_arrive(empty_a + b);
        }
        // ---- the previous chunk's outputs -----------------------------------------------
        if (c > 0 && (stop = !write_outputs(c - 1))) break;
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
  CUtensorMap mo, mv;
  // V: one box of d_v x 64 tokens, used for L2 prefetch only
  if (!encode_bthd_bf16(&mv, a.v, TB, a.T, a.H, a.dv, a.dv, kC, false)) return cudaErrorInvalidValue;
  // output boxes of 16 KB: 64 tokens of bf16 or 32 of fp32
  const bool out_ok =
      sizeof(Tout) == 2 ? encode_bthd_bf16(&mo, a.o, TB, a.T, a.H, a.dv, a.dv, 64, false)
                        : encode_bthd_f32(&mo, (const float*)a.o, TB, a.T, a.H, a.dv, a.dv, 32);
  if (!out_ok) return cudaErrorInvalidValue;
  auto carry = chain_carry_kernel<Tout>;
  cudaError_t e = cudaFuncSetAttribute(carry, cudaFuncAttributeMaxDynamicSharedMemorySize, K_SMEM);
  if (e != cudaSuccess) return e;
  carry<<<m.nseq * a.H, K_THREADS, K_SMEM, stream>>>(mo, mv, (const __nv_bfloat16*)a.v,
                                                     (const unsigned char*)a.workspace,
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
