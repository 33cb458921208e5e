// Which state carry a two-kernel prefill runs (carry_sliced.cu, carry_rows.cu, or
// carry_rows.cu in two segments followed by carry_segfix.cu), and the size of one chunk's
// operand image they read.  The timing aid's marks after the carry's kernels are set here
// (slot 1, and slot 2 after the two-segment fix-up).

#include <stdlib.h>

#include "chunk_image.cuh"
#include "chunkmap.cuh"
#include "gdr.h"
#include "launch.h"

namespace gdr {

// The value-sliced carry while one 32-column slice per CTA still fits a single wave of
// SMs (a few long chains: several SMs share each head), else the per-head carry (it
// spends a quarter of the SM time per chunk).  GDR_CARRY=rows or GDR_CARRY=sliced picks
// one regardless.
//
// A dense batch of few long chains may instead take the two-segment carry (each chain's
// chunks in two halves run at once by three per-head CTAs, then carry_segfix.cu adds the
// first half's state to the second half) when the workspace holds its buffers
// (gdr_prefill_workspace_bytes counts them).  It is not picked on its own: on the B1 H32
// T4096 prefills it measured 0.143 ms (the per-head carry over 32 chunks) + 0.040 ms (the
// fix-up) against 0.173 ms for the value-sliced carry.  GDR_CARRY=seg picks it.
constexpr bool kSegAuto = false;
constexpr int kSegMinChunks = 16;

cudaError_t launch_chunk_carry(const PrefillArgs& a, const ChunkMap& m, uint32_t spin_limit,
                               cudaStream_t stream) {
  const char* pick = getenv("GDR_CARRY");
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long chains = (long)m.nseq * a.H;
  // the two-segment buffers follow the chunk images
  const size_t seg_bytes = m.cu ? 0 : segment_workspace_bytes(m.nseq, m.T, a.H);
  const size_t seg_off = m.img_base + (size_t)a.H * m.nck * img::kChunkWs;
  const bool seg_ok = seg_bytes > 0 && a.ws_bytes >= seg_off + seg_bytes;
  bool seg = false, rows;
  if (pick && pick[0] == 'r') {
    rows = true;
  } else if (pick && pick[0] == 's' && pick[1] == 'e') {
    seg = seg_ok;
    rows = true;
  } else if (pick && pick[0] == 's') {
    rows = false;
  } else {
    rows = chains * (a.dv / 32) > sms;
    seg = kSegAuto && !rows && seg_ok && 3 * chains <= sms && m.nchunks >= kSegMinChunks;
  }
  if (seg) {
    SegmentBuffers sb;
    sb.states = reinterpret_cast<float*>(static_cast<unsigned char*>(a.workspace) + seg_off);
    sb.outputs = sb.states + 3 * chains * 128 * 128;
    sb.t1p = (m.nchunks - ((m.nchunks + 1) >> 1)) * GDR_CHUNK;
    cudaError_t e = launch_carry_rows(a, m, spin_limit, stream, &sb);
    if (e != cudaSuccess) return e;
    timing_mark(stream, 1);
    e = launch_segment_fixup(a, m, spin_limit, stream, sb);
    if (e == cudaSuccess) timing_mark(stream, 2);
    return e;
  }
  const cudaError_t e = rows ? launch_carry_rows(a, m, spin_limit, stream)
                             : launch_carry_sliced(a, m, spin_limit, stream);
  if (e == cudaSuccess) timing_mark(stream, 1);
  return e;
}

size_t chunk_image_bytes() { return img::kChunkWs; }

}  // namespace gdr
