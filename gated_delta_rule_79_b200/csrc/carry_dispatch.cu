// Which state carry a two-kernel prefill runs (carry_sliced.cu or carry_rows.cu), and the
// size of one chunk's operand image both read.  The timing aid's mark after the carry is
// set here.

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
  const cudaError_t e = rows ? launch_carry_rows(a, m, spin_limit, stream)
                             : launch_carry_sliced(a, m, spin_limit, stream);
  if (e == cudaSuccess) timing_mark(stream, 1);
  return e;
}

size_t chunk_image_bytes() { return img::kChunkWs; }

}  // namespace gdr
