// Which state carry a two-kernel prefill runs (carry_chain.cu, carry_rows.cu or
// carry_sliced.cu), and the size of one chunk's operand image they read.  The timing
// aid's mark after the carry is set here.

#include <stdlib.h>

#include "chunk_image.cuh"
#include "chunkmap.cuh"
#include "gdr.h"
#include "launch.h"

namespace gdr {

// The chained carry (one CTA per (sequence, head), products fed from tensor memory) while
// the chains fit one wave of SMs; with more chains than SMs every carry is bound by the
// chunk images it reads, and the per-head carry takes them.  GDR_CARRY=chain, =rows or
// =sliced picks one regardless (the value-sliced carry spreads each head over several SMs).
cudaError_t launch_chunk_carry(const PrefillArgs& a, const ChunkMap& m, uint32_t spin_limit,
                               cudaStream_t stream) {
  const char* pick = getenv("GDR_CARRY");
  char which;
  if (pick && (pick[0] == 'c' || pick[0] == 'r' || pick[0] == 's')) {
    which = pick[0];
  } else {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    which = (long)m.nseq * a.H > sms ? 'r' : 'c';
  }
  const cudaError_t e = which == 'c'   ? launch_carry_chain(a, m, spin_limit, stream)
                        : which == 'r' ? launch_carry_rows(a, m, spin_limit, stream)
                                       : launch_carry_sliced(a, m, spin_limit, stream);
  if (e == cudaSuccess) timing_mark(stream, 1);
  return e;
}

size_t chunk_image_bytes() { return img::kChunkWs; }

}  // namespace gdr
