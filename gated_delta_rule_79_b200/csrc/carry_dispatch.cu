// Which state carry a two-kernel prefill runs (carry_chain.cu, carry_rows.cu or
// carry_sliced.cu), and the size of one chunk's operand image they read.  The timing
// aid's mark after the carry is set here.

#include <stdlib.h>

#include "chunk_image.cuh"
#include "chunkmap.cuh"
#include "gdr.h"
#include "launch.h"

namespace gdr {

// The chained carry (one CTA per (sequence, head), products fed from tensor memory)
// unless GDR_CARRY=rows or =sliced picks the per-head or the value-sliced carry: it was
// the fastest of the three on every shape measured, from 32 long chains (0.124 against
// 0.173 ms sliced) to 2048 short ones (packed prompts, 0.376 against 0.424 ms per-head).
cudaError_t launch_chunk_carry(const PrefillArgs& a, const ChunkMap& m, uint32_t spin_limit,
                               cudaStream_t stream) {
  const char* pick = getenv("GDR_CARRY");
  const char which = (pick && (pick[0] == 'r' || pick[0] == 's')) ? pick[0] : 'c';
  const cudaError_t e = which == 'c'   ? launch_carry_chain(a, m, spin_limit, stream)
                        : which == 'r' ? launch_carry_rows(a, m, spin_limit, stream)
                                       : launch_carry_sliced(a, m, spin_limit, stream);
  if (e == cudaSuccess) timing_mark(stream, 1);
  return e;
}

size_t chunk_image_bytes() { return img::kChunkWs; }

}  // namespace gdr
