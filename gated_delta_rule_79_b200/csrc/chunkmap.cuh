// Where the chunks of a prefill lie: a dense batch ([B, T, H, *] tensors, every
// sequence T tokens) or packed sequences of different lengths ([1, total, H, *]
// tensors with token offsets).  Both two-kernel prefills number the chunks of all
// sequences globally ("gc"), keep one workspace image per (head, gc), and find a
// chunk's sequence, first token and length through this map.
//
// In the GDR_CHECKS build (checks.cuh) the three functions below also test what they
// derive from device data against the tensors' extents; a failed test is recorded in
// *checks and the result is made harmless (an invalid chunk of length 0, an empty chunk
// range, a state index of -1 that the carries skip).
#pragma once

#include "checks.cuh"

namespace gdr {

struct ChunkMap {
  const int* cu;       // packed: [nseq + 1] token offsets of the sequences; null: dense
  const int* cseq;     // packed: sequence of each global chunk
  const int* cstart;   // packed: [nseq + 1] first global chunk of each sequence
  const int* slots;    // packed: state slot of each sequence (null: the sequence index)
  int nseq;            // sequences (dense: B)
  int T;               // tokens per sequence (dense) or in total (packed): the tensors' T
  int nchunks;         // dense: chunks per sequence
  int nck;             // global chunks per head: B * nchunks, or an upper bound (packed)
  size_t img_base;     // byte offset of the first chunk image in the workspace
  unsigned int* checks;  // GDR_CHECKS build: the device word failed index checks set
};

struct ChunkLoc {
  int seq;    // sequence
  int b;      // batch coordinate of the chunk's rows in the tensors
  int t0;     // first token of the chunk along the tensors' T axis
  int L;      // tokens of the chunk (1..64); rows past L belong to no token of it
  bool valid;
};

__device__ __forceinline__ ChunkLoc chunk_locate(const ChunkMap& m, int gc) {
  ChunkLoc r;
  if (!m.cu) {
    r.seq = gc / m.nchunks;
    const int c = gc - r.seq * m.nchunks;
    r.b = r.seq;
    r.t0 = c * 64;
    r.L = min(64, m.T - r.t0);
    r.valid = r.seq < m.nseq;
  } else {
    r.valid = gc < m.cstart[m.nseq];
    if (!r.valid) {
      r.seq = r.b = r.t0 = 0;
      r.L = 0;
      return r;
    }
#ifdef GDR_CHECKS
    if (!dcheck(gc >= 0 && gc < m.nck, m.checks, kCheckChunk)) {
      r.seq = r.b = r.t0 = r.L = 0;
      r.valid = false;
      return r;
    }
#endif
    r.seq = m.cseq[gc];
#ifdef GDR_CHECKS
    if (!dcheck(r.seq >= 0 && r.seq < m.nseq, m.checks, kCheckChunk)) {
      r.seq = r.b = r.t0 = r.L = 0;
      r.valid = false;
      return r;
    }
#endif
    const int c = gc - m.cstart[r.seq];
    r.b = 0;
    r.t0 = m.cu[r.seq] + 64 * c;
    r.L = min(64, m.cu[r.seq + 1] - r.t0);
  }
#ifdef GDR_CHECKS
  if (r.valid && !dcheck(gc >= 0 && gc < m.nck && r.t0 >= 0 && r.L >= 1 && r.L <= 64 &&
                             r.t0 + r.L <= m.T && r.seq < m.nseq,
                         m.checks, kCheckChunk)) {
    r.seq = r.b = r.t0 = r.L = 0;
    r.valid = false;
  }
#endif
  return r;
}

// Global chunks [first, first + count) of sequence `seq`.
__device__ __forceinline__ void chunk_range(const ChunkMap& m, int seq, int& first, int& count) {
#ifdef GDR_CHECKS
  if (!dcheck(seq >= 0 && seq < m.nseq, m.checks, kCheckChunk)) {
    first = 0;
    count = 0;
    return;
  }
#endif
  if (!m.cu) {
    first = seq * m.nchunks;
    count = m.nchunks;
  } else {
    first = m.cstart[seq];
    count = m.cstart[seq + 1] - first;
  }
#ifdef GDR_CHECKS
  if (!dcheck(first >= 0 && count >= 0 && first + count <= m.nck, m.checks, kCheckChunk)) {
    first = 0;
    count = 0;
  }
#endif
}

// Index of the state of sequence `seq` in the state tensors ([*, H, d_v, d_k]); the
// carries neither read nor write a state whose index is negative.
__device__ __forceinline__ int chunk_state_index(const ChunkMap& m, int seq) {
#ifdef GDR_CHECKS
  if (!dcheck(seq >= 0 && seq < m.nseq, m.checks, kCheckState)) return -1;
#endif
  const int i = (m.cu && m.slots) ? m.slots[seq] : seq;
#ifdef GDR_CHECKS
  // a pool's size is not known here: slots are checked for sign, batch entries fully
  if (!dcheck(i >= 0 && (m.slots != nullptr || i < m.nseq), m.checks, kCheckState)) return -1;
#endif
  return i;
}

}  // namespace gdr
