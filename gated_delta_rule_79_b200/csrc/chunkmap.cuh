// Where the chunks of a prefill lie: a dense batch ([B, T, H, *] tensors, every
// sequence T tokens) or packed sequences of different lengths ([1, total, H, *]
// tensors with token offsets).  Both two-kernel prefills number the chunks of all
// sequences globally ("gc"), keep one workspace image per (head, gc), and find a
// chunk's sequence, first token and length through this map.
#pragma once

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
    r.seq = m.cseq[gc];
    const int c = gc - m.cstart[r.seq];
    r.b = 0;
    r.t0 = m.cu[r.seq] + 64 * c;
    r.L = min(64, m.cu[r.seq + 1] - r.t0);
  }
  return r;
}

// Global chunks [first, first + count) of sequence `seq`.
__device__ __forceinline__ void chunk_range(const ChunkMap& m, int seq, int& first, int& count) {
  if (!m.cu) {
    first = seq * m.nchunks;
    count = m.nchunks;
  } else {
    first = m.cstart[seq];
    count = m.cstart[seq + 1] - first;
  }
}

// Index of the state of sequence `seq` in the state tensors ([*, H, d_v, d_k]).
__device__ __forceinline__ int chunk_state_index(const ChunkMap& m, int seq) {
  return (m.cu && m.slots) ? m.slots[seq] : seq;
}

}  // namespace gdr
