// Device-side index checks of the GDR_CHECKS debug build.
//
// The library is also built as libgdr_checks.so with -DGDR_CHECKS (build.py).  In that
// build the kernels test the indices they derive from device data (packed-sequence
// offsets, chunk numbers, state slots) and from their own launch layout before using
// them; a failed test sets a bit in one device word per GPU (gdr_check_status reads and
// clears it) and the access is skipped, so a bad index shows up as a status bit rather
// than as a memory fault.  In the product build dcheck() is `true` and costs nothing.
#pragma once

#include <stdint.h>

namespace gdr {

enum : unsigned {
  kCheckChunk = 1u,    // a chunk's sequence, first token or length outside the tensors
  kCheckState = 2u,    // a state index (batch entry or pool slot) outside the state tensor
  kCheckImage = 4u,    // a chunk image outside the workspace's image area
  kCheckLayout = 8u,   // a decode / verify thread mapped outside its state rows
};

// True when `ok` holds.  Otherwise, in the checks build, records `bit` in *word (when
// the host passed one) and returns false so that the caller skips the access.
__device__ __forceinline__ bool dcheck(bool ok, unsigned int* word, unsigned bit) {
#ifdef GDR_CHECKS
  if (!ok) {
    if (word) atomicOr(word, bit);
    return false;
  }
  return true;
#else
  (void)ok;
  (void)word;
  (void)bit;
  return true;
#endif
}

}  // namespace gdr
