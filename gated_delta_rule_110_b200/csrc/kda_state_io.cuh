// kda_state_io.cuh -- where each sequence's recurrent state is read from and
// written to.  Either dense rows (sequence n <-> row n of S0 / S_T), or slots
// of a caller-owned state pool addressed through an int32 index per sequence
// (continuous batching, prefix-cached states, prefill resumed from a cached
// state).  Shared by every kernel of the library.
#pragma once

#include "kda_ptx.cuh"

namespace kda {

struct StateIO {
  const float* S0 = nullptr;        // initial states [rows, H, dk, dv], or nullptr (zeros)
  float* S_T = nullptr;             // final states, or nullptr (not written)
  const int32_t* slots = nullptr;   // nullptr: row n; else the pool slot of sequence n (< 0: padding)
  const uint8_t* has_init = nullptr;  // with slots: per sequence, 0 = start from zeros (nullptr = all 1)
  int num_slots = 0;                // with slots: rows of the pool; larger indices are refused
};

// Resolves sequence n to a state row and says whether to read the initial
// state from it and whether to write the final state back.  A slot past the
// pool is treated as padding (nothing read or written) and recorded as
// KDA_ERR_ARGUMENT in the device error word.
__device__ __forceinline__ int state_row(const StateIO& io, int n, bool* read, bool* write) {
  if (io.slots == nullptr) {
    *read = io.S0 != nullptr;
    *write = io.S_T != nullptr;
    return n;
  }
  const int s = io.slots[n];
  if (s < 0 || s >= io.num_slots) {
    if (s >= io.num_slots) record_error(-10 /* KDA_ERR_ARGUMENT */);
    *read = *write = false;
    return -1;
  }
  *read = io.S0 != nullptr && (io.has_init == nullptr || io.has_init[n] != 0);
  *write = io.S_T != nullptr;
  return s;
}

}  // namespace kda
