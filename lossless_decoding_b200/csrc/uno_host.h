// Host-side helpers shared by the Uno entry points.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "uno.h"

namespace uno_host {

inline bool aligned(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

// UNO_OK when the current device is an sm_100 part (compute capability 10.0),
// UNO_ERR_DEVICE otherwise, UNO_ERR_CUDA when the runtime cannot say. The
// answer is cached per device ordinal.
int check_device();

// One inverse-CDF draw per softmax row (draft_sample.cu): row n of sequence b
// (logits + ((b * rows_per_seq + n) * V)) draws with the uniform of Philox
// word `word` of the block (b, row_key[b][n] or n, step); rows with
// n >= n_rows[b] are skipped and get -1 (n_rows null: all rows are used); a
// row with no finite logit gets -1. Arguments are checked by the caller.
struct RowDraws {
  const void* logits;
  int B, rows_per_seq, V, dtype;
  int seq_rows = 0;  // rows from one sequence's block to the next (0: rows_per_seq)
  const int32_t* row_key;
  const int32_t* n_rows;
  int word;
  uint64_t seed, step;
  int32_t* out;
};
int sample_rows(const RowDraws& r, cudaStream_t st);

}  // namespace uno_host
