// Whole-token persistent decode kernel (batch-1 hot path): placeholder sizes until
// the kernel lands; the multi-launch layer path in kernels.cuh is complete on its own.
#pragma once

#include "common.cuh"

namespace dfssm {

constexpr int kMaxLayers = 64;

// Scratch for the LM-head argmax partials (value + id per block per batch row).
inline size_t persistent_scratch_bytes(int batch, int d_model, int d_inner, int in_rows, int head_blocks) {
  (void)d_model; (void)d_inner; (void)in_rows;
  return size_t(8) * batch * (head_blocks > 0 ? head_blocks : 1);
}

}  // namespace dfssm
