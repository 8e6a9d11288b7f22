// One launch that writes the same finalized frames into several layer caches.
#pragma once

#include "kvcr_internal.h"

namespace kvcr {

constexpr int kMaxBatchPairs = 256;  // (cache, frame) pairs of one batched append

// Pair i copies one frame of K (rotated when rotate_a) and V from src_*[i] to
// dst_*[i] (each T x H x D elements); its t-axis angles are row tframe[i] of
// ttab.  Every cache of a batch has the same T, H, D, dtype and RoPE, so the
// (h, w) tables of one of them serve all.
struct RopeCopyBatchParams {
  const void* src_a[kMaxBatchPairs];
  const void* src_b[kMaxBatchPairs];
  void* dst_a[kMaxBatchPairs];
  void* dst_b[kMaxBatchPairs];
  int tframe[kMaxBatchPairs];
  int n, T, H, D, grid_w;
  int rotate_a;
  int pairs_t, pairs_h, pairs_w;
  const float2* htab;
  const float2* wtab;
  float2 ttab[kMaxFrames][kMaxPairsT];
};

cudaError_t launch_rope_copy_batch(const RopeCopyBatchParams& p, kvcr_dtype dtype, cudaStream_t s,
                                   int n_sm);

}  // namespace kvcr
