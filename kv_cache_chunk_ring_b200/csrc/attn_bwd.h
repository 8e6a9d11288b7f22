// Declarations of the MoBA attention backward kernels (host library <-> kernels).
#pragma once

#include "kvcr_internal.h"

namespace kvcr {

// Work order of one backward launch: 128-row tiles (key tiles for dK / dV,
// query tiles for dQ), heaviest first.  CTA b runs tile order[b % n_units] of
// head b / n_units (head-major, so co-resident CTAs share one head's tiles in L2).
struct MobaBwdSched {
  int n_chunks, chunk_tokens, n_bidir;
  int L;
  int n_units;                     // 128-row tiles
  uint16_t order[kMobaMaxTiles];
};

struct MobaBwdParams {
  CUtensorMap tm_q;    // 3D (D, H, L), box 64 x 1 x 128, 128-byte swizzle
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  CUtensorMap tm_do;
  const float* ws;     // [H][n_units][2][128]: lse * log2 e, then rowsum(dO o O), of a tile's rows
  void* dq;            // [L][H][D] bf16
  void* dk;
  void* dv;
  int H;
  int Lpad;
  float scale;         // softmax scale
  float scale_log2;    // softmax scale * log2 e
  int inject;          // test hook: 1 = one P-ready arrival is never made
  long long wait_ns;   // bound of every device wait
  MobaBwdSched s;
};

struct MobaBwdPrepParams {
  const void* o;       // [L][H][D] bf16
  const void* d_o;
  const float* lse;    // [H][L], natural log
  float* ws;           // [H][Lpad / 128][2][128]
  int L, Lpad, H;
};

cudaError_t launch_moba_bwd_prep(const MobaBwdPrepParams& p, int head_dim, cudaStream_t s);
cudaError_t launch_moba_bwd_dkdv_sm100(const MobaBwdParams& p, int head_dim, cudaStream_t s);
cudaError_t launch_moba_bwd_dq_sm100(const MobaBwdParams& p, int head_dim, cudaStream_t s);
cudaError_t read_and_clear_status_bwd(int* st, cudaStream_t s);

}  // namespace kvcr
