// Internal declarations shared by the host library and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kvcr.h"

namespace kvcr {

// ----------------------------------------------------------------- limits --
constexpr int kMaxSlots = 32;        // sinks + window
constexpr int kMaxFrames = 16;       // frames of one append / one current chunk
constexpr int kMaxPairsT = 32;       // rotary pairs on the t axis
constexpr int kTile = 128;           // query rows per attention tile (MoBA class granularity)
constexpr int kKeyTile = 128;        // keys per K / V tile of the attention kernel
constexpr int kMobaMaxTiles = 4096;  // MoBA sequence length <= 4096 * 128 tokens
constexpr long long kWaitTimeoutNs = 2000000000LL;  // bounded device waits: 2 s

// ------------------------------------------------------- rope / copy pass --
// One launch moves n_frames frames of two tensors (a and b) of shape
// [T][H][D] each from contiguous sources to per-frame destinations, rotating
// a (and b when rotate_b) with the 3D rotary embedding.  src_b = NULL moves a
// alone (single-cache kernel).
struct RopeCopyParams {
  const void* src_a;
  const void* src_b;
  void* dst_a;
  void* dst_b;
  long long dst_frame_off[kMaxFrames];  // element offset of frame f's destination
  int src_frame[kMaxFrames];            // which source frame feeds destination f
  int n_frames, T, H, D, grid_w;
  int rotate_a, rotate_b;
  int pairs_t, pairs_h, pairs_w;
  const float2* htab;                   // [grid_h][pairs_h] (cos, sin)
  const float2* wtab;                   // [grid_w][pairs_w] (cos, sin)
  float2 ttab[kMaxFrames][kMaxPairsT];  // per destination frame, t-axis (cos, sin)
};

cudaError_t launch_rope_copy(const RopeCopyParams& p, kvcr_dtype dtype, cudaStream_t s,
                             int n_sm);

// ------------------------------------------------------------- attention --
struct ChunkSched {
  int T;             // tokens per cached frame
  int n_vis;         // cached frames read, in slot order
  int tiles_per_slot;
  int n_cur;         // current-chunk keys
  int cur_tiles;
  int slots[kMaxSlots];
};

struct MobaSched {
  int n_chunks, chunk_tokens, n_bidir;
  int L;
  int n_row_tiles;                    // work units per head: pairs of 128-row query tiles
  uint16_t order[kMobaMaxTiles / 2];  // units, heaviest first
};

struct AttnCommon {
  void* o;
  float* lse;
  int n_q;
  int H;
  float scale_log2;   // softmax scale * log2(e)
  int inject;         // test hook: 1 = one P-ready arrival is never made (a wait runs out)
  long long wait_ns;  // bound of every device wait
};

// Test hook for the failure path (set by kvcr_debug_inject, read at launch).
struct InjectState {
  int kind;
  long long wait_ns;
};
InjectState inject_state();

struct ChunkAttnParams {
  CUtensorMap tm_q;   // 3D (D, H, n_q)
  CUtensorMap tm_kc;  // 4D (D, H, T, slots) cached K
  CUtensorMap tm_vc;  // 4D cached V
  CUtensorMap tm_kn;  // 3D (D, H, n_cur) current K
  CUtensorMap tm_vn;  // 3D current V
  AttnCommon c;
  ChunkSched s;
  // e4m3 QK^T only (tm_q, tm_kc, tm_kn then map the e4m3 codes): scale of each
  // 128-token block and head, [block][H] (cached keys: [slot][block][H])
  const float* q_scale;
  const float* kc_scale;
  const float* kn_scale;
};

struct MobaAttnParams {
  CUtensorMap tm_q;   // 3D (D, H, L)
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  AttnCommon c;
  MobaSched s;
};

cudaError_t launch_chunk_attn_sm100(const ChunkAttnParams& p, int head_dim, int n_q_tiles,
                                    cudaStream_t s, bool qk_e4m3 = false);
cudaError_t launch_moba_attn_sm100(const MobaAttnParams& p, int head_dim, cudaStream_t s);

// fp32 CUDA-core attention over the same key sequence (cached slots + current)
struct F32AttnParams {
  const float* q;       // [n_q][H][D]
  const float* kc;      // cache K area [slots][T][H][D]
  const float* vc;
  const float* kn;      // current K [n_cur][H][D]
  const float* vn;
  float* o;
  float* lse;
  int n_q, H, D, T, n_vis, n_cur;
  float scale;
  int slots[kMaxSlots];
};
cudaError_t launch_attn_f32(const F32AttnParams& p, cudaStream_t s);

// ------------------------------------------------- e4m3 block quantization --
// Segment i: src[i] bf16 [n_tok[i]][H][D] -> dst[i] e4m3 codes (same layout, one
// byte each) and scale[i] fp32 [ceil(n_tok[i] / 128)][H]; the blocks of segment i
// are grid blocks tile0[i] .. tile0[i] + ceil(n_tok[i] / 128) - 1.
constexpr int kMaxQuantSegs = 256;
struct QuantParams {
  const void* src[kMaxQuantSegs];
  void* dst[kMaxQuantSegs];
  float* scale[kMaxQuantSegs];
  int n_tok[kMaxQuantSegs];
  int tile0[kMaxQuantSegs];
  int n_seg, H;
};
cudaError_t launch_quant_e4m3(const QuantParams& p, int head_dim, cudaStream_t s);

// device status words (one per kernel translation unit)
cudaError_t read_and_clear_status_attn(int* st, cudaStream_t s);
cudaError_t read_and_clear_status_f32(int* st, cudaStream_t s);

}  // namespace kvcr
