// Tensor-core attention for sm_100a: chunk attention over the slot-indirected
// KV cache, and MoBA block-sparse attention.
//
// What it computes (per head): O = softmax(scale * Q K^T) V and
// LSE = log sum exp(scale * Q K^T) over the keys a query may read, with fp32
// accumulation.  Chunk attention reads every cached frame (anchors + window,
// in slot order) then the current chunk ("LingBot-World-Infinity: The
// Open-Source World Model That Refuses to Forget", "How the cache keeps the
// world alive"; "Westlake AGI Lab's 'World in World' ...", second paragraph:
// 6 anchor + 8 recent + 4 current latent frames).  MoBA reads keys by the
// teacher-forcing + bidirectional rule ("Infinite Worlds with Versatile
// Interactions", causal-pretraining paragraph) and skips empty 128 x 128 tiles.
//
// Design (one CTA = two 128-query tiles of one head, 384 threads = 3 warpgroups;
// the producer warpgroup gives registers to the two softmax warpgroups):
//   warp 8      TMA producer: Q0 and Q1 once, then K and V tiles (128 keys x D)
//               through a 2-stage ring shared by both query tiles; cached-frame
//               tiles come from a 4D tensor map (D, H, T, slot) so a tile never
//               crosses a slot and the frame's ragged tail is zero-filled.
//   warp 9      MMA issuer (one thread), tcgen05.mma kind::f16, fp32 in TMEM:
//                 S_t = Q_t K_j^T          (A, B from shared memory)
//                 O_t += P_t V_j           (A = P_t from TMEM, B = V from smem)
//               issued in the order  PV_0(j), S_0(j+1), PV_1(j), S_1(j+1), so the
//               tensor core works on one tile while the other tile's softmax
//               runs.  P_t overwrites S_t in TMEM (bf16 pairs packed in 32-bit
//               columns); MMAs of one thread execute in issue order, so S_t(j+1)
//               is written only after PV_t(j) has read P_t(j).
//   warps 0-3   softmax of tile 0, warps 4-7 softmax of tile 1: thread r owns
//               query row r = TMEM lane r, so the row max / sum stay in-thread;
//               exp2 with the scale folded in (packed fp32x2 arithmetic); P is
//               released to the MMA in two 64-key halves and the row sum is
//               accumulated after the release, off the path to the MMA; the
//               running max only moves (and O_t is rescaled in TMEM) when it
//               grows by more than 2^8, and the final normalisation uses the same
//               stale max, so the result is exact.
//   epilogue    each softmax warpgroup: O_t / l -> bf16 -> global, LSE.
// Every wait is bounded: after 2 s a thread records KVCR_ETIMEOUT in the device
// status word, raises the CTA abort flag and the CTA drains its in-flight
// copies and MMAs before freeing TMEM and returning.
#include <cuda_bf16.h>
#include <math.h>

#include "kvcr_internal.h"
#include "moba_layout.h"
#include "sm100_ptx.cuh"

namespace kvcr {

__device__ int g_attn_status = 0;

namespace {
using namespace ptx;

constexpr int kMaxDevices = 64;

constexpr int kStages = 2;
constexpr int kThreads = 384;
// Register budgets after setmaxnreg: launch 384 x 168; producer warpgroup
// (TMA warp, MMA warp, two idle warps) 80, softmax warpgroups 208 each:
// 128 x (208 + 208 + 80) = 63488 <= 384 x 168 = 64512.
constexpr uint32_t kRegsProducer = 80;
constexpr uint32_t kRegsSoftmax = 208;
constexpr int kWarpTma = 8;
constexpr int kWarpMma = 9;
constexpr float kRescaleLog2 = 8.0f;
// P of a tile is released to the MMA in this many parts of 128 / kPParts keys.
constexpr int kPParts = 2;
// Of the 16 key pairs in each 32-key group, pairs [0, kExpSfuPairs) take exp2 on
// the SFU and the rest on the FMA pipe.  With bf16 QK^T all go to the SFU (1 or 2
// of 16 on the FMA pipe measured the same or ~1 % slower); with the e4m3 QK^T
// (half the S product time) 4 of 16 on the FMA pipe measured fastest per 832x464
// call: 0.768 ms against 0.780 with 2 of 16, 0.786 with 6 of 16, 0.81-0.82 with none.
constexpr int kExpSfuPairs = 16;
constexpr int kExpSfuPairsE4m3 = 12;
constexpr uint32_t kTmemCols = 512;
// TMEM columns: S_t / P_t at t * 128, O_t at 256 + t * 128.
constexpr uint32_t kTmemS = 0;
constexpr uint32_t kTmemO = 256;

struct __align__(8) Ctl {
  uint64_t q_full;
  uint64_t k_full[kStages], k_empty[kStages], v_full[kStages], v_empty[kStages];
  uint64_t s_full[2], p_full[2][kPParts], o_done[2];  // p_full[tile][key part]
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int n_tiles;
  int pad;
  unsigned long long wait_ns;  // bound of every wait (from the launch parameters)
  uint16_t tiles[kMobaMaxTiles];  // MoBA: key tile | class(tile 0) << 12 | class(tile 1) << 14
};

// kFp8: Q and K tiles hold e4m3 codes (one 128-byte box per 128-element row);
// V stays bf16.
template <int HD, bool kFp8>
struct Smem {
  static_assert(!kFp8 || HD == 128, "e4m3 QK^T tiles need head_dim 128");
  static constexpr int kBoxes = HD / 64;          // 64-element (128-byte) bf16 boxes per row
  static constexpr int kBoxBytes = 128 * 128;     // 128 rows x 128 bytes
  static constexpr int kTileBytes = kBoxes * kBoxBytes;                   // V tile
  static constexpr int kQKBoxes = kFp8 ? HD / 128 : kBoxes;              // Q / K boxes per row
  static constexpr int kQKBoxElems = kFp8 ? 128 : 64;
  static constexpr int kQKTileBytes = kQKBoxes * kBoxBytes;               // Q / K tile
  static constexpr int kQ = 0;                    // Q0, Q1
  static constexpr int kK = kQ + 2 * kQKTileBytes;
  static constexpr int kV = kK + kStages * kQKTileBytes;
  static constexpr int kCtl = kV + kStages * kTileBytes;
  static constexpr int kBytes = kCtl + (int)sizeof(Ctl) + 1024;  // + 1024 B alignment slack
};

struct TileRef {
  int map;    // 0 = cached slots (4D) / MoBA keys, 1 = current chunk
  int slot;   // cache slot (map 0, chunk attention)
  int row0;   // first key row of the tile within its tensor
  int valid;  // keys of the tile inside the tensor
  int cls0;   // class for query tile 0 / 1 (kTileFull: no mask needed)
  int cls1;
};

__device__ __forceinline__ TileRef tile_ref(const ChunkAttnParams& p, const Ctl*, int j) {
  TileRef t;
  const int n_cached = p.s.n_vis * p.s.tiles_per_slot;
  if (j < n_cached) {
    const int si = j / p.s.tiles_per_slot;
    const int tt = j - si * p.s.tiles_per_slot;
    t.map = 0;
    t.slot = p.s.slots[si];
    t.row0 = tt * kTile;
    t.valid = min(kTile, p.s.T - t.row0);
  } else {
    const int tt = j - n_cached;
    t.map = 1;
    t.slot = 0;
    t.row0 = tt * kTile;
    t.valid = min(kTile, p.s.n_cur - t.row0);
  }
  t.cls0 = t.cls1 = kTileFull;
  return t;
}

__device__ __forceinline__ TileRef tile_ref(const MobaAttnParams& p, const Ctl* ctl, int j) {
  TileRef t;
  const uint32_t e = ctl->tiles[j];
  t.map = 0;
  t.slot = 0;
  t.row0 = (int)(e & 0xFFFu) * kTile;
  t.valid = min(kTile, p.s.L - t.row0);
  t.cls0 = (int)((e >> 12) & 3u);
  t.cls1 = (int)((e >> 14) & 3u);
  return t;
}

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, Ctl* ctl) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (*reinterpret_cast<volatile int*>(&ctl->abort)) return false;
    if (globaltimer() - t0 > ctl->wait_ns) {
      atomicExch(&g_attn_status, (int)KVCR_ETIMEOUT);
      *reinterpret_cast<volatile int*>(&ctl->abort) = 1;
      return false;
    }
  }
  return true;
}

// Same contract as wait_bar, for the single MMA-issuing thread: it polls with the
// non-suspending test so it reacts to a completed phase without a sleep quantum.
__device__ __forceinline__ bool spin_bar(uint64_t* bar, uint32_t parity, Ctl* ctl) {
  if (mbar_test_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  uint32_t n = 0;
  while (!mbar_test_wait(bar, parity)) {
    if ((++n & 255u) == 0u) {
      if (*reinterpret_cast<volatile int*>(&ctl->abort)) return false;
      if (globaltimer() - t0 > ctl->wait_ns) {
        atomicExch(&g_attn_status, (int)KVCR_ETIMEOUT);
        *reinterpret_cast<volatile int*>(&ctl->abort) = 1;
        return false;
      }
    }
  }
  return true;
}

// Wait used while draining after an abort: ignores the abort flag, bounded.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > (uint64_t)kWaitTimeoutNs) return;
  }
}

template <int HD, bool kFp8>
__device__ __forceinline__ void load_kv_tile(const ChunkAttnParams& p, const TileRef& t, bool is_v,
                                             uint8_t* dst, uint64_t* bar, int h) {
  using L = Smem<HD, kFp8>;
  const int n_box = is_v ? L::kBoxes : L::kQKBoxes;
  const int box_elems = is_v ? 64 : L::kQKBoxElems;
#pragma unroll
  for (int b = 0; b < L::kBoxes; ++b) {
    if (b >= n_box) break;
    uint8_t* d = dst + b * L::kBoxBytes;
    if (t.map == 0)
      tma_load_4d(d, is_v ? &p.tm_vc : &p.tm_kc, bar, b * box_elems, h, t.row0, t.slot);
    else
      tma_load_3d(d, is_v ? &p.tm_vn : &p.tm_kn, bar, b * box_elems, h, t.row0);
  }
}

template <int HD, bool kFp8>
__device__ __forceinline__ void load_kv_tile(const MobaAttnParams& p, const TileRef& t, bool is_v,
                                             uint8_t* dst, uint64_t* bar, int h) {
#pragma unroll
  for (int b = 0; b < Smem<HD, false>::kBoxes; ++b)
    tma_load_3d(dst + b * Smem<HD, false>::kBoxBytes, is_v ? &p.tm_v : &p.tm_k, bar, b * 64, h,
                t.row0);
}

__device__ __forceinline__ void prefetch_maps(const ChunkAttnParams& p) {
  prefetch_tmap(&p.tm_q);
  prefetch_tmap(&p.tm_kc);
  prefetch_tmap(&p.tm_vc);
  prefetch_tmap(&p.tm_kn);
  prefetch_tmap(&p.tm_vn);
}
__device__ __forceinline__ void prefetch_maps(const MobaAttnParams& p) {
  prefetch_tmap(&p.tm_q);
  prefetch_tmap(&p.tm_k);
  prefetch_tmap(&p.tm_v);
}

// MoBA: list the key tiles that are non-empty for query tile 2u or 2u + 1
// (one warp), with each tile's class for both query tiles.
__device__ void build_moba_list(const MobaAttnParams& p, int unit, Ctl* ctl, int lane) {
  const MobaLay lay{p.s.n_chunks, p.s.chunk_tokens, p.s.n_bidir, p.s.L};
  const int qt0 = 2 * unit;
  const int r0 = qt0 * kTile;
  const int r1 = min(r0 + 2 * kTile, p.s.L);
  int lo, hi;
  moba_row_bounds(lay, r0, r1, lo, hi);
  const int kt0 = lo / kTile, kt1 = (hi + kTile - 1) / kTile;
  int count = 0;
  for (int base = kt0; base < kt1; base += 32) {
    const int kt = base + lane;
    int c0 = kTileEmpty, c1 = kTileEmpty;
    if (kt < kt1) {
      c0 = moba_classify(lay, qt0, kt, kTile);
      c1 = moba_classify(lay, qt0 + 1, kt, kTile);
    }
    const bool keep = c0 != kTileEmpty || c1 != kTileEmpty;
    const unsigned ball = __ballot_sync(0xFFFFFFFFu, keep);
    if (keep)
      ctl->tiles[count + __popc(ball & ((1u << lane) - 1u))] =
          (uint16_t)(kt | (c0 << 12) | (c1 << 14));
    count += __popc(ball);
  }
  if (lane == 0) ctl->n_tiles = count;
}

// Bits [lo, hi) of a 32-bit word, the range clipped to [0, 32).
__device__ __forceinline__ uint32_t bit_range(int lo, int hi) {
  lo = max(lo, 0);
  hi = min(hi, 32);
  if (hi <= lo) return 0u;
  const uint32_t upto_hi = hi >= 32 ? 0xFFFFFFFFu : ((1u << hi) - 1u);
  return upto_hi & ~((1u << lo) - 1u);
}

// max(a, b, c) in one instruction (sm_100 three-input max).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 2^x on the SFU (MUFU.EX2); -inf -> +0.
__device__ __forceinline__ float ex2_sfu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x on the FMA / integer pipes for two values at once (keeps the SFU free).
// Cody-Waite style range reduction x = n + f, n = round(x) taken from the low
// mantissa bits of x + 1.5 * 2^23, f in [-1/2, 1/2]; 2^f by the cubic
// 1 + f (c1 + f (c2 + f c3)) fitted here to 2^f on [-1/2, 1/2] for least
// maximum relative error (Lawson-weighted least squares; max relative error
// 1.02e-4, below the bf16 rounding of P); n is added to the exponent field.
// x is clamped at -127, where the result is exactly +0 (p(0) = 1), so masked
// scores give 0.  The arithmetic uses packed fp32x2 instructions.
constexpr float kExpC1 = 0.6932829022f, kExpC2 = 0.2422103733f, kExpC3 = 0.0550085828f;
__device__ __forceinline__ float2 ex2_fma2(float2 x) {
  const float2 kShift = make_float2(12582912.0f, 12582912.0f);
  const float2 kNegShift = make_float2(-12582912.0f, -12582912.0f);
  const float2 one = make_float2(1.0f, 1.0f);
  const float2 c1 = make_float2(kExpC1, kExpC1);
  const float2 c2 = make_float2(kExpC2, kExpC2);
  const float2 c3 = make_float2(kExpC3, kExpC3);
  x.x = fmaxf(x.x, -127.0f);
  x.y = fmaxf(x.y, -127.0f);
  const float2 t = fadd2(x, kShift);
  const float2 n = fadd2(t, kNegShift);
  const float2 f = ffma2(n, make_float2(-1.0f, -1.0f), x);
  const float2 p = ffma2(f, ffma2(f, ffma2(f, c3, c2), c1), one);
  return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Scale of the e4m3 key block of tile t for head h (chunk attention).
__device__ __forceinline__ float key_block_scale(const ChunkAttnParams& p, const TileRef& t, int h) {
  const int blk = t.row0 >> 7;
  return t.map == 0 ? __ldg(p.kc_scale + ((size_t)t.slot * p.s.tiles_per_slot + blk) * p.c.H + h)
                    : __ldg(p.kn_scale + (size_t)blk * p.c.H + h);
}
__device__ __forceinline__ float key_block_scale(const MobaAttnParams&, const TileRef&, int) {
  return 1.f;
}
__device__ __forceinline__ float query_block_scale(const ChunkAttnParams& p, int q_tile, int h) {
  return q_tile * kTile < p.c.n_q ? __ldg(p.q_scale + (size_t)q_tile * p.c.H + h) : 0.f;
}
__device__ __forceinline__ float query_block_scale(const MobaAttnParams&, int, int) { return 1.f; }

template <int HD, bool kMoba, bool kFp8, typename Params>
__global__ void __launch_bounds__(kThreads, 1) attn_fwd_kernel(const __grid_constant__ Params p) {
  static_assert(!(kMoba && kFp8), "the MoBA kernel is bf16 only");
  using L = Smem<HD, kFp8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  Ctl* ctl = reinterpret_cast<Ctl*>(smem + L::kCtl);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  int unit, h;  // unit = pair of query tiles (rows [256 unit, 256 unit + 256))
  if constexpr (kMoba) {
    h = blockIdx.x / p.s.n_row_tiles;
    unit = p.s.order[blockIdx.x - h * p.s.n_row_tiles];
  } else {
    unit = blockIdx.x;
    h = blockIdx.y;
  }
  const int q0 = unit * 2 * kTile;

  if (threadIdx.x == 0) {
    mbar_init(&ctl->q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ctl->k_full[s], 1);
      mbar_init(&ctl->k_empty[s], 1);
      mbar_init(&ctl->v_full[s], 1);
      mbar_init(&ctl->v_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&ctl->s_full[t], 1);
      for (int q = 0; q < kPParts; ++q) mbar_init(&ctl->p_full[t][q], 128);
      mbar_init(&ctl->o_done[t], 1);
    }
    mbar_init(&ctl->drain, 1);
    ctl->abort = 0;
    ctl->wait_ns = p.c.wait_ns > 0 ? (unsigned long long)p.c.wait_ns
                                   : (unsigned long long)kWaitTimeoutNs;
    if constexpr (!kMoba) ctl->n_tiles = p.s.n_vis * p.s.tiles_per_slot + p.s.cur_tiles;
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(&ctl->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if constexpr (kMoba) {
    if (warp == kWarpTma) build_moba_list(p, unit, ctl, lane);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  const int n_tiles = ctl->n_tiles;

  if (warp >= 8) {
  setmaxnreg_dec<kRegsProducer>();
  if (warp == kWarpTma) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0 && n_tiles > 0) {
      prefetch_maps(p);
      mbar_arrive_expect_tx(&ctl->q_full, 2 * L::kQKTileBytes);
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int b = 0; b < L::kQKBoxes; ++b)
          tma_load_3d(smem + L::kQ + t * L::kQKTileBytes + b * L::kBoxBytes, &p.tm_q,
                      &ctl->q_full, b * L::kQKBoxElems, h, q0 + t * kTile);
      int issued = 0;  // tiles whose K and V loads were issued
      bool ok = true;
      for (int j = 0; j < n_tiles; ++j) {
        const int st = j % kStages;
        const uint32_t ph = (uint32_t)(j / kStages) & 1u;
        const TileRef t = tile_ref(p, ctl, j);
        if (!(ok = wait_bar(&ctl->k_empty[st], ph ^ 1u, ctl))) break;
        mbar_arrive_expect_tx(&ctl->k_full[st], L::kQKTileBytes);
        load_kv_tile<HD, kFp8>(p, t, false, smem + L::kK + st * L::kQKTileBytes, &ctl->k_full[st],
                               h);
        if (!(ok = wait_bar(&ctl->v_empty[st], ph ^ 1u, ctl))) {
          issued = j;
          drain_wait(&ctl->k_full[st], ph);
          break;
        }
        mbar_arrive_expect_tx(&ctl->v_full[st], L::kTileBytes);
        load_kv_tile<HD, kFp8>(p, t, true, smem + L::kV + st * L::kTileBytes, &ctl->v_full[st], h);
        issued = j + 1;
      }
      if (!ok) {
        // Let every issued copy land before the CTA can exit.
        drain_wait(&ctl->q_full, 0);
        for (int j = issued - kStages < 0 ? 0 : issued - kStages; j < issued; ++j) {
          const int st = j % kStages;
          const uint32_t ph = (uint32_t)(j / kStages) & 1u;
          drain_wait(&ctl->k_full[st], ph);
          drain_wait(&ctl->v_full[st], ph);
        }
      }
    }
  } else if (warp == kWarpMma) {
    // -------------------------------------------------------- MMA issuer --
    if (lane == 0 && n_tiles > 0) {
      constexpr uint32_t kIdescS =
          kFp8 ? idesc_e4m3_f32(128, 128) : idesc_bf16_f32(128, 128, false);
      constexpr uint32_t kIdescO = idesc_bf16_f32(128, HD, true);
      const uint32_t sQ = smem_u32(smem + L::kQ);
      const uint32_t sK = smem_u32(smem + L::kK);
      const uint32_t sV = smem_u32(smem + L::kV);
      // S_t(j) = Q_t K_j^T: K steps of 32 bytes (16 bf16 or 32 e4m3 elements) inside
      // each 128-byte swizzled row
      auto issue_s = [&](int t, int j) {
        const uint32_t d = tmem + kTmemS + (uint32_t)t * 128u;
        const uint32_t qb = sQ + t * L::kQKTileBytes;
        const uint32_t kb = sK + (j % kStages) * L::kQKTileBytes;
#pragma unroll
        for (int kk = 0; kk < HD / (kFp8 ? 32 : 16); ++kk) {
          const uint32_t off = (kk >> 2) * L::kBoxBytes + (kk & 3) * 32;
          if constexpr (kFp8)
            umma_ss_f8(d, sdesc_sw128(qb + off, 16, 1024), sdesc_sw128(kb + off, 16, 1024),
                       kIdescS, kk > 0 ? 1u : 0u);
          else
            umma_ss(d, sdesc_sw128(qb + off, 16, 1024), sdesc_sw128(kb + off, 16, 1024), kIdescS,
                    kk > 0 ? 1u : 0u);
        }
      };
      // O_t += P_t(j) V_j over part hf of the keys, P_t in TMEM (8 packed columns
      // per 16 keys)
      auto issue_pv = [&](int t, int j, int hf) {
        const uint32_t pa = tmem + kTmemS + (uint32_t)t * 128u;
        const uint32_t d = tmem + kTmemO + (uint32_t)t * 128u;
        const uint32_t vb = sV + (j % kStages) * L::kTileBytes;
#pragma unroll
        for (int k4 = 0; k4 < 8 / kPParts; ++k4) {
          const int kk = (8 / kPParts) * hf + k4;
          umma_ts(d, pa + kk * 8, sdesc_sw128(vb + kk * 16 * 128, L::kBoxBytes, 1024), kIdescO,
                  (j > 0 || kk > 0) ? 1u : 0u);
        }
      };
      bool ok = spin_bar(&ctl->q_full, 0, ctl) && spin_bar(&ctl->k_full[0], 0, ctl);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        umma_commit(&ctl->s_full[0]);
        issue_s(1, 0);
        umma_commit(&ctl->s_full[1]);
        umma_commit(&ctl->k_empty[0]);
      }
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int st = j % kStages;
        const bool more = j + 1 < n_tiles;
        // tile 0: PV_0(j) half by half as P arrives, then S_0(j+1)
        if (!(ok = spin_bar(&ctl->v_full[st], (uint32_t)(j / kStages) & 1u, ctl))) break;
        for (int q = 0; ok && q < kPParts; ++q) {
          if (!(ok = spin_bar(&ctl->p_full[0][q], (uint32_t)j & 1u, ctl))) break;
          tc_fence_after();
          issue_pv(0, j, q);
        }
        if (!ok) break;
        if (more) {
          if (!(ok = spin_bar(&ctl->k_full[(j + 1) % kStages],
                              (uint32_t)((j + 1) / kStages) & 1u, ctl)))
            break;
          tc_fence_after();
          issue_s(0, j + 1);
          umma_commit(&ctl->s_full[0]);
        } else {
          umma_commit(&ctl->o_done[0]);
        }
        // tile 1: PV_1(j), then S_1(j+1)
        for (int q = 0; ok && q < kPParts; ++q) {
          if (!(ok = spin_bar(&ctl->p_full[1][q], (uint32_t)j & 1u, ctl))) break;
          tc_fence_after();
          issue_pv(1, j, q);
        }
        if (!ok) break;
        umma_commit(&ctl->v_empty[st]);
        if (more) {
          issue_s(1, j + 1);
          umma_commit(&ctl->s_full[1]);
          umma_commit(&ctl->k_empty[(j + 1) % kStages]);
        } else {
          umma_commit(&ctl->o_done[1]);
        }
      }
      if (!ok) {
        umma_commit(&ctl->drain);
        drain_wait(&ctl->drain, 0);
      }
    }
  }
  } else {
    setmaxnreg_inc<kRegsSoftmax>();
    // --------------------------------------------- softmax + epilogue ----
    const int tq = warp >> 2;                        // query tile of this warpgroup
    const int r = threadIdx.x & 127;                 // row in the tile = TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t s_addr = tmem + lane_base + kTmemS + (uint32_t)tq * 128u;
    const uint32_t o_addr = tmem + lane_base + kTmemO + (uint32_t)tq * 128u;
    const float sl2 = p.c.scale_log2;
    // e4m3 QK^T: S holds code products; a tile's true scores are S * (q scale * k scale)
    const float q_blk_scale = kFp8 ? query_block_scale(p, 2 * unit + tq, h) : 1.f;
    const int row_g = q0 + tq * kTile + r;           // global query row
    float m_ref = -INFINITY;                        // running (possibly stale) max, log2 units
    float l_sum = 0.f;
    bool ok = true;

    // MoBA: the keys this row may read form at most two intervals [a0,b0) u [a1,b1).
    int a0 = 0, b0 = 0, a1 = 0, b1 = 0;
    if constexpr (kMoba) {
      const MobaLay lay{p.s.n_chunks, p.s.chunk_tokens, p.s.n_bidir, p.s.L};
      const int row = min(row_g, p.s.L - 1);
      int lo[2] = {0, 0}, hi[2] = {0, 0};
      moba_row_intervals(lay, row, row + 1, lo, hi, 2);
      a0 = lo[0]; b0 = hi[0]; a1 = lo[1]; b1 = hi[1];
    }

    for (int j = 0; j < n_tiles; ++j) {
      const TileRef t = tile_ref(p, ctl, j);        // independent of S: before the wait
      float sl2t = sl2;                              // log2-domain factor of this tile's S
      if constexpr (kFp8) {
        // a zero block scale gives zero scores: keep the factor positive so that the
        // masked -inf entries stay -inf
        sl2t = fmaxf(sl2 * q_blk_scale * key_block_scale(p, t, h), 1.17549435e-38f);
      }
      ok = wait_bar(&ctl->s_full[tq], (uint32_t)j & 1u, ctl);
      if (!__all_sync(0xFFFFFFFFu, ok)) {  // leave the loop warp-uniformly
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t s[128];
      tmem_ld_32x32b_x32(s_addr + 0, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
      tmem_ld_32x32b_x32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
      tmem_ld_32x32b_x32(s_addr + 64, *reinterpret_cast<uint32_t(*)[32]>(&s[64]));
      tmem_ld_32x32b_x32(s_addr + 96, *reinterpret_cast<uint32_t(*)[32]>(&s[96]));
      tmem_ld_wait();

      const int cls = tq == 0 ? t.cls0 : t.cls1;
      if (t.valid < kTile || (kMoba && cls != kTileFull)) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int base = t.row0 + 32 * c;
          uint32_t keep = bit_range(0, t.valid - 32 * c);
          if (kMoba && cls != kTileFull)
            keep &= bit_range(a0 - base, b0 - base) | bit_range(a1 - base, b1 - base);
#pragma unroll
          for (int n = 0; n < 32; ++n)
            if (!((keep >> n) & 1u)) s[32 * c + n] = __float_as_uint(-INFINITY);
        }
      }
      // row max with three-input max: 16 independent chains, then a tree (72 max
      // instructions for 128 keys)
      float mx[16];
#pragma unroll
      for (int k = 0; k < 16; ++k)
        mx[k] = fmax3(__uint_as_float(s[k]), __uint_as_float(s[16 + k]),
                      __uint_as_float(s[32 + k]));
#pragma unroll
      for (int n = 48; n < 112; n += 32)
#pragma unroll
        for (int k = 0; k < 16; ++k)
          mx[k] = fmax3(mx[k], __uint_as_float(s[n + k]), __uint_as_float(s[n + 16 + k]));
#pragma unroll
      for (int k = 0; k < 16; ++k) mx[k] = fmaxf(mx[k], __uint_as_float(s[112 + k]));
      float mt[6];
#pragma unroll
      for (int k = 0; k < 5; ++k) mt[k] = fmax3(mx[3 * k], mx[3 * k + 1], mx[3 * k + 2]);
      mt[5] = mx[15];
      const float row_max = fmaxf(fmax3(mt[0], mt[1], mt[2]), fmax3(mt[3], mt[4], mt[5]));
      const float m_new = fmaxf(m_ref, row_max * sl2t);

      // O_t is stable here: S_t(j) was committed after PV_t(j-1).
      const bool grow = m_new > m_ref + kRescaleLog2;
      if (__any_sync(0xFFFFFFFFu, grow)) {
        const float alpha = (m_ref == -INFINITY) ? 0.f : ex2_sfu(m_ref - m_new);
        if (j >= 1) {
#pragma unroll 1
          for (int c = 0; c < HD / 32; ++c) {
            uint32_t o[32];
            tmem_ld_32x32b_x32(o_addr + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int n = 0; n < 32; ++n) o[n] = __float_as_uint(__uint_as_float(o[n]) * alpha);
            tmem_st_32x32b_x32(o_addr + c * 32, o);
          }
        }
        l_sum *= alpha;
        if (m_new != -INFINITY) m_ref = m_new;
      }
      const float msub = (m_ref == -INFINITY) ? 0.f : m_ref;
      const float2 sl2x2 = make_float2(sl2t, sl2t);
      const float2 negm = make_float2(-msub, -msub);
#pragma unroll
      for (int c = 0; c < 4; ++c) {                 // 4 groups of 32 keys -> 16 packed columns
        uint32_t packed[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float2 sv = make_float2(__uint_as_float(s[32 * c + 2 * e]),
                                        __uint_as_float(s[32 * c + 2 * e + 1]));
          const float2 x = ffma2(sv, sl2x2, negm);
          float2 pv;
          if (e >= (kFp8 ? kExpSfuPairsE4m3 : kExpSfuPairs)) {  // this share on the FMA pipe
            pv = ex2_fma2(x);
          } else {
            pv = make_float2(ex2_sfu(x.x), ex2_sfu(x.y));
          }
          s[32 * c + 2 * e] = __float_as_uint(pv.x); // kept for the row sum below
          s[32 * c + 2 * e + 1] = __float_as_uint(pv.y);
          __nv_bfloat162 b2 = __floats2bfloat162_rn(pv.x, pv.y);
          packed[e] = *reinterpret_cast<uint32_t*>(&b2);
        }
        tmem_st_32x32b_x16(s_addr + c * 16, packed);
        if (((c + 1) % (4 / kPParts)) == 0) {       // part c / (4 / kPParts) of P is ready
          tmem_st_wait();
          tc_fence_before();
          // test hook: tile 1 withholds its first P-ready arrival, so the MMA issuer's
          // wait runs out and the whole CTA takes the timeout path
          if (!(p.c.inject == 1 && tq == 1 && j == 0 && c == 4 / kPParts - 1))
            mbar_arrive(&ctl->p_full[tq][c / (4 / kPParts)]);
        }
      }
      // the row sum is off the path to the MMA: accumulated after P is released
      float2 lacc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                        make_float2(0.f, 0.f)};
#pragma unroll
      for (int n = 0; n < 128; n += 2)
        lacc[(n >> 1) & 3] = fadd2(lacc[(n >> 1) & 3],
                                   make_float2(__uint_as_float(s[n]), __uint_as_float(s[n + 1])));
      l_sum += ((lacc[0].x + lacc[0].y) + (lacc[1].x + lacc[1].y)) +
               ((lacc[2].x + lacc[2].y) + (lacc[3].x + lacc[3].y));
    }

    // ---------------------------------------------------------- epilogue --
    if (ok && n_tiles > 0) ok = wait_bar(&ctl->o_done[tq], 0, ctl);
    ok = __all_sync(0xFFFFFFFFu, ok);
    tc_fence_after();
    // a CTA that gave up on a wait writes NaN rows (and NaN LSE): its outputs are
    // invalid, and a caller that missed kvcr_check_status() still sees it
    const bool row_ok = row_g < p.c.n_q;
    const float inv_l = !ok ? __int_as_float(0x7FC00000) : (l_sum > 0.f ? 1.f / l_sum : 0.f);
    __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.c.o) + ((size_t)row_g * p.c.H + h) * HD;
#pragma unroll 1
    for (int c = 0; c < HD / 32; ++c) {
      uint32_t o[32];
      if (n_tiles > 0 && ok) {
        tmem_ld_32x32b_x32(o_addr + c * 32, o);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int n = 0; n < 32; ++n) o[n] = 0u;
      }
      if (row_ok) {
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(o[g * 8 + 2 * e]) * inv_l,
                                                      __uint_as_float(o[g * 8 + 2 * e + 1]) * inv_l);
            w[e] = *reinterpret_cast<uint32_t*>(&b2);
          }
          *reinterpret_cast<uint4*>(orow + c * 32 + g * 8) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
    if (row_ok && p.c.lse != nullptr) {
      const float lse = !ok ? __int_as_float(0x7FC00000)
                            : (l_sum > 0.f ? (m_ref + log2f(l_sum)) * 0.6931471805599453f
                                           : -INFINITY);
      p.c.lse[(size_t)h * p.c.n_q + row_g] = lse;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int HD, bool kMoba, bool kFp8, typename Params>
cudaError_t launch_impl(const Params& p, dim3 grid, cudaStream_t s) {
  auto kern = attn_fwd_kernel<HD, kMoba, kFp8, Params>;
  // the shared-memory limit is a per-device attribute of the function
  static bool attr_set[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Smem<HD, kFp8>::kBytes);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  kern<<<grid, kThreads, Smem<HD, kFp8>::kBytes, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_attn_sm100(const ChunkAttnParams& p, int head_dim, int n_q_tiles,
                                    cudaStream_t s, bool qk_e4m3) {
  dim3 grid((unsigned)((n_q_tiles + 1) / 2), (unsigned)p.c.H);
  if (qk_e4m3) {
    if (head_dim == 128) return launch_impl<128, false, true>(p, grid, s);
    return cudaErrorInvalidValue;
  }
  if (head_dim == 128) return launch_impl<128, false, false>(p, grid, s);
  if (head_dim == 64) return launch_impl<64, false, false>(p, grid, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_moba_attn_sm100(const MobaAttnParams& p, int head_dim, cudaStream_t s) {
  dim3 grid((unsigned)(p.s.n_row_tiles * p.c.H));
  if (head_dim == 128) return launch_impl<128, true, false>(p, grid, s);
  if (head_dim == 64) return launch_impl<64, true, false>(p, grid, s);
  return cudaErrorInvalidValue;
}

cudaError_t read_and_clear_status_attn(int* st, cudaStream_t s) {
  int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(st, g_attn_status, sizeof(int), 0,
                                            cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return e;
  e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return e;
  if (*st != 0) e = cudaMemcpyToSymbol(g_attn_status, &zero, sizeof(int));
  return e;
}

}  // namespace kvcr
