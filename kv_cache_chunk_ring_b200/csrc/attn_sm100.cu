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
// Design (one CTA = one 128-query tile of one head, 192 threads):
//   warp 4      TMA producer: Q once, then K and V tiles (128 keys x D) through
//               a 2-stage ring; cached-frame tiles come from a 4D tensor map
//               (D, H, T, slot) so a tile never crosses a slot and the frame's
//               ragged tail is zero-filled.
//   warp 5      MMA issuer (one thread): S_j = Q K_j^T into one of two TMEM
//               S buffers (128 columns fp32 each), O += P_j V_j into TMEM O.
//               UMMA 128 x 128 x 16 (S) and 128 x D x 16 (PV), bf16 in, fp32 out.
//   warps 0-3   softmax: thread r owns query row r = TMEM lane r, so the row
//               max / sum are in-thread; exp2 with the scale folded in; P is
//               written bf16 into a 128B-swizzled shared tile (the UMMA A
//               operand); the running max is only moved (and O rescaled in
//               TMEM) when it grows by more than 2^8, and the final
//               normalisation uses the same stale max, so the result is exact.
//   epilogue    O / l -> bf16 -> global, LSE = (m + log2 l) ln 2.
// Every wait is bounded: after 2 s a thread records KVCR_ETIMEOUT in the
// device status word, raises the CTA abort flag and the CTA drains its
// in-flight copies and MMAs before freeing TMEM and returning.
#include <cuda_bf16.h>
#include <math.h>

#include "kvcr_internal.h"
#include "moba_layout.h"
#include "sm100_ptx.cuh"

namespace kvcr {

__device__ int g_attn_status = 0;

namespace {
using namespace ptx;

constexpr int kStages = 2;
constexpr int kThreads = 192;
constexpr int kWarpTma = 4;
constexpr int kWarpMma = 5;
constexpr float kRescaleLog2 = 8.0f;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 256;  // O accumulator columns [256, 256 + D)

struct __align__(8) Ctl {
  uint64_t q_full;
  uint64_t k_full[kStages], k_empty[kStages], v_full[kStages], v_empty[kStages];
  uint64_t s_full[2];
  uint64_t p_full;
  uint64_t o_done;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int n_tiles;
  int pad;
  uint16_t tiles[kMobaMaxTiles];  // MoBA: key tile | class << 12
};

template <int HD>
struct Smem {
  static constexpr int kBoxes = HD / 64;          // 64-element (128-byte) boxes per row
  static constexpr int kBoxBytes = 128 * 128;     // 128 rows x 128 bytes
  static constexpr int kTileBytes = kBoxes * kBoxBytes;
  static constexpr int kPBytes = 2 * kBoxBytes;   // 128 x 128 bf16
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTileBytes;
  static constexpr int kV = kK + kStages * kTileBytes;
  static constexpr int kP = kV + kStages * kTileBytes;
  static constexpr int kCtl = kP + kPBytes;
  static constexpr int kBytes = kCtl + (int)sizeof(Ctl) + 1024;  // + 1024 B alignment slack
};

struct TileRef {
  int map;    // 0 = cached slots (4D) / MoBA keys, 1 = current chunk
  int slot;   // cache slot (map 0, chunk attention)
  int row0;   // first key row of the tile within its tensor
  int valid;  // keys of the tile inside the tensor
  int cls;    // kTileFull / kTilePartial
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
  t.cls = kTileFull;
  return t;
}

__device__ __forceinline__ TileRef tile_ref(const MobaAttnParams& p, const Ctl* ctl, int j) {
  TileRef t;
  const uint32_t e = ctl->tiles[j];
  t.map = 0;
  t.slot = 0;
  t.row0 = (int)(e & 0xFFFu) * kTile;
  t.valid = min(kTile, p.s.L - t.row0);
  t.cls = (int)(e >> 12);
  return t;
}

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, Ctl* ctl) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (*reinterpret_cast<volatile int*>(&ctl->abort)) return false;
    if (globaltimer() - t0 > (uint64_t)kWaitTimeoutNs) {
      atomicExch(&g_attn_status, (int)KVCR_ETIMEOUT);
      *reinterpret_cast<volatile int*>(&ctl->abort) = 1;
      return false;
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

template <int HD>
__device__ __forceinline__ void load_kv_tile(const ChunkAttnParams& p, const TileRef& t, bool is_v,
                                             uint8_t* dst, uint64_t* bar, int h) {
#pragma unroll
  for (int b = 0; b < Smem<HD>::kBoxes; ++b) {
    uint8_t* d = dst + b * Smem<HD>::kBoxBytes;
    if (t.map == 0)
      tma_load_4d(d, is_v ? &p.tm_vc : &p.tm_kc, bar, b * 64, h, t.row0, t.slot);
    else
      tma_load_3d(d, is_v ? &p.tm_vn : &p.tm_kn, bar, b * 64, h, t.row0);
  }
}

template <int HD>
__device__ __forceinline__ void load_kv_tile(const MobaAttnParams& p, const TileRef& t, bool is_v,
                                             uint8_t* dst, uint64_t* bar, int h) {
#pragma unroll
  for (int b = 0; b < Smem<HD>::kBoxes; ++b)
    tma_load_3d(dst + b * Smem<HD>::kBoxBytes, is_v ? &p.tm_v : &p.tm_k, bar, b * 64, h, t.row0);
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

// MoBA: list the non-empty key tiles of query tile qt (one warp).
__device__ void build_moba_list(const MobaAttnParams& p, int qt, Ctl* ctl, int lane) {
  const MobaLay lay{p.s.n_chunks, p.s.chunk_tokens, p.s.n_bidir, p.s.L};
  const int r0 = qt * kTile;
  const int r1 = min(r0 + kTile, p.s.L);
  int lo, hi;
  moba_row_bounds(lay, r0, r1, lo, hi);
  const int kt0 = lo / kTile, kt1 = (hi + kTile - 1) / kTile;
  int count = 0;
  for (int base = kt0; base < kt1; base += 32) {
    const int kt = base + lane;
    const int cls = kt < kt1 ? moba_classify(lay, qt, kt, kTile) : (int)kTileEmpty;
    const unsigned ball = __ballot_sync(0xFFFFFFFFu, cls != kTileEmpty);
    if (cls != kTileEmpty)
      ctl->tiles[count + __popc(ball & ((1u << lane) - 1u))] = (uint16_t)(kt | (cls << 12));
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

// 2^x on the SFU (MUFU.EX2); -inf -> +0.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

template <int HD, bool kMoba, typename Params>
__global__ void __launch_bounds__(kThreads, 1) attn_fwd_kernel(const __grid_constant__ Params p) {
  using L = Smem<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  Ctl* ctl = reinterpret_cast<Ctl*>(smem + L::kCtl);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  int qt, h;
  if constexpr (kMoba) {
    h = blockIdx.x / p.s.n_row_tiles;
    qt = p.s.order[blockIdx.x - h * p.s.n_row_tiles];
  } else {
    qt = blockIdx.x;
    h = blockIdx.y;
  }
  const int q0 = qt * kTile;

  if (threadIdx.x == 0) {
    mbar_init(&ctl->q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ctl->k_full[s], 1);
      mbar_init(&ctl->k_empty[s], 1);
      mbar_init(&ctl->v_full[s], 1);
      mbar_init(&ctl->v_empty[s], 1);
    }
    mbar_init(&ctl->s_full[0], 1);
    mbar_init(&ctl->s_full[1], 1);
    mbar_init(&ctl->p_full, 128);
    mbar_init(&ctl->o_done, 1);
    mbar_init(&ctl->drain, 1);
    ctl->abort = 0;
    if constexpr (!kMoba) ctl->n_tiles = p.s.n_vis * p.s.tiles_per_slot + p.s.cur_tiles;
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(&ctl->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if constexpr (kMoba) {
    if (warp == kWarpTma) build_moba_list(p, qt, ctl, lane);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  const int n_tiles = ctl->n_tiles;

  if (warp == kWarpTma) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0 && n_tiles > 0) {
      prefetch_maps(p);
      mbar_arrive_expect_tx(&ctl->q_full, L::kTileBytes);
#pragma unroll
      for (int b = 0; b < L::kBoxes; ++b)
        tma_load_3d(smem + L::kQ + b * L::kBoxBytes, &p.tm_q, &ctl->q_full, b * 64, h, q0);
      int issued = 0;  // tiles whose K and V loads were issued
      bool ok = true;
      for (int j = 0; j < n_tiles; ++j) {
        const int st = j % kStages;
        const uint32_t ph = (uint32_t)(j / kStages) & 1u;
        const TileRef t = tile_ref(p, ctl, j);
        if (!(ok = wait_bar(&ctl->k_empty[st], ph ^ 1u, ctl))) break;
        mbar_arrive_expect_tx(&ctl->k_full[st], L::kTileBytes);
        load_kv_tile<HD>(p, t, false, smem + L::kK + st * L::kTileBytes, &ctl->k_full[st], h);
        if (!(ok = wait_bar(&ctl->v_empty[st], ph ^ 1u, ctl))) {
          issued = j;  // K of tile j in flight: drained below with the V side skipped
          drain_wait(&ctl->k_full[st], ph);
          break;
        }
        mbar_arrive_expect_tx(&ctl->v_full[st], L::kTileBytes);
        load_kv_tile<HD>(p, t, true, smem + L::kV + st * L::kTileBytes, &ctl->v_full[st], h);
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
      constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t kIdescO = idesc_bf16_f32(128, HD, true);
      const uint32_t sQ = smem_u32(smem + L::kQ);
      const uint32_t sK = smem_u32(smem + L::kK);
      const uint32_t sV = smem_u32(smem + L::kV);
      const uint32_t sP = smem_u32(smem + L::kP);
      bool ok = wait_bar(&ctl->q_full, 0, ctl);
      tc_fence_after();
      for (int j = 0; ok && j <= n_tiles; ++j) {
        if (j < n_tiles) {
          const int st = j % kStages;
          if (!(ok = wait_bar(&ctl->k_full[st], (uint32_t)(j / kStages) & 1u, ctl))) break;
          tc_fence_after();
          const uint32_t d = tmem + (uint32_t)(j & 1) * 128u;
          const uint32_t kb = sK + st * L::kTileBytes;
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            const uint32_t off = (kk >> 2) * L::kBoxBytes + (kk & 3) * 32;
            umma_ss(d, sdesc_sw128(sQ + off, 16, 1024), sdesc_sw128(kb + off, 16, 1024), kIdescS,
                    kk > 0 ? 1u : 0u);
          }
          umma_commit(&ctl->s_full[j & 1]);
          umma_commit(&ctl->k_empty[st]);
        }
        if (j >= 1) {
          const int jj = j - 1;
          const int st = jj % kStages;
          if (!(ok = wait_bar(&ctl->p_full, (uint32_t)jj & 1u, ctl))) break;
          if (!(ok = wait_bar(&ctl->v_full[st], (uint32_t)(jj / kStages) & 1u, ctl))) break;
          tc_fence_after();
          const uint32_t vb = sV + st * L::kTileBytes;
#pragma unroll
          for (int kk = 0; kk < 128 / 16; ++kk) {
            const uint32_t poff = (kk >> 2) * L::kBoxBytes + (kk & 3) * 32;
            umma_ss(tmem + kTmemO, sdesc_sw128(sP + poff, 16, 1024),
                    sdesc_sw128(vb + kk * 16 * 128, L::kBoxBytes, 1024), kIdescO,
                    (jj > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&ctl->o_done);
          umma_commit(&ctl->v_empty[st]);
        }
      }
      if (!ok) {
        umma_commit(&ctl->drain);
        drain_wait(&ctl->drain, 0);
      }
    }
  } else {
    // --------------------------------------------- softmax + epilogue ----
    const int r = threadIdx.x;                      // query row in the tile = TMEM lane
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const float sl2 = p.c.scale_log2;
    uint8_t* sP = smem + L::kP;
    float m_ref = -INFINITY;                        // running (possibly stale) max, log2 units
    float l_sum = 0.f;
    bool ok = true;

    // MoBA: the keys this row may read form at most two intervals [a0,b0) u [a1,b1).
    int a0 = 0, b0 = 0, a1 = 0, b1 = 0;
    if constexpr (kMoba) {
      const MobaLay lay{p.s.n_chunks, p.s.chunk_tokens, p.s.n_bidir, p.s.L};
      const int row = min(q0 + r, p.s.L - 1);
      int lo[2] = {0, 0}, hi[2] = {0, 0};
      moba_row_intervals(lay, row, row + 1, lo, hi, 2);
      a0 = lo[0]; b0 = hi[0]; a1 = lo[1]; b1 = hi[1];
    }

    for (int j = 0; j < n_tiles; ++j) {
      ok = wait_bar(&ctl->s_full[j & 1], (uint32_t)(j >> 1) & 1u, ctl);
      if (!__all_sync(0xFFFFFFFFu, ok)) {  // leave the loop warp-uniformly
        ok = false;
        break;
      }
      tc_fence_after();
      __syncwarp();
      uint32_t s[128];
      const uint32_t sbase = tmem + lane_base + (uint32_t)(j & 1) * 128u;
      tmem_ld_32x32b_x32(sbase + 0, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
      tmem_ld_32x32b_x32(sbase + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
      tmem_ld_32x32b_x32(sbase + 64, *reinterpret_cast<uint32_t(*)[32]>(&s[64]));
      tmem_ld_32x32b_x32(sbase + 96, *reinterpret_cast<uint32_t(*)[32]>(&s[96]));
      tmem_ld_wait();

      const TileRef t = tile_ref(p, ctl, j);
      if (t.valid < kTile || (kMoba && t.cls == kTilePartial)) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int base = t.row0 + 32 * c;
          uint32_t keep = bit_range(0, t.valid - 32 * c);
          if (kMoba && t.cls == kTilePartial)
            keep &= bit_range(a0 - base, b0 - base) | bit_range(a1 - base, b1 - base);
#pragma unroll
          for (int n = 0; n < 32; ++n)
            if (!((keep >> n) & 1u)) s[32 * c + n] = __float_as_uint(-INFINITY);
        }
      }
      float mx = -INFINITY;
#pragma unroll
      for (int n = 0; n < 128; ++n) mx = fmaxf(mx, __uint_as_float(s[n]));
      const float m_new = fmaxf(m_ref, mx * sl2);

      // PV of the previous tile must be done before P is overwritten or O rescaled.
      if (j >= 1) {
        ok = wait_bar(&ctl->o_done, (uint32_t)(j - 1) & 1u, ctl);
        if (!__all_sync(0xFFFFFFFFu, ok)) {
          ok = false;
          break;
        }
        tc_fence_after();
      }
      const bool grow = m_new > m_ref + kRescaleLog2;
      if (__any_sync(0xFFFFFFFFu, grow)) {
        const float alpha = (m_ref == -INFINITY) ? 0.f : ex2(m_ref - m_new);
        if (j >= 1) {
          __syncwarp();
#pragma unroll 1
          for (int c = 0; c < HD / 32; ++c) {
            uint32_t o[32];
            const uint32_t oaddr = tmem + lane_base + kTmemO + c * 32;
            tmem_ld_32x32b_x32(oaddr, o);
            tmem_ld_wait();
#pragma unroll
            for (int n = 0; n < 32; ++n) o[n] = __float_as_uint(__uint_as_float(o[n]) * alpha);
            tmem_st_32x32b_x32(oaddr, o);
          }
          tmem_st_wait();
        }
        l_sum *= alpha;
        if (m_new != -INFINITY) m_ref = m_new;
      }
      const float msub = (m_ref == -INFINITY) ? 0.f : m_ref;
#pragma unroll
      for (int g = 0; g < 16; ++g) {                // 16 groups of 8 keys
        uint32_t packed[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float p0 = ex2(fmaf(__uint_as_float(s[g * 8 + 2 * e]), sl2, -msub));
          const float p1 = ex2(fmaf(__uint_as_float(s[g * 8 + 2 * e + 1]), sl2, -msub));
          l_sum += p0 + p1;
          __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
          packed[e] = *reinterpret_cast<uint32_t*>(&b2);
        }
        const int box = g >> 3, c16 = g & 7;
        uint8_t* dst = sP + box * L::kBoxBytes + r * 128 + ((c16 ^ (r & 7)) << 4);
        *reinterpret_cast<uint4*>(dst) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&ctl->p_full);
    }

    // ---------------------------------------------------------- epilogue --
    if (ok && n_tiles > 0) ok = wait_bar(&ctl->o_done, (uint32_t)(n_tiles - 1) & 1u, ctl);
    ok = __all_sync(0xFFFFFFFFu, ok);
    tc_fence_after();
    __syncwarp();
    const int row = q0 + r;
    const bool row_ok = ok && row < p.c.n_q;
    const float inv_l = l_sum > 0.f ? 1.f / l_sum : 0.f;
    __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.c.o) + ((size_t)row * p.c.H + h) * HD;
#pragma unroll 1
    for (int c = 0; c < HD / 32; ++c) {
      uint32_t o[32];
      if (n_tiles > 0 && ok) {
        tmem_ld_32x32b_x32(tmem + lane_base + kTmemO + c * 32, o);
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
      const float lse = l_sum > 0.f ? (m_ref + log2f(l_sum)) * 0.6931471805599453f : -INFINITY;
      p.c.lse[(size_t)h * p.c.n_q + row] = lse;
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

template <int HD, bool kMoba, typename Params>
cudaError_t launch_impl(const Params& p, dim3 grid, cudaStream_t s) {
  auto kern = attn_fwd_kernel<HD, kMoba, Params>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Smem<HD>::kBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  kern<<<grid, kThreads, Smem<HD>::kBytes, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_attn_sm100(const ChunkAttnParams& p, int head_dim, int n_q_tiles,
                                    cudaStream_t s) {
  dim3 grid((unsigned)n_q_tiles, (unsigned)p.c.H);
  if (head_dim == 128) return launch_impl<128, false>(p, grid, s);
  if (head_dim == 64) return launch_impl<64, false>(p, grid, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_moba_attn_sm100(const MobaAttnParams& p, int head_dim, cudaStream_t s) {
  dim3 grid((unsigned)(p.s.n_row_tiles * p.c.H));
  if (head_dim == 128) return launch_impl<128, true>(p, grid, s);
  if (head_dim == 64) return launch_impl<64, true>(p, grid, s);
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
