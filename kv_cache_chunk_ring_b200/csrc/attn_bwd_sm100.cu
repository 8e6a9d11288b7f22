// Backward pass of MoBA attention on sm_100a: dQ, dK, dV.
//
// What it computes (per head, over the keys each query may read under the
// teacher-forcing + bidirectional rule of "Infinite Worlds with Versatile
// Interactions", causal-pretraining paragraph -- the mask the model is trained
// with; "Mix Forcing", "Mix the training modes"), with P the forward's
// attention probabilities, recomputed from the saved LSE:
//   P_ij = exp(scale * q_i . k_j - LSE_i)        (0 where j is not allowed)
//   dV   = P^T dO        dP = dO V^T        D_i = rowsum(dO o O)_i
//   dS   = P o (dP - D)  dQ = scale * dS K   dK = scale * dS^T Q
// in fp32 on the tensor cores (bf16 operands), written back as bf16.
//
// Three launches, no atomics (the result does not depend on scheduling):
//   prep   per head and 128-row tile: -LSE_i * log2 e of its rows, then -D_i of
//          them (ws[h][t][0][r], ws[h][t][1][r]; negated so that they enter the
//          packed fma and add as they are); rows past L get (-inf, 0), so their
//          probabilities are exactly 0.
//   dK/dV  one CTA per (head, 128-key tile), head-major and heaviest tiles first
//          within a head; K_j, V_j stay in shared memory and
//          the query tiles that may read them stream through a 2-stage ring
//          (Q_i copied first, under a barrier of its own):
//            S^T  = K_j Q_i^T            (SS)       TMEM cols   0-127
//            dP^T = V_j dO_i^T           (SS)       TMEM cols 128-255
//            dV  += P^T dO_i             (TS: P^T in TMEM, dO_i MN-major)  256-383
//            dK  += dS^T Q_i             (TS: dS^T in TMEM, Q_i MN-major)  384-511
//          Thread r of each warpgroup owns key r (TMEM lane r); warpgroup w
//          handles query columns [64 w, 64 w + 64), so LSE and D are per column,
//          staged per stage in shared memory (one 1 KB bulk copy).  Once a
//          warpgroup has read its half of S^T and of dP^T into registers, it
//          writes P^T (bf16 pairs) into the first 32 and dS^T into the last 32
//          of its 64 dP^T columns.  The S^T columns are then free, so S^T(i+1)
//          is issued as soon as they are read and stage i+1 has landed, ahead
//          of dV_i when it can, and overlaps tile i's exponentials; dP^T(i+1)
//          follows dK_i (MMAs of one thread run in issue order).
//   dQ     one CTA per (head, 128-query tile), the key tiles it may read
//          streaming K_j through three slots and V_j through two (the producer
//          warp finds the tiles 32 per ballot and hands them on in a ring):
//            S  = Q K_j^T (SS, cols 0-127)   dP = dO V_j^T (SS, cols 128-255)
//            dQ += dS K_j (TS: dS in TMEM, K_j MN-major; cols 256-383)
//          Thread r owns query r; LSE and D are per row (registers).
// Roles as in the forward kernel: warp 8 issues the TMA copies, warp 9 the MMAs
// (one elected lane of the converged warp; elect.sync picks the same lane every
// time, so its products run in issue order and its commits track them), warps
// 0-7 (two warpgroups, registers raised with setmaxnreg) the elementwise work
// and the epilogue.  Every wait is bounded (2 s): a thread
// that gives up records KVCR_ETIMEOUT, raises the CTA abort flag, and the CTA
// drains its copies and MMAs before freeing TMEM.
#include <cuda_bf16.h>
#include <math.h>

#include <type_traits>

#include "attn_bwd.h"
#include "moba_layout.h"
#include "sm100_ptx.cuh"

namespace kvcr {

__device__ int g_bwd_status = 0;

namespace {
using namespace ptx;

constexpr int kMaxDevices = 64;

constexpr int kStages = 2;
constexpr int kThreads = 384;
// launch 384 x 168 registers; producer warpgroup 80, the two work warpgroups
// 208 each: 128 x (80 + 208 + 208) = 63488 <= 64512.
constexpr uint32_t kRegsProducer = 80;
constexpr uint32_t kRegsWork = 208;
constexpr int kWarpTma = 8;
constexpr int kWarpMma = 9;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemS = 0;     // S^T / P^T (dK/dV kernel), S (dQ kernel)
constexpr uint32_t kTmemDP = 128;  // dP^T / dS^T, dP / dS
constexpr uint32_t kTmemAcc0 = 256;  // dV (dK/dV kernel), dQ (dQ kernel)
constexpr uint32_t kTmemAcc1 = 384;  // dK
constexpr int kWsBytes = kTile * 8;  // (lse, D) of one 128-row tile

struct __align__(8) BwdCtl {
  uint64_t fixed_full;                         // the CTA's own two tiles
  uint64_t x_full[kStages];                    // stage: Q_i
  uint64_t st_full[kStages], st_empty[kStages];  // the rest of the stage; the whole stage
  uint64_t s_full, dp_full, s_free;
  uint64_t p_full[2], ds_full[2];              // per warpgroup (column half)
  uint64_t acc_done;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int n_tiles;
  int pad;
  unsigned long long wait_ns;
  uint16_t tiles[kMobaMaxTiles];               // streamed tile | class << 12
};

template <int HD>
struct BwdSmem {
  static constexpr int kBoxes = HD / 64;
  static constexpr int kBoxBytes = 128 * 128;
  static constexpr int kTileBytes = kBoxes * kBoxBytes;
  static constexpr int kA = 0;                              // K_j   (dK/dV kernel)
  static constexpr int kB = kA + kTileBytes;                // V_j
  static constexpr int kX = kB + kTileBytes;                // stages: Q_i
  static constexpr int kY = kX + kStages * kTileBytes;      // stages: dO_i
  static constexpr int kW = kY + kStages * kTileBytes;      // stages: (lse, D) of Q_i
  static constexpr int kCtl = kW + kStages * kWsBytes;
  static constexpr int kBytes = kCtl + (int)sizeof(BwdCtl) + 1024;
};

// dQ kernel: K_j streams through three slots, so the copy of K_{j+1} is not held
// up until dQ_{j-1} has read K_{j-1}; V_j through two (freed after dP_j).  The
// key-tile list is a ring the producer fills as it goes.  224 KB of tiles.
constexpr int kKStages = 3;
constexpr int kVStages = 2;
constexpr int kRing = 8;

struct __align__(8) DqCtl {
  uint64_t fixed_full;                         // Q_i, dO_i
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t v_full[kVStages], v_empty[kVStages];
  uint64_t s_full, dp_full, s_free;
  uint64_t ds_full[2];                         // per warpgroup (column half)
  uint64_t acc_done;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int n_tiles;
  int pad;
  unsigned long long wait_ns;
  uint16_t tiles[kRing];                       // key tile | class << 12, by j % kRing
};

// Offsets from the first 1024-byte aligned address of the dynamic shared memory;
// the launch asks for at most the per-CTA limit, and the kernel checks the fit.
template <int HD>
struct DqSmem {
  static constexpr int kTileBytes = BwdSmem<HD>::kTileBytes;
  static constexpr int kQ = 0;
  static constexpr int kDO = kQ + kTileBytes;
  static constexpr int kK = kDO + kTileBytes;
  static constexpr int kV = kK + kKStages * kTileBytes;
  static constexpr int kCtl = kV + kVStages * kTileBytes;
  static constexpr int kUsed = kCtl + (int)sizeof(DqCtl);
  static constexpr int kBytes = kUsed + 1024 < 227 * 1024 ? kUsed + 1024 : 227 * 1024;
};
static_assert(DqSmem<128>::kUsed <= 227 * 1024, "dQ shared memory exceeds the per-CTA limit");

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// 1D bulk copy global -> shared, completion counted on an mbarrier
// (addresses 16-byte aligned, size a multiple of 16).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

template <class Ctl>
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, Ctl* ctl) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (*reinterpret_cast<volatile int*>(&ctl->abort)) return false;
    if (globaltimer() - t0 > ctl->wait_ns) {
      atomicExch(&g_bwd_status, (int)KVCR_ETIMEOUT);
      *reinterpret_cast<volatile int*>(&ctl->abort) = 1;
      return false;
    }
  }
  return true;
}

// wait_bar for the MMA-issuing warp: non-suspending polls.
template <class Ctl>
__device__ __forceinline__ bool spin_bar(uint64_t* bar, uint32_t parity, Ctl* ctl) {
  if (mbar_test_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  uint32_t n = 0;
  while (!mbar_test_wait(bar, parity)) {
    if ((++n & 255u) == 0u) {
      if (*reinterpret_cast<volatile int*>(&ctl->abort)) return false;
      if (globaltimer() - t0 > ctl->wait_ns) {
        atomicExch(&g_bwd_status, (int)KVCR_ETIMEOUT);
        *reinterpret_cast<volatile int*>(&ctl->abort) = 1;
        return false;
      }
    }
  }
  return true;
}

// Time / abort check of a hand-written poll loop: true when the CTA is aborting or
// the wait that began at t0 ran out (recording KVCR_ETIMEOUT and raising abort).
template <class Ctl>
__device__ __forceinline__ bool poll_expired(Ctl* ctl, uint64_t t0) {
  if (*reinterpret_cast<volatile int*>(&ctl->abort)) return true;
  if (globaltimer() - t0 > ctl->wait_ns) {
    atomicExch(&g_bwd_status, (int)KVCR_ETIMEOUT);
    *reinterpret_cast<volatile int*>(&ctl->abort) = 1;
    return true;
  }
  return false;
}

// spin_bar for the whole MMA warp: every lane polls (a completed phase stays
// completed until the warp's own later products let the next one finish), and the
// lanes agree on the outcome before the warp goes on, converged.
template <class Ctl>
__device__ __forceinline__ bool spin_bar_w(uint64_t* bar, uint32_t parity, Ctl* ctl) {
  const bool ok = spin_bar(bar, parity, ctl);
  return __all_sync(0xFFFFFFFFu, ok);
}

// Wait used while draining after an abort: ignores the abort flag, bounded.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > (uint64_t)kWaitTimeoutNs) return;
  }
}

__device__ __forceinline__ uint32_t bit_range(int lo, int hi) {
  lo = max(lo, 0);
  hi = min(hi, 32);
  if (hi <= lo) return 0u;
  const uint32_t upto_hi = hi >= 32 ? 0xFFFFFFFFu : ((1u << hi) - 1u);
  return upto_hi & ~((1u << lo) - 1u);
}

__device__ __forceinline__ float ex2_sfu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Packed two-lane fp32 product (sm_100): one instruction for two values.
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

template <int HD>
__device__ __forceinline__ void load_tile(const CUtensorMap* m, uint8_t* dst, uint64_t* bar, int h,
                                          int row0) {
#pragma unroll
  for (int b = 0; b < BwdSmem<HD>::kBoxes; ++b)
    tma_load_3d(dst + b * BwdSmem<HD>::kBoxBytes, m, bar, b * 64, h, row0);
}

// Bounding range [u0, u1) of the tiles streamed past tile t: for the dK/dV kernel
// (kByKey) the query tiles that may read key tile t, for the dQ kernel the key
// tiles query tile t may read.
template <bool kByKey>
__device__ __forceinline__ void list_range(const MobaBwdParams& p, int t, int& u0, int& u1) {
  const MobaLay lay{p.s.n_chunks, p.s.chunk_tokens, p.s.n_bidir, p.s.L};
  const int r0 = t * kTile;
  const int r1 = min(r0 + kTile, p.s.L);
  int lo, hi;
  if (kByKey)
    moba_col_bounds(lay, r0, r1, lo, hi);
  else
    moba_row_bounds(lay, r0, r1, lo, hi);
  u0 = lo / kTile;
  u1 = hi > lo ? (hi + kTile - 1) / kTile : u0;
}

// Class of the pair (tile t, streamed tile u).
template <bool kByKey>
__device__ __forceinline__ int pair_class(const MobaBwdParams& p, int t, int u) {
  const MobaLay lay{p.s.n_chunks, p.s.chunk_tokens, p.s.n_bidir, p.s.L};
  return kByKey ? moba_classify(lay, u, t, kTile) : moba_classify(lay, t, u, kTile);
}

// Count (one warp) the non-empty tiles of that range and, when `tiles` is given,
// list them in order, each with its class (u | class << 12).
template <bool kByKey>
__device__ int build_list(const MobaBwdParams& p, int t, uint16_t* tiles, int lane) {
  int u0, u1;
  list_range<kByKey>(p, t, u0, u1);
  int count = 0;
  for (int base = u0; base < u1; base += 32) {
    const int u = base + lane;
    const int c = u < u1 ? pair_class<kByKey>(p, t, u) : (int)kTileEmpty;
    const bool keep = c != kTileEmpty;
    const unsigned ball = __ballot_sync(0xFFFFFFFFu, keep);
    if (keep && tiles) tiles[count + __popc(ball & ((1u << lane) - 1u))] = (uint16_t)(u | (c << 12));
    count += __popc(ball);
  }
  return count;
}

// The non-empty streamed tiles of [u0, u1) in order, found by the whole warp 32
// candidates at a time (one ballot per block of 32, as build_list); every lane
// gets the same (u, class) from next().
template <bool kByKey>
struct TileFeeder {
  const MobaBwdParams& p;
  int t, lane, base, u1, cls;
  unsigned mask;
  __device__ __forceinline__ TileFeeder(const MobaBwdParams& p_, int t_, int lane_)
      : p(p_), t(t_), lane(lane_), cls(kTileEmpty), mask(0u) {
    int u0;
    list_range<kByKey>(p, t, u0, u1);
    base = u0 - 32;
  }
  // false when the range is exhausted
  __device__ __forceinline__ bool next(int& u, int& c) {
    while (mask == 0u) {
      base += 32;
      if (base >= u1) return false;
      const int v = base + lane;
      cls = v < u1 ? pair_class<kByKey>(p, t, v) : (int)kTileEmpty;
      mask = __ballot_sync(0xFFFFFFFFu, cls != kTileEmpty);
    }
    const int bit = __ffs(mask) - 1;
    mask &= mask - 1u;
    u = base + bit;
    c = __shfl_sync(0xFFFFFFFFu, cls, bit);
    return true;
  }
};

// Prologue of the dK/dV kernel: barriers, TMEM, the list of streamed query tiles.
__device__ __forceinline__ void dkdv_setup(const MobaBwdParams& p, BwdCtl* ctl, int tile,
                                           int warp, int lane) {
  if (threadIdx.x == 0) {
    mbar_init(&ctl->fixed_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ctl->x_full[s], 1);
      mbar_init(&ctl->st_full[s], 1);
      mbar_init(&ctl->st_empty[s], 1);
    }
    mbar_init(&ctl->s_full, 1);
    mbar_init(&ctl->dp_full, 1);
    mbar_init(&ctl->s_free, 256);
    for (int w = 0; w < 2; ++w) {
      mbar_init(&ctl->p_full[w], 128);
      mbar_init(&ctl->ds_full[w], 128);
    }
    mbar_init(&ctl->acc_done, 1);
    mbar_init(&ctl->drain, 1);
    ctl->abort = 0;
    ctl->wait_ns =
        p.wait_ns > 0 ? (unsigned long long)p.wait_ns : (unsigned long long)kWaitTimeoutNs;
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(&ctl->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kWarpTma) {
    const int n = build_list<true>(p, tile, ctl->tiles, lane);
    if (lane == 0) ctl->n_tiles = n;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
}

// TMA producer of the dK/dV kernel (one thread): K_j and V_j, then per streamed
// query tile its Q_i, dO_i and the 1 KB of (lse, D) of its rows.
template <int HD>
__device__ void dkdv_producer(const MobaBwdParams& p, BwdCtl* ctl, uint8_t* smem, int h,
                              int tile) {
  using L = BwdSmem<HD>;
  const int n_tiles = ctl->n_tiles;
  prefetch_tmap(&p.tm_q);
  prefetch_tmap(&p.tm_k);
  prefetch_tmap(&p.tm_v);
  prefetch_tmap(&p.tm_do);
  mbar_arrive_expect_tx(&ctl->fixed_full, 2 * L::kTileBytes);
  load_tile<HD>(&p.tm_k, smem + L::kA, &ctl->fixed_full, h, tile * kTile);
  load_tile<HD>(&p.tm_v, smem + L::kB, &ctl->fixed_full, h, tile * kTile);
  // Q_i is copied first and has a barrier of its own: the next S^T needs only it,
  // and starts before dO_i and (lse, D) land
  constexpr uint32_t kRestBytes = L::kTileBytes + kWsBytes;
  int issued = 0;
  bool ok = true;
  for (int i = 0; i < n_tiles; ++i) {
    const int st = i % kStages;
    const uint32_t ph = (uint32_t)(i / kStages) & 1u;
    const int u = (int)(ctl->tiles[i] & 0xFFFu);
    if (!(ok = wait_bar(&ctl->st_empty[st], ph ^ 1u, ctl))) break;
    mbar_arrive_expect_tx(&ctl->x_full[st], L::kTileBytes);
    load_tile<HD>(&p.tm_q, smem + L::kX + st * L::kTileBytes, &ctl->x_full[st], h, u * kTile);
    mbar_arrive_expect_tx(&ctl->st_full[st], kRestBytes);
    load_tile<HD>(&p.tm_do, smem + L::kY + st * L::kTileBytes, &ctl->st_full[st], h, u * kTile);
    bulk_load(smem + L::kW + st * kWsBytes, p.ws + ((size_t)h * p.s.n_units + u) * 2 * kTile,
              kWsBytes, &ctl->st_full[st]);
    issued = i + 1;
  }
  if (!ok) {
    drain_wait(&ctl->fixed_full, 0);
    for (int i = issued - kStages < 0 ? 0 : issued - kStages; i < issued; ++i) {
      drain_wait(&ctl->x_full[i % kStages], (uint32_t)(i / kStages) & 1u);
      drain_wait(&ctl->st_full[i % kStages], (uint32_t)(i / kStages) & 1u);
    }
  }
}

// S-type product (SS, both K-major over the head dim): D = A(fixed) * B(stage)^T.
template <int HD>
__device__ __forceinline__ void mma_ss_tiles(uint32_t d, uint32_t a, uint32_t b) {
  constexpr uint32_t kIdesc = idesc_bf16_f32(128, 128, false);
#pragma unroll
  for (int kk = 0; kk < HD / 16; ++kk) {
    const uint32_t off = (kk >> 2) * BwdSmem<HD>::kBoxBytes + (kk & 3) * 32;
    umma_ss_w(d, sdesc_sw128(a + off, 16, 1024), sdesc_sw128(b + off, 16, 1024), kIdesc,
              kk > 0 ? 1u : 0u);
  }
}

// Accumulating product over one 64-row half of the streamed tile:
// D += A(TMEM, bf16 pairs of warpgroup `half`) * B(stage rows, MN-major).
template <int HD>
__device__ __forceinline__ void mma_ts_half(uint32_t d, uint32_t a_base, uint32_t b, int half,
                                            bool first) {
  constexpr uint32_t kIdesc = idesc_bf16_f32(128, HD, true);
#pragma unroll
  for (int k4 = 0; k4 < 4; ++k4) {
    const int kk = 4 * half + k4;
    umma_ts_w(d, a_base + (uint32_t)(half * 64 + k4 * 8),
              sdesc_sw128(b + kk * 16 * 128, BwdSmem<HD>::kBoxBytes, 1024), kIdesc,
              (first && kk == 0) ? 0u : 1u);
  }
}

// ------------------------------------------------------------------ dK / dV --
template <int HD>
__global__ void __launch_bounds__(kThreads, 1) moba_dkdv_kernel(const __grid_constant__ MobaBwdParams p) {
  using L = BwdSmem<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  BwdCtl* ctl = reinterpret_cast<BwdCtl*>(smem + L::kCtl);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int h = blockIdx.x / p.s.n_units;             // head-major: co-resident CTAs
  const int kt = p.s.order[blockIdx.x - h * p.s.n_units];  // share one head in L2
  const int k0 = kt * kTile;

  dkdv_setup(p, ctl, kt, warp, lane);
  const uint32_t tmem = ctl->tmem_base;
  const int n_tiles = ctl->n_tiles;

  if (warp >= 8) {
    setmaxnreg_dec<kRegsProducer>();
    if (warp == kWarpTma) {
      if (lane == 0 && n_tiles > 0) dkdv_producer<HD>(p, ctl, smem, h, kt);
    } else if (warp == kWarpMma) {
      if (n_tiles > 0) {          // the whole warp: operands stay warp-uniform
        const uint32_t sK = smem_u32(smem + L::kA), sV = smem_u32(smem + L::kB);
        const uint32_t sQ = smem_u32(smem + L::kX), sDO = smem_u32(smem + L::kY);
        bool ok = spin_bar_w(&ctl->fixed_full, 0, ctl) && spin_bar_w(&ctl->x_full[0], 0, ctl);
        if (ok) {
          tc_fence_after();
          mma_ss_tiles<HD>(tmem + kTmemS, sK, sQ);      // S^T(0)
          umma_commit_w(&ctl->s_full);
          ok = spin_bar_w(&ctl->st_full[0], 0, ctl);
        }
        if (ok) {
          tc_fence_after();
          mma_ss_tiles<HD>(tmem + kTmemDP, sV, sDO);    // dP^T(0)
          umma_commit_w(&ctl->dp_full);
        }
        for (int i = 0; ok && i < n_tiles; ++i) {
          const int st = i % kStages;
          const int sn = (i + 1) % kStages;
          const bool more = i + 1 < n_tiles;
          const uint32_t ph = (uint32_t)i & 1u;
          const uint32_t phn = (uint32_t)((i + 1) / kStages) & 1u;
          // S^T(i+1) goes as soon as the softmax has read S^T(i) and stage i+1 has
          // landed, ahead of dV_i if it can: P^T(i) lives in the dP^T columns, so
          // the S^T columns are free once read, and the next S^T overlaps this
          // tile's exponentials instead of following its dV.
          bool s_pending = more;
          for (int w = 0; ok && w < 2; ++w) {           // dV += P^T dO_i
            const uint64_t t0 = globaltimer();
            uint32_t n = 0;
            for (;;) {
              if (s_pending &&
                  __all_sync(0xFFFFFFFFu, mbar_test_wait(&ctl->s_free, ph) &&
                                              mbar_test_wait(&ctl->x_full[sn], phn))) {
                tc_fence_after();
                mma_ss_tiles<HD>(tmem + kTmemS, sK, sQ + sn * L::kTileBytes);   // S^T(i+1)
                umma_commit_w(&ctl->s_full);
                s_pending = false;
              }
              if (__all_sync(0xFFFFFFFFu, mbar_test_wait(&ctl->p_full[w], ph))) break;
              if ((++n & 255u) == 0u && __any_sync(0xFFFFFFFFu, poll_expired(ctl, t0))) {
                ok = false;
                break;
              }
            }
            if (!ok) break;
            tc_fence_after();
            mma_ts_half<HD>(tmem + kTmemAcc0, tmem + kTmemDP, sDO + st * L::kTileBytes, w, i == 0);
          }
          if (!ok) break;
          if (s_pending) {
            if (!(ok = spin_bar_w(&ctl->s_free, ph, ctl) && spin_bar_w(&ctl->x_full[sn], phn, ctl)))
              break;
            tc_fence_after();
            mma_ss_tiles<HD>(tmem + kTmemS, sK, sQ + sn * L::kTileBytes);   // S^T(i+1)
            umma_commit_w(&ctl->s_full);
          }
          for (int w = 0; ok && w < 2; ++w) {           // dK += dS^T Q_i
            if (!(ok = spin_bar_w(&ctl->ds_full[w], ph, ctl))) break;
            tc_fence_after();
            mma_ts_half<HD>(tmem + kTmemAcc1, tmem + kTmemDP + 32u, sQ + st * L::kTileBytes, w,
                            i == 0);
          }
          if (!ok) break;
          umma_commit_w(&ctl->st_empty[st]);
          if (more) {
            if (!(ok = spin_bar_w(&ctl->st_full[sn], phn, ctl))) break;
            tc_fence_after();
            mma_ss_tiles<HD>(tmem + kTmemDP, sV, sDO + sn * L::kTileBytes);  // dP^T(i+1)
            umma_commit_w(&ctl->dp_full);
          } else {
            umma_commit_w(&ctl->acc_done);
          }
        }
        if (!ok) {
          umma_commit_w(&ctl->drain);
          drain_wait(&ctl->drain, 0);
        }
      }
    }
  } else {
    setmaxnreg_inc<kRegsWork>();
    const int wg = warp >> 2;                       // query columns [64 wg, 64 wg + 64)
    const int r = threadIdx.x & 127;                // key row = TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t s_addr = tmem + lane_base + kTmemS + (uint32_t)wg * 64u;
    const uint32_t dp_addr = tmem + lane_base + kTmemDP + (uint32_t)wg * 64u;
    const float sl2 = p.scale_log2;
    const MobaLay lay{p.s.n_chunks, p.s.chunk_tokens, p.s.n_bidir, p.s.L};
    int a[2], b[2];
    moba_col_intervals(lay, min(k0 + r, p.s.L - 1), a, b);
    bool ok = true;

    for (int i = 0; i < n_tiles; ++i) {
      const uint32_t e = ctl->tiles[i];
      const int qt = (int)(e & 0xFFFu);
      const int cls = (int)((e >> 12) & 3u);
      const int st = i % kStages;
      ok = wait_bar(&ctl->st_full[st], (uint32_t)(i / kStages) & 1u, ctl) &&
           wait_bar(&ctl->s_full, (uint32_t)i & 1u, ctl);
      if (!__all_sync(0xFFFFFFFFu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t s[64];
      tmem_ld_32x32b_x32(s_addr, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
      tmem_ld_32x32b_x32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&ctl->s_free);                    // S^T columns may take S^T(i+1)
      // -lse * log2 e (l4) and -D (d4) of columns 4m .. 4m + 3 of this warpgroup
      const float4* l4 = reinterpret_cast<const float4*>(smem + L::kW + st * kWsBytes) + wg * 16;
      const float4* d4 = l4 + kTile / 4;
      uint32_t keep[2] = {0xFFFFFFFFu, 0xFFFFFFFFu};
      if (cls != kTileFull) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int base = qt * kTile + wg * 64 + 32 * c;
          keep[c] = bit_range(a[0] - base, b[0] - base) | bit_range(a[1] - base, b[1] - base);
        }
      }
      float pr[64];
      const float2 sl2x2 = make_float2(sl2, sl2);
      // full tiles (most of them) skip the per-element mask
      auto exps = [&](auto masked_c) {
        constexpr bool kMasked = decltype(masked_c)::value;
#pragma unroll
        for (int n = 0; n < 64; n += 2) {
          const float4 lv = l4[n >> 2];
          const float2 x = ffma2(make_float2(__uint_as_float(s[n]), __uint_as_float(s[n + 1])),
                                 sl2x2, (n & 2) ? make_float2(lv.z, lv.w)
                                                : make_float2(lv.x, lv.y));
          float p0 = ex2_sfu(x.x), p1 = ex2_sfu(x.y);
          if (kMasked) {
            if (!((keep[n >> 5] >> (n & 31)) & 1u)) p0 = 0.f;
            if (!((keep[n >> 5] >> ((n + 1) & 31)) & 1u)) p1 = 0.f;
          }
          pr[n] = p0;
          pr[n + 1] = p1;
        }
      };
      if (cls == kTileFull) exps(std::false_type{});
      else exps(std::true_type{});

      ok = wait_bar(&ctl->dp_full, (uint32_t)i & 1u, ctl);
      if (!__all_sync(0xFFFFFFFFu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      tmem_ld_32x32b_x32(dp_addr, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
      tmem_ld_32x32b_x32(dp_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
      tmem_ld_wait();
      // This warpgroup's dP^T half is in registers now: P^T (bf16 pairs) takes
      // its first 32 columns, dS^T its last 32.
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t packed[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) packed[q] = pack_bf16(pr[32 * c + 2 * q], pr[32 * c + 2 * q + 1]);
        tmem_st_32x32b_x16(dp_addr + c * 16, packed);
      }
      tmem_st_wait();
      tc_fence_before();
      // test hook: warpgroup 1 withholds its first P-ready arrival
      if (!(p.inject == 1 && wg == 1 && i == 0)) mbar_arrive(&ctl->p_full[wg]);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t packed[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const int n = 32 * c + 2 * q;
          const float4 nd = d4[n >> 2];                 // -D of the columns
          const float2 t = fadd2(make_float2(__uint_as_float(s[n]), __uint_as_float(s[n + 1])),
                                 (q & 1) ? make_float2(nd.z, nd.w) : make_float2(nd.x, nd.y));
          const float2 d = fmul2(make_float2(pr[n], pr[n + 1]), t);
          packed[q] = pack_bf16(d.x, d.y);
        }
        tmem_st_32x32b_x16(dp_addr + 32 + c * 16, packed);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&ctl->ds_full[wg]);
    }

    // ---------------------------------------------------------- epilogue --
    if (ok && n_tiles > 0) ok = wait_bar(&ctl->acc_done, 0, ctl);
    ok = __all_sync(0xFFFFFFFFu, ok);
    tc_fence_after();
    const int row = k0 + r;
    const bool row_ok = ok && row < p.s.L;
    const uint32_t acc = tmem + lane_base + (wg == 0 ? kTmemAcc0 : kTmemAcc1);
    const float mul = wg == 0 ? 1.f : p.scale;
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(wg == 0 ? p.dv : p.dk) +
                         ((size_t)row * p.H + h) * HD;
#pragma unroll 1
    for (int c = 0; c < HD / 32; ++c) {
      uint32_t v[32];
      if (n_tiles > 0 && ok) {
        tmem_ld_32x32b_x32(acc + c * 32, v);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int n = 0; n < 32; ++n) v[n] = 0u;
      }
      if (row_ok) {
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          uint32_t w[4];
#pragma unroll
          for (int q = 0; q < 4; ++q)
            w[q] = pack_bf16(__uint_as_float(v[g * 8 + 2 * q]) * mul,
                             __uint_as_float(v[g * 8 + 2 * q + 1]) * mul);
          *reinterpret_cast<uint4*>(out + c * 32 + g * 8) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
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

// ----------------------------------------------------------------------- dQ --
// Prologue of the dQ kernel: barriers, TMEM, the count of streamed key tiles.
__device__ __forceinline__ void dq_setup(const MobaBwdParams& p, DqCtl* ctl, int qt, int warp,
                                         int lane) {
  if (threadIdx.x == 0) {
    mbar_init(&ctl->fixed_full, 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&ctl->k_full[s], 1);
      mbar_init(&ctl->k_empty[s], 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&ctl->v_full[s], 1);
      mbar_init(&ctl->v_empty[s], 1);
    }
    mbar_init(&ctl->s_full, 1);
    mbar_init(&ctl->dp_full, 1);
    mbar_init(&ctl->s_free, 256);
    for (int w = 0; w < 2; ++w) mbar_init(&ctl->ds_full[w], 128);
    mbar_init(&ctl->acc_done, 1);
    mbar_init(&ctl->drain, 1);
    ctl->abort = 0;
    ctl->wait_ns =
        p.wait_ns > 0 ? (unsigned long long)p.wait_ns : (unsigned long long)kWaitTimeoutNs;
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(&ctl->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kWarpTma) {
    const int n = build_list<false>(p, qt, nullptr, lane);
    if (lane == 0) ctl->n_tiles = n;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
}

// TMA producer of the dQ kernel (warp 8; lane 0 issues the copies): Q_i and dO_i,
// then, for each key tile query tile i may read in order, its ring entry, K_j into
// slot j % 3 and V_j into slot j % 2.
template <int HD>
__device__ void dq_producer(const MobaBwdParams& p, DqCtl* ctl, uint8_t* smem, int h, int qt,
                            int lane) {
  using L = DqSmem<HD>;
  const int n_tiles = ctl->n_tiles;
  if (lane == 0) {
    prefetch_tmap(&p.tm_q);
    prefetch_tmap(&p.tm_k);
    prefetch_tmap(&p.tm_v);
    prefetch_tmap(&p.tm_do);
    mbar_arrive_expect_tx(&ctl->fixed_full, 2 * L::kTileBytes);
    load_tile<HD>(&p.tm_q, smem + L::kQ, &ctl->fixed_full, h, qt * kTile);
    load_tile<HD>(&p.tm_do, smem + L::kDO, &ctl->fixed_full, h, qt * kTile);
  }
  TileFeeder<false> feed(p, qt, lane);
  int nk = 0, nv = 0;  // copies issued
  bool ok = true;
  for (int j = 0; j < n_tiles; ++j) {
    int u, c;
    if (!feed.next(u, c)) {  // unreachable: n_tiles counts the same classification
      if (lane == 0) {
        atomicExch(&g_bwd_status, (int)KVCR_ESTATE);
        *reinterpret_cast<volatile int*>(&ctl->abort) = 1;
      }
      ok = false;
      break;
    }
    const int ks = j % kKStages;
    ok = __all_sync(0xFFFFFFFFu,
                    wait_bar(&ctl->k_empty[ks], ((uint32_t)(j / kKStages) & 1u) ^ 1u, ctl));
    if (!ok) break;
    if (lane == 0) {
      ctl->tiles[j % kRing] = (uint16_t)(u | (c << 12));
      mbar_arrive_expect_tx(&ctl->k_full[ks], L::kTileBytes);
      load_tile<HD>(&p.tm_k, smem + L::kK + ks * L::kTileBytes, &ctl->k_full[ks], h, u * kTile);
    }
    nk = j + 1;
    const int vs = j % kVStages;
    ok = __all_sync(0xFFFFFFFFu,
                    wait_bar(&ctl->v_empty[vs], ((uint32_t)(j / kVStages) & 1u) ^ 1u, ctl));
    if (!ok) break;
    if (lane == 0) {
      mbar_arrive_expect_tx(&ctl->v_full[vs], L::kTileBytes);
      load_tile<HD>(&p.tm_v, smem + L::kV + vs * L::kTileBytes, &ctl->v_full[vs], h, u * kTile);
    }
    nv = j + 1;
  }
  if (!ok && lane == 0) {
    // let every issued copy land before the CTA can exit
    drain_wait(&ctl->fixed_full, 0);
    for (int j = nk - kKStages < 0 ? 0 : nk - kKStages; j < nk; ++j)
      drain_wait(&ctl->k_full[j % kKStages], (uint32_t)(j / kKStages) & 1u);
    for (int j = nv - kVStages < 0 ? 0 : nv - kVStages; j < nv; ++j)
      drain_wait(&ctl->v_full[j % kVStages], (uint32_t)(j / kVStages) & 1u);
  }
}

template <int HD>
__global__ void __launch_bounds__(kThreads, 1) moba_dq_kernel(const __grid_constant__ MobaBwdParams p) {
  using L = DqSmem<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  if ((int)(smem - smem_raw) + L::kUsed > L::kBytes) {  // uniform: before any barrier
    if (threadIdx.x == 0) atomicExch(&g_bwd_status, (int)KVCR_EUNSUPPORTED);
    return;
  }
  DqCtl* ctl = reinterpret_cast<DqCtl*>(smem + L::kCtl);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int h = blockIdx.x / p.s.n_units;             // head-major: co-resident CTAs
  const int qt = p.s.order[blockIdx.x - h * p.s.n_units];  // share one head in L2
  const int q0 = qt * kTile;

  dq_setup(p, ctl, qt, warp, lane);
  const uint32_t tmem = ctl->tmem_base;
  const int n_tiles = ctl->n_tiles;

  if (warp >= 8) {
    setmaxnreg_dec<kRegsProducer>();
    if (warp == kWarpTma) {
      if (n_tiles > 0) dq_producer<HD>(p, ctl, smem, h, qt, lane);
    } else if (warp == kWarpMma) {
      if (n_tiles > 0) {          // the whole warp: operands stay warp-uniform
        const uint32_t sQ = smem_u32(smem + L::kQ), sDO = smem_u32(smem + L::kDO);
        const uint32_t sK = smem_u32(smem + L::kK), sV = smem_u32(smem + L::kV);
        bool ok = spin_bar_w(&ctl->fixed_full, 0, ctl) && spin_bar_w(&ctl->k_full[0], 0, ctl);
        if (ok) {
          tc_fence_after();
          mma_ss_tiles<HD>(tmem + kTmemS, sQ, sK);      // S(0)
          umma_commit_w(&ctl->s_full);
          ok = spin_bar_w(&ctl->v_full[0], 0, ctl);
        }
        if (ok) {
          tc_fence_after();
          mma_ss_tiles<HD>(tmem + kTmemDP, sDO, sV);    // dP(0)
          umma_commit_w(&ctl->dp_full);
          umma_commit_w(&ctl->v_empty[0]);              // last read of V_0
        }
        for (int j = 0; ok && j < n_tiles; ++j) {
          const bool more = j + 1 < n_tiles;
          const uint32_t ph = (uint32_t)j & 1u;
          const int ks = j % kKStages, kn = (j + 1) % kKStages;
          const int vn = (j + 1) % kVStages;
          if (!(ok = spin_bar_w(&ctl->s_free, ph, ctl))) break;
          if (more) {
            if (!(ok = spin_bar_w(&ctl->k_full[kn], (uint32_t)((j + 1) / kKStages) & 1u, ctl)))
              break;
            tc_fence_after();
            mma_ss_tiles<HD>(tmem + kTmemS, sQ, sK + kn * L::kTileBytes);   // S(j+1)
            umma_commit_w(&ctl->s_full);
          }
          for (int w = 0; ok && w < 2; ++w) {           // dQ += dS K_j
            if (!(ok = spin_bar_w(&ctl->ds_full[w], ph, ctl))) break;
            tc_fence_after();
            mma_ts_half<HD>(tmem + kTmemAcc0, tmem + kTmemDP, sK + ks * L::kTileBytes, w, j == 0);
          }
          if (!ok) break;
          umma_commit_w(&ctl->k_empty[ks]);             // last read of K_j
          if (more) {
            if (!(ok = spin_bar_w(&ctl->v_full[vn], (uint32_t)((j + 1) / kVStages) & 1u, ctl)))
              break;
            tc_fence_after();
            mma_ss_tiles<HD>(tmem + kTmemDP, sDO, sV + vn * L::kTileBytes);  // dP(j+1)
            umma_commit_w(&ctl->dp_full);
            umma_commit_w(&ctl->v_empty[vn]);           // last read of V_{j+1}
          } else {
            umma_commit_w(&ctl->acc_done);
          }
        }
        if (!ok) {
          umma_commit_w(&ctl->drain);
          drain_wait(&ctl->drain, 0);
        }
      }
    }
  } else {
    setmaxnreg_inc<kRegsWork>();
    const int wg = warp >> 2;                       // key columns [64 wg, 64 wg + 64)
    const int r = threadIdx.x & 127;                // query row = TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t s_addr = tmem + lane_base + kTmemS + (uint32_t)wg * 64u;
    const uint32_t dp_addr = tmem + lane_base + kTmemDP + (uint32_t)wg * 64u;
    const float sl2 = p.scale_log2;
    const MobaLay lay{p.s.n_chunks, p.s.chunk_tokens, p.s.n_bidir, p.s.L};
    const float* wt = p.ws + ((size_t)h * p.s.n_units + qt) * 2 * kTile;
    const float2 wrow = make_float2(wt[r], wt[kTile + r]);   // (-lse * log2 e, -D) of row q0 + r
    const float2 neg_d = make_float2(wrow.y, wrow.y);
    const float2 sl2x2 = make_float2(sl2, sl2);
    const float2 neg_lse = make_float2(wrow.x, wrow.x);
    int a[2] = {0, 0}, b[2] = {0, 0};
    {
      const int row = min(q0 + r, p.s.L - 1);
      moba_row_intervals(lay, row, row + 1, a, b, 2);
    }
    bool ok = true;

    for (int j = 0; j < n_tiles; ++j) {
      // K_j's copy (and with it this ring entry) has landed, and S(j) is in TMEM
      ok = wait_bar(&ctl->k_full[j % kKStages], (uint32_t)(j / kKStages) & 1u, ctl) &&
           wait_bar(&ctl->s_full, (uint32_t)j & 1u, ctl);
      if (!__all_sync(0xFFFFFFFFu, ok)) {
        ok = false;
        break;
      }
      const uint32_t e = ctl->tiles[j % kRing];
      const int kt = (int)(e & 0xFFFu);
      const int cls = (int)((e >> 12) & 3u);
      tc_fence_after();
      uint32_t s[64];
      tmem_ld_32x32b_x32(s_addr, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
      tmem_ld_32x32b_x32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&ctl->s_free);
      const int col0 = kt * kTile + wg * 64;
      uint32_t keep[2];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int base = col0 + 32 * c;
        keep[c] = bit_range(0, p.s.L - base);
        if (cls != kTileFull)
          keep[c] &= bit_range(a[0] - base, b[0] - base) | bit_range(a[1] - base, b[1] - base);
      }
      float pr[64];
      // full tiles inside the sequence (most of them) skip the per-element mask
      auto exps = [&](auto masked_c) {
        constexpr bool kMasked = decltype(masked_c)::value;
#pragma unroll
        for (int n = 0; n < 64; n += 2) {
          const float2 x = ffma2(make_float2(__uint_as_float(s[n]), __uint_as_float(s[n + 1])),
                                 sl2x2, neg_lse);
          float p0 = ex2_sfu(x.x), p1 = ex2_sfu(x.y);
          if (kMasked) {
            if (!((keep[n >> 5] >> (n & 31)) & 1u)) p0 = 0.f;
            if (!((keep[n >> 5] >> ((n + 1) & 31)) & 1u)) p1 = 0.f;
          }
          pr[n] = p0;
          pr[n + 1] = p1;
        }
      };
      if (cls == kTileFull && (kt + 1) * kTile <= p.s.L) exps(std::false_type{});
      else exps(std::true_type{});

      ok = wait_bar(&ctl->dp_full, (uint32_t)j & 1u, ctl);
      if (!__all_sync(0xFFFFFFFFu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      tmem_ld_32x32b_x32(dp_addr, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
      tmem_ld_32x32b_x32(dp_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t packed[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const int n = 32 * c + 2 * q;
          const float2 t = fadd2(make_float2(__uint_as_float(s[n]), __uint_as_float(s[n + 1])),
                                 neg_d);
          const float2 d = fmul2(make_float2(pr[n], pr[n + 1]), t);
          packed[q] = pack_bf16(d.x, d.y);
        }
        tmem_st_32x32b_x16(dp_addr + c * 16, packed);
      }
      tmem_st_wait();
      tc_fence_before();
      // test hook: warpgroup 1 withholds its first dS-ready arrival
      if (!(p.inject == 1 && wg == 1 && j == 0)) mbar_arrive(&ctl->ds_full[wg]);
    }

    // ---------------------------------------------------------- epilogue --
    if (ok && n_tiles > 0) ok = wait_bar(&ctl->acc_done, 0, ctl);
    ok = __all_sync(0xFFFFFFFFu, ok);
    tc_fence_after();
    const int row = q0 + r;
    const bool row_ok = ok && row < p.s.L;
    // warpgroup wg writes dQ columns [wg * HD / 2, (wg + 1) * HD / 2)
    const uint32_t acc = tmem + lane_base + kTmemAcc0 + (uint32_t)(wg * (HD / 2));
    __nv_bfloat16* out =
        static_cast<__nv_bfloat16*>(p.dq) + ((size_t)row * p.H + h) * HD + wg * (HD / 2);
#pragma unroll 1
    for (int c = 0; c < HD / 64; ++c) {
      uint32_t v[32];
      if (n_tiles > 0 && ok) {
        tmem_ld_32x32b_x32(acc + c * 32, v);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int n = 0; n < 32; ++n) v[n] = 0u;
      }
      if (row_ok) {
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          uint32_t w[4];
#pragma unroll
          for (int q = 0; q < 4; ++q)
            w[q] = pack_bf16(__uint_as_float(v[g * 8 + 2 * q]) * p.scale,
                             __uint_as_float(v[g * 8 + 2 * q + 1]) * p.scale);
          *reinterpret_cast<uint4*>(out + c * 32 + g * 8) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
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

// --------------------------------------------------------------------- prep --
// HD / 8 threads per (head, row): each reads 8 bf16 of O and of dO (16 bytes).
template <int HD>
__global__ void __launch_bounds__(256) moba_bwd_prep_kernel(const MobaBwdPrepParams p) {
  constexpr int kTpr = HD / 8;
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long item = gid / kTpr;                // h * Lpad + row
  const int part = (int)(gid % kTpr);
  const long long n_items = (long long)p.H * p.Lpad;
  const int h = (int)(item / p.Lpad);
  const int row = (int)(item - (long long)h * p.Lpad);
  const bool live = item < n_items && row < p.L;
  float acc = 0.f;
  if (live) {
    const size_t off = ((size_t)row * p.H + h) * HD + part * 8;
    const uint4 a = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.o) + off);
    const uint4 b = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.d_o) + off);
    const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 x = __bfloat1622float2(a2[q]);
      const float2 y = __bfloat1622float2(b2[q]);
      acc = fmaf(x.x, y.x, acc);
      acc = fmaf(x.y, y.y, acc);
    }
  }
#pragma unroll
  for (int w = kTpr / 2; w >= 1; w >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, w);
  if (part == 0 && item < n_items) {
    float lse2 = INFINITY;                          // rows past L (or with no key): P = 0
    if (row < p.L) {
      const float v = p.lse[(size_t)h * p.L + row];
      if (v != -INFINITY) lse2 = v * 1.4426950408889634f;
    }
    float* wt = p.ws + ((size_t)h * (p.Lpad / kTile) + row / kTile) * 2 * kTile;
    wt[row % kTile] = -lse2;                        // stored negated, as -D below
    wt[kTile + row % kTile] = live ? -acc : 0.f;
  }
}

template <int HD>
cudaError_t launch_dkdv(const MobaBwdParams& p, cudaStream_t s) {
  auto kern = moba_dkdv_kernel<HD>;
  // the shared-memory limit is a per-device attribute of the function
  static bool attr_set[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, BwdSmem<HD>::kBytes);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  kern<<<(unsigned)(p.s.n_units * p.H), kThreads, BwdSmem<HD>::kBytes, s>>>(p);
  return cudaGetLastError();
}

template <int HD>
cudaError_t launch_dq(const MobaBwdParams& p, cudaStream_t s) {
  auto kern = moba_dq_kernel<HD>;
  // the shared-memory limit is a per-device attribute of the function
  static bool attr_set[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, DqSmem<HD>::kBytes);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  kern<<<(unsigned)(p.s.n_units * p.H), kThreads, DqSmem<HD>::kBytes, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_moba_bwd_prep(const MobaBwdPrepParams& p, int head_dim, cudaStream_t s) {
  const long long threads = (long long)p.H * p.Lpad * (head_dim / 8);
  const unsigned blocks = (unsigned)((threads + 255) / 256);
  if (head_dim == 128) moba_bwd_prep_kernel<128><<<blocks, 256, 0, s>>>(p);
  else if (head_dim == 64) moba_bwd_prep_kernel<64><<<blocks, 256, 0, s>>>(p);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_moba_bwd_dkdv_sm100(const MobaBwdParams& p, int head_dim, cudaStream_t s) {
  if (head_dim == 128) return launch_dkdv<128>(p, s);
  if (head_dim == 64) return launch_dkdv<64>(p, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_moba_bwd_dq_sm100(const MobaBwdParams& p, int head_dim, cudaStream_t s) {
  if (head_dim == 128) return launch_dq<128>(p, s);
  if (head_dim == 64) return launch_dq<64>(p, s);
  return cudaErrorInvalidValue;
}

cudaError_t read_and_clear_status_bwd(int* st, cudaStream_t s) {
  int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(st, g_bwd_status, sizeof(int), 0,
                                            cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return e;
  e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return e;
  if (*st != 0) e = cudaMemcpyToSymbol(g_bwd_status, &zero, sizeof(int));
  return e;
}

}  // namespace kvcr
