// Host side of the C ABI declared in include/kvcr.h: argument validation, the
// per-layer slot table (anchors + sliding window), device-storage layout,
// rotary angle tables, TMA tensor-map encoding, kernel launches and tracing.
//
// Slot rules ("LingBot-World-Infinity: The Open-Source World Model That
// Refuses to Forget", "The trick: treat video like a causal stream" and "How
// the cache keeps the world alive"; "Westlake AGI Lab's 'World in World'
// Steers Frozen Video Models", second paragraph):
//   - the first `sinks` finalized frames are the anchors, slot i for the i-th;
//     anchors are never evicted;
//   - a later frame that finds `window` non-anchor frames cached evicts the
//     oldest of them and takes its slot, else it takes the lowest free window
//     slot;
//   - kv_cache_evict(keep) drops the oldest non-anchor frames down to `keep`
//     (the dynamic KV-cache scheduler of "Infinite Worlds with Versatile
//     Interactions", deployment paragraph).
// Bookkeeping never reads device memory, so every call stays asynchronous.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <deque>
#include <memory>
#include <mutex>
#include <string>
#include <vector>

#include "attn_bwd.h"
#include "kvcr_internal.h"
#include "moba_layout.h"
#include "rope_batch.h"
#include "static_scratch.h"

using namespace kvcr;

namespace {

thread_local std::string g_err;

int fail(int code, const std::string& msg) {
  g_err = msg;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(KVCR_ECUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

// ------------------------------------------------------------ tensor maps --
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Tiled map over a tensor [..][tokens][H][D] of bf16 (box 64 elements wide) or
// of e4m3 codes as bytes (box 128 wide), innermost first: D, H, tokens[,
// slots]; box = 128 bytes x 1 x box_rows (x 1), 128-byte swizzle, zero fill.
int encode_map(CUtensorMap* m, bool codes, const void* base, int rank, const uint64_t* dims,
               int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(KVCR_ECUDA, "cuTensorMapEncodeTiled not available from the driver");
  cuuint64_t gdim[4];
  cuuint64_t gstride[3];
  cuuint32_t box[4] = {codes ? 128u : 64u, 1, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  uint64_t stride = codes ? 1 : 2;
  for (int i = 0; i < rank; ++i) {
    gdim[i] = dims[i];
    if (i > 0) gstride[i - 1] = stride;
    stride *= dims[i];
  }
  CUresult r = fn(m, codes ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                  (cuuint32_t)rank, const_cast<void*>(base), gdim, gstride, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(KVCR_ECUDA, "cuTensorMapEncodeTiled failed (" +
                                                     std::to_string((int)r) + ")");
  return KVCR_OK;
}

int encode_bf16_map(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
                    int box_rows) {
  return encode_map(m, false, base, rank, dims, box_rows);
}

// --------------------------------------------------------- failure hook --
std::atomic<int> g_inject_kind{0};
std::atomic<long long> g_inject_wait_ns{0};

// ----------------------------------------------------------------- tracing --
std::atomic<long long> g_launches{0};
std::mutex g_trace_mu;
bool g_trace_on = false;
struct TraceRec {
  int kid;
  cudaEvent_t a, b;
};
std::vector<TraceRec> g_recs;
std::vector<cudaEvent_t> g_pool;

cudaEvent_t pool_event() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

// Brackets one launch with events on its stream when tracing is on.
class LaunchScope {
 public:
  LaunchScope(int kid, cudaStream_t s) : kid_(kid), s_(s) {
    g_launches.fetch_add(1);
    std::lock_guard<std::mutex> g(g_trace_mu);
    if (g_trace_on) {
      a_ = pool_event();
      b_ = pool_event();
      if (a_ && b_) cudaEventRecord(a_, s_);
    }
  }
  ~LaunchScope() {
    if (!a_ || !b_) return;
    cudaEventRecord(b_, s_);
    std::lock_guard<std::mutex> g(g_trace_mu);
    g_recs.push_back({kid_, a_, b_});
  }

 private:
  int kid_;
  cudaStream_t s_;
  cudaEvent_t a_ = nullptr, b_ = nullptr;
};

// -------------------------------------------------------------- device info --
int device_sm_count(int* n_sm, int* cc_major) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  e = cudaDeviceGetAttribute(n_sm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
  e = cudaDeviceGetAttribute(cc_major, cudaDevAttrComputeCapabilityMajor, dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
  return KVCR_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct StorageLayout {
  size_t k_off, v_off, q_off, ks_off, h_off, w_off;
  // e4m3 copies (KVCR_CACHE_FP8_K): cached K codes and their block scales, then the
  // codes and scales of one chunk's queries and current keys
  size_t k8_off, k8s_off, q8_off, q8s_off, c8_off, c8s_off;
  size_t total;
};

int blocks_of(long long n) { return (int)((n + 127) / 128); }

bool make_layout(int S, int W, int A, int T, int H, int D, int F, bool rope, size_t esize,
                 StorageLayout* L, bool fp8 = false, bool spare = false) {
  const int n_phys = S + W + A + (spare ? F : 0);
  if (S < 0 || W < 0 || A < 0 || S + W < 1 || n_phys > kMaxSlots || T < 1 || H < 1 || D < 1 ||
      F < 1 || F > kMaxFrames)
    return false;
  const size_t frame = (size_t)T * H * D * esize;
  const size_t slots = (size_t)n_phys;  // anchors, window, auxiliary, spare
  size_t off = 0;
  L->k_off = off;
  off = align_up(off + slots * frame, 256);
  L->v_off = off;
  off = align_up(off + slots * frame, 256);
  L->q_off = L->ks_off = L->h_off = L->w_off = off;
  if (rope) {
    L->q_off = off;
    off = align_up(off + (size_t)F * frame, 256);
    L->ks_off = off;
    off = align_up(off + (size_t)F * frame, 256);
    // angle tables: at most T rows x D/2 pairs each for h and w
    L->h_off = off;
    off = align_up(off + (size_t)T * (D / 2) * sizeof(float2), 256);
    L->w_off = off;
    off = align_up(off + (size_t)T * (D / 2) * sizeof(float2), 256);
  }
  L->k8_off = L->k8s_off = L->q8_off = L->q8s_off = L->c8_off = L->c8s_off = off;
  if (fp8) {
    const size_t codes = (size_t)T * H * D;                      // bytes per frame
    const size_t chunk_codes = (size_t)F * T * H * D;
    L->k8_off = off;
    off = align_up(off + slots * codes, 256);
    L->k8s_off = off;
    off = align_up(off + slots * blocks_of(T) * H * sizeof(float), 256);
    L->q8_off = off;
    off = align_up(off + chunk_codes, 256);
    L->q8s_off = off;
    off = align_up(off + (size_t)blocks_of((long long)F * T) * H * sizeof(float), 256);
    L->c8_off = off;
    off = align_up(off + chunk_codes, 256);
    L->c8s_off = off;
    off = align_up(off + (size_t)blocks_of((long long)F * T) * H * sizeof(float), 256);
  }
  L->total = off;
  return true;
}

}  // namespace

// ====================================================================== cache
struct kvcr_cache {
  int S, W, T, H, D, F;
  int A;      // auxiliary slots (physical slots S + W .. S + W + A - 1)
  int n_aux;  // auxiliary frames visible to the current chunk's attention
  kvcr_dtype dtype;
  size_t esize;
  bool rope;
  kvcr_rope rp;
  bool has_storage;
  uint8_t* storage;
  StorageLayout lay;
  int n_sm, cc_major;
  CUtensorMap tm_kc, tm_vc;
  bool fp8;             // e4m3 K copies kept (KVCR_CACHE_FP8_K)
  CUtensorMap tm_kc8;   // 4D map over the e4m3 K copies
  // Physical frame slot of each anchor / window slot (the identity unless
  // chunk_attention_fwd_finalize() relabelled them) and the spare physical slots
  // (KVCR_CACHE_FUSED_FINALIZE: chunk_frames of them, after the auxiliary slots).
  bool fused;
  std::vector<int> phys;
  std::vector<int> spare;
  // slot table
  std::vector<int> slot_frame;
  int n_sinks_filled;
  std::deque<int> recent;  // non-anchor frames, oldest first
  int last_frame;
  std::vector<int> last_slots, last_evicted;
};

namespace kvcr {
InjectState inject_state() { return InjectState{g_inject_kind.load(), g_inject_wait_ns.load()}; }
}  // namespace kvcr

namespace {

struct SlotState {
  std::vector<int> slot_frame;
  int n_sinks_filled;
  std::deque<int> recent;
  int last_frame;
  std::vector<int> phys, spare;
};

SlotState snapshot(const kvcr_cache* c) {
  return SlotState{c->slot_frame, c->n_sinks_filled, c->recent, c->last_frame, c->phys, c->spare};
}

void restore(kvcr_cache* c, const SlotState& s) {
  c->slot_frame = s.slot_frame;
  c->n_sinks_filled = s.n_sinks_filled;
  c->recent = s.recent;
  c->last_frame = s.last_frame;
  c->phys = s.phys;
  c->spare = s.spare;
}

// Physical frame slot of a slot index (anchor / window slots through the
// relabelling table, auxiliary slots as they are).
int phys_of(const kvcr_cache* c, int slot) {
  return slot < c->S + c->W ? c->phys[slot] : slot;
}

// Visible frames of the next attention call as physical slots: cached frames in
// slot order, then the auxiliary frames.
int visible_slots(const kvcr_cache* c, int* slots) {
  int n = 0;
  for (int i = 0; i < c->S + c->W; ++i)
    if (c->slot_frame[i] >= 0) slots[n++] = c->phys[i];
  for (int i = 0; i < c->n_aux; ++i) slots[n++] = c->S + c->W + i;
  return n;
}

// Apply the slot rules to one frame; returns its slot (-1 = not retained) and
// appends evicted frames.
int place_frame(kvcr_cache* c, int f, std::vector<int>& evicted) {
  int s;
  c->last_frame = f;
  if (c->n_sinks_filled < c->S) {
    s = c->n_sinks_filled++;
  } else if (c->W == 0) {
    evicted.push_back(f);
    return -1;
  } else if ((int)c->recent.size() == c->W) {
    const int old = c->recent.front();
    c->recent.pop_front();
    s = -1;
    for (int i = c->S; i < c->S + c->W; ++i)
      if (c->slot_frame[i] == old) s = i;
    c->slot_frame[s] = -1;
    evicted.push_back(old);
    c->recent.push_back(f);
  } else {
    s = -1;
    for (int i = c->S; i < c->S + c->W && s < 0; ++i)
      if (c->slot_frame[i] == -1) s = i;
    c->recent.push_back(f);
  }
  c->slot_frame[s] = f;
  return s;
}

void fill_ttab(const kvcr_cache* c, RopeCopyParams& p, const int32_t* frames, int n) {
  for (int f = 0; f < n; ++f)
    for (int j = 0; j < c->rp.pairs_t; ++j) {
      const double ang =
          (double)frames[f] * std::pow(c->rp.base, -(2.0 * j) / (2.0 * c->rp.pairs_t));
      p.ttab[f][j] = make_float2((float)std::cos(ang), (float)std::sin(ang));
    }
}

void fill_common(const kvcr_cache* c, RopeCopyParams& p) {
  p.T = c->T;
  p.H = c->H;
  p.D = c->D;
  p.grid_w = c->rope ? c->rp.grid_w : 1;
  p.pairs_t = c->rope ? c->rp.pairs_t : 0;
  p.pairs_h = c->rope ? c->rp.pairs_h : 0;
  p.pairs_w = c->rope ? c->rp.pairs_w : 0;
  p.htab = c->rope ? reinterpret_cast<const float2*>(c->storage + c->lay.h_off) : nullptr;
  p.wtab = c->rope ? reinterpret_cast<const float2*>(c->storage + c->lay.w_off) : nullptr;
}

// Segment i of a quantization launch: the bf16 K of physical slot `slot` of cache c
// to its e4m3 copy and block scales.
void quant_segment_of_slot(const kvcr_cache* c, int slot, QuantParams& p, int i, int tile0) {
  const size_t codes = (size_t)c->T * c->H * c->D;
  slot = phys_of(c, slot);
  p.src[i] = c->storage + c->lay.k_off + (size_t)slot * codes * c->esize;
  p.dst[i] = c->storage + c->lay.k8_off + (size_t)slot * codes;
  p.scale[i] = reinterpret_cast<float*>(c->storage + c->lay.k8s_off) +
               (size_t)slot * blocks_of(c->T) * c->H;
  p.n_tok[i] = c->T;
  p.tile0[i] = tile0;
}

// e4m3 copies of the K of the listed physical slots of an e4m3 cache (their bf16 K
// written earlier on the same stream).
cudaError_t quant_slots(const kvcr_cache* c, const std::vector<int>& slots, cudaStream_t s) {
  if (!c->fp8 || slots.empty()) return cudaSuccess;
  std::unique_ptr<QuantParams> p(new QuantParams());
  std::memset(p.get(), 0, sizeof(QuantParams));
  for (size_t i = 0; i < slots.size(); ++i)
    quant_segment_of_slot(c, slots[i], *p, (int)i, (int)i * blocks_of(c->T));
  p->n_seg = (int)slots.size();
  p->H = c->H;
  LaunchScope scope(KVCR_K_QUANT_E4M3, s);
  return launch_quant_e4m3(*p, c->D, s);
}

int check_frames(const kvcr_cache* c, const int32_t* frames, int n, const char* what) {
  if (n > 0 && frames == nullptr) return fail(KVCR_EINVAL, std::string(what) + ": frame indices are NULL");
  int prev = c->last_frame;
  for (int i = 0; i < n; ++i) {
    if (frames[i] < 0) return fail(KVCR_EINVAL, std::string(what) + ": negative frame index");
    if (frames[i] <= prev)
      return fail(KVCR_ESTATE, std::string(what) +
                                   ": frame indices must increase and exceed every cached frame");
    prev = frames[i];
  }
  return KVCR_OK;
}

}  // namespace

extern "C" {

const char* kvcr_last_error(void) { return g_err.c_str(); }

size_t kv_cache_storage_bytes_ex(int sinks, int window, int aux_frames, int tokens_per_frame,
                                 int heads, int head_dim, int chunk_frames, int with_rope,
                                 kvcr_dtype dtype, unsigned flags) {
  if (dtype != KVCR_BF16 && dtype != KVCR_F32) return 0;
  if (flags & ~(unsigned)(KVCR_CACHE_FP8_K | KVCR_CACHE_FUSED_FINALIZE)) return 0;
  if ((flags & KVCR_CACHE_FP8_K) && (flags & KVCR_CACHE_FUSED_FINALIZE)) return 0;
  StorageLayout L;
  if (!make_layout(sinks, window, aux_frames, tokens_per_frame, heads, head_dim, chunk_frames,
                   with_rope != 0, dtype == KVCR_BF16 ? 2 : 4, &L,
                   (flags & KVCR_CACHE_FP8_K) != 0, (flags & KVCR_CACHE_FUSED_FINALIZE) != 0))
    return 0;
  return L.total;
}

size_t kv_cache_storage_bytes_aux(int sinks, int window, int aux_frames, int tokens_per_frame,
                                  int heads, int head_dim, int chunk_frames, int with_rope,
                                  kvcr_dtype dtype) {
  return kv_cache_storage_bytes_ex(sinks, window, aux_frames, tokens_per_frame, heads, head_dim,
                                   chunk_frames, with_rope, dtype, 0u);
}

size_t kv_cache_storage_bytes(int sinks, int window, int tokens_per_frame, int heads, int head_dim,
                              int chunk_frames, int with_rope, kvcr_dtype dtype) {
  return kv_cache_storage_bytes_aux(sinks, window, 0, tokens_per_frame, heads, head_dim,
                                    chunk_frames, with_rope, dtype);
}

int kv_cache_init(kvcr_cache** out, int sinks, int window, int tokens_per_frame, int heads,
                  int head_dim, int chunk_frames, const kvcr_rope* rope, kvcr_dtype dtype,
                  void* device_storage, size_t storage_bytes) {
  return kv_cache_init_aux(out, sinks, window, 0, tokens_per_frame, heads, head_dim, chunk_frames,
                           rope, dtype, device_storage, storage_bytes);
}

int kv_cache_init_aux(kvcr_cache** out, int sinks, int window, int aux_frames,
                      int tokens_per_frame, int heads, int head_dim, int chunk_frames,
                      const kvcr_rope* rope, kvcr_dtype dtype, void* device_storage,
                      size_t storage_bytes) {
  return kv_cache_init_ex(out, sinks, window, aux_frames, tokens_per_frame, heads, head_dim,
                          chunk_frames, rope, dtype, 0u, device_storage, storage_bytes);
}

int kv_cache_init_ex(kvcr_cache** out, int sinks, int window, int aux_frames,
                     int tokens_per_frame, int heads, int head_dim, int chunk_frames,
                     const kvcr_rope* rope, kvcr_dtype dtype, unsigned flags,
                     void* device_storage, size_t storage_bytes) {
  if (out == nullptr) return fail(KVCR_EINVAL, "kv_cache_init: out is NULL");
  *out = nullptr;
  if (dtype != KVCR_BF16 && dtype != KVCR_F32) return fail(KVCR_EINVAL, "kv_cache_init: bad dtype");
  if (head_dim != 64 && head_dim != 128)
    return fail(KVCR_EUNSUPPORTED, "kv_cache_init: head_dim must be 64 or 128");
  if (flags & ~(unsigned)(KVCR_CACHE_FP8_K | KVCR_CACHE_FUSED_FINALIZE))
    return fail(KVCR_EINVAL, "kv_cache_init: unknown flags");
  const bool fp8 = (flags & KVCR_CACHE_FP8_K) != 0;
  const bool fused = (flags & KVCR_CACHE_FUSED_FINALIZE) != 0;
  if (fp8 && fused)
    return fail(KVCR_EINVAL, "kv_cache_init: KVCR_CACHE_FP8_K and KVCR_CACHE_FUSED_FINALIZE "
                             "cannot be combined");
  if (fp8 && (dtype != KVCR_BF16 || head_dim != 128))
    return fail(KVCR_EUNSUPPORTED, "kv_cache_init: e4m3 K copies need bf16 and head_dim 128");
  if (fused && dtype != KVCR_BF16)
    return fail(KVCR_EUNSUPPORTED, "kv_cache_init: fused finalize needs bf16");
  if (sinks < 0 || window < 0 || aux_frames < 0 || sinks + window < 1 ||
      sinks + window + aux_frames + (fused ? chunk_frames : 0) > kMaxSlots)
    return fail(KVCR_ESHAPE, "kv_cache_init: need 1 <= sinks + window and sinks + window + "
                             "aux_frames (+ chunk_frames spare slots) <= 32");
  if (tokens_per_frame < 1 || heads < 1 || chunk_frames < 1 || chunk_frames > kMaxFrames)
    return fail(KVCR_ESHAPE, "kv_cache_init: bad tokens_per_frame / heads / chunk_frames (<= 16)");
  if ((long long)chunk_frames * tokens_per_frame > (1LL << 30) ||
      (long long)tokens_per_frame * heads * head_dim > (1LL << 31) / 4)
    return fail(KVCR_ESHAPE, "kv_cache_init: frame too large");
  if (rope) {
    if ((long long)rope->grid_h * rope->grid_w != tokens_per_frame || rope->grid_h < 1 ||
        rope->grid_w < 1)
      return fail(KVCR_ESHAPE, "kv_cache_init: rope grid_h * grid_w != tokens_per_frame");
    if (rope->pairs_t < 0 || rope->pairs_h < 0 || rope->pairs_w < 0 ||
        rope->pairs_t + rope->pairs_h + rope->pairs_w != head_dim / 2 ||
        rope->pairs_t > kMaxPairsT)
      return fail(KVCR_ESHAPE, "kv_cache_init: rope pairs must sum to head_dim/2 (pairs_t <= 32)");
    if (!(rope->base > 0.0)) return fail(KVCR_EINVAL, "kv_cache_init: rope base must be > 0");
  }
  const size_t esize = dtype == KVCR_BF16 ? 2 : 4;
  StorageLayout L;
  if (!make_layout(sinks, window, aux_frames, tokens_per_frame, heads, head_dim, chunk_frames,
                   rope != nullptr, esize, &L, fp8, fused))
    return fail(KVCR_ESHAPE, "kv_cache_init: bad sizes");
  const bool has_storage = device_storage != nullptr;
  if (!has_storage && storage_bytes != 0)
    return fail(KVCR_ESTORAGE, "kv_cache_init: storage is NULL but storage_bytes != 0");
  int n_sm = 0, cc = 0;
  if (has_storage) {
    if (storage_bytes < L.total)
      return fail(KVCR_ESTORAGE, "kv_cache_init: storage smaller than kv_cache_storage_bytes()");
    if ((reinterpret_cast<uintptr_t>(device_storage) & 255u) != 0)
      return fail(KVCR_ESTORAGE, "kv_cache_init: storage must be 256-byte aligned");
    int rc = device_sm_count(&n_sm, &cc);
    if (rc) return rc;
    if (dtype == KVCR_BF16 && cc != 10)
      return fail(KVCR_EUNSUPPORTED, "kv_cache_init: the bf16 path needs an sm_100 GPU");
  }
  kvcr_cache* c = new kvcr_cache();
  c->S = sinks;
  c->W = window;
  c->A = aux_frames;
  c->n_aux = 0;
  c->T = tokens_per_frame;
  c->H = heads;
  c->D = head_dim;
  c->F = chunk_frames;
  c->dtype = dtype;
  c->esize = esize;
  c->rope = rope != nullptr;
  if (rope) c->rp = *rope;
  c->has_storage = has_storage;
  c->storage = static_cast<uint8_t*>(device_storage);
  c->lay = L;
  c->n_sm = n_sm;
  c->cc_major = cc;
  c->fp8 = fp8;
  c->fused = fused;
  c->phys.resize(sinks + window);
  for (int i = 0; i < sinks + window; ++i) c->phys[i] = i;
  if (fused)
    for (int f = 0; f < chunk_frames; ++f) c->spare.push_back(sinks + window + aux_frames + f);
  c->slot_frame.assign(sinks + window, -1);
  c->n_sinks_filled = 0;
  c->last_frame = -1;
  if (has_storage) {
    if (c->rope) {
      // (h, w) angle tables in double precision, stored as fp32 (cos, sin).
      std::vector<float2> ht((size_t)rope->grid_h * std::max(rope->pairs_h, 1));
      std::vector<float2> wt((size_t)rope->grid_w * std::max(rope->pairs_w, 1));
      for (int y = 0; y < rope->grid_h; ++y)
        for (int j = 0; j < rope->pairs_h; ++j) {
          const double a = (double)y * std::pow(rope->base, -(2.0 * j) / (2.0 * rope->pairs_h));
          ht[(size_t)y * rope->pairs_h + j] = make_float2((float)std::cos(a), (float)std::sin(a));
        }
      for (int x = 0; x < rope->grid_w; ++x)
        for (int j = 0; j < rope->pairs_w; ++j) {
          const double a = (double)x * std::pow(rope->base, -(2.0 * j) / (2.0 * rope->pairs_w));
          wt[(size_t)x * rope->pairs_w + j] = make_float2((float)std::cos(a), (float)std::sin(a));
        }
      cudaError_t e = cudaMemcpy(c->storage + L.h_off, ht.data(), ht.size() * sizeof(float2),
                                 cudaMemcpyHostToDevice);
      if (e == cudaSuccess)
        e = cudaMemcpy(c->storage + L.w_off, wt.data(), wt.size() * sizeof(float2),
                       cudaMemcpyHostToDevice);
      if (e != cudaSuccess) {
        delete c;
        return cuda_fail(e, "kv_cache_init: writing angle tables");
      }
    }
    if (dtype == KVCR_BF16) {
      const uint64_t dims[4] = {(uint64_t)head_dim, (uint64_t)heads, (uint64_t)tokens_per_frame,
                                (uint64_t)(sinks + window + aux_frames +
                                           (fused ? chunk_frames : 0))};
      int rc = encode_bf16_map(&c->tm_kc, c->storage + L.k_off, 4, dims, kKeyTile);
      if (!rc) rc = encode_bf16_map(&c->tm_vc, c->storage + L.v_off, 4, dims, kKeyTile);
      if (!rc && fp8) rc = encode_map(&c->tm_kc8, true, c->storage + L.k8_off, 4, dims, kKeyTile);
      if (rc) {
        delete c;
        return rc;
      }
    }
  }
  *out = c;
  return KVCR_OK;
}

void kv_cache_destroy(kvcr_cache* c) { delete c; }

int kv_cache_append_rope(kvcr_cache* c, const void* k, const void* v, const int32_t* frame_idx,
                         int n_frames, void* stream) {
  if (c == nullptr) return fail(KVCR_EINVAL, "kv_cache_append_rope: cache is NULL");
  if (n_frames < 0 || n_frames > kMaxFrames)
    return fail(KVCR_ESHAPE, "kv_cache_append_rope: n_frames must be in [0, 16]");
  if (n_frames == 0) {
    c->last_slots.clear();
    c->last_evicted.clear();
    c->n_aux = 0;
    return KVCR_OK;
  }
  int rc = check_frames(c, frame_idx, n_frames, "kv_cache_append_rope");
  if (rc) return rc;
  if (c->has_storage) {
    if (k == nullptr || v == nullptr) return fail(KVCR_EINVAL, "kv_cache_append_rope: k/v NULL");
    if (!aligned16(k) || !aligned16(v))
      return fail(KVCR_EINVAL, "kv_cache_append_rope: k/v must be 16-byte aligned");
  } else if (k != nullptr || v != nullptr) {
    return fail(KVCR_ESTATE, "kv_cache_append_rope: bookkeeping-only cache takes k = v = NULL");
  }
  const SlotState before = snapshot(c);
  std::vector<int> slots(n_frames), evicted;
  for (int i = 0; i < n_frames; ++i) slots[i] = place_frame(c, frame_idx[i], evicted);
  if (c->has_storage) {
    RopeCopyParams p;
    std::memset(&p, 0, sizeof(p));
    fill_common(c, p);
    p.src_a = k;
    p.src_b = v;
    p.dst_a = c->storage + c->lay.k_off;
    p.dst_b = c->storage + c->lay.v_off;
    p.rotate_a = c->rope ? 1 : 0;
    p.rotate_b = 0;
    const long long frame_elems = (long long)c->T * c->H * c->D;
    int n = 0;
    std::vector<int32_t> written;
    std::vector<int> written_slots;
    for (int i = 0; i < n_frames; ++i) {
      // skip frames not retained, or evicted again by a later frame of this call
      if (slots[i] < 0 || c->slot_frame[slots[i]] != frame_idx[i]) continue;
      p.dst_frame_off[n] = (long long)phys_of(c, slots[i]) * frame_elems;
      p.src_frame[n] = i;
      written.push_back(frame_idx[i]);
      written_slots.push_back(slots[i]);
      ++n;
    }
    p.n_frames = n;
    if (c->rope) fill_ttab(c, p, written.data(), n);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    {
      LaunchScope scope(KVCR_K_APPEND_ROPE, s);
      e = launch_rope_copy(p, c->dtype, s, c->n_sm);
    }
    if (e == cudaSuccess) e = quant_slots(c, written_slots, s);
    if (e != cudaSuccess) {
      restore(c, before);
      return cuda_fail(e, "kv_cache_append_rope: launch");
    }
  }
  c->last_slots = slots;
  c->last_evicted = evicted;
  c->n_aux = 0;  // the chunk is finalized: its auxiliary frames are dropped
  return KVCR_OK;
}

int kv_cache_append_rope_batch(kvcr_cache* const* caches, int n_caches, const void* const* k,
                               const void* const* v, const int32_t* frame_idx, int n_frames,
                               void* stream) {
  const char* fn = "kv_cache_append_rope_batch";
  if (caches == nullptr || n_caches < 1) return fail(KVCR_EINVAL, std::string(fn) + ": no caches");
  if (n_frames < 0 || n_frames > kMaxFrames)
    return fail(KVCR_ESHAPE, std::string(fn) + ": n_frames must be in [0, 16]");
  if ((long long)n_caches * n_frames > kMaxBatchPairs)
    return fail(KVCR_ESHAPE, std::string(fn) + ": n_caches * n_frames must be <= 256");
  const kvcr_cache* c0 = caches[0];
  for (int i = 0; i < n_caches; ++i) {
    const kvcr_cache* c = caches[i];
    if (c == nullptr) return fail(KVCR_EINVAL, std::string(fn) + ": a cache is NULL");
    for (int j = 0; j < i; ++j)
      if (caches[j] == c) return fail(KVCR_EINVAL, std::string(fn) + ": a cache is listed twice");
    if (c->T != c0->T || c->H != c0->H || c->D != c0->D || c->dtype != c0->dtype ||
        c->rope != c0->rope || c->has_storage != c0->has_storage ||
        (c->rope && (c->rp.grid_h != c0->rp.grid_h || c->rp.grid_w != c0->rp.grid_w ||
                     c->rp.pairs_t != c0->rp.pairs_t || c->rp.pairs_h != c0->rp.pairs_h ||
                     c->rp.pairs_w != c0->rp.pairs_w || c->rp.base != c0->rp.base)))
      return fail(KVCR_ESHAPE, std::string(fn) +
                                   ": caches differ in frame shape, dtype, RoPE or storage");
    int rc = check_frames(c, frame_idx, n_frames, fn);
    if (rc) return rc;
    if (c->has_storage && n_frames > 0) {
      if (k == nullptr || v == nullptr || k[i] == nullptr || v[i] == nullptr)
        return fail(KVCR_EINVAL, std::string(fn) + ": k/v NULL");
      if (!aligned16(k[i]) || !aligned16(v[i]))
        return fail(KVCR_EINVAL, std::string(fn) + ": k/v must be 16-byte aligned");
    } else if (!c->has_storage && k != nullptr && v != nullptr && (k[i] != nullptr || v[i] != nullptr)) {
      return fail(KVCR_ESTATE, std::string(fn) + ": bookkeeping-only caches take k = v = NULL");
    }
  }
  if (n_frames == 0) {
    for (int i = 0; i < n_caches; ++i) {
      caches[i]->last_slots.clear();
      caches[i]->last_evicted.clear();
      caches[i]->n_aux = 0;
    }
    return KVCR_OK;
  }
  std::vector<SlotState> before;
  std::vector<std::vector<int>> slots(n_caches), evicted(n_caches);
  for (int i = 0; i < n_caches; ++i) {
    before.push_back(snapshot(caches[i]));
    slots[i].resize(n_frames);
    for (int f = 0; f < n_frames; ++f) slots[i][f] = place_frame(caches[i], frame_idx[f], evicted[i]);
  }
  if (c0->has_storage) {
    RopeCopyBatchParams* p = new RopeCopyBatchParams();
    std::memset(p, 0, sizeof(*p));
    p->T = c0->T;
    p->H = c0->H;
    p->D = c0->D;
    p->grid_w = c0->rope ? c0->rp.grid_w : 1;
    p->rotate_a = c0->rope ? 1 : 0;
    p->pairs_t = c0->rope ? c0->rp.pairs_t : 0;
    p->pairs_h = c0->rope ? c0->rp.pairs_h : 0;
    p->pairs_w = c0->rope ? c0->rp.pairs_w : 0;
    p->htab = c0->rope ? reinterpret_cast<const float2*>(c0->storage + c0->lay.h_off) : nullptr;
    p->wtab = c0->rope ? reinterpret_cast<const float2*>(c0->storage + c0->lay.w_off) : nullptr;
    if (c0->rope)
      for (int f = 0; f < n_frames; ++f)
        for (int j = 0; j < c0->rp.pairs_t; ++j) {
          const double ang = (double)frame_idx[f] *
                             std::pow(c0->rp.base, -(2.0 * j) / (2.0 * c0->rp.pairs_t));
          p->ttab[f][j] = make_float2((float)std::cos(ang), (float)std::sin(ang));
        }
    const size_t frame_bytes = (size_t)c0->T * c0->H * c0->D * c0->esize;
    int n = 0;
    std::unique_ptr<QuantParams> qp(new QuantParams());
    std::memset(qp.get(), 0, sizeof(QuantParams));
    for (int i = 0; i < n_caches; ++i) {
      const kvcr_cache* c = caches[i];
      for (int f = 0; f < n_frames; ++f) {
        // skip frames not retained, or evicted again by a later frame of this call
        if (slots[i][f] < 0 || c->slot_frame[slots[i][f]] != frame_idx[f]) continue;
        if (c->fp8) {                              // its e4m3 copy, after the batch
          quant_segment_of_slot(c, slots[i][f], *qp, qp->n_seg, qp->n_seg * blocks_of(c->T));
          ++qp->n_seg;
        }
        p->src_a[n] = static_cast<const uint8_t*>(k[i]) + (size_t)f * frame_bytes;
        p->src_b[n] = static_cast<const uint8_t*>(v[i]) + (size_t)f * frame_bytes;
        p->dst_a[n] = c->storage + c->lay.k_off + (size_t)phys_of(c, slots[i][f]) * frame_bytes;
        p->dst_b[n] = c->storage + c->lay.v_off + (size_t)phys_of(c, slots[i][f]) * frame_bytes;
        p->tframe[n] = f;
        ++n;
      }
    }
    p->n = n;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    {
      LaunchScope scope(KVCR_K_APPEND_BATCH, s);
      e = launch_rope_copy_batch(*p, c0->dtype, s, c0->n_sm);
    }
    delete p;
    if (e == cudaSuccess && qp->n_seg > 0) {
      qp->H = c0->H;
      LaunchScope scope(KVCR_K_QUANT_E4M3, s);
      e = launch_quant_e4m3(*qp, c0->D, s);
    }
    if (e != cudaSuccess) {
      for (int i = 0; i < n_caches; ++i) restore(caches[i], before[i]);
      return cuda_fail(e, "kv_cache_append_rope_batch: launch");
    }
  }
  for (int i = 0; i < n_caches; ++i) {
    caches[i]->last_slots = slots[i];
    caches[i]->last_evicted = evicted[i];
    caches[i]->n_aux = 0;
  }
  return KVCR_OK;
}

int kv_cache_evict(kvcr_cache* c, int keep_recent, int32_t* evicted_out, int evicted_cap,
                   int* n_evicted) {
  if (c == nullptr) return fail(KVCR_EINVAL, "kv_cache_evict: cache is NULL");
  if (keep_recent < 0 || keep_recent > c->W)
    return fail(KVCR_EINVAL, "kv_cache_evict: keep_recent must be in [0, window]");
  int n = 0;
  while ((int)c->recent.size() > keep_recent) {
    const int old = c->recent.front();
    c->recent.pop_front();
    for (int i = c->S; i < c->S + c->W; ++i)
      if (c->slot_frame[i] == old) c->slot_frame[i] = -1;
    if (evicted_out && n < evicted_cap) evicted_out[n] = old;
    ++n;
  }
  if (n_evicted) *n_evicted = n;
  return KVCR_OK;
}

int kv_cache_slot_map(const kvcr_cache* c, int32_t* frame_of_slot, int cap) {
  if (c == nullptr || frame_of_slot == nullptr) return fail(KVCR_EINVAL, "kv_cache_slot_map: NULL");
  if (cap < c->S + c->W) return fail(KVCR_ESHAPE, "kv_cache_slot_map: cap < sinks + window");
  for (int i = 0; i < c->S + c->W; ++i) frame_of_slot[i] = c->slot_frame[i];
  return KVCR_OK;
}

int kv_cache_last_append(const kvcr_cache* c, int32_t* slots, int slots_cap, int32_t* evicted,
                         int evicted_cap, int* n_evicted) {
  if (c == nullptr) return fail(KVCR_EINVAL, "kv_cache_last_append: NULL");
  if (slots)
    for (int i = 0; i < (int)c->last_slots.size() && i < slots_cap; ++i) slots[i] = c->last_slots[i];
  if (evicted)
    for (int i = 0; i < (int)c->last_evicted.size() && i < evicted_cap; ++i)
      evicted[i] = c->last_evicted[i];
  if (n_evicted) *n_evicted = (int)c->last_evicted.size();
  return KVCR_OK;
}

int kv_cache_num_cached(const kvcr_cache* c, int* n) {
  if (c == nullptr || n == nullptr) return fail(KVCR_EINVAL, "kv_cache_num_cached: NULL");
  int k = 0;
  for (int f : c->slot_frame) k += f >= 0;
  *n = k;
  return KVCR_OK;
}

int kv_cache_slot_data(const kvcr_cache* c, int slot, const void** k, const void** v) {
  if (c == nullptr || k == nullptr || v == nullptr)
    return fail(KVCR_EINVAL, "kv_cache_slot_data: NULL");
  if (!c->has_storage) return fail(KVCR_ESTATE, "kv_cache_slot_data: bookkeeping-only cache");
  if (slot < 0 || slot >= c->S + c->W + c->A)
    return fail(KVCR_EINVAL, "kv_cache_slot_data: bad slot");
  const size_t frame = (size_t)c->T * c->H * c->D * c->esize;
  const int ph = phys_of(c, slot);
  *k = c->storage + c->lay.k_off + (size_t)ph * frame;
  *v = c->storage + c->lay.v_off + (size_t)ph * frame;
  return KVCR_OK;
}

int kv_cache_slot_data_fp8(const kvcr_cache* c, int slot, const void** k_codes,
                           const float** k_scales) {
  if (c == nullptr || k_codes == nullptr || k_scales == nullptr)
    return fail(KVCR_EINVAL, "kv_cache_slot_data_fp8: NULL");
  if (!c->has_storage || !c->fp8)
    return fail(KVCR_ESTATE, "kv_cache_slot_data_fp8: the cache keeps no e4m3 K copies");
  if (slot < 0 || slot >= c->S + c->W + c->A)
    return fail(KVCR_EINVAL, "kv_cache_slot_data_fp8: bad slot");
  const int ph = phys_of(c, slot);
  *k_codes = c->storage + c->lay.k8_off + (size_t)ph * c->T * c->H * c->D;
  *k_scales = reinterpret_cast<const float*>(c->storage + c->lay.k8s_off) +
              (size_t)ph * blocks_of(c->T) * c->H;
  return KVCR_OK;
}

int kv_cache_set_aux(kvcr_cache* c, const void* k, const void* v, const int32_t* aux_pos,
                     int n_frames, void* stream) {
  const char* fn = "kv_cache_set_aux";
  if (c == nullptr) return fail(KVCR_EINVAL, std::string(fn) + ": cache is NULL");
  if (n_frames < 0 || n_frames > c->A || n_frames > kMaxFrames)
    return fail(KVCR_ESHAPE, std::string(fn) + ": n_frames must be in [0, aux_frames] (<= 16)");
  if (aux_pos != nullptr)
    for (int i = 0; i < n_frames; ++i)
      if (aux_pos[i] < 0) return fail(KVCR_EINVAL, std::string(fn) + ": negative position");
  if (c->has_storage && n_frames > 0) {
    if (k == nullptr || v == nullptr) return fail(KVCR_EINVAL, std::string(fn) + ": k/v NULL");
    if (!aligned16(k) || !aligned16(v))
      return fail(KVCR_EINVAL, std::string(fn) + ": k/v must be 16-byte aligned");
  } else if (!c->has_storage && (k != nullptr || v != nullptr)) {
    return fail(KVCR_ESTATE, std::string(fn) + ": bookkeeping-only cache takes k = v = NULL");
  }
  if (c->has_storage && n_frames > 0) {
    RopeCopyParams p;
    std::memset(&p, 0, sizeof(p));
    fill_common(c, p);
    p.src_a = k;
    p.src_b = v;
    p.dst_a = c->storage + c->lay.k_off;
    p.dst_b = c->storage + c->lay.v_off;
    p.rotate_a = (c->rope && aux_pos != nullptr) ? 1 : 0;
    p.rotate_b = 0;
    p.n_frames = n_frames;
    const long long frame_elems = (long long)c->T * c->H * c->D;
    for (int f = 0; f < n_frames; ++f) {
      p.dst_frame_off[f] = (long long)(c->S + c->W + f) * frame_elems;
      p.src_frame[f] = f;
    }
    if (p.rotate_a) fill_ttab(c, p, aux_pos, n_frames);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    {
      LaunchScope scope(KVCR_K_SET_AUX, s);
      e = launch_rope_copy(p, c->dtype, s, c->n_sm);
    }
    if (e == cudaSuccess && c->fp8) {
      std::vector<int> aux_slots;
      for (int f = 0; f < n_frames; ++f) aux_slots.push_back(c->S + c->W + f);
      e = quant_slots(c, aux_slots, s);
    }
    if (e != cudaSuccess) return cuda_fail(e, "kv_cache_set_aux: launch");
  }
  c->n_aux = n_frames;
  return KVCR_OK;
}

// ==================================================== host state checkpoint
// Layout (int32 words): magic, version, then the configuration (S, W, A, T, H, D, F,
// dtype, rope, grid_h, grid_w, pairs_t, pairs_h, pairs_w, base as two words, fp8,
// fused), then the state: slot_frame[S + W], n_sinks_filled, last_frame, n_aux,
// phys[S + W], n_spare, spare[], n_recent, recent[], n_last_slots, last_slots[],
// n_last_evicted, last_evicted[].
namespace {
constexpr int32_t kStateMagic = 0x5243564B;  // "KVCR"
constexpr int32_t kStateVersion = 1;

void config_words(const kvcr_cache* c, std::vector<int32_t>& w) {
  int32_t base[2];
  std::memcpy(base, &c->rp.base, sizeof(double));
  const int32_t cfg[] = {c->S, c->W, c->A, c->T, c->H, c->D, c->F, (int32_t)c->dtype,
                         c->rope ? 1 : 0, c->rope ? c->rp.grid_h : 0, c->rope ? c->rp.grid_w : 0,
                         c->rope ? c->rp.pairs_t : 0, c->rope ? c->rp.pairs_h : 0,
                         c->rope ? c->rp.pairs_w : 0, c->rope ? base[0] : 0,
                         c->rope ? base[1] : 0, c->fp8 ? 1 : 0, c->fused ? 1 : 0};
  w.insert(w.end(), std::begin(cfg), std::end(cfg));
}

void state_words(const kvcr_cache* c, std::vector<int32_t>& w) {
  w.push_back(kStateMagic);
  w.push_back(kStateVersion);
  config_words(c, w);
  w.insert(w.end(), c->slot_frame.begin(), c->slot_frame.end());
  w.push_back(c->n_sinks_filled);
  w.push_back(c->last_frame);
  w.push_back(c->n_aux);
  w.insert(w.end(), c->phys.begin(), c->phys.end());
  w.push_back((int32_t)c->spare.size());
  w.insert(w.end(), c->spare.begin(), c->spare.end());
  w.push_back((int32_t)c->recent.size());
  w.insert(w.end(), c->recent.begin(), c->recent.end());
  w.push_back((int32_t)c->last_slots.size());
  w.insert(w.end(), c->last_slots.begin(), c->last_slots.end());
  w.push_back((int32_t)c->last_evicted.size());
  w.insert(w.end(), c->last_evicted.begin(), c->last_evicted.end());
}
}  // namespace

int kv_cache_export_state(const kvcr_cache* c, void* buf, size_t cap, size_t* size) {
  if (c == nullptr || size == nullptr) return fail(KVCR_EINVAL, "kv_cache_export_state: NULL");
  std::vector<int32_t> w;
  state_words(c, w);
  *size = w.size() * sizeof(int32_t);
  if (buf == nullptr) return KVCR_OK;
  if (cap < *size) return fail(KVCR_ESTORAGE, "kv_cache_export_state: buffer too small");
  std::memcpy(buf, w.data(), *size);
  return KVCR_OK;
}

int kv_cache_import_state(kvcr_cache* c, const void* buf, size_t size) {
  const char* fn = "kv_cache_import_state";
  if (c == nullptr || buf == nullptr) return fail(KVCR_EINVAL, std::string(fn) + ": NULL");
  if (size % sizeof(int32_t) != 0) return fail(KVCR_EINVAL, std::string(fn) + ": truncated");
  const size_t n = size / sizeof(int32_t);
  std::vector<int32_t> w(n);
  std::memcpy(w.data(), buf, size);
  size_t at = 0;
  bool short_buf = false;
  auto next = [&]() -> int32_t {
    if (at >= n) {
      short_buf = true;
      return 0;
    }
    return w[at++];
  };
  auto bad = [&](const char* why) { return fail(KVCR_EINVAL, std::string(fn) + ": " + why); };
  if (next() != kStateMagic || next() != kStateVersion)
    return bad("not a cache state of this version");
  std::vector<int32_t> cfg_want;
  config_words(c, cfg_want);
  for (int32_t v : cfg_want)
    if (next() != v || short_buf)
      return fail(KVCR_ESHAPE, std::string(fn) + ": the state belongs to a cache of another "
                                                 "configuration");
  const int SW = c->S + c->W;
  std::vector<int> slot_frame(SW), phys(SW), spare, recent_v, last_slots, last_evicted;
  for (int i = 0; i < SW; ++i) slot_frame[i] = next();
  const int n_sinks_filled = next();
  const int last_frame = next();
  const int n_aux = next();
  for (int i = 0; i < SW; ++i) phys[i] = next();
  auto read_list = [&](std::vector<int>& out, int limit) -> bool {
    const int k = next();
    if (short_buf || k < 0 || k > limit) return false;
    out.resize(k);
    for (int i = 0; i < k; ++i) out[i] = next();
    return !short_buf;
  };
  if (!read_list(spare, kMaxSlots) || !read_list(recent_v, c->W) ||
      !read_list(last_slots, kMaxFrames) || !read_list(last_evicted, kMaxSlots + kMaxFrames))
    return bad("malformed lists");
  if (short_buf || at != n) return bad("wrong length");
  // consistency of the slot table
  if (n_sinks_filled < 0 || n_sinks_filled > c->S) return bad("anchor count out of range");
  if (n_aux < 0 || n_aux > c->A) return bad("auxiliary count out of range");
  int max_cached = -1;
  std::vector<int> cached;
  for (int i = 0; i < SW; ++i) {
    const int f = slot_frame[i];
    if (f < -1) return bad("negative frame");
    if (i < c->S && ((i < n_sinks_filled) != (f >= 0))) return bad("anchor slots inconsistent");
    if (f >= 0) {
      cached.push_back(f);
      max_cached = std::max(max_cached, f);
    }
  }
  std::sort(cached.begin(), cached.end());
  if (std::adjacent_find(cached.begin(), cached.end()) != cached.end())
    return bad("a frame is cached twice");
  if (last_frame < max_cached) return bad("last frame below a cached frame");
  for (size_t i = 0; i < recent_v.size(); ++i) {
    if (i > 0 && recent_v[i] <= recent_v[i - 1]) return bad("window frames not increasing");
    int hits = 0;
    for (int s = c->S; s < SW; ++s) hits += slot_frame[s] == recent_v[i];
    if (hits != 1) return bad("window frame not in exactly one window slot");
  }
  int window_used = 0;
  for (int s = c->S; s < SW; ++s) window_used += slot_frame[s] >= 0;
  if (window_used != (int)recent_v.size()) return bad("window slots and recency list differ");
  // the physical relabelling: a permutation of the non-auxiliary frame slots
  const int n_phys = SW + c->A + (c->fused ? c->F : 0);
  std::vector<int> seen(n_phys, 0);
  if ((int)spare.size() != (c->fused ? c->F : 0)) return bad("spare slot count");
  for (int v : phys) {
    if (v < 0 || v >= n_phys || (v >= SW && v < SW + c->A)) return bad("physical slot range");
    seen[v]++;
  }
  for (int v : spare) {
    if (v < 0 || v >= n_phys || (v >= SW && v < SW + c->A)) return bad("spare slot range");
    seen[v]++;
  }
  for (int v = 0; v < n_phys; ++v)
    if ((v >= SW && v < SW + c->A) ? seen[v] != 0 : seen[v] != 1)
      return bad("physical slots are not a permutation");
  for (int v : last_slots)
    if (v < -1 || v >= SW) return bad("appended slot out of range");
  for (int v : last_evicted)
    if (v < 0) return bad("negative evicted frame");
  // commit
  c->slot_frame = slot_frame;
  c->n_sinks_filled = n_sinks_filled;
  c->last_frame = last_frame;
  c->n_aux = n_aux;
  c->phys = phys;
  c->spare = spare;
  c->recent.assign(recent_v.begin(), recent_v.end());
  c->last_slots = last_slots;
  c->last_evicted = last_evicted;
  return KVCR_OK;
}

int kv_cache_num_aux(const kvcr_cache* c, int* n) {
  if (c == nullptr || n == nullptr) return fail(KVCR_EINVAL, "kv_cache_num_aux: NULL");
  *n = c->n_aux;
  return KVCR_OK;
}

int chunk_attention_fwd(kvcr_cache* c, const void* q, int n_q, const void* k_cur,
                        const void* v_cur, const int32_t* cur_frame_idx, int n_cur_frames,
                        float softmax_scale, void* o, float* lse, void* stream) {
  if (c == nullptr) return fail(KVCR_EINVAL, "chunk_attention_fwd: cache is NULL");
  if (!c->has_storage) return fail(KVCR_ESTATE, "chunk_attention_fwd: bookkeeping-only cache");
  if (n_cur_frames < 1 || n_cur_frames > c->F)
    return fail(KVCR_ESHAPE, "chunk_attention_fwd: n_cur_frames must be in [1, chunk_frames]");
  if (n_q < 0) return fail(KVCR_ESHAPE, "chunk_attention_fwd: n_q < 0");
  const int n_cur = n_cur_frames * c->T;
  if (c->rope && n_q != n_cur)
    return fail(KVCR_ESHAPE, "chunk_attention_fwd: with RoPE n_q must be n_cur_frames * T");
  int rc = check_frames(c, cur_frame_idx, n_cur_frames, "chunk_attention_fwd");
  if (rc) return rc;
  if (n_q == 0) return KVCR_OK;
  if (!q || !k_cur || !v_cur || !o) return fail(KVCR_EINVAL, "chunk_attention_fwd: NULL tensor");
  if (!aligned16(q) || !aligned16(k_cur) || !aligned16(v_cur) || !aligned16(o))
    return fail(KVCR_EINVAL, "chunk_attention_fwd: tensors must be 16-byte aligned");
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u))
    return fail(KVCR_EINVAL, "chunk_attention_fwd: lse must be 4-byte aligned");
  if ((long long)n_q * c->H * c->D > (1LL << 31) - 1)
    return fail(KVCR_ESHAPE, "chunk_attention_fwd: n_q too large");
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt((float)c->D);
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  // visible cached frames, in slot order
  int slots[kMaxSlots];
  const int n_vis = visible_slots(c, slots);

  const void* q_src = q;
  const void* k_src = k_cur;
  if (c->rope) {
    RopeCopyParams p;
    std::memset(&p, 0, sizeof(p));
    fill_common(c, p);
    p.src_a = q;
    p.src_b = k_cur;
    p.dst_a = c->storage + c->lay.q_off;
    p.dst_b = c->storage + c->lay.ks_off;
    p.rotate_a = 1;
    p.rotate_b = 1;
    p.n_frames = n_cur_frames;
    const long long frame_elems = (long long)c->T * c->H * c->D;
    for (int f = 0; f < n_cur_frames; ++f) {
      p.dst_frame_off[f] = f * frame_elems;
      p.src_frame[f] = f;
    }
    fill_ttab(c, p, cur_frame_idx, n_cur_frames);
    cudaError_t e;
    {
      LaunchScope scope(KVCR_K_ROPE_STAGE, s);
      e = launch_rope_copy(p, c->dtype, s, c->n_sm);
    }
    if (e != cudaSuccess) return cuda_fail(e, "chunk_attention_fwd: rope stage launch");
    q_src = c->storage + c->lay.q_off;
    k_src = c->storage + c->lay.ks_off;
  }

  if (c->dtype == KVCR_BF16) {
    ChunkAttnParams p;
    std::memset(&p, 0, sizeof(p));
    const uint64_t dq[3] = {(uint64_t)c->D, (uint64_t)c->H, (uint64_t)n_q};
    const uint64_t dn[3] = {(uint64_t)c->D, (uint64_t)c->H, (uint64_t)n_cur};
    rc = encode_bf16_map(&p.tm_q, q_src, 3, dq, kTile);
    if (!rc) rc = encode_bf16_map(&p.tm_kn, k_src, 3, dn, kKeyTile);
    if (!rc) rc = encode_bf16_map(&p.tm_vn, v_cur, 3, dn, kKeyTile);
    if (rc) return rc;
    p.tm_kc = c->tm_kc;
    p.tm_vc = c->tm_vc;
    p.c.o = o;
    p.c.lse = lse;
    p.c.n_q = n_q;
    p.c.H = c->H;
    p.c.scale_log2 = (float)(scale * 1.4426950408889634);
    p.c.inject = inject_state().kind;
    p.c.wait_ns = inject_state().wait_ns;
    p.s.T = c->T;
    p.s.n_vis = n_vis;
    p.s.tiles_per_slot = (c->T + kKeyTile - 1) / kKeyTile;
    p.s.n_cur = n_cur;
    p.s.cur_tiles = (n_cur + kKeyTile - 1) / kKeyTile;
    for (int i = 0; i < n_vis; ++i) p.s.slots[i] = slots[i];
    cudaError_t e;
    {
      LaunchScope scope(KVCR_K_CHUNK_ATTN, s);
      e = launch_chunk_attn_sm100(p, c->D, (n_q + kTile - 1) / kTile, s);
    }
    if (e != cudaSuccess) return cuda_fail(e, "chunk_attention_fwd: attention launch");
  } else {
    F32AttnParams p;
    std::memset(&p, 0, sizeof(p));
    p.q = static_cast<const float*>(q_src);
    p.kc = reinterpret_cast<const float*>(c->storage + c->lay.k_off);
    p.vc = reinterpret_cast<const float*>(c->storage + c->lay.v_off);
    p.kn = static_cast<const float*>(k_src);
    p.vn = static_cast<const float*>(v_cur);
    p.o = static_cast<float*>(o);
    p.lse = lse;
    p.n_q = n_q;
    p.H = c->H;
    p.D = c->D;
    p.T = c->T;
    p.n_vis = n_vis;
    p.n_cur = n_cur;
    p.scale = scale;
    for (int i = 0; i < n_vis; ++i) p.slots[i] = slots[i];
    cudaError_t e;
    {
      LaunchScope scope(KVCR_K_ATTN_F32, s);
      e = launch_attn_f32(p, s);
    }
    if (e != cudaSuccess) return cuda_fail(e, "chunk_attention_fwd: fp32 attention launch");
  }
  return KVCR_OK;
}

// ====================================== chunk attention + finalize in one pass
// The chunk's rotated K and its V go once into spare physical slots (one rope
// copy launch), the queries are rotated into the scratch, the attention reads
// the chunk's keys from the spare slots (as cached-frame tiles), and the append
// is done by relabelling: each retained frame's anchor / window slot points at
// the spare slot holding it, and the physical slot it replaced becomes spare.
int chunk_attention_fwd_finalize(kvcr_cache* c, const void* q, int n_q, const void* k_cur,
                                 const void* v_cur, const int32_t* cur_frame_idx,
                                 int n_cur_frames, float softmax_scale, void* o, float* lse,
                                 void* stream) {
  const char* fn = "chunk_attention_fwd_finalize";
  if (c == nullptr) return fail(KVCR_EINVAL, std::string(fn) + ": cache is NULL");
  if (!c->has_storage) return fail(KVCR_ESTATE, std::string(fn) + ": bookkeeping-only cache");
  if (!c->fused)
    return fail(KVCR_ESTATE, std::string(fn) + ": the cache has no spare slots "
                                               "(create it with KVCR_CACHE_FUSED_FINALIZE)");
  if (n_cur_frames < 1 || n_cur_frames > c->F)
    return fail(KVCR_ESHAPE, std::string(fn) + ": n_cur_frames must be in [1, chunk_frames]");
  if (n_q < 0) return fail(KVCR_ESHAPE, std::string(fn) + ": n_q < 0");
  const int n_cur = n_cur_frames * c->T;
  if (c->rope && n_q != n_cur)
    return fail(KVCR_ESHAPE, std::string(fn) + ": with RoPE n_q must be n_cur_frames * T");
  int rc = check_frames(c, cur_frame_idx, n_cur_frames, fn);
  if (rc) return rc;
  if (!k_cur || !v_cur || (n_q > 0 && (!q || !o)))
    return fail(KVCR_EINVAL, std::string(fn) + ": NULL tensor");
  if (!aligned16(k_cur) || !aligned16(v_cur) || (n_q > 0 && (!aligned16(q) || !aligned16(o))))
    return fail(KVCR_EINVAL, std::string(fn) + ": tensors must be 16-byte aligned");
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u))
    return fail(KVCR_EINVAL, std::string(fn) + ": lse must be 4-byte aligned");
  if ((long long)n_q * c->H * c->D > (1LL << 31) - 1)
    return fail(KVCR_ESHAPE, std::string(fn) + ": n_q too large");
  if ((int)c->spare.size() < n_cur_frames)
    return fail(KVCR_ESTATE, std::string(fn) + ": not enough spare slots");
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt((float)c->D);
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  // keys of this call: the visible cached / auxiliary frames, then the chunk's
  // own frames from the spare slots they are written to
  int slots[kMaxSlots];
  int n_vis = visible_slots(c, slots);
  for (int f = 0; f < n_cur_frames; ++f) slots[n_vis++] = c->spare[f];
  const long long frame_elems = (long long)c->T * c->H * c->D;
  cudaError_t e;
  {  // rotated K and V of the chunk into the spare slots
    RopeCopyParams p;
    std::memset(&p, 0, sizeof(p));
    fill_common(c, p);
    p.src_a = k_cur;
    p.src_b = v_cur;
    p.dst_a = c->storage + c->lay.k_off;
    p.dst_b = c->storage + c->lay.v_off;
    p.rotate_a = c->rope ? 1 : 0;
    p.rotate_b = 0;
    p.n_frames = n_cur_frames;
    for (int f = 0; f < n_cur_frames; ++f) {
      p.dst_frame_off[f] = (long long)c->spare[f] * frame_elems;
      p.src_frame[f] = f;
    }
    if (c->rope) fill_ttab(c, p, cur_frame_idx, n_cur_frames);
    LaunchScope scope(KVCR_K_APPEND_ROPE, s);
    e = launch_rope_copy(p, c->dtype, s, c->n_sm);
  }
  if (e != cudaSuccess) return cuda_fail(e, "chunk_attention_fwd_finalize: write launch");
  const void* q_src = q;
  if (c->rope && n_q > 0) {  // rotated queries into the scratch
    RopeCopyParams p;
    std::memset(&p, 0, sizeof(p));
    fill_common(c, p);
    p.src_a = q;
    p.dst_a = c->storage + c->lay.q_off;
    p.rotate_a = 1;
    p.n_frames = n_cur_frames;
    for (int f = 0; f < n_cur_frames; ++f) {
      p.dst_frame_off[f] = f * frame_elems;
      p.src_frame[f] = f;
    }
    fill_ttab(c, p, cur_frame_idx, n_cur_frames);
    LaunchScope scope(KVCR_K_ROPE_STAGE, s);
    e = launch_rope_copy(p, c->dtype, s, c->n_sm);
    if (e != cudaSuccess) return cuda_fail(e, "chunk_attention_fwd_finalize: stage launch");
    q_src = c->storage + c->lay.q_off;
  }
  if (n_q > 0) {
    ChunkAttnParams p;
    std::memset(&p, 0, sizeof(p));
    const uint64_t dq[3] = {(uint64_t)c->D, (uint64_t)c->H, (uint64_t)n_q};
    const uint64_t dn[3] = {(uint64_t)c->D, (uint64_t)c->H, (uint64_t)n_cur};
    rc = encode_bf16_map(&p.tm_q, q_src, 3, dq, kTile);
    // no current-chunk tiles are read; the maps stay valid for the prefetch
    if (!rc) rc = encode_bf16_map(&p.tm_kn, k_cur, 3, dn, kKeyTile);
    if (!rc) rc = encode_bf16_map(&p.tm_vn, v_cur, 3, dn, kKeyTile);
    if (rc) return rc;
    p.tm_kc = c->tm_kc;
    p.tm_vc = c->tm_vc;
    p.c.o = o;
    p.c.lse = lse;
    p.c.n_q = n_q;
    p.c.H = c->H;
    p.c.scale_log2 = (float)(scale * 1.4426950408889634);
    p.c.inject = inject_state().kind;
    p.c.wait_ns = inject_state().wait_ns;
    p.s.T = c->T;
    p.s.n_vis = n_vis;
    p.s.tiles_per_slot = (c->T + kKeyTile - 1) / kKeyTile;
    p.s.n_cur = 0;
    p.s.cur_tiles = 0;
    for (int i = 0; i < n_vis; ++i) p.s.slots[i] = slots[i];
    LaunchScope scope(KVCR_K_CHUNK_ATTN, s);
    e = launch_chunk_attn_sm100(p, c->D, (n_q + kTile - 1) / kTile, s);
    if (e != cudaSuccess) return cuda_fail(e, "chunk_attention_fwd_finalize: attention launch");
  }

  // the append, by relabelling
  std::vector<int> placed(n_cur_frames), evicted;
  for (int i = 0; i < n_cur_frames; ++i) {
    placed[i] = place_frame(c, cur_frame_idx[i], evicted);
    if (placed[i] >= 0) std::swap(c->phys[placed[i]], c->spare[i]);
  }
  c->last_slots = placed;
  c->last_evicted = evicted;
  c->n_aux = 0;
  return KVCR_OK;
}

// ============================================== chunk attention, e4m3 QK^T
// Stage (RoPE) as chunk_attention_fwd(), quantize the staged queries and current
// keys to e4m3 blocks of 128 tokens, then the tensor-core kernel with the QK^T
// product in e4m3 over the cache's e4m3 K copies and the P V product in bf16.
int chunk_attention_fwd_fp8(kvcr_cache* c, const void* q, int n_q, const void* k_cur,
                            const void* v_cur, const int32_t* cur_frame_idx, int n_cur_frames,
                            float softmax_scale, void* o, float* lse, void* stream) {
  const char* fn = "chunk_attention_fwd_fp8";
  if (c == nullptr) return fail(KVCR_EINVAL, std::string(fn) + ": cache is NULL");
  if (!c->has_storage) return fail(KVCR_ESTATE, std::string(fn) + ": bookkeeping-only cache");
  if (!c->fp8)
    return fail(KVCR_ESTATE, std::string(fn) + ": the cache keeps no e4m3 K copies "
                                               "(create it with KVCR_CACHE_FP8_K)");
  if (n_cur_frames < 1 || n_cur_frames > c->F)
    return fail(KVCR_ESHAPE, std::string(fn) + ": n_cur_frames must be in [1, chunk_frames]");
  if (n_q < 0) return fail(KVCR_ESHAPE, std::string(fn) + ": n_q < 0");
  const int n_cur = n_cur_frames * c->T;
  if (c->rope && n_q != n_cur)
    return fail(KVCR_ESHAPE, std::string(fn) + ": with RoPE n_q must be n_cur_frames * T");
  if (!c->rope && (long long)n_q > (long long)c->F * c->T)
    return fail(KVCR_ESHAPE, std::string(fn) + ": n_q larger than the query staging "
                                               "(chunk_frames * tokens_per_frame)");
  int rc = check_frames(c, cur_frame_idx, n_cur_frames, fn);
  if (rc) return rc;
  if (n_q == 0) return KVCR_OK;
  if (!q || !k_cur || !v_cur || !o) return fail(KVCR_EINVAL, std::string(fn) + ": NULL tensor");
  if (!aligned16(q) || !aligned16(k_cur) || !aligned16(v_cur) || !aligned16(o))
    return fail(KVCR_EINVAL, std::string(fn) + ": tensors must be 16-byte aligned");
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u))
    return fail(KVCR_EINVAL, std::string(fn) + ": lse must be 4-byte aligned");
  if ((long long)n_q * c->H * c->D > (1LL << 31) - 1)
    return fail(KVCR_ESHAPE, std::string(fn) + ": n_q too large");
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt((float)c->D);
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  int slots[kMaxSlots];
  const int n_vis = visible_slots(c, slots);

  const void* q_src = q;
  const void* k_src = k_cur;
  cudaError_t e;
  if (c->rope) {
    RopeCopyParams p;
    std::memset(&p, 0, sizeof(p));
    fill_common(c, p);
    p.src_a = q;
    p.src_b = k_cur;
    p.dst_a = c->storage + c->lay.q_off;
    p.dst_b = c->storage + c->lay.ks_off;
    p.rotate_a = 1;
    p.rotate_b = 1;
    p.n_frames = n_cur_frames;
    const long long frame_elems = (long long)c->T * c->H * c->D;
    for (int f = 0; f < n_cur_frames; ++f) {
      p.dst_frame_off[f] = f * frame_elems;
      p.src_frame[f] = f;
    }
    fill_ttab(c, p, cur_frame_idx, n_cur_frames);
    {
      LaunchScope scope(KVCR_K_ROPE_STAGE, s);
      e = launch_rope_copy(p, c->dtype, s, c->n_sm);
    }
    if (e != cudaSuccess) return cuda_fail(e, "chunk_attention_fwd_fp8: rope stage launch");
    q_src = c->storage + c->lay.q_off;
    k_src = c->storage + c->lay.ks_off;
  }
  uint8_t* q8 = c->storage + c->lay.q8_off;
  uint8_t* k8 = c->storage + c->lay.c8_off;
  float* q8s = reinterpret_cast<float*>(c->storage + c->lay.q8s_off);
  float* k8s = reinterpret_cast<float*>(c->storage + c->lay.c8s_off);
  {
    std::unique_ptr<QuantParams> qp(new QuantParams());
    std::memset(qp.get(), 0, sizeof(QuantParams));
    qp->src[0] = q_src;
    qp->dst[0] = q8;
    qp->scale[0] = q8s;
    qp->n_tok[0] = n_q;
    qp->tile0[0] = 0;
    qp->src[1] = k_src;
    qp->dst[1] = k8;
    qp->scale[1] = k8s;
    qp->n_tok[1] = n_cur;
    qp->tile0[1] = blocks_of(n_q);
    qp->n_seg = 2;
    qp->H = c->H;
    LaunchScope scope(KVCR_K_QUANT_E4M3, s);
    e = launch_quant_e4m3(*qp, c->D, s);
  }
  if (e != cudaSuccess) return cuda_fail(e, "chunk_attention_fwd_fp8: quantization launch");

  ChunkAttnParams p;
  std::memset(&p, 0, sizeof(p));
  const uint64_t dq[3] = {(uint64_t)c->D, (uint64_t)c->H, (uint64_t)n_q};
  const uint64_t dn[3] = {(uint64_t)c->D, (uint64_t)c->H, (uint64_t)n_cur};
  rc = encode_map(&p.tm_q, true, q8, 3, dq, kTile);
  if (!rc) rc = encode_map(&p.tm_kn, true, k8, 3, dn, kKeyTile);
  if (!rc) rc = encode_bf16_map(&p.tm_vn, v_cur, 3, dn, kKeyTile);
  if (rc) return rc;
  p.tm_kc = c->tm_kc8;
  p.tm_vc = c->tm_vc;
  p.q_scale = q8s;
  p.kc_scale = reinterpret_cast<const float*>(c->storage + c->lay.k8s_off);
  p.kn_scale = k8s;
  p.c.o = o;
  p.c.lse = lse;
  p.c.n_q = n_q;
  p.c.H = c->H;
  p.c.scale_log2 = (float)(scale * 1.4426950408889634);
  p.c.inject = inject_state().kind;
  p.c.wait_ns = inject_state().wait_ns;
  p.s.T = c->T;
  p.s.n_vis = n_vis;
  p.s.tiles_per_slot = (c->T + kKeyTile - 1) / kKeyTile;
  p.s.n_cur = n_cur;
  p.s.cur_tiles = (n_cur + kKeyTile - 1) / kKeyTile;
  for (int i = 0; i < n_vis; ++i) p.s.slots[i] = slots[i];
  {
    LaunchScope scope(KVCR_K_CHUNK_ATTN_FP8, s);
    e = launch_chunk_attn_sm100(p, c->D, (n_q + kTile - 1) / kTile, s, true);
  }
  if (e != cudaSuccess) return cuda_fail(e, "chunk_attention_fwd_fp8: attention launch");
  return KVCR_OK;
}

// ============================================= chunk attention, static scratch
// Same computation as chunk_attention_fwd(); the rotated queries and current
// keys are staged in the library's fixed device array instead of the cache's
// scratch region, so the call needs no memory beyond its inputs, outputs and
// the cache.  The first call on a device looks the array's address up (once
// per device); make that first call before any stream capture.
int chunk_attention_fwd_static_scratch(kvcr_cache* c, const void* q, int n_q, const void* k_cur,
                                       const void* v_cur, const int32_t* cur_frame_idx,
                                       int n_cur_frames, float softmax_scale, void* o, float* lse,
                                       void* stream) {
  const char* fn = "chunk_attention_fwd_static_scratch";
  if (c == nullptr) return fail(KVCR_EINVAL, std::string(fn) + ": cache is NULL");
  if (!c->has_storage) return fail(KVCR_ESTATE, std::string(fn) + ": bookkeeping-only cache");
  if (n_cur_frames < 1 || n_cur_frames > c->F)
    return fail(KVCR_ESHAPE, std::string(fn) + ": n_cur_frames must be in [1, chunk_frames]");
  if (n_q < 0) return fail(KVCR_ESHAPE, std::string(fn) + ": n_q < 0");
  const int n_cur = n_cur_frames * c->T;
  if (c->rope && n_q != n_cur)
    return fail(KVCR_ESHAPE, std::string(fn) + ": with RoPE n_q must be n_cur_frames * T");
  int rc = check_frames(c, cur_frame_idx, n_cur_frames, fn);
  if (rc) return rc;
  if (n_q == 0) return KVCR_OK;
  if (!q || !k_cur || !v_cur || !o) return fail(KVCR_EINVAL, std::string(fn) + ": NULL tensor");
  if (!aligned16(q) || !aligned16(k_cur) || !aligned16(v_cur) || !aligned16(o))
    return fail(KVCR_EINVAL, std::string(fn) + ": tensors must be 16-byte aligned");
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u))
    return fail(KVCR_EINVAL, std::string(fn) + ": lse must be 4-byte aligned");
  if ((long long)n_q * c->H * c->D > (1LL << 31) - 1)
    return fail(KVCR_ESHAPE, std::string(fn) + ": n_q too large");
  // staging needs: rotated Q then rotated current K, each 256-byte aligned
  const size_t half = align_up((size_t)n_cur * c->H * c->D * c->esize, 256);
  if (c->rope && 2 * half > kStaticScratchBytes)
    return fail(KVCR_ESHAPE, std::string(fn) + ": the chunk needs " + std::to_string(2 * half) +
                                 " bytes of staging, more than the fixed " +
                                 std::to_string(kStaticScratchBytes) + "-byte array");
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt((float)c->D);
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  int slots[kMaxSlots];
  const int n_vis = visible_slots(c, slots);

  const void* q_src = q;
  const void* k_src = k_cur;
  if (c->rope) {
    void* scratch = nullptr;
    cudaError_t e = static_scratch_address(&scratch);
    if (e != cudaSuccess) return cuda_fail(e, "chunk_attention_fwd_static_scratch: array address");
    uint8_t* qs = static_cast<uint8_t*>(scratch);
    uint8_t* ks = qs + half;
    RopeCopyParams p;
    std::memset(&p, 0, sizeof(p));
    fill_common(c, p);
    p.src_a = q;
    p.src_b = k_cur;
    p.dst_a = qs;
    p.dst_b = ks;
    p.rotate_a = 1;
    p.rotate_b = 1;
    p.n_frames = n_cur_frames;
    const long long frame_elems = (long long)c->T * c->H * c->D;
    for (int f = 0; f < n_cur_frames; ++f) {
      p.dst_frame_off[f] = f * frame_elems;
      p.src_frame[f] = f;
    }
    fill_ttab(c, p, cur_frame_idx, n_cur_frames);
    {
      LaunchScope scope(KVCR_K_ROPE_STAGE, s);
      e = launch_rope_copy(p, c->dtype, s, c->n_sm);
    }
    if (e != cudaSuccess) return cuda_fail(e, "chunk_attention_fwd_static_scratch: stage launch");
    q_src = qs;
    k_src = ks;
  }

  if (c->dtype == KVCR_BF16) {
    ChunkAttnParams p;
    std::memset(&p, 0, sizeof(p));
    const uint64_t dq[3] = {(uint64_t)c->D, (uint64_t)c->H, (uint64_t)n_q};
    const uint64_t dn[3] = {(uint64_t)c->D, (uint64_t)c->H, (uint64_t)n_cur};
    rc = encode_bf16_map(&p.tm_q, q_src, 3, dq, kTile);
    if (!rc) rc = encode_bf16_map(&p.tm_kn, k_src, 3, dn, kKeyTile);
    if (!rc) rc = encode_bf16_map(&p.tm_vn, v_cur, 3, dn, kKeyTile);
    if (rc) return rc;
    p.tm_kc = c->tm_kc;
    p.tm_vc = c->tm_vc;
    p.c.o = o;
    p.c.lse = lse;
    p.c.n_q = n_q;
    p.c.H = c->H;
    p.c.scale_log2 = (float)(scale * 1.4426950408889634);
    p.c.inject = inject_state().kind;
    p.c.wait_ns = inject_state().wait_ns;
    p.s.T = c->T;
    p.s.n_vis = n_vis;
    p.s.tiles_per_slot = (c->T + kKeyTile - 1) / kKeyTile;
    p.s.n_cur = n_cur;
    p.s.cur_tiles = (n_cur + kKeyTile - 1) / kKeyTile;
    for (int i = 0; i < n_vis; ++i) p.s.slots[i] = slots[i];
    cudaError_t e;
    {
      LaunchScope scope(KVCR_K_CHUNK_ATTN, s);
      e = launch_chunk_attn_sm100(p, c->D, (n_q + kTile - 1) / kTile, s);
    }
    if (e != cudaSuccess) return cuda_fail(e, "chunk_attention_fwd_static_scratch: attention launch");
  } else {
    F32AttnParams p;
    std::memset(&p, 0, sizeof(p));
    p.q = static_cast<const float*>(q_src);
    p.kc = reinterpret_cast<const float*>(c->storage + c->lay.k_off);
    p.vc = reinterpret_cast<const float*>(c->storage + c->lay.v_off);
    p.kn = static_cast<const float*>(k_src);
    p.vn = static_cast<const float*>(v_cur);
    p.o = static_cast<float*>(o);
    p.lse = lse;
    p.n_q = n_q;
    p.H = c->H;
    p.D = c->D;
    p.T = c->T;
    p.n_vis = n_vis;
    p.n_cur = n_cur;
    p.scale = scale;
    for (int i = 0; i < n_vis; ++i) p.slots[i] = slots[i];
    cudaError_t e;
    {
      LaunchScope scope(KVCR_K_ATTN_F32, s);
      e = launch_attn_f32(p, s);
    }
    if (e != cudaSuccess)
      return cuda_fail(e, "chunk_attention_fwd_static_scratch: fp32 attention launch");
  }
  return KVCR_OK;
}

// ======================================================================= MoBA
static int moba_check_layout(const kvcr_moba_layout* layout, MobaLay* out) {
  if (layout == nullptr) return fail(KVCR_EINVAL, "moba: layout is NULL");
  if (layout->n_chunks < 1 || layout->chunk_tokens < 1 || layout->n_bidir_chunks < 0)
    return fail(KVCR_ESHAPE, "moba: need n_chunks >= 1, chunk_tokens >= 1, n_bidir_chunks >= 0");
  const long long L =
      (2LL * layout->n_chunks + layout->n_bidir_chunks) * (long long)layout->chunk_tokens;
  if (L > (long long)kMobaMaxTiles * kTile)
    return fail(KVCR_ESHAPE, "moba: sequence longer than 4096 * 128 tokens");
  *out = MobaLay{layout->n_chunks, layout->chunk_tokens, layout->n_bidir_chunks, (int)L};
  return KVCR_OK;
}

int moba_classify_tiles(const kvcr_moba_layout* layout, int tile, uint8_t* cls, size_t cap) {
  MobaLay l;
  int rc = moba_check_layout(layout, &l);
  if (rc) return rc;
  if (tile < 1) return fail(KVCR_EINVAL, "moba_classify_tiles: tile < 1");
  const long long nt = ((long long)l.L + tile - 1) / tile;
  if (cls == nullptr || (long long)cap < nt * nt)
    return fail(KVCR_ESHAPE, "moba_classify_tiles: output smaller than nt * nt");
  for (long long i = 0; i < nt; ++i)
    for (long long j = 0; j < nt; ++j)
      cls[i * nt + j] = (uint8_t)moba_classify(l, (int)i, (int)j, tile);
  return KVCR_OK;
}

namespace {
// Number of 128-key tiles hit by the union of intervals [lo[k], hi[k]).
int tiles_hit(const int* lo, const int* hi, int n) {
  std::vector<std::pair<int, int>> iv;
  for (int k = 0; k < n; ++k)
    if (hi[k] > lo[k]) iv.push_back({lo[k] / kTile, (hi[k] - 1) / kTile});
  std::sort(iv.begin(), iv.end());
  int count = 0, cur_lo = -1, cur_hi = -2;
  for (auto& t : iv) {
    if (t.first > cur_hi) {
      if (cur_hi >= cur_lo && cur_lo >= 0) count += cur_hi - cur_lo + 1;
      cur_lo = t.first;
      cur_hi = t.second;
    } else {
      cur_hi = std::max(cur_hi, t.second);
    }
  }
  if (cur_lo >= 0) count += cur_hi - cur_lo + 1;
  return count;
}

// Units ordered heaviest first (stable on ties).
void order_by_work(const std::vector<int>& work, std::vector<uint16_t>& order) {
  order.resize(work.size());
  for (size_t i = 0; i < work.size(); ++i) order[i] = (uint16_t)i;
  std::stable_sort(order.begin(), order.end(),
                   [&](uint16_t a, uint16_t b) { return work[a] > work[b]; });
}

// Forward work units are pairs of 128-row query tiles (one CTA each).  A unit's
// work is the number of key tiles hit by the union of its rows' allowed key
// intervals.
void moba_order(const MobaLay& l, std::vector<uint16_t>& order) {
  constexpr int kUnitRows = 2 * kTile;
  const int nt = (l.L + kUnitRows - 1) / kUnitRows;
  std::vector<int> work(nt);
  constexpr int kCap = 2 * kUnitRows + 8;
  int lo[kCap], hi[kCap];
  for (int i = 0; i < nt; ++i) {
    const int r0 = i * kUnitRows, r1 = std::min(r0 + kUnitRows, l.L);
    work[i] = tiles_hit(lo, hi, moba_row_intervals(l, r0, r1, lo, hi, kCap));
  }
  order_by_work(work, order);
}

// Backward work units are single 128-row tiles: query tiles for dQ (work = key
// tiles read), key tiles for dK / dV (work = query tiles that read them).
void moba_bwd_orders(const MobaLay& l, std::vector<uint16_t>& by_query,
                     std::vector<uint16_t>& by_key) {
  const int nt = (l.L + kTile - 1) / kTile;
  std::vector<int> wq(nt), wk(nt);
  constexpr int kCap = 2 * kTile + 8;
  int lo[kCap], hi[kCap];
  for (int i = 0; i < nt; ++i) {
    const int r0 = i * kTile, r1 = std::min(r0 + kTile, l.L);
    wq[i] = tiles_hit(lo, hi, moba_row_intervals(l, r0, r1, lo, hi, kCap));
    int n = 0, kk, ki, ks, ke;
    for (int cp = r0; cp < r1 && n + 2 <= kCap; cp = ke) {
      moba_block(l, cp, kk, ki, ks, ke);
      n += moba_col_intervals(l, cp, lo + n, hi + n);
    }
    wk[i] = tiles_hit(lo, hi, n);
  }
  order_by_work(wq, by_query);
  order_by_work(wk, by_key);
}
}  // namespace

int moba_attention_fwd(const void* q, const void* k, const void* v,
                       const kvcr_moba_layout* layout, int heads, int head_dim, kvcr_dtype dtype,
                       float softmax_scale, void* o, float* lse, void* stream) {
  MobaLay l;
  int rc = moba_check_layout(layout, &l);
  if (rc) return rc;
  if (dtype != KVCR_BF16) return fail(KVCR_EUNSUPPORTED, "moba_attention_fwd: bf16 only");
  if (head_dim != 64 && head_dim != 128)
    return fail(KVCR_EUNSUPPORTED, "moba_attention_fwd: head_dim must be 64 or 128");
  if (heads < 1) return fail(KVCR_ESHAPE, "moba_attention_fwd: heads < 1");
  if ((long long)l.L * heads * head_dim > (1LL << 31) - 1)
    return fail(KVCR_ESHAPE, "moba_attention_fwd: tensor too large");
  if (!q || !k || !v || !o) return fail(KVCR_EINVAL, "moba_attention_fwd: NULL tensor");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return fail(KVCR_EINVAL, "moba_attention_fwd: tensors must be 16-byte aligned");
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u))
    return fail(KVCR_EINVAL, "moba_attention_fwd: lse must be 4-byte aligned");
  int n_sm = 0, cc = 0;
  rc = device_sm_count(&n_sm, &cc);
  if (rc) return rc;
  if (cc != 10) return fail(KVCR_EUNSUPPORTED, "moba_attention_fwd: needs an sm_100 GPU");

  static std::mutex mu;
  static MobaLay last{0, 0, 0, 0};
  static std::vector<uint16_t> last_order;
  MobaAttnParams* p = new MobaAttnParams();
  std::memset(p, 0, sizeof(*p));
  {
    std::lock_guard<std::mutex> g(mu);
    if (!(last.n == l.n && last.c == l.c && last.m == l.m)) {
      moba_order(l, last_order);
      last = l;
    }
    for (size_t i = 0; i < last_order.size(); ++i) p->s.order[i] = last_order[i];
  }
  const uint64_t d3[3] = {(uint64_t)head_dim, (uint64_t)heads, (uint64_t)l.L};
  rc = encode_bf16_map(&p->tm_q, q, 3, d3, kTile);
  if (!rc) rc = encode_bf16_map(&p->tm_k, k, 3, d3, kKeyTile);
  if (!rc) rc = encode_bf16_map(&p->tm_v, v, 3, d3, kKeyTile);
  if (rc) {
    delete p;
    return rc;
  }
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt((float)head_dim);
  p->c.o = o;
  p->c.lse = lse;
  p->c.n_q = l.L;
  p->c.H = heads;
  p->c.scale_log2 = (float)(scale * 1.4426950408889634);
  p->c.inject = inject_state().kind;
  p->c.wait_ns = inject_state().wait_ns;
  p->s.n_chunks = l.n;
  p->s.chunk_tokens = l.c;
  p->s.n_bidir = l.m;
  p->s.L = l.L;
  p->s.n_row_tiles = (l.L + 2 * kTile - 1) / (2 * kTile);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  {
    LaunchScope scope(KVCR_K_MOBA_ATTN, s);
    e = launch_moba_attn_sm100(*p, head_dim, s);
  }
  delete p;
  if (e != cudaSuccess) return cuda_fail(e, "moba_attention_fwd: launch");
  return KVCR_OK;
}

size_t moba_attention_bwd_workspace_bytes(const kvcr_moba_layout* layout, int heads) {
  MobaLay l;
  if (moba_check_layout(layout, &l) != KVCR_OK || heads < 1) return 0;
  const size_t lpad = (size_t)((l.L + kTile - 1) / kTile) * kTile;
  return lpad * (size_t)heads * 2 * sizeof(float);
}

int moba_attention_bwd(const void* q, const void* k, const void* v, const void* o,
                       const void* d_o, const float* lse, const kvcr_moba_layout* layout,
                       int heads, int head_dim, kvcr_dtype dtype, float softmax_scale, void* dq,
                       void* dk, void* dv, void* workspace, size_t workspace_bytes,
                       void* stream) {
  MobaLay l;
  int rc = moba_check_layout(layout, &l);
  if (rc) return rc;
  if (dtype != KVCR_BF16) return fail(KVCR_EUNSUPPORTED, "moba_attention_bwd: bf16 only");
  if (head_dim != 64 && head_dim != 128)
    return fail(KVCR_EUNSUPPORTED, "moba_attention_bwd: head_dim must be 64 or 128");
  if (heads < 1) return fail(KVCR_ESHAPE, "moba_attention_bwd: heads < 1");
  if ((long long)l.L * heads * head_dim > (1LL << 31) - 1)
    return fail(KVCR_ESHAPE, "moba_attention_bwd: tensor too large");
  if (!q || !k || !v || !o || !d_o || !lse || !dq || !dk || !dv || !workspace)
    return fail(KVCR_EINVAL, "moba_attention_bwd: NULL pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(d_o) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(workspace))
    return fail(KVCR_EINVAL, "moba_attention_bwd: tensors and workspace must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(lse) & 3u)
    return fail(KVCR_EINVAL, "moba_attention_bwd: lse must be 4-byte aligned");
  if (workspace_bytes < moba_attention_bwd_workspace_bytes(layout, heads))
    return fail(KVCR_ESTORAGE, "moba_attention_bwd: workspace smaller than "
                               "moba_attention_bwd_workspace_bytes()");
  int n_sm = 0, cc = 0;
  rc = device_sm_count(&n_sm, &cc);
  if (rc) return rc;
  if (cc != 10) return fail(KVCR_EUNSUPPORTED, "moba_attention_bwd: needs an sm_100 GPU");

  const int nt = (l.L + kTile - 1) / kTile;
  static std::mutex mu;
  static MobaLay last{0, 0, 0, 0};
  static std::vector<uint16_t> by_query, by_key;
  MobaBwdParams* p = new MobaBwdParams();
  std::memset(p, 0, sizeof(*p));
  const uint64_t d3[3] = {(uint64_t)head_dim, (uint64_t)heads, (uint64_t)l.L};
  rc = encode_bf16_map(&p->tm_q, q, 3, d3, kTile);
  if (!rc) rc = encode_bf16_map(&p->tm_k, k, 3, d3, kTile);
  if (!rc) rc = encode_bf16_map(&p->tm_v, v, 3, d3, kTile);
  if (!rc) rc = encode_bf16_map(&p->tm_do, d_o, 3, d3, kTile);
  if (rc) {
    delete p;
    return rc;
  }
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt((float)head_dim);
  float* ws = static_cast<float*>(workspace);
  p->ws = ws;
  p->dq = dq;
  p->dk = dk;
  p->dv = dv;
  p->H = heads;
  p->Lpad = nt * kTile;
  p->scale = scale;
  p->scale_log2 = (float)(scale * 1.4426950408889634);
  p->inject = inject_state().kind;
  p->wait_ns = inject_state().wait_ns;
  p->s.n_chunks = l.n;
  p->s.chunk_tokens = l.c;
  p->s.n_bidir = l.m;
  p->s.L = l.L;
  p->s.n_units = nt;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  MobaBwdPrepParams pp{o, d_o, lse, ws, l.L, nt * kTile, heads};
  cudaError_t e;
  {
    LaunchScope scope(KVCR_K_MOBA_BWD_PREP, s);
    e = launch_moba_bwd_prep(pp, head_dim, s);
  }
  if (e == cudaSuccess) {
    std::lock_guard<std::mutex> g(mu);
    if (!(last.n == l.n && last.c == l.c && last.m == l.m)) {
      moba_bwd_orders(l, by_query, by_key);
      last = l;
    }
    for (int i = 0; i < nt; ++i) p->s.order[i] = by_key[i];
    {
      LaunchScope scope(KVCR_K_MOBA_BWD_DKDV, s);
      e = launch_moba_bwd_dkdv_sm100(*p, head_dim, s);
    }
    if (e == cudaSuccess) {
      for (int i = 0; i < nt; ++i) p->s.order[i] = by_query[i];
      LaunchScope scope(KVCR_K_MOBA_BWD_DQ, s);
      e = launch_moba_bwd_dq_sm100(*p, head_dim, s);
    }
  }
  delete p;
  if (e != cudaSuccess) return cuda_fail(e, "moba_attention_bwd: launch");
  return KVCR_OK;
}

// ===================================================================== status
int kvcr_check_status(void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int a = 0, b = 0, c = 0;
  cudaError_t e = read_and_clear_status_attn(&a, s);
  if (e == cudaSuccess) e = read_and_clear_status_f32(&b, s);
  if (e == cudaSuccess) e = read_and_clear_status_bwd(&c, s);
  if (e != cudaSuccess) return cuda_fail(e, "kvcr_check_status");
  if (a != 0 || b != 0 || c != 0) return fail(KVCR_ETIMEOUT, "a kernel gave up on a bounded wait");
  return KVCR_OK;
}

long long kvcr_launch_count(void) { return g_launches.load(); }

int kvcr_debug_inject(int kind, long long wait_ns) {
  if (kind < 0 || kind > 1 || wait_ns < 0) return fail(KVCR_EINVAL, "kvcr_debug_inject: bad argument");
  g_inject_kind.store(kind);
  g_inject_wait_ns.store(wait_ns);
  return KVCR_OK;
}

int kvcr_trace_enable(int on) {
  std::lock_guard<std::mutex> g(g_trace_mu);
  g_trace_on = on != 0;
  return KVCR_OK;
}

int kvcr_trace_reset(void) {
  std::lock_guard<std::mutex> g(g_trace_mu);
  for (auto& r : g_recs) {
    cudaEventSynchronize(r.b);
    g_pool.push_back(r.a);
    g_pool.push_back(r.b);
  }
  g_recs.clear();
  return KVCR_OK;
}

int kvcr_trace_read(int kernel_id, long long* launches, double* total_ms) {
  if (kernel_id < 0 || kernel_id >= KVCR_K_COUNT) return fail(KVCR_EINVAL, "kvcr_trace_read: id");
  std::lock_guard<std::mutex> g(g_trace_mu);
  long long n = 0;
  double ms = 0.0;
  for (auto& r : g_recs) {
    if (r.kid != kernel_id) continue;
    cudaError_t e = cudaEventSynchronize(r.b);
    if (e != cudaSuccess) return cuda_fail(e, "kvcr_trace_read");
    float t = 0.f;
    e = cudaEventElapsedTime(&t, r.a, r.b);
    if (e != cudaSuccess) return cuda_fail(e, "kvcr_trace_read");
    ms += t;
    ++n;
  }
  if (launches) *launches = n;
  if (total_ms) *total_ms = ms;
  return KVCR_OK;
}

}  // extern "C"
