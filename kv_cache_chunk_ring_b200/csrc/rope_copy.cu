// Cache write and query staging: 3D rotary embedding fused into a streaming copy.
//
// What it computes: each destination frame f receives the tokens of source
// frame src_frame[f]; tensor a (K, or Q when staging) is rotated pair by pair
// with the 3D (t, h, w) RoPE at the frame's absolute index t and each token's
// patch row / column, tensor b (V, or the current K when staging) is copied or
// rotated.  The rotation of pair i is (x0 c - x1 s, x0 s + x1 c) with (c, s)
// from host-computed double-precision angle tables; arithmetic is fp32, the
// result is rounded once to the storage dtype.  (RoPE is named among the fused
// elementwise kernels of kaarelkaarelson.com/lingbot, step table, "Kernel
// fusion" row; the split and base come from the 832x464 workload statement.)
//
// Roofline: HBM-bound streaming pass.  Algorithmic bytes per frame =
// 2 tensors x (read + write) x T x H x D x sizeof(elem); the angle tables are
// a few KB and stay in L1/L2.
//
// Layout: a warp moves one token (all heads) at a time with coalesced 16-byte
// loads and stores, several vectors in flight per lane; a lane's vectors all
// cover the same rotary pairs, so their (cos, sin) are fetched once per token.
// The grid is one wave of resident CTAs (a multiple of the SM count).
#include <cuda_bf16.h>

#include "kvcr_internal.h"
#include "rope_batch.h"

namespace kvcr {
namespace {

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void st_vec(void* p, uint4 v) {
  asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

__device__ __forceinline__ void rot(float& x0, float& x1, float2 cs) {
  const float y0 = x0 * cs.x - x1 * cs.y;
  const float y1 = x0 * cs.y + x1 * cs.x;
  x0 = y0;
  x1 = y1;
}

template <int kPairs>
__device__ __forceinline__ uint4 rotate_vec(uint4 v, const float2 (&cs)[4]);

// 8 bf16 = 4 pairs
template <>
__device__ __forceinline__ uint4 rotate_vec<4>(uint4 v, const float2 (&cs)[4]) {
  uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    __nv_bfloat162 b2 = *reinterpret_cast<__nv_bfloat162*>(&w[k]);
    float2 f = __bfloat1622float2(b2);
    rot(f.x, f.y, cs[k]);
    b2 = __floats2bfloat162_rn(f.x, f.y);
    w[k] = *reinterpret_cast<uint32_t*>(&b2);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// 4 fp32 = 2 pairs
template <>
__device__ __forceinline__ uint4 rotate_vec<2>(uint4 v, const float2 (&cs)[4]) {
  float f[4] = {__uint_as_float(v.x), __uint_as_float(v.y), __uint_as_float(v.z),
                __uint_as_float(v.w)};
  rot(f[0], f[1], cs[0]);
  rot(f[2], f[3], cs[1]);
  return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                    __float_as_uint(f[3]));
}

// One warp moves one token (H x D elements of a and of b) at a time.  A token
// is H * D / kPerVec 16-byte vectors; lane l takes vectors l, l + 32, ..., and
// because D / kPerVec divides 32, every vector of a lane covers the same
// kPairsPerVec rotary pairs: the lane fetches their (cos, sin) once per token
// (t-axis pairs once per frame) and reuses them for every head.  `ttab` is the
// frame's row of t-axis (cos, sin); `cta`, `n_cta` split the frame's tokens.
template <typename Elem, int D>
__device__ __forceinline__ void copy_frame(const Elem* src_a, const Elem* src_b, Elem* dst_a,
                                           Elem* dst_b, const float2* ttab, int T, int H,
                                           int grid_w, int pairs_t, int pairs_h, int pairs_w,
                                           const float2* htab, const float2* wtab, int rotate_a,
                                           int rotate_b, int cta, int n_cta) {
  constexpr int kPerVec = 16 / sizeof(Elem);          // elements per 16-byte vector
  constexpr int kPairsPerVec = kPerVec / 2;
  constexpr int kVecPerRow = D / kPerVec;             // vectors per (token, head)
  constexpr int kBatch = 6;                           // vectors in flight per lane and tensor
  const int lane = threadIdx.x & 31;
  const int vpt = H * kVecPerRow;                     // vectors per token
  const int n_mine = (vpt - lane + 31) / 32;          // vectors of this lane per token
  const int pair0 = (lane % kVecPerRow) * kPairsPerVec;
  const long long tok_elems = (long long)H * D;

  // axis and index of this lane's pairs; t-axis (cos, sin) are per frame
  int axis[4], jx[4];
  float2 cs_t[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    int i = pair0 + k;
    axis[k] = i < pairs_t ? 0 : (i < pairs_t + pairs_h ? 1 : 2);
    jx[k] = axis[k] == 0 ? i : (axis[k] == 1 ? i - pairs_t : i - pairs_t - pairs_h);
    cs_t[k] = (k < kPairsPerVec && axis[k] == 0 && (rotate_a || rotate_b))
                  ? ttab[jx[k] < kMaxPairsT ? jx[k] : 0]
                  : make_float2(1.f, 0.f);
  }
  const int warps_total = n_cta * (blockDim.x / 32);
  for (int tok = cta * (blockDim.x / 32) + (threadIdx.x >> 5); tok < T; tok += warps_total) {
    float2 cs[4];
    if (rotate_a || rotate_b) {
      const int hh = tok / grid_w;
      const int ww = tok - hh * grid_w;
#pragma unroll
      for (int k = 0; k < kPairsPerVec; ++k) {
        if (axis[k] == 0) cs[k] = cs_t[k];
        else if (axis[k] == 1) cs[k] = htab[hh * pairs_h + jx[k]];
        else cs[k] = wtab[ww * pairs_w + jx[k]];
      }
    }
    const long long base = (long long)tok * tok_elems;
    for (int k0 = 0; k0 < n_mine; k0 += kBatch) {
      uint4 a[kBatch], b[kBatch];
#pragma unroll
      for (int k = 0; k < kBatch; ++k) {
        if (k0 + k < n_mine) {
          const long long off = base + (long long)(lane + 32 * (k0 + k)) * kPerVec;
          a[k] = ld_stream(src_a + off);
          b[k] = ld_stream(src_b + off);
        }
      }
#pragma unroll
      for (int k = 0; k < kBatch; ++k) {
        if (k0 + k < n_mine) {
          const long long off = base + (long long)(lane + 32 * (k0 + k)) * kPerVec;
          uint4 ra = a[k], rb = b[k];
          if (rotate_a) ra = rotate_vec<kPairsPerVec>(ra, cs);
          if (rotate_b) rb = rotate_vec<kPairsPerVec>(rb, cs);
          st_vec(dst_a + off, ra);
          st_vec(dst_b + off, rb);
        }
      }
    }
  }
}

// The single-cache kernel keeps its own copy of the loop: reading the frame's
// parameters straight from the kernel parameters measured ~5 % faster than
// passing them to copy_frame().
template <typename Elem, int D>
__global__ void __launch_bounds__(256) rope_copy_kernel(const __grid_constant__ RopeCopyParams p) {
  constexpr int kPerVec = 16 / sizeof(Elem);          // elements per 16-byte vector
  constexpr int kPairsPerVec = kPerVec / 2;
  constexpr int kVecPerRow = D / kPerVec;             // vectors per (token, head)
  constexpr int kBatch = 6;                           // vectors in flight per lane and tensor
  const int f = blockIdx.y;                           // destination frame
  const int lane = threadIdx.x & 31;
  const int vpt = p.H * kVecPerRow;                   // vectors per token
  const int n_mine = (vpt - lane + 31) / 32;          // vectors of this lane per token
  const int pair0 = (lane % kVecPerRow) * kPairsPerVec;
  const long long tok_elems = (long long)p.H * D;
  const Elem* src_a = static_cast<const Elem*>(p.src_a) + (long long)p.src_frame[f] * p.T * tok_elems;
  const bool has_b = p.src_b != nullptr;             // tensor b is optional
  const Elem* src_b = static_cast<const Elem*>(p.src_b) + (long long)p.src_frame[f] * p.T * tok_elems;
  Elem* dst_a = static_cast<Elem*>(p.dst_a) + p.dst_frame_off[f];
  Elem* dst_b = static_cast<Elem*>(p.dst_b) + p.dst_frame_off[f];

  // axis and index of this lane's pairs; t-axis (cos, sin) are per frame
  int axis[4], jx[4];
  float2 cs_t[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    int i = pair0 + k;
    axis[k] = i < p.pairs_t ? 0 : (i < p.pairs_t + p.pairs_h ? 1 : 2);
    jx[k] = axis[k] == 0 ? i : (axis[k] == 1 ? i - p.pairs_t : i - p.pairs_t - p.pairs_h);
    cs_t[k] = (k < kPairsPerVec && axis[k] == 0 && (p.rotate_a || p.rotate_b))
                  ? p.ttab[f][jx[k] < kMaxPairsT ? jx[k] : 0]
                  : make_float2(1.f, 0.f);
  }
  const int warps_total = gridDim.x * (blockDim.x / 32);
  for (int tok = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5); tok < p.T;
       tok += warps_total) {
    float2 cs[4];
    if (p.rotate_a || p.rotate_b) {
      const int hh = tok / p.grid_w;
      const int ww = tok - hh * p.grid_w;
#pragma unroll
      for (int k = 0; k < kPairsPerVec; ++k) {
        if (axis[k] == 0) cs[k] = cs_t[k];
        else if (axis[k] == 1) cs[k] = p.htab[hh * p.pairs_h + jx[k]];
        else cs[k] = p.wtab[ww * p.pairs_w + jx[k]];
      }
    }
    const long long base = (long long)tok * tok_elems;
    for (int k0 = 0; k0 < n_mine; k0 += kBatch) {
      uint4 a[kBatch], b[kBatch];
#pragma unroll
      for (int k = 0; k < kBatch; ++k) {
        if (k0 + k < n_mine) {
          const long long off = base + (long long)(lane + 32 * (k0 + k)) * kPerVec;
          a[k] = ld_stream(src_a + off);
          if (has_b) b[k] = ld_stream(src_b + off);
        }
      }
#pragma unroll
      for (int k = 0; k < kBatch; ++k) {
        if (k0 + k < n_mine) {
          const long long off = base + (long long)(lane + 32 * (k0 + k)) * kPerVec;
          uint4 ra = a[k];
          if (p.rotate_a) ra = rotate_vec<kPairsPerVec>(ra, cs);
          st_vec(dst_a + off, ra);
          if (has_b) {
            uint4 rb = b[k];
            if (p.rotate_b) rb = rotate_vec<kPairsPerVec>(rb, cs);
            st_vec(dst_b + off, rb);
          }
        }
      }
    }
  }
}


// Several caches at once: blockIdx.y = one (cache, frame) pair of the batch.
template <typename Elem, int D>
__global__ void __launch_bounds__(256)
    rope_copy_batch_kernel(const __grid_constant__ RopeCopyBatchParams p) {
  const int i = blockIdx.y;
  copy_frame<Elem, D>(static_cast<const Elem*>(p.src_a[i]), static_cast<const Elem*>(p.src_b[i]),
                      static_cast<Elem*>(p.dst_a[i]), static_cast<Elem*>(p.dst_b[i]),
                      p.ttab[p.tframe[i]], p.T, p.H, p.grid_w, p.pairs_t, p.pairs_h, p.pairs_w,
                      p.htab, p.wtab, p.rotate_a, 0, blockIdx.x, gridDim.x);
}

}  // namespace

namespace {
template <typename Elem, int D>
cudaError_t launch_one(const RopeCopyParams& p, cudaStream_t s, int n_sm) {
  static int per_sm = 0;  // resident CTAs per SM, from the occupancy calculator
  if (per_sm == 0) {
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, rope_copy_kernel<Elem, D>,
                                                                  256, 0);
    if (e != cudaSuccess || per_sm < 1) per_sm = 1;
  }
  // One wave: every resident CTA slot busy, split evenly over the frames; each
  // of a CTA's 8 warps takes one token at a time.
  const long long want = (p.T + 7) / 8;
  long long gx = ((long long)n_sm * per_sm + p.n_frames - 1) / p.n_frames;
  if (want < gx) gx = want;
  if (gx < 1) gx = 1;
  rope_copy_kernel<Elem, D><<<dim3((unsigned)gx, (unsigned)p.n_frames), 256, 0, s>>>(p);
  return cudaGetLastError();
}

template <typename Elem, int D>
cudaError_t launch_batch(const RopeCopyBatchParams& p, cudaStream_t s, int n_sm) {
  static int per_sm = 0;
  if (per_sm == 0) {
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
        &per_sm, rope_copy_batch_kernel<Elem, D>, 256, 0);
    if (e != cudaSuccess || per_sm < 1) per_sm = 1;
  }
  const long long want = (p.T + 7) / 8;
  long long gx = ((long long)n_sm * per_sm + p.n - 1) / p.n;
  if (want < gx) gx = want;
  if (gx < 1) gx = 1;
  rope_copy_batch_kernel<Elem, D><<<dim3((unsigned)gx, (unsigned)p.n), 256, 0, s>>>(p);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_rope_copy_batch(const RopeCopyBatchParams& p, kvcr_dtype dtype, cudaStream_t s,
                                   int n_sm) {
  if (p.n <= 0 || p.T <= 0) return cudaSuccess;
  if (dtype == KVCR_BF16)
    return p.D == 128 ? launch_batch<__nv_bfloat16, 128>(p, s, n_sm)
                      : launch_batch<__nv_bfloat16, 64>(p, s, n_sm);
  return p.D == 128 ? launch_batch<float, 128>(p, s, n_sm) : launch_batch<float, 64>(p, s, n_sm);
}

cudaError_t launch_rope_copy(const RopeCopyParams& p, kvcr_dtype dtype, cudaStream_t s, int n_sm) {
  if (p.n_frames <= 0 || p.T <= 0) return cudaSuccess;
  if (dtype == KVCR_BF16)
    return p.D == 128 ? launch_one<__nv_bfloat16, 128>(p, s, n_sm)
                      : launch_one<__nv_bfloat16, 64>(p, s, n_sm);
  return p.D == 128 ? launch_one<float, 128>(p, s, n_sm) : launch_one<float, 64>(p, s, n_sm);
}

}  // namespace kvcr
