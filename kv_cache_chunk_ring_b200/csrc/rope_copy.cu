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
// Layout: one thread owns one 16-byte vector of a and the matching vector of
// b (8 bf16 = 4 pairs, or 4 fp32 = 2 pairs), so loads and stores are
// coalesced 16-byte accesses; a grid-stride loop over (frame, token, head,
// vector) keeps the grid at a multiple of the SM count.
#include <cuda_bf16.h>

#include "kvcr_internal.h"

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

// (cos, sin) of pair i for a token at (frame slot fr, row hh, col ww)
__device__ __forceinline__ float2 angle_cs(const RopeCopyParams& p, int fr, int hh, int ww, int i) {
  if (i < p.pairs_t) return p.ttab[fr][i];
  i -= p.pairs_t;
  if (i < p.pairs_h) return p.htab[hh * p.pairs_h + i];
  i -= p.pairs_h;
  return p.wtab[ww * p.pairs_w + i];
}

__device__ __forceinline__ void rot(float& x0, float& x1, float2 cs) {
  const float y0 = x0 * cs.x - x1 * cs.y;
  const float y1 = x0 * cs.y + x1 * cs.x;
  x0 = y0;
  x1 = y1;
}

__device__ __forceinline__ uint4 rotate_bf16x8(uint4 v, const RopeCopyParams& p, int fr, int hh,
                                               int ww, int pair0) {
  uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    __nv_bfloat162 b2 = *reinterpret_cast<__nv_bfloat162*>(&w[k]);
    float2 f = __bfloat1622float2(b2);
    rot(f.x, f.y, angle_cs(p, fr, hh, ww, pair0 + k));
    b2 = __floats2bfloat162_rn(f.x, f.y);
    w[k] = *reinterpret_cast<uint32_t*>(&b2);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ uint4 rotate_f32x4(uint4 v, const RopeCopyParams& p, int fr, int hh,
                                              int ww, int pair0) {
  float f[4] = {__uint_as_float(v.x), __uint_as_float(v.y), __uint_as_float(v.z),
                __uint_as_float(v.w)};
  rot(f[0], f[1], angle_cs(p, fr, hh, ww, pair0));
  rot(f[2], f[3], angle_cs(p, fr, hh, ww, pair0 + 1));
  return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                    __float_as_uint(f[3]));
}

template <typename Elem, int D>
__global__ void __launch_bounds__(256) rope_copy_kernel(const __grid_constant__ RopeCopyParams p) {
  constexpr int kPerVec = 16 / sizeof(Elem);          // elements per 16-byte vector
  constexpr int kPairsPerVec = kPerVec / 2;
  constexpr int kVecPerRow = D / kPerVec;             // vectors per (token, head)
  const int f = blockIdx.y;                           // destination frame
  const unsigned vec_per_frame = (unsigned)p.T * p.H * kVecPerRow;
  const long long in_base = (long long)p.src_frame[f] * p.T * p.H * D;
  const long long out_base = p.dst_frame_off[f];
  const Elem* src_a = static_cast<const Elem*>(p.src_a) + in_base;
  const Elem* src_b = static_cast<const Elem*>(p.src_b) + in_base;
  Elem* dst_a = static_cast<Elem*>(p.dst_a) + out_base;
  Elem* dst_b = static_cast<Elem*>(p.dst_b) + out_base;
  for (unsigned r = blockIdx.x * blockDim.x + threadIdx.x; r < vec_per_frame;
       r += gridDim.x * blockDim.x) {
    const unsigned row = r / kVecPerRow;              // token * H + head
    const int vi = (int)(r - row * kVecPerRow);
    const int tok = (int)(row / (unsigned)p.H);
    const int hh = tok / p.grid_w;
    const int ww = tok - hh * p.grid_w;
    const int pair0 = vi * kPairsPerVec;
    uint4 a = ld_stream(src_a + (size_t)r * kPerVec);
    uint4 b = ld_stream(src_b + (size_t)r * kPerVec);
    if constexpr (sizeof(Elem) == 2) {
      if (p.rotate_a) a = rotate_bf16x8(a, p, f, hh, ww, pair0);
      if (p.rotate_b) b = rotate_bf16x8(b, p, f, hh, ww, pair0);
    } else {
      if (p.rotate_a) a = rotate_f32x4(a, p, f, hh, ww, pair0);
      if (p.rotate_b) b = rotate_f32x4(b, p, f, hh, ww, pair0);
    }
    st_vec(dst_a + (size_t)r * kPerVec, a);
    st_vec(dst_b + (size_t)r * kPerVec, b);
  }
}

}  // namespace

cudaError_t launch_rope_copy(const RopeCopyParams& p, kvcr_dtype dtype, cudaStream_t s, int n_sm) {
  if (p.n_frames <= 0) return cudaSuccess;
  const int per_vec = dtype == KVCR_BF16 ? 8 : 4;
  const long long per_frame = (long long)p.T * p.H * (p.D / per_vec);
  if (per_frame == 0) return cudaSuccess;
  // About 8 resident 256-thread CTAs per SM in total, split over the frames.
  long long want = (per_frame + 255) / 256;
  long long gx = ((long long)n_sm * 8 + p.n_frames - 1) / p.n_frames;
  if (want < gx) gx = want;
  dim3 grid((unsigned)gx, (unsigned)p.n_frames);
  if (dtype == KVCR_BF16) {
    if (p.D == 128) rope_copy_kernel<__nv_bfloat16, 128><<<grid, 256, 0, s>>>(p);
    else rope_copy_kernel<__nv_bfloat16, 64><<<grid, 256, 0, s>>>(p);
  } else {
    if (p.D == 128) rope_copy_kernel<float, 128><<<grid, 256, 0, s>>>(p);
    else rope_copy_kernel<float, 64><<<grid, 256, 0, s>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace kvcr
