// Block quantization of bf16 Q / K to e4m3 for the low-precision QK^T product.
//
// What it computes (the attention's 8-bit QK^T of kaarelkaarelson.com/lingbot,
// kernel table, "SageAttention" row, here in the tensor cores' e4m3 format):
// for every block of 128 consecutive tokens of a segment and one head,
//   amax  = max |x| over the block (x the bf16 values, exact in fp32),
//   inv   = 448 / amax,  scale = amax / 448        (fp32 divisions, round to nearest),
//   code  = e4m3(x * inv)                          (fp32 product, round to nearest even,
//                                                   saturating at +-448),
// and the block dequantizes to code * scale; amax = 0 gives zero codes and a zero
// scale.  A segment is one tensor [n_tok][H][D] (a cached frame, the chunk's
// rotated queries, the chunk's rotated keys); blocks never cross segments, so
// they are the attention kernel's key and query tiles.
//
// One CTA per (block, head): 256 threads, two per token, each owning 64 (D = 128)
// or 32 (D = 64) contiguous elements; the amax is a warp-shuffle and then a
// shared-memory reduction.  Traffic per block: read 2 * 128 * D bytes, write
// 128 * D bytes of codes and one fp32 scale.
#include <cuda_bf16.h>

#include "kvcr_internal.h"

namespace kvcr {
namespace {

// Two fp32 values to two e4m3 codes: lo goes to the lower byte.
__device__ __forceinline__ uint16_t cvt_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

template <int D>
__global__ void __launch_bounds__(256) quant_e4m3_kernel(const __grid_constant__ QuantParams p) {
  constexpr int kPer = D / 2;            // elements of one thread (half a token's head row)
  constexpr int kVec = kPer / 8;         // 16-byte loads of 8 bf16
  __shared__ float red[8];
  // segment and block of this CTA
  int seg = 0;
  while (seg + 1 < p.n_seg && (int)blockIdx.x >= p.tile0[seg + 1]) ++seg;
  const int blk = blockIdx.x - p.tile0[seg];
  const int h = blockIdx.y;
  const int n_tok = p.n_tok[seg];
  const int tok = blk * 128 + (threadIdx.x >> 1);
  const int half = threadIdx.x & 1;
  const bool live = tok < n_tok;
  const long long off = ((long long)tok * p.H + h) * D + half * kPer;

  uint4 v[kVec];
  float amax = 0.f;
  if (live) {
    const uint4* src = reinterpret_cast<const uint4*>(
        static_cast<const __nv_bfloat16*>(p.src[seg]) + off);
#pragma unroll
    for (int i = 0; i < kVec; ++i) v[i] = src[i];
#pragma unroll
    for (int i = 0; i < kVec; ++i) {
      const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[k]));
        amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
      }
    }
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) amax = fmaxf(amax, red[w]);

  const float inv = amax > 0.f ? __fdiv_rn(448.0f, amax) : 0.f;
  if (threadIdx.x == 0) p.scale[seg][(long long)blk * p.H + h] = __fdiv_rn(amax, 448.0f);
  if (!live) return;
  uint8_t* dst = static_cast<uint8_t*>(p.dst[seg]) + off;
#pragma unroll
  for (int i = 0; i < kVec; i += 2) {          // 16 elements -> one 16-byte store
    uint32_t out[4];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const uint32_t w[4] = {v[i + j].x, v[i + j].y, v[i + j].z, v[i + j].w};
      uint32_t c[2];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[2 * k]));
        const float2 b =
            __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[2 * k + 1]));
        const uint32_t lo = cvt_e4m3x2(__fmul_rn(a.x, inv), __fmul_rn(a.y, inv));
        const uint32_t hi = cvt_e4m3x2(__fmul_rn(b.x, inv), __fmul_rn(b.y, inv));
        c[k] = lo | (hi << 16);
      }
      out[2 * j] = c[0];
      out[2 * j + 1] = c[1];
    }
    *reinterpret_cast<uint4*>(dst + i * 8) = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

}  // namespace

cudaError_t launch_quant_e4m3(const QuantParams& p, int head_dim, cudaStream_t s) {
  if (p.n_seg <= 0) return cudaSuccess;
  const int tiles = p.tile0[p.n_seg - 1] + (p.n_tok[p.n_seg - 1] + 127) / 128;
  if (tiles <= 0) return cudaSuccess;
  const dim3 grid((unsigned)tiles, (unsigned)p.H);
  if (head_dim == 128) quant_e4m3_kernel<128><<<grid, 256, 0, s>>>(p);
  else if (head_dim == 64) quant_e4m3_kernel<64><<<grid, 256, 0, s>>>(p);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace kvcr
