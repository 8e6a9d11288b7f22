// fp32 chunk attention on the CUDA cores (the cache dtype fp32 path).
//
// Same key sequence and the same result as the tensor-core kernel (every
// cached frame in slot order, then the current chunk; O = softmax(scale Q K^T) V,
// LSE = log sum exp), computed with fp32 FMAs and expf so the fp32 workload
// keeps fp32 arithmetic end to end.
//
// Layout: a CTA holds 32 query rows of one head; each row is split over a
// quad of 4 threads (D/4 elements of q and of the output accumulator each);
// the quad's partial dot products are summed with two warp shuffles.  K and V
// tiles of 32 keys are staged in shared memory with 16-byte loads.  Online
// softmax with the running max moved on every tile (fp32 has the range).
#include <math.h>

#include "kvcr_internal.h"

namespace kvcr {

__device__ int g_f32_status = 0;

namespace {

constexpr int kRows = 32;      // query rows per CTA
constexpr int kKeys = 32;      // keys per shared-memory tile
constexpr int kThreads = 128;  // 32 rows x 4 threads

__device__ __forceinline__ const float* key_ptr(const F32AttnParams& p, const float* cached,
                                                const float* cur, int kidx, int h) {
  const int n_cached = p.n_vis * p.T;
  if (kidx < n_cached) {
    const int si = kidx / p.T;
    const int tok = kidx - si * p.T;
    return cached + (((size_t)p.slots[si] * p.T + tok) * p.H + h) * p.D;
  }
  return cur + ((size_t)(kidx - n_cached) * p.H + h) * p.D;
}

template <int D>
__global__ void __launch_bounds__(kThreads) attn_f32_kernel(const __grid_constant__ F32AttnParams p) {
  constexpr int kPer = D / 4;  // elements per thread
  __shared__ __align__(16) float sk[kKeys][D];
  __shared__ __align__(16) float sv[kKeys][D];
  const int h = blockIdx.y;
  const int row = blockIdx.x * kRows + threadIdx.x / 4;
  const int part = threadIdx.x & 3;
  const bool row_ok = row < p.n_q;

  float q[kPer], acc[kPer];
  const float* qrow = p.q + ((size_t)(row_ok ? row : 0) * p.H + h) * D + part * kPer;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    q[i] = row_ok ? qrow[i] : 0.f;
    acc[i] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  const int n_keys = p.n_vis * p.T + p.n_cur;

  for (int k0 = 0; k0 < n_keys; k0 += kKeys) {
    __syncthreads();
    // stage up to 32 keys: kKeys * D / 4 float4 per tensor
    for (int i = threadIdx.x; i < kKeys * D / 4; i += kThreads) {
      const int key = i / (D / 4);
      const int c4 = i - key * (D / 4);
      float4 kv = make_float4(0.f, 0.f, 0.f, 0.f), vv = kv;
      if (k0 + key < n_keys) {
        kv = reinterpret_cast<const float4*>(key_ptr(p, p.kc, p.kn, k0 + key, h))[c4];
        vv = reinterpret_cast<const float4*>(key_ptr(p, p.vc, p.vn, k0 + key, h))[c4];
      }
      reinterpret_cast<float4*>(&sk[key][0])[c4] = kv;
      reinterpret_cast<float4*>(&sv[key][0])[c4] = vv;
    }
    __syncthreads();
    const int nk = min(kKeys, n_keys - k0);
    float sc[kKeys];
    float mt = -INFINITY;
#pragma unroll
    for (int j = 0; j < kKeys; ++j) {
      float d = 0.f;
#pragma unroll
      for (int i = 0; i < kPer; ++i) d = fmaf(q[i], sk[j][part * kPer + i], d);
      d += __shfl_xor_sync(0xFFFFFFFFu, d, 1);
      d += __shfl_xor_sync(0xFFFFFFFFu, d, 2);
      sc[j] = j < nk ? d * p.scale : -INFINITY;
      mt = fmaxf(mt, sc[j]);
    }
    const float m_new = fmaxf(m, mt);
    const float alpha = (m == -INFINITY) ? 0.f : expf(m - m_new);
    l *= alpha;
#pragma unroll
    for (int i = 0; i < kPer; ++i) acc[i] *= alpha;
#pragma unroll
    for (int j = 0; j < kKeys; ++j) {
      const float pj = (sc[j] == -INFINITY) ? 0.f : expf(sc[j] - m_new);
      l += pj;
#pragma unroll
      for (int i = 0; i < kPer; ++i) acc[i] = fmaf(pj, sv[j][part * kPer + i], acc[i]);
    }
    m = m_new;
  }
  if (row_ok) {
    const float inv = l > 0.f ? 1.f / l : 0.f;
    float* orow = p.o + ((size_t)row * p.H + h) * D + part * kPer;
#pragma unroll
    for (int i = 0; i < kPer; ++i) orow[i] = acc[i] * inv;
    if (p.lse != nullptr && part == 0) p.lse[(size_t)h * p.n_q + row] = l > 0.f ? m + logf(l) : -INFINITY;
  }
}

}  // namespace

cudaError_t launch_attn_f32(const F32AttnParams& p, cudaStream_t s) {
  dim3 grid((unsigned)((p.n_q + kRows - 1) / kRows), (unsigned)p.H);
  if (p.D == 128) attn_f32_kernel<128><<<grid, kThreads, 0, s>>>(p);
  else if (p.D == 64) attn_f32_kernel<64><<<grid, kThreads, 0, s>>>(p);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t read_and_clear_status_f32(int* st, cudaStream_t s) {
  int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(st, g_f32_status, sizeof(int), 0,
                                            cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return e;
  e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return e;
  if (*st != 0) e = cudaMemcpyToSymbol(g_f32_status, &zero, sizeof(int));
  return e;
}

}  // namespace kvcr
