// Row-wise kernels of the model step around the Flash-Cache layer: RMSNorm
// (LLaMA-style pre-norm of the LLaDA decoder layer; optionally gathering the
// rows the LM head scores) and the merge of the LM head's per-tile softmax
// statistics into each row's top token, its confidence and the Flash-Verify
// acceptance (confidence >= threshold; paper-digest page, Flash-Verify).
#include <cuda_bf16.h>

#include "fc_internal.h"
#include "ptx.cuh"

namespace fc {
namespace {

constexpr int NORM_THREADS = 256;

// y[i] = x[r] / sqrt(mean(x[r]^2) + eps) * g with r = rows ? rows[i] : i; one
// CTA per output row, fp32 arithmetic, bf16 in and out.  D % 8 == 0.
__global__ void __launch_bounds__(NORM_THREADS) rmsnorm_kernel(
    const __nv_bfloat16* __restrict__ x, const int32_t* __restrict__ rows, int D,
    const __nv_bfloat16* __restrict__ g, float eps, __nv_bfloat16* __restrict__ y) {
  ptx::griddep_launch_dependents();
  ptx::griddep_wait();
  const int i = blockIdx.x;
  const int r = rows ? rows[i] : i;
  const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)r * D);
  const uint4* gr = reinterpret_cast<const uint4*>(g);
  uint4* yr = reinterpret_cast<uint4*>(y + (size_t)i * D);
  const int n8 = D / 8;
  float ss = 0.f;
  for (int c = threadIdx.x; c < n8; c += NORM_THREADS) {
    const uint4 v = xr[c];
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(p[e]);
      ss += f.x * f.x + f.y * f.y;
    }
  }
  __shared__ float red[NORM_THREADS / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < NORM_THREADS / 32; ++w) tot += red[w];
  const float inv = rsqrtf(tot / (float)D + eps);
  for (int c = threadIdx.x; c < n8; c += NORM_THREADS) {
    const uint4 v = xr[c], gv = gr[c];
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
    const __nv_bfloat162* q = reinterpret_cast<const __nv_bfloat162*>(&gv);
    uint4 o;
    uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(p[e]), w = __bfloat1622float2(q[e]);
      const __nv_bfloat162 b = __floats2bfloat162_rn(f.x * inv * w.x, f.y * inv * w.y);
      ow[e] = *reinterpret_cast<const uint32_t*>(&b);
    }
    yr[c] = o;
  }
}

// One warp per row: merge (max, sum exp(x - max), argmax) over the row's
// column tiles.  Equal maxima keep the lowest tile, i.e. the lowest column.
__global__ void __launch_bounds__(256) lmhead_reduce_kernel(
    const float* __restrict__ partials, int R, int num_n, float threshold,
    int32_t* __restrict__ token, float* __restrict__ confidence, uint8_t* __restrict__ accept) {
  ptx::griddep_launch_dependents();
  ptx::griddep_wait();
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= R) return;
  const float* pr = partials + (size_t)row * num_n * 3;
  float mx = -INFINITY;
  int arg = 0x7fffffff;
  for (int t = lane; t < num_n; t += 32) {
    const float m = pr[3 * t];
    if (m > mx) {  // tiles visited in increasing order: the first maximum stays
      mx = m;
      arg = __float_as_int(pr[3 * t + 2]);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float om = __shfl_xor_sync(0xffffffffu, mx, o);
    const int oa = __shfl_xor_sync(0xffffffffu, arg, o);
    if (om > mx || (om == mx && oa < arg)) {
      mx = om;
      arg = oa;
    }
  }
  float s = 0.f;
  for (int t = lane; t < num_n; t += 32) s += pr[3 * t + 1] * __expf(pr[3 * t] - mx);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) {
    const float conf = 1.f / s;
    token[row] = arg;
    confidence[row] = conf;
    accept[row] = conf >= threshold ? 1 : 0;
  }
}

}  // namespace

cudaError_t launch_rmsnorm(cudaStream_t st, const __nv_bfloat16* x, const int32_t* rows, int n_rows,
                           int D, const __nv_bfloat16* g, float eps, __nv_bfloat16* y) {
  if (n_rows <= 0) return cudaSuccess;
  return launch_pdl(rmsnorm_kernel, dim3(n_rows), dim3(NORM_THREADS), 0, st, x, rows, D, g, eps, y);
}

cudaError_t launch_lmhead_reduce(cudaStream_t st, const float* partials, int R, int num_n,
                                 float threshold, int32_t* token, float* confidence,
                                 uint8_t* accept) {
  if (R <= 0) return cudaSuccess;
  return launch_pdl(lmhead_reduce_kernel, dim3((R + 7) / 8), dim3(256), 0, st, partials, R, num_n,
                    threshold, token, confidence, accept);
}

}  // namespace fc
