// CUDA-core (SIMT) path of the Flash-Cache step, fp32 arithmetic throughout.
//
// It serves the fp32 configuration (tensor-core tf32 cannot meet a 1e-5
// relative tolerance) and any bf16 shape outside the tensor-core path
// (head_dim != 128, hidden not a multiple of 64).  It computes exactly what the
// tensor-core path computes:
//   qkv_rope_scatter_simt: [q|k|v] = W_qkv x, RoPE on q and k at the row's
//     position, q (scaled by log2(e)/sqrt(d)) to the Q buffer, k and v rounded
//     into the cache at cu_seqlens_k[b] + q_pos[r];
//   attn_simt: two passes over the sequence's cache per (sequence, head,
//     query tile): pass 1 finds each row's max and normaliser, pass 2 forms the
//     final probabilities, accumulates P V and adds the column sums of P to the
//     fixed-point importance accumulator.
// (Flash-dLLM: infernews post "Flash-dLLM: IO-aware KV caching and parallel
// decoding", Flash-Cache paragraph; paper-digest page, Fig. 2 caption.)
#include <cuda_bf16.h>

#include "fc_internal.h"

namespace fc {
namespace {

template <typename T>
__device__ __forceinline__ float to_f(T v);
template <>
__device__ __forceinline__ float to_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T>
__device__ __forceinline__ T from_f(float v);
template <>
__device__ __forceinline__ float from_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// ---------------------------------------------------------------------------
// QKV projection over "pair columns": pair p = (head slot hs, i < d/2) owns the
// output columns hs*d + i and hs*d + i + d/2, so one thread holds both halves
// of a RoPE rotation.  Head slots 0..H-1 are Q heads, H..2H-1 K, 2H..3H-1 V.
constexpr int GM = 64, GP = 32, GK = 16;

template <typename T>
__global__ void __launch_bounds__(256) qkv_rope_scatter_simt(
    StepShape s, const T* __restrict__ x, const T* __restrict__ w,
    const int32_t* __restrict__ q_pos, const int32_t* __restrict__ row_dst,
    const float* __restrict__ rcos, const float* __restrict__ rsin, T* __restrict__ q_buf,
    T* __restrict__ k_cache, T* __restrict__ v_cache, float q_scale) {
  __shared__ float xs[GK][GM + 1];
  __shared__ float wsm[GK][2 * GP + 1];
  const int tid = threadIdx.x;
  const int half = s.d / 2;
  const int P = 3 * s.H * half;
  const int r0 = blockIdx.x * GM, p0 = blockIdx.y * GP;
  const int ty = tid / 16, tx = tid % 16;

  float acc[4][2][2];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 2; ++b) acc[a][b][0] = acc[a][b][1] = 0.f;

  for (int k0 = 0; k0 < s.D; k0 += GK) {
    for (int e = tid; e < GM * GK; e += 256) {
      int rr = e / GK, kk = e % GK;
      int r = r0 + rr, k = k0 + kk;
      xs[kk][rr] = (r < s.T && k < s.D) ? to_f(x[(size_t)r * s.D + k]) : 0.f;
    }
    for (int e = tid; e < 2 * GP * GK; e += 256) {
      int c = e / GK, kk = e % GK;
      int p = p0 + (c % GP), hi = c / GP, k = k0 + kk;
      float v = 0.f;
      if (p < P && k < s.D) {
        int hs = p / half, i = p % half;
        size_t wrow = (size_t)hs * s.d + i + hi * half;
        v = to_f(w[wrow * s.D + k]);
      }
      wsm[kk][c] = v;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < GK; ++kk) {
      float xv[4], wv[2][2];
#pragma unroll
      for (int a = 0; a < 4; ++a) xv[a] = xs[kk][ty * 4 + a];
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        wv[b][0] = wsm[kk][tx * 2 + b];
        wv[b][1] = wsm[kk][GP + tx * 2 + b];
      }
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          acc[a][b][0] = fmaf(xv[a], wv[b][0], acc[a][b][0]);
          acc[a][b][1] = fmaf(xv[a], wv[b][1], acc[a][b][1]);
        }
    }
    __syncthreads();
  }

#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int r = r0 + ty * 4 + a;
    if (r >= s.T) continue;
    const int dst = row_dst[r];
    const bool valid = dst >= 0 && dst < s.S;
    const int pos = valid ? q_pos[r] : 0;
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      const int p = p0 + tx * 2 + b;
      if (p >= P) continue;
      const int hs = p / half, i = p % half;
      const int region = hs / s.H, hh = hs % s.H;
      float u0 = acc[a][b][0], u1 = acc[a][b][1];
      if (region < 2) {
        const float c = rcos[(size_t)pos * half + i], sn = rsin[(size_t)pos * half + i];
        const float v0 = u0 * c - u1 * sn;
        const float v1 = u1 * c + u0 * sn;
        u0 = v0;
        u1 = v1;
      }
      if (region == 0) {
        T* qrow = q_buf + ((size_t)r * s.H + hh) * s.d;
        qrow[i] = from_f<T>(valid ? u0 * q_scale : 0.f);
        qrow[i + half] = from_f<T>(valid ? u1 * q_scale : 0.f);
      } else if (valid) {
        T* dstp = (region == 1 ? k_cache : v_cache) + ((size_t)dst * s.H + hh) * s.d;
        dstp[i] = from_f<T>(u0);
        dstp[i + half] = from_f<T>(u1);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Attention: one CTA of 4 warps per work item (sequence, head, 16-row query
// tile); each warp owns 4 query rows; keys stream through shared memory in
// tiles of 32.  Scores are in the log2 domain (q was pre-scaled by
// log2(e)/sqrt(d)), so p = exp2(s - m) / l.
constexpr int AK = 32;        // keys per tile
constexpr int AMAXD = 256;    // largest head_dim
constexpr int AROWS = kSimtQTile;

template <typename T>
__global__ void __launch_bounds__(128) attn_simt(
    StepShape s, const WorkItem* __restrict__ items, int32_t* __restrict__ sched,
    const int32_t* __restrict__ cu_q, const int32_t* __restrict__ cu_k,
    const T* __restrict__ q_buf, const T* __restrict__ k_cache, const T* __restrict__ v_cache,
    T* __restrict__ out, unsigned long long* __restrict__ imp_acc, int want_imp) {
  extern __shared__ float sm[];
  const int d = s.d;
  float* qs = sm;                    // [AROWS][d]
  float* ks = qs + AROWS * d;        // [AK][d + 1]
  float* vs = ks + AK * (d + 1);     // [AK][d]
  float* cs = vs + AK * d;           // [4][AK]
  __shared__ int item_sh;

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int n_items = sched[0];
  const int ndl = (d + 31) / 32;  // dims per lane

  for (;;) {
    if (tid == 0) item_sh = atomicAdd(&sched[1], 1);
    __syncthreads();
    const int it = item_sh;
    __syncthreads();
    if (it >= n_items) break;
    const WorkItem wi = items[it];
    const int b = wi.seq, qt = wi.tile_head >> 8, hh = wi.tile_head & 0xFF;
    const int q0 = cu_q[b], n = cu_q[b + 1] - q0, k0 = cu_k[b], L = cu_k[b + 1] - k0;
    const int rbeg = qt * AROWS;
    const int nrows = min(AROWS, n - rbeg);

    for (int e = tid; e < AROWS * d; e += 128) {
      int rr = e / d, c = e % d;
      qs[e] = rr < nrows ? to_f(q_buf[((size_t)(q0 + rbeg + rr) * s.H + hh) * d + c]) : 0.f;
    }

    float m[4], l[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      m[a] = -INFINITY;
      l[a] = 0.f;
    }
    // ---- pass 1: row max and normaliser (online)
    for (int kt = 0; kt < L; kt += AK) {
      __syncthreads();
      for (int e = tid; e < AK * d; e += 128) {
        int j = e / d, c = e % d;
        ks[j * (d + 1) + c] =
            (kt + j < L) ? to_f(k_cache[((size_t)(k0 + kt + j) * s.H + hh) * d + c]) : 0.f;
      }
      __syncthreads();
      const bool kvalid = kt + lane < L;
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const int rr = warp * 4 + a;
        float sc = 0.f;
        for (int c = 0; c < d; ++c) sc = fmaf(qs[rr * d + c], ks[lane * (d + 1) + c], sc);
        sc = kvalid ? sc : -INFINITY;
        float tmax = sc;
        for (int o = 16; o; o >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
        const float mn = fmaxf(m[a], tmax);
        float e = kvalid ? exp2f(sc - mn) : 0.f;
        for (int o = 16; o; o >>= 1) e += __shfl_xor_sync(0xffffffffu, e, o);
        l[a] = l[a] * exp2f(m[a] - mn) + e;
        m[a] = mn;
      }
    }
    float inv_l[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) inv_l[a] = 1.f / l[a];

    // ---- pass 2: final probabilities, P V and column sums
    float o[4][AMAXD / 32];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int t = 0; t < AMAXD / 32; ++t) o[a][t] = 0.f;
    for (int kt = 0; kt < L; kt += AK) {
      __syncthreads();
      for (int e = tid; e < AK * d; e += 128) {
        int j = e / d, c = e % d;
        bool kv = kt + j < L;
        size_t g = ((size_t)(k0 + kt + j) * s.H + hh) * d + c;
        ks[j * (d + 1) + c] = kv ? to_f(k_cache[g]) : 0.f;
        vs[j * d + c] = kv ? to_f(v_cache[g]) : 0.f;
      }
      __syncthreads();
      const bool kvalid = kt + lane < L;
      float colsum = 0.f;
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const int rr = warp * 4 + a;
        float sc = 0.f;
        for (int c = 0; c < d; ++c) sc = fmaf(qs[rr * d + c], ks[lane * (d + 1) + c], sc);
        const bool live = kvalid && rr < nrows;
        const float p = live ? exp2f(sc - m[a]) * inv_l[a] : 0.f;
        colsum += p;
        for (int j = 0; j < AK; ++j) {
          const float pj = __shfl_sync(0xffffffffu, p, j);
#pragma unroll
          for (int t = 0; t < AMAXD / 32; ++t) {
            const int c = lane + 32 * t;
            if (t < ndl && c < d) o[a][t] = fmaf(pj, vs[j * d + c], o[a][t]);
          }
        }
      }
      if (want_imp) {
        cs[warp * AK + lane] = colsum;
        __syncthreads();
        if (tid < AK && kt + tid < L) {
          const float tot = ((cs[tid] + cs[AK + tid]) + cs[2 * AK + tid]) + cs[3 * AK + tid];
          const unsigned long long fx = (unsigned long long)__double2ll_rn((double)tot * kImpScale);
          atomicAdd(&imp_acc[k0 + kt + tid], fx);
        }
      }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int rr = warp * 4 + a;
      if (rr >= nrows) continue;
      T* orow = out + ((size_t)(q0 + rbeg + rr) * s.H + hh) * d;
#pragma unroll
      for (int t = 0; t < AMAXD / 32; ++t) {
        const int c = lane + 32 * t;
        if (t < ndl && c < d) orow[c] = from_f<T>(o[a][t]);
      }
    }
  }
}

}  // namespace

cudaError_t launch_qkv_simt(const fc_handle* h, cudaStream_t st, const StepShape& s,
                            const void* x, const int32_t* q_pos, void* k_cache, void* v_cache) {
  const int P = 3 * s.H * (s.d / 2);
  dim3 grid((s.T + GM - 1) / GM, (P + GP - 1) / GP);
  const float q_scale = (float)(1.4426950408889634 / sqrt((double)s.d));
  if (h->cfg.dtype == FC_DTYPE_FP32) {
    qkv_rope_scatter_simt<float><<<grid, 256, 0, st>>>(
        s, (const float*)x, (const float*)h->w_qkv, q_pos, h->ws.row_dst, h->ws.rope_cos,
        h->ws.rope_sin, (float*)h->ws.q_buf, (float*)k_cache, (float*)v_cache, q_scale);
  } else {
    qkv_rope_scatter_simt<__nv_bfloat16><<<grid, 256, 0, st>>>(
        s, (const __nv_bfloat16*)x, (const __nv_bfloat16*)h->w_qkv, q_pos, h->ws.row_dst,
        h->ws.rope_cos, h->ws.rope_sin, (__nv_bfloat16*)h->ws.q_buf, (__nv_bfloat16*)k_cache,
        (__nv_bfloat16*)v_cache, q_scale);
  }
  return cudaGetLastError();
}

cudaError_t launch_attn_simt(const fc_handle* h, cudaStream_t st, const StepShape& s,
                             const int32_t* cu_q, const int32_t* cu_k, const void* k_cache,
                             const void* v_cache, void* out, bool want_importance) {
  const int d = s.d;
  size_t smem = sizeof(float) * (AROWS * d + AK * (d + 1) + AK * d + 4 * AK);
  const int grid = h->num_sms * 8;
  cudaError_t e;
  if (h->cfg.dtype == FC_DTYPE_FP32) {
    if (smem > 48 * 1024) {
      e = cudaFuncSetAttribute(attn_simt<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)smem);
      if (e != cudaSuccess) return e;
    }
    attn_simt<float><<<grid, 128, smem, st>>>(s, h->ws.items, h->ws.sched, cu_q, cu_k,
                                              (const float*)h->ws.q_buf, (const float*)k_cache,
                                              (const float*)v_cache, (float*)out, h->ws.imp_acc,
                                              want_importance ? 1 : 0);
  } else {
    if (smem > 48 * 1024) {
      e = cudaFuncSetAttribute(attn_simt<__nv_bfloat16>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
    }
    attn_simt<__nv_bfloat16><<<grid, 128, smem, st>>>(
        s, h->ws.items, h->ws.sched, cu_q, cu_k, (const __nv_bfloat16*)h->ws.q_buf,
        (const __nv_bfloat16*)k_cache, (const __nv_bfloat16*)v_cache, (__nv_bfloat16*)out,
        h->ws.imp_acc, want_importance ? 1 : 0);
  }
  return cudaGetLastError();
}

}  // namespace fc
