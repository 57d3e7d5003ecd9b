// fc_attention_noalloc: attention with importance for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc: code that runs where the allocator is
// not theirs to use (an embedding runtime that owns all device memory, a
// plug-in loaded into someone else's process, a context that has handed its
// whole pool to a caching allocator).  fc_create needs a workspace, so such
// callers cannot create a handle.  This entry point needs none: the scratch
// it uses (the fixed-point importance accumulator and a completion counter)
// lives in file-scope __device__ arrays of a fixed size, which every GPU that
// loads the library holds until the process exits.
//
// It computes, for query rows that are already projected and rotated, the
// bidirectional attention over each sequence's whole cache and the per-key
// importance (sum over heads and query rows of the softmax probability), the
// same quantities fc_step produces after its projection.  One kernel does the
// work; its last CTA converts the accumulator into `importance`.
#include <cuda_bf16.h>

#include <algorithm>
#include <mutex>

#include "fc_internal.h"

namespace {

constexpr int NA_ROWS = 16;     // query rows per CTA
constexpr int NA_KEYS = 32;     // keys per shared-memory tile
constexpr int NA_MAXD = 256;

// The scratch: one fixed-point (2^-40) accumulator per key plus a ticket
// counter.  Shared by every call on a device; calls that overlap on the GPU
// race on it.
static __device__ __align__(256) unsigned long long g_noalloc_acc[FC_NOALLOC_MAX_KEYS + 32];

template <typename T>
__device__ __forceinline__ float ld_f(const T* p);
template <>
__device__ __forceinline__ float ld_f<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float ld_f<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}
template <typename T>
__device__ __forceinline__ T st_f(float v);
template <>
__device__ __forceinline__ float st_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 st_f<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// grid = (X, H, B); block = 128 threads (4 warps x 4 query rows).  CTA
// (x, h, b) takes the 16-row query tiles x, x + X, x + 2X, ... of sequence b
// and head h.  acc[0 .. S) must be zero and acc[S] (the ticket) zero at launch.
template <typename T>
__global__ void __launch_bounds__(128) attn_noalloc_kernel(
    int B, int H, int d, int Ttot, int Stot, float qk_scale_log2, const T* __restrict__ q,
    const int32_t* __restrict__ cu_q, const int32_t* __restrict__ cu_k, const T* __restrict__ kc,
    const T* __restrict__ vc, T* __restrict__ out, float* __restrict__ importance,
    unsigned long long* __restrict__ acc) {
  extern __shared__ float sm[];
  float* qs = sm;                      // [16][d]
  float* ks = qs + NA_ROWS * d;        // [32][d + 1]
  float* vs = ks + NA_KEYS * (d + 1);  // [32][d]
  float* cs = vs + NA_KEYS * d;        // [4][32]
  __shared__ bool last_cta;
  unsigned long long* ticket = acc + Stot;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int hh = blockIdx.y, b = blockIdx.z;
  const int q0 = cu_q[b], n = cu_q[b + 1] - q0, k0 = cu_k[b], L = cu_k[b + 1] - k0;
  const bool ok = q0 >= 0 && n >= 0 && q0 + n <= Ttot && k0 >= 0 && L >= 0 && k0 + L <= Stot;
  for (int qt = blockIdx.x; ok && qt * NA_ROWS < n; qt += gridDim.x) {
    const int rbeg = qt * NA_ROWS;
    const int nrows = min(NA_ROWS, n - rbeg);
    if (L == 0) {  // no key to attend: the rows' output is an empty sum, zero
      for (int e = tid; e < nrows * d; e += 128)
        out[((size_t)(q0 + rbeg + e / d) * H + hh) * d + e % d] = st_f<T>(0.f);
      continue;
    }
    for (int e = tid; e < NA_ROWS * d; e += 128) {
      const int rr = e / d, c = e % d;
      qs[e] = rr < nrows ? ld_f(q + ((size_t)(q0 + rbeg + rr) * H + hh) * d + c) * qk_scale_log2 : 0.f;
    }
    float m[4], l[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      m[a] = -INFINITY;
      l[a] = 0.f;
    }
    for (int kt = 0; kt < L; kt += NA_KEYS) {  // pass 1: max and normaliser
      __syncthreads();
      for (int e = tid; e < NA_KEYS * d; e += 128) {
        const int j = e / d, c = e % d;
        ks[j * (d + 1) + c] = kt + j < L ? ld_f(kc + ((size_t)(k0 + kt + j) * H + hh) * d + c) : 0.f;
      }
      __syncthreads();
      const bool kv = kt + lane < L;
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const int rr = warp * 4 + a;
        float s = 0.f;
        for (int c = 0; c < d; ++c) s = fmaf(qs[rr * d + c], ks[lane * (d + 1) + c], s);
        s = kv ? s : -INFINITY;
        float mx = s;
        for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        const float mn = fmaxf(m[a], mx);
        float e = kv ? exp2f(s - mn) : 0.f;
        for (int o = 16; o; o >>= 1) e += __shfl_xor_sync(0xffffffffu, e, o);
        l[a] = l[a] * exp2f(m[a] - mn) + e;
        m[a] = mn;
      }
    }
    float o[4][NA_MAXD / 32];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int t = 0; t < NA_MAXD / 32; ++t) o[a][t] = 0.f;
    for (int kt = 0; kt < L; kt += NA_KEYS) {  // pass 2: probabilities, P V, column sums
      __syncthreads();
      for (int e = tid; e < NA_KEYS * d; e += 128) {
        const int j = e / d, c = e % d;
        const bool kv = kt + j < L;
        const size_t g = ((size_t)(k0 + kt + j) * H + hh) * d + c;
        ks[j * (d + 1) + c] = kv ? ld_f(kc + g) : 0.f;
        vs[j * d + c] = kv ? ld_f(vc + g) : 0.f;
      }
      __syncthreads();
      const bool kv = kt + lane < L;
      float col = 0.f;
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const int rr = warp * 4 + a;
        float s = 0.f;
        for (int c = 0; c < d; ++c) s = fmaf(qs[rr * d + c], ks[lane * (d + 1) + c], s);
        const float pr = (kv && rr < nrows) ? exp2f(s - m[a]) / l[a] : 0.f;
        col += pr;
        for (int j = 0; j < NA_KEYS; ++j) {
          const float pj = __shfl_sync(0xffffffffu, pr, j);
#pragma unroll
          for (int t = 0; t < NA_MAXD / 32; ++t) {
            const int c = lane + 32 * t;
            if (c < d) o[a][t] = fmaf(pj, vs[j * d + c], o[a][t]);
          }
        }
      }
      cs[warp * NA_KEYS + lane] = col;
      __syncthreads();
      if (tid < NA_KEYS && kt + tid < L) {
        const float tot = ((cs[tid] + cs[NA_KEYS + tid]) + cs[2 * NA_KEYS + tid]) + cs[3 * NA_KEYS + tid];
        atomicAdd(&acc[k0 + kt + tid],
                  (unsigned long long)__double2ll_rn((double)tot * fc::kImpScale));
      }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int rr = warp * 4 + a;
      if (rr >= nrows) continue;
      T* orow = out + ((size_t)(q0 + rbeg + rr) * H + hh) * d;
#pragma unroll
      for (int t = 0; t < NA_MAXD / 32; ++t) {
        const int c = lane + 32 * t;
        if (c < d) orow[c] = st_f<T>(o[a][t]);
      }
    }
    __syncthreads();  // the shared tiles are reused by the next query tile
  }

  // the last CTA to finish turns the accumulator into floats
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const unsigned long long total =
        (unsigned long long)gridDim.x * gridDim.y * gridDim.z;
    last_cta = atomicAdd(ticket, 1ull) == total - 1ull;
  }
  __syncthreads();
  if (last_cta) {
    __threadfence();
    for (int j = tid; j < Stot; j += 128)
      importance[j] = (float)((double)(long long)__ldcg(&acc[j]) * fc::kImpInvScale);
  }
}

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

std::mutex g_mu;
// (context, device address of the scratch in it), one entry per context seen
constexpr int kMaxCtx = 64;
CUcontext g_ctx[kMaxCtx] = {};
void* g_scratch[kMaxCtx] = {};
int g_nctx = 0;

CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (CtxGetCurrentFn)p;
  }
  return fn;
}

// Device address of the scratch array in the current context, looked up the
// first time a context calls (host code cannot use the array's name as a
// device address).  Keyed by context, so a process that creates its own
// contexts gets each one's copy of the array.
void* scratch_address() {
  std::lock_guard<std::mutex> lk(g_mu);
  CtxGetCurrentFn get = ctx_get_current();
  CUcontext ctx = nullptr;
  if (!get || get(&ctx) != CUDA_SUCCESS) return nullptr;
  if (!ctx) {  // no context bound yet: the runtime's device, primary context
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaSetDevice(dev) != cudaSuccess ||
        get(&ctx) != CUDA_SUCCESS || !ctx) {
      cudaGetLastError();
      return nullptr;
    }
  }
  for (int i = 0; i < g_nctx; ++i)
    if (g_ctx[i] == ctx) return g_scratch[i];
  if (g_nctx == kMaxCtx) return nullptr;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_acc) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  g_ctx[g_nctx] = ctx;
  g_scratch[g_nctx] = p;
  ++g_nctx;
  return p;
}

}  // namespace

extern "C" fc_status fc_attention_noalloc(void* stream, int dtype, int batch, int n_heads,
                                          int head_dim, const void* q,
                                          const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                                          int total_q, int total_k, const void* k_cache,
                                          const void* v_cache, void* out, float* importance) {
  if (dtype != FC_DTYPE_BF16 && dtype != FC_DTYPE_FP32) return FC_ERR_INVALID_ARG;
  if (batch < 1 || batch > 65535 || n_heads < 1 || n_heads > 65535 || head_dim < 1 ||
      total_q < 0 || total_k < 0)
    return FC_ERR_INVALID_ARG;
  if (head_dim > NA_MAXD || total_k > FC_NOALLOC_MAX_KEYS) return FC_ERR_UNSUPPORTED;
  // a key's importance is at most (heads x query rows); the signed 2^-40 fixed
  // point accumulator holds sums below 2^23
  if ((long long)n_heads * total_q >= (1ll << 23)) return FC_ERR_UNSUPPORTED;
  if (!cu_seqlens_q || !cu_seqlens_k || !importance) return FC_ERR_INVALID_ARG;
  if (total_q > 0 && (!q || !k_cache || !v_cache || !out)) return FC_ERR_INVALID_ARG;
  unsigned long long* acc = static_cast<unsigned long long*>(scratch_address());
  if (!acc) return FC_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  // accumulator of the keys in use and the ticket counter start at zero
  if (cudaMemsetAsync(acc, 0, ((size_t)total_k + 1) * sizeof(unsigned long long), st) != cudaSuccess)
    return FC_ERR_CUDA;
  // query tiles per (sequence, head) CTA column: the batch's average tile
  // count, so the grid holds about as many CTAs as there are tiles; a longer
  // sequence's CTAs loop over its further tiles
  const long long tiles = (total_q + NA_ROWS - 1) / NA_ROWS;
  const int gx = (int)std::max(1ll, (tiles + batch - 1) / batch);
  dim3 grid(gx, n_heads, batch);
  const int d = head_dim;
  const size_t smem = sizeof(float) * (NA_ROWS * d + NA_KEYS * (d + 1) + NA_KEYS * d + 4 * NA_KEYS);
  const float scale = (float)(1.4426950408889634 / sqrt((double)d));
  if (dtype == FC_DTYPE_FP32) {
    if (smem > 48 * 1024 && cudaFuncSetAttribute(attn_noalloc_kernel<float>,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)smem) != cudaSuccess)
      return FC_ERR_CUDA;
    attn_noalloc_kernel<float><<<grid, 128, smem, st>>>(
        batch, n_heads, d, total_q, total_k, scale, (const float*)q, cu_seqlens_q, cu_seqlens_k,
        (const float*)k_cache, (const float*)v_cache, (float*)out, importance, acc);
  } else {
    if (smem > 48 * 1024 && cudaFuncSetAttribute(attn_noalloc_kernel<__nv_bfloat16>,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)smem) != cudaSuccess)
      return FC_ERR_CUDA;
    attn_noalloc_kernel<__nv_bfloat16><<<grid, 128, smem, st>>>(
        batch, n_heads, d, total_q, total_k, scale, (const __nv_bfloat16*)q, cu_seqlens_q,
        cu_seqlens_k, (const __nv_bfloat16*)k_cache, (const __nv_bfloat16*)v_cache,
        (__nv_bfloat16*)out, importance, acc);
  }
  return cudaGetLastError() == cudaSuccess ? FC_OK : FC_ERR_CUDA;
}
