// QKV projection for small query counts: split-K over a thread-block cluster,
// with RoPE and the K/V cache write fused into the epilogue (Flash-dLLM,
// infernews post "Flash-dLLM: IO-aware KV caching and parallel decoding",
// Flash-Cache paragraph: one pass does the QKV projection, the rotary
// embedding and the cache writes).
//
// With few query rows (one sequence of 128 rows, say) the pair kernel
// (qkv_tc.cu) has one 256-row block and 48 column tiles: half of every tile is
// empty and 52 of 148 SMs idle, while each busy SM streams all of X and its
// share of W.  Here a 128 x 256 output tile (two heads) is computed by a
// cluster of S CTAs, each over 1/S of the reduction (D / 64 steps of 64):
//   warp 0     TMA producer: X (128 x 64) and W (256 x 64) slices into a
//              4-stage ring (128-byte swizzle);
//   warp 1     TMEM allocation (256 columns) and tcgen05.mma issue (M = 128,
//              N = 256, K = 16);
//   warps 2-5  epilogue: the partial accumulator (TMEM) -> this CTA's shared
//              memory (fp32, over the drained ring); after a cluster barrier
//              each CTA takes 1/S of the tile's rows, sums the S partials
//              through distributed shared memory, applies RoPE and stores q
//              (scaled by log2(e)/sqrt(d)) to the Q buffer and k, v (bf16) to
//              their cache rows, as the pair kernel does.
// A second cluster barrier keeps every CTA's shared memory alive until the
// other CTAs have read it.
//
// Measured on one B200 (128 x 4096 query, W 12288 x 4096): 42.5 us at split 2
// (48 clusters, 96 CTAs) against 41.3 us for the pair kernel; at splits 3-8
// only 45, 33, 22 and 15 clusters fit at once, so 48 tiles take two or more
// waves (66-146 us).  A plain TMA stream of the same W into shared memory,
// without any math, takes 26-29 us on 96-148 CTAs, so both kernels are within
// 1.5x of what streaming W once allows.  The kernel is therefore selected only
// on request (fc_set_option); the default is the pair kernel.
#include <cuda_bf16.h>

#include "fc_internal.h"
#include "ptx.cuh"

namespace fc {
namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int HD = 128;
constexpr uint32_t A_BYTES = BM * BK * 2;  // 16 KiB
constexpr uint32_t B_BYTES = BN * BK * 2;  // 32 KiB
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int PSTRIDE = BN + 4;  // floats per row of the partial (16-byte rows, no bank aliasing)
static_assert((uint32_t)BM * PSTRIDE * 4 <= STAGES * STAGE_BYTES, "partial must fit the ring");
static_assert(kQkvXBoxRows == BM && kQkvWBoxRows == BN / 2, "TMA boxes of the host");
constexpr uint32_t IDESC = ptx::idesc_bf16_f32(BM, BN, 0, 0);
constexpr int THREADS = 192;

struct SplitParams {
  int T, S, H;
  int num_m, num_n, num_k, split;  // row blocks of 128, column tiles, K steps, CTAs per tile
  const int32_t* q_pos;
  const int32_t* row_dst;
  const float* rcos;
  const float* rsin;
  __nv_bfloat16* q_buf;
  size_t q_rs, q_hs;
  __nv_bfloat16* k_cache;
  __nv_bfloat16* v_cache;
  float q_scale;
  int32_t* err;
};

struct __align__(8) Bars {
  unsigned long long full[STAGES], empty[STAGES], acc, drain;
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ void store32(__nv_bfloat16* dst, const float* v) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 w;
    w.x = pack_bf16(v[8 * q + 0], v[8 * q + 1]);
    w.y = pack_bf16(v[8 * q + 2], v[8 * q + 3]);
    w.z = pack_bf16(v[8 * q + 4], v[8 * q + 5]);
    w.w = pack_bf16(v[8 * q + 6], v[8 * q + 7]);
    d4[q] = w;
  }
}

__device__ __forceinline__ float4 ld_dsmem_f4(uint32_t cluster_addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(cluster_addr)
               : "memory");
  return v;
}

__global__ void __launch_bounds__(THREADS, 1)
    qkv_splitk_kernel(const __grid_constant__ CUtensorMap tm_x,
                      const __grid_constant__ CUtensorMap tm_w, SplitParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = ptx::smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  Bars* bars = reinterpret_cast<Bars*>(smem + STAGES * STAGE_BYTES);
  volatile int* abort_flag = &bars->abort_flag;
  auto bar = [](unsigned long long& b) { return ptx::smem_u32(&b); };
  auto sA = [&](int s) { return base + s * STAGE_BYTES; };
  auto sB = [&](int s) { return base + s * STAGE_BYTES + A_BYTES; };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  ptx::griddep_launch_dependents();
  const int rank = (int)ptx::cluster_ctarank();
  const int tile = blockIdx.x / p.split;
  const int m = tile % p.num_m, n = tile / p.num_m;
  // this CTA's K steps
  const int kb0 = rank * p.num_k / p.split, kb1 = (rank + 1) * p.num_k / p.split;

  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(bar(bars->full[s]), 1);
      ptx::mbar_init(bar(bars->empty[s]), 1);
    }
    ptx::mbar_init(bar(bars->acc), 1);
    ptx::mbar_init(bar(bars->drain), 1);
    bars->abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tm_x);
    ptx::prefetch_tmap(&tm_w);
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_u32(&bars->tmem_base), 256);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  bool failed = false;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      int issued_phase[STAGES];
      for (int s = 0; s < STAGES; ++s) issued_phase[s] = -1;
      for (int kb = kb0, i = 0; kb < kb1; ++kb, ++i) {
        const int s = i % STAGES;
        const uint32_t ph = (uint32_t)(i / STAGES) & 1u;
        if (!ptx::mbar_wait(bar(bars->empty[s]), ph ^ 1u, abort_flag)) {
          failed = true;
          break;
        }
        ptx::mbar_arrive_expect_tx(bar(bars->full[s]), STAGE_BYTES);
        ptx::tma_load_2d(sA(s), &tm_x, kb * BK, m * BM, bar(bars->full[s]));
        ptx::tma_load_2d(sB(s), &tm_w, kb * BK, n * BN, bar(bars->full[s]));
        ptx::tma_load_2d(sB(s) + B_BYTES / 2, &tm_w, kb * BK, n * BN + BN / 2, bar(bars->full[s]));
        issued_phase[s] = (int)ph;
      }
      if (failed) {
        *abort_flag = 1;
        const unsigned long long t0 = ptx::globaltimer();
        for (int s = 0; s < STAGES; ++s)
          if (issued_phase[s] >= 0)
            while (!ptx::mbar_try_wait(bar(bars->full[s]), (uint32_t)issued_phase[s]) &&
                   ptx::globaltimer() - t0 < ptx::kWaitLimitNs) {
            }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      for (int kb = kb0, i = 0; kb < kb1; ++kb, ++i) {
        const int s = i % STAGES;
        const uint32_t ph = (uint32_t)(i / STAGES) & 1u;
        if (!ptx::mbar_wait(bar(bars->full[s]), ph, abort_flag)) {
          failed = true;
          break;
        }
        ptx::tc_fence_after();
#pragma unroll
        for (int k = 0; k < BK / 16; ++k) {
          const uint64_t ad = ptx::smem_desc(sA(s) + k * 32, 16, 1024);
          const uint64_t bd = ptx::smem_desc(sB(s) + k * 32, 16, 1024);
          ptx::mma_bf16_ss(tmem, ad, bd, IDESC, (i | k) != 0 ? 1u : 0u);
        }
        ptx::mma_commit(bar(bars->empty[s]));
      }
      if (failed) {
        *abort_flag = 1;
        ptx::mma_commit(bar(bars->drain));
        const unsigned long long t0 = ptx::globaltimer();
        while (!ptx::mbar_try_wait(bar(bars->drain), 0u) &&
               ptx::globaltimer() - t0 < ptx::kWaitLimitNs) {
        }
      } else {
        ptx::mma_commit(bar(bars->acc));  // the partial accumulator is complete
      }
    }
  } else {
    // ---------------- epilogue, phase 1: partial accumulator -> shared memory
    // (the ring is drained once every MMA has completed)
    const int quad = warp & 3;
    const int rl = quad * 32 + lane;
    if (ptx::mbar_wait(bar(bars->acc), 0u, abort_flag)) {
      ptx::tc_fence_after();
      float* part = reinterpret_cast<float*>(smem) + (size_t)rl * PSTRIDE;
#pragma unroll 1
      for (int c = 0; c < BN; c += 32) {
        uint32_t r[32];
        ptx::tmem_ld32(tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)c, r);
        ptx::tmem_wait_ld();
        float4* d4 = reinterpret_cast<float4*>(part + c);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          d4[q] = make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                              __uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3]));
      }
    } else {
      *abort_flag = 1;
    }
  }
  // every CTA's partial is in its shared memory
  __syncwarp();
  ptx::tc_fence_before();
  ptx::cluster_sync();
  ptx::tc_fence_after();

  if (warp >= 2) {
    // ---------------- epilogue, phase 2: this CTA's rows of the tile, both heads
    ptx::griddep_wait();  // the row map comes from the preparation kernel
    const int per = (BM + p.split - 1) / p.split;
    const int u = tid - 64;  // 0..127: a row (u / 2) and one of the tile's two heads (u % 2)
    const int j = u & 1;
    const int row_end = min(BM, (rank + 1) * per);
#pragma unroll 1
    for (int row = rank * per + (u >> 1); row < row_end; row += 64) {
      const int g = m * BM + row;
      if (g >= p.T) break;
      const int dst = p.row_dst[g];
      const bool valid = dst >= 0 && dst < p.S;
      const int pos = valid ? p.q_pos[g] : 0;
      const int hs = n * 2 + j;
      const int region = hs / p.H, hh = hs - region * p.H;
      const int half = HD / 2;
      const uint32_t my_row = base + (uint32_t)(row * PSTRIDE + j * HD) * 4u;
#pragma unroll 1
      for (int c = 0; c < half; c += 32) {
        float lo[32], hi[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) lo[e] = hi[e] = 0.f;
#pragma unroll 1
        for (int src = 0; src < p.split; ++src) {
          const uint32_t at = ptx::mapa_shared(my_row, (uint32_t)src);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float4 a = ld_dsmem_f4(at + (uint32_t)(c + 4 * q) * 4u);
            const float4 b = ld_dsmem_f4(at + (uint32_t)(half + c + 4 * q) * 4u);
            lo[4 * q] += a.x, lo[4 * q + 1] += a.y, lo[4 * q + 2] += a.z, lo[4 * q + 3] += a.w;
            hi[4 * q] += b.x, hi[4 * q + 1] += b.y, hi[4 * q + 2] += b.z, hi[4 * q + 3] += b.w;
          }
        }
        if (region < 2) {  // RoPE, rotate-half pairs (i, i + 64)
          const float4* cp = reinterpret_cast<const float4*>(p.rcos + (size_t)pos * half + c);
          const float4* sp = reinterpret_cast<const float4*>(p.rsin + (size_t)pos * half + c);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float4 cc = __ldg(cp + q), ss = __ldg(sp + q);
            const float cv[4] = {cc.x, cc.y, cc.z, cc.w};
            const float sv[4] = {ss.x, ss.y, ss.z, ss.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float u0 = lo[4 * q + e], u1 = hi[4 * q + e];
              lo[4 * q + e] = u0 * cv[e] - u1 * sv[e];
              hi[4 * q + e] = u1 * cv[e] + u0 * sv[e];
            }
          }
        }
        if (region == 0) {
          const float sc = valid ? p.q_scale : 0.f;
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            lo[e] *= sc;
            hi[e] *= sc;
          }
          __nv_bfloat16* qrow = p.q_buf + (size_t)g * p.q_rs + (size_t)hh * p.q_hs;
          store32(qrow + c, lo);
          store32(qrow + half + c, hi);
        } else if (valid) {
          __nv_bfloat16* crow = (region == 1 ? p.k_cache : p.v_cache) + ((size_t)dst * p.H + hh) * HD;
          store32(crow + c, lo);
          store32(crow + half + c, hi);
        }
      }
    }
  }
  // the other CTAs have read this CTA's partial
  __syncwarp();
  ptx::cluster_sync();
  if (tid == 0 && bars->abort_flag) atomicOr(p.err, FC_DEVERR_TIMEOUT);
  if (warp == 1) ptx::tmem_dealloc(tmem, 256);
}

}  // namespace

size_t qkv_splitk_smem_bytes() { return STAGES * STAGE_BYTES + sizeof(Bars) + 1024; }

int qkv_splitk_max_clusters(int split) {
  const size_t smem = qkv_splitk_smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(qkv_splitk_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return -(int)e;
  }
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)split;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3((unsigned)split, 1, 1);
  cfg.blockDim = dim3(THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  e = cudaOccupancyMaxActiveClusters(&n, qkv_splitk_kernel, &cfg);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return -(int)e;
  }
  return n;
}

cudaError_t launch_qkv_splitk(const fc_handle* h, cudaStream_t st, const StepShape& s,
                              const CUtensorMap& tm_x, const CUtensorMap& tm_w,
                              const int32_t* q_pos, void* k_cache, void* v_cache, int split) {
  SplitParams p;
  p.T = s.T;
  p.S = s.S;
  p.H = s.H;
  p.num_m = (s.T + BM - 1) / BM;
  p.num_n = 3 * s.H * HD / BN;
  p.num_k = s.D / BK;
  p.split = split;
  p.q_pos = q_pos;
  p.row_dst = h->ws.row_dst;
  p.rcos = h->ws.rope_cos;
  p.rsin = h->ws.rope_sin;
  p.q_buf = (__nv_bfloat16*)h->ws.q_buf;
  if (h->tc_attn) {  // [H, max_T, d]: one head's query rows contiguous for TMA
    p.q_rs = HD;
    p.q_hs = (size_t)h->cfg.max_total_q * HD;
  } else {
    p.q_rs = (size_t)s.H * HD;
    p.q_hs = HD;
  }
  p.k_cache = (__nv_bfloat16*)k_cache;
  p.v_cache = (__nv_bfloat16*)v_cache;
  p.q_scale = (float)(1.4426950408889634 / sqrt((double)HD));
  p.err = h->ws.err;
  const size_t smem = qkv_splitk_smem_bytes();
  cudaError_t e = smem_attr(qkv_splitk_kernel, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)split;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3((unsigned)(p.num_m * p.num_n * split), 1, 1);
  cfg.blockDim = dim3(THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = h->pdl ? 2 : 1;
  e = cudaLaunchKernelEx(&cfg, qkv_splitk_kernel, tm_x, tm_w, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace fc
