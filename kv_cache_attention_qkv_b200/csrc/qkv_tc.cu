// QKV projection on the 5th-generation tensor cores with RoPE and the K/V
// cache write fused into the epilogue (Flash-dLLM, infernews post "Flash-dLLM:
// IO-aware KV caching and parallel decoding", Flash-Cache paragraph: one pass
// does the QKV projection, the rotary embedding and the cache writes).
//
// C[T, 3*H*128] = X[T, D] * W_qkv[3*H*128, D]^T is never written: each
// 128 x 256 output tile (two heads) lives in TMEM, and the epilogue rotates q
// and k by RoPE at the row's position and stores
//   q * log2(e)/sqrt(d) -> Q buffer (bf16; [H, max_T, d] when the tensor-core
//     attention reads it, else [T, H, d]),
//   k, v (bf16, round to nearest even) -> cache row cu_seqlens_k[b] + q_pos[r].
//
// Structure: CTA pairs (clusters of two), each pair persistent over 256 x 256
// output tiles; one tcgen05.mma.cta_group::2 (M=256, N=256, K=16) covers the
// pair, each CTA holding 128 rows of X and 128 rows of W per stage, so each SM
// streams half of the W tile through its shared memory.
//   warp 0     TMA producer (both CTAs): X and W slices (64 wide, 128-byte
//              swizzle) into a 6-stage ring; completion is counted on the
//              leader CTA's barrier;
//   warp 1     allocates 512 TMEM columns (pair allocation); in the leader CTA
//              it issues the MMAs into one of two TMEM accumulators and
//              releases stages and accumulators to both CTAs (multicast commit);
//   warps 2-5  epilogue (both CTAs): tcgen05.ld of its 32-row quadrant, RoPE,
//              stores, while the MMA warp already fills the other accumulator.
#include <cuda_bf16.h>

#include <algorithm>

#include "fc_internal.h"
#include "ptx.cuh"

namespace fc {
namespace {

constexpr int BM = 128;                         // rows of X per CTA
constexpr int PM = 256;                         // rows per pair tile
constexpr int BN = 256, BK = 64, STAGES = 6;
constexpr int HD = 128;                         // head_dim of this path
constexpr uint32_t A_BYTES = BM * BK * 2;       // 16 KiB
constexpr uint32_t B_BYTES = (BN / 2) * BK * 2; // 16 KiB: this CTA's half of the W tile
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
static_assert(kQkvXBoxRows == BM && kQkvWBoxRows == BN / 2,
              "the host's TMA boxes must match the per-CTA tiles");
constexpr uint32_t IDESC = ptx::idesc_bf16_f32(PM, BN, 0, 0);
constexpr int THREADS = 192;

struct QkvParams {
  int T, S, D, H;
  int num_m, num_n, num_tiles, num_k;
  int group_m;  // tile raster: groups of this many pair row blocks
  const int32_t* q_pos;
  const int32_t* row_dst;
  const float* rcos;
  const float* rsin;
  __nv_bfloat16* q_buf;
  size_t q_rs, q_hs;  // element strides of a query row and of a head in the Q buffer
  __nv_bfloat16* k_cache;
  __nv_bfloat16* v_cache;
  float q_scale;
  int32_t* err;
};

struct __align__(8) Bars {
  unsigned long long full[STAGES], empty[STAGES], tfull[2], tempty[2], drain;
  uint32_t tmem_base;
  int abort_flag;
};

// Tile t of the raster: row blocks vary fastest inside a group of group_m of
// them, which sweeps every column block of W before the next group starts, so
// a group's rows of X stay in L2 while W streams through once per group.
__device__ __forceinline__ void tile_coords(int t, int num_m, int num_n, int group_m, int& m,
                                            int& n) {
  const int per_group = group_m * num_n;
  const int g = t / per_group;
  const int first_m = g * group_m;
  const int gsize = min(num_m - first_m, group_m);
  const int r = t - g * per_group;
  m = first_m + r % gsize;
  n = r / gsize;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Store 32 consecutive bf16 (from 32 floats) at dst (64 bytes, 16-byte aligned).
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

__global__ void __launch_bounds__(THREADS, 1)
    qkv_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                  QkvParams p) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte-swizzled tiles
  const uint32_t raw = ptx::smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  Bars* bars = reinterpret_cast<Bars*>(smem + STAGES * STAGE_BYTES);
  volatile int* abort_flag = &bars->abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  auto sA = [&](int s) { return base + s * STAGE_BYTES; };
  auto sB = [&](int s) { return base + s * STAGE_BYTES + A_BYTES; };
  auto bar = [](unsigned long long& b) { return ptx::smem_u32(&b); };

  ptx::griddep_launch_dependents();
  const uint32_t rank = ptx::cluster_ctarank();  // 0 = leader of the pair
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(bar(bars->full[s]), 1);
      ptx::mbar_init(bar(bars->empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(bar(bars->tfull[a]), 1);
      ptx::mbar_init(bar(bars->tempty[a]), 8);  // 4 epilogue warps in each CTA
    }
    ptx::mbar_init(bar(bars->drain), 1);
    bars->abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tm_x);
    ptx::prefetch_tmap(&tm_w);
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(ptx::smem_u32(&bars->tmem_base), 512);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();  // both CTAs' barriers exist before any cross-CTA traffic
  ptx::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  bool failed = false;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      int stage = 0;
      uint32_t phase = 0;
      int issued_phase[STAGES];
      for (int s = 0; s < STAGES; ++s) issued_phase[s] = -1;
      // X is reused by every column block of its group, W once per group
      const uint64_t pol_x = ptx::l2_policy_evict_last(), pol_w = ptx::l2_policy_evict_first();
      for (int t = pair; t < p.num_tiles && !failed; t += npairs) {
        int m, n;
        tile_coords(t, p.num_m, p.num_n, p.group_m, m, n);
        for (int kb = 0; kb < p.num_k; ++kb) {
          if (!ptx::mbar_wait(bar(bars->empty[stage]), phase ^ 1u, abort_flag)) {
            failed = true;
            break;
          }
          // the leader's barrier counts both CTAs' bytes
          if (leader) ptx::mbar_arrive_expect_tx(bar(bars->full[stage]), 2 * STAGE_BYTES);
          const uint32_t lbar = ptx::mapa_shared(bar(bars->full[stage]), 0);
          ptx::tma_load_2d_pair_hint(sA(stage), &tm_x, kb * BK, m * PM + (int)rank * BM, lbar,
                                     pol_x);
          ptx::tma_load_2d_pair_hint(sB(stage), &tm_w, kb * BK, n * BN + (int)rank * (BN / 2),
                                     lbar, pol_w);
          issued_phase[stage] = (int)phase;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (failed && leader) {
        // let the copies already in flight land before the CTA exits (the
        // leader's barriers also count the other CTA's copies)
        *abort_flag = 1;
        for (int s = 0; s < STAGES; ++s)
          if (issued_phase[s] >= 0) {
            const unsigned long long t0 = ptx::globaltimer();
            while (!ptx::mbar_try_wait(bar(bars->full[s]), (uint32_t)issued_phase[s]) &&
                   ptx::globaltimer() - t0 < ptx::kWaitLimitNs) {
            }
          }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- MMA issuer (leader CTA only)
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      for (int t = pair; t < p.num_tiles && !failed; t += npairs, ++it) {
        const int a = it & 1;
        const uint32_t u = (uint32_t)(it >> 1);
        if (!ptx::mbar_wait(bar(bars->tempty[a]), (u & 1u) ^ 1u, abort_flag)) {
          failed = true;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(a * BN);
        for (int kb = 0; kb < p.num_k; ++kb) {
          if (!ptx::mbar_wait(bar(bars->full[stage]), phase, abort_flag)) {
            failed = true;
            break;
          }
          ptx::tc_fence_after();
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t ad = ptx::smem_desc(sA(stage) + k * 32, 16, 1024);
            const uint64_t bd = ptx::smem_desc(sB(stage) + k * 32, 16, 1024);
            ptx::mma_bf16_ss_pair(d, ad, bd, IDESC, (kb | k) != 0 ? 1u : 0u);
          }
          ptx::mma_commit_pair_mc(bar(bars->empty[stage]), 0x3);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (failed) break;
        ptx::mma_commit_pair_mc(bar(bars->tfull[a]), 0x3);
      }
      if (failed) {
        *abort_flag = 1;
        ptx::mma_commit_pair_mc(bar(bars->drain), 0x1);
        const unsigned long long t0 = ptx::globaltimer();
        while (!ptx::mbar_try_wait(bar(bars->drain), 0u) &&
               ptx::globaltimer() - t0 < ptx::kWaitLimitNs) {
        }
      }
    }
  } else {
    // ---------------- epilogue: warps 2..5, TMEM lane quadrant = warp % 4
    const int quad = warp & 3;
    const int half = HD / 2;
    int it = 0;
    ptx::griddep_wait();  // the row map comes from the preparation kernel
    const uint32_t tempty_leader0 = ptx::mapa_shared(bar(bars->tempty[0]), 0);
    const uint32_t tempty_leader1 = ptx::mapa_shared(bar(bars->tempty[1]), 0);
    for (int t = pair; t < p.num_tiles; t += npairs, ++it) {
      int m, n;
      tile_coords(t, p.num_m, p.num_n, p.group_m, m, n);
      const int a = it & 1;
      const uint32_t u = (uint32_t)(it >> 1);
      if (!ptx::mbar_wait(bar(bars->tfull[a]), u & 1u, abort_flag)) {
        failed = true;
        *abort_flag = 1;
        break;
      }
      ptx::tc_fence_after();
      const int row = m * PM + (int)rank * BM + quad * 32 + lane;
      const bool in = row < p.T;
      const int dst = in ? p.row_dst[row] : -1;
      const bool valid = dst >= 0 && dst < p.S;
      const int pos = valid ? p.q_pos[row] : 0;
      const uint32_t tb = tmem + (uint32_t)(a * BN) + ((uint32_t)(quad * 32) << 16);
#pragma unroll 1
      for (int j = 0; j < 2; ++j) {
        const int hs = n * 2 + j;
        const int region = hs / p.H, hh = hs - region * p.H;
#pragma unroll 1
        for (int c = 0; c < half; c += 32) {
          uint32_t rl[32], rh[32];
          ptx::tmem_ld32(tb + j * HD + c, rl);
          ptx::tmem_ld32(tb + j * HD + half + c, rh);
          ptx::tmem_wait_ld();
          float lo[32], hi[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            lo[e] = __uint_as_float(rl[e]);
            hi[e] = __uint_as_float(rh[e]);
          }
          if (region < 2) {
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
            if (in) {
              const float sc = valid ? p.q_scale : 0.f;
#pragma unroll
              for (int e = 0; e < 32; ++e) {
                lo[e] *= sc;
                hi[e] *= sc;
              }
              __nv_bfloat16* qrow = p.q_buf + (size_t)row * p.q_rs + (size_t)hh * p.q_hs;
              store32(qrow + c, lo);
              store32(qrow + half + c, hi);
            }
          } else if (valid) {
            __nv_bfloat16* crow = (region == 1 ? p.k_cache : p.v_cache) + ((size_t)dst * p.H + hh) * HD;
            store32(crow + c, lo);
            store32(crow + half + c, hi);
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive_cluster(a ? tempty_leader1 : tempty_leader0);
    }
  }

  __syncwarp();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();  // the pair's MMAs and cross-CTA arrivals are all done
  ptx::tc_fence_after();
  if (tid == 0 && bars->abort_flag) atomicOr(p.err, FC_DEVERR_TIMEOUT);
  if (warp == 1) ptx::tmem_dealloc_pair(tmem, 512);
}

}  // namespace

size_t qkv_tc_smem_bytes() { return STAGES * STAGE_BYTES + sizeof(Bars) + 1024; }

cudaError_t launch_qkv_tc(const fc_handle* h, cudaStream_t st, const StepShape& s,
                          const CUtensorMap& tm_x, const CUtensorMap& tm_w, const int32_t* q_pos,
                          void* k_cache, void* v_cache) {
  QkvParams p;
  p.T = s.T;
  p.S = s.S;
  p.D = s.D;
  p.H = s.H;
  p.num_m = (s.T + PM - 1) / PM;
  p.num_n = 3 * s.H * HD / BN;
  p.num_tiles = p.num_m * p.num_n;
  p.num_k = s.D / BK;
  // as many row blocks per group as keep about 48 MiB of X in L2
  const size_t x_block_bytes = (size_t)PM * s.D * 2;
  p.group_m = (int)std::max<size_t>(1, std::min<size_t>((size_t)p.num_m,
                                                        (48ull << 20) / x_block_bytes));
  p.q_pos = q_pos;
  p.row_dst = h->ws.row_dst;
  p.rcos = h->ws.rope_cos;
  p.rsin = h->ws.rope_sin;
  p.q_buf = (__nv_bfloat16*)h->ws.q_buf;
  if (h->tc_attn) {  // [H, max_T, d]: one head's query rows contiguous for TMA
    p.q_rs = HD;
    p.q_hs = (size_t)h->cfg.max_total_q * HD;
  } else {  // [T, H, d]
    p.q_rs = (size_t)s.H * HD;
    p.q_hs = HD;
  }
  p.k_cache = (__nv_bfloat16*)k_cache;
  p.v_cache = (__nv_bfloat16*)v_cache;
  p.q_scale = (float)(1.4426950408889634 / sqrt((double)HD));
  p.err = h->ws.err;
  const size_t smem = qkv_tc_smem_bytes();
  cudaError_t e = smem_attr(qkv_tc_kernel, smem);
  if (e != cudaSuccess) return e;
  int pairs = h->num_sms / 2;
  if (p.num_tiles < pairs) pairs = p.num_tiles;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int max_clusters = 0;
  cfg.numAttrs = 1;  // occupancy query with the cluster shape only
  const bool occ_ok = cudaOccupancyMaxActiveClusters(&max_clusters, qkv_tc_kernel, &cfg) == cudaSuccess;
  cfg.numAttrs = h->pdl ? 2 : 1;
  if (occ_ok &&
      max_clusters > 0 && max_clusters < pairs) {
    pairs = max_clusters;
    cfg.gridDim = dim3(2 * pairs, 1, 1);
  }
  cudaGetLastError();
  e = cudaLaunchKernelEx(&cfg, qkv_tc_kernel, tm_x, tm_w, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace fc
