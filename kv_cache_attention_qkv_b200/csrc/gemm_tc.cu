// The decoder's other projections on the 5th-generation tensor cores, with
// their elementwise follow-ups fused into the epilogue (LLaMA-style decoder
// layer around the Flash-Cache attention, as in LLaDA-8B, the model the
// Flash-dLLM pages evaluate):
//   GEMM_RESID   out = resid + A . B^T          (attention output projection,
//                                                 MLP down projection; in place)
//   GEMM_SWIGLU  out = silu(A . Wg^T) * (A . Wu^T) (MLP gate and up projections)
//   GEMM_LMHEAD  per row and 256-column tile of A . W^T: the largest logit, its
//                column and the sum of exp(logit - largest); the logits
//                themselves are never written.
//
// Same structure as the QKV projection: CTA pairs (clusters of two), each
// persistent over 256 x 256 output tiles, one tcgen05.mma.cta_group::2
// (M=256, N=256, K=16) per 16-wide K step; each CTA holds 128 rows of A and
// 128 rows of B per stage of a 6-stage TMA ring (128-byte swizzle), two TMEM
// accumulators so that the epilogue of a tile overlaps the next main loop.
// For GEMM_SWIGLU the pair's 256 B rows are 128 gate rows (from the leader's
// ring) and the same 128 features' up rows (from the other CTA's ring), so
// each CTA's accumulator holds gate and up of its rows side by side.
//   warp 0     TMA producer (both CTAs);
//   warp 1     MMA issue (leader CTA), TMEM allocation (pair);
//   warps 2-5  epilogue (both CTAs): tcgen05.ld of its 32-row quadrant.
#include <cuda_bf16.h>

#include <algorithm>

#include "fc_internal.h"
#include "ptx.cuh"

namespace fc {
namespace {

constexpr int BM = 128;                          // rows of A per CTA
constexpr int PM = 256;                          // rows per pair tile
constexpr int BN = 256, BK = 64, STAGES = 6;
constexpr uint32_t A_BYTES = BM * BK * 2;        // 16 KiB
constexpr uint32_t B_BYTES = (BN / 2) * BK * 2;  // 16 KiB: this CTA's half of the B tile
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
constexpr uint32_t IDESC = ptx::idesc_bf16_f32(PM, BN, 0, 0);
constexpr int THREADS = 192;
static_assert(kGemmBoxRows == BM && kGemmBoxRows == BN / 2, "TMA boxes must match the tiles");

struct __align__(8) Bars {
  unsigned long long full[STAGES], empty[STAGES], tfull[2], tempty[2], drain;
  uint32_t tmem_base;
  int abort_flag;
};

// Tile t of the raster: row blocks vary fastest inside a group of group_m of
// them, which sweeps every column block of B before the next group starts, so
// a group's rows of A stay in L2 while B streams through once per group.
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

__device__ __forceinline__ float silu(float g) { return __fdividef(g, 1.f + __expf(-g)); }

__global__ void __launch_bounds__(THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b0,
                   const __grid_constant__ CUtensorMap tm_b1, GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
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
    ptx::prefetch_tmap(&tm_a);
    ptx::prefetch_tmap(&tm_b0);
    ptx::prefetch_tmap(&tm_b1);
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
  // A is the previous kernel's output
  ptx::griddep_wait();

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      int stage = 0;
      uint32_t phase = 0;
      int issued_phase[STAGES];
      for (int s = 0; s < STAGES; ++s) issued_phase[s] = -1;
      const CUtensorMap* tm_b = (p.mode == GEMM_SWIGLU && rank == 1) ? &tm_b1 : &tm_b0;
      for (int t = pair; t < p.num_tiles && !failed; t += npairs) {
        int m, n;
        tile_coords(t, p.num_m, p.num_n, p.group_m, m, n);
        // B rows of this CTA: its half of a 256-row tile, or for SwiGLU the
        // tile's 128 features of its own matrix (gate on the leader, up on the other)
        const int brow = p.mode == GEMM_SWIGLU ? n * (BN / 2) : n * BN + (int)rank * (BN / 2);
        for (int kb = 0; kb < p.num_k; ++kb) {
          if (!ptx::mbar_wait(bar(bars->empty[stage]), phase ^ 1u, abort_flag)) {
            failed = true;
            break;
          }
          if (leader) ptx::mbar_arrive_expect_tx(bar(bars->full[stage]), 2 * STAGE_BYTES);
          const uint32_t lbar = ptx::mapa_shared(bar(bars->full[stage]), 0);
          ptx::tma_load_2d_pair(sA(stage), &tm_a, kb * BK, m * PM + (int)rank * BM, lbar);
          ptx::tma_load_2d_pair(sB(stage), tm_b, kb * BK, brow, lbar);
          issued_phase[stage] = (int)phase;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (failed && leader) {
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
    int it = 0;
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
      const bool in = row < p.M;
      const uint32_t tb = tmem + (uint32_t)(a * BN) + ((uint32_t)(quad * 32) << 16);
      if (p.mode == GEMM_RESID) {
        // out[row, n*256 + c] = resid + acc  (resid may be out itself)
        const size_t off = (size_t)row * p.ldo + (size_t)n * BN;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t r[32];
          ptx::tmem_ld32(tb + c, r);
          ptx::tmem_wait_ld();
          if (in) {
            const uint4* src = reinterpret_cast<const uint4*>(p.resid + off + c);
            uint4* dst = reinterpret_cast<uint4*>(p.out + off + c);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint4 rv = src[q];
              const uint32_t rw[4] = {rv.x, rv.y, rv.z, rv.w};
              uint32_t ow[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const __nv_bfloat162 b2 = *reinterpret_cast<const __nv_bfloat162*>(&rw[e]);
                const float2 f = __bfloat1622float2(b2);
                ow[e] = pack_bf16(f.x + __uint_as_float(r[8 * q + 2 * e]),
                                  f.y + __uint_as_float(r[8 * q + 2 * e + 1]));
              }
              dst[q] = make_uint4(ow[0], ow[1], ow[2], ow[3]);
            }
          }
        }
      } else if (p.mode == GEMM_SWIGLU) {
        // accumulator columns 0..127 = gate, 128..255 = up of features n*128 ..
        const size_t off = (size_t)row * p.ldo + (size_t)n * (BN / 2);
#pragma unroll 1
        for (int c = 0; c < BN / 2; c += 32) {
          uint32_t g[32], v[32];
          ptx::tmem_ld32(tb + c, g);
          ptx::tmem_ld32(tb + BN / 2 + c, v);
          ptx::tmem_wait_ld();
          if (in) {
            uint4* dst = reinterpret_cast<uint4*>(p.out + off + c);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint32_t ow[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int j = 8 * q + 2 * e;
                ow[e] = pack_bf16(silu(__uint_as_float(g[j])) * __uint_as_float(v[j]),
                                  silu(__uint_as_float(g[j + 1])) * __uint_as_float(v[j + 1]));
              }
              dst[q] = make_uint4(ow[0], ow[1], ow[2], ow[3]);
            }
          }
        }
      } else {
        // GEMM_LMHEAD: running max / argmax / sum of exp over the tile's valid columns
        float mx = -INFINITY, se = 0.f;
        int arg = -1;
        const int c_end = min(BN, p.N - n * BN);
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t r[32];
          ptx::tmem_ld32(tb + c, r);
          ptx::tmem_wait_ld();
          if (c >= c_end) continue;
          float cm = -INFINITY;
          int ca = -1;
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float x = __uint_as_float(r[e]);
            if (c + e < c_end && x > cm) {  // strict: the first maximum wins
              cm = x;
              ca = c + e;
            }
          }
          if (cm > mx) {
            se = mx == -INFINITY ? 0.f : se * __expf(mx - cm);
            mx = cm;
            arg = ca;
          }
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (c + e < c_end) se += __expf(__uint_as_float(r[e]) - mx);
        }
        if (in) {
          float* part = p.partials + ((size_t)row * p.num_n + n) * 3;
          part[0] = mx;
          part[1] = se;
          part[2] = __int_as_float(n * BN + arg);
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

size_t gemm_tc_smem_bytes() { return STAGES * STAGE_BYTES + sizeof(Bars) + 1024; }

cudaError_t launch_gemm_tc(int num_sms, cudaStream_t st, const CUtensorMap& tm_a,
                           const CUtensorMap& tm_b0, const CUtensorMap& tm_b1, GemmParams p) {
  p.num_m = (p.M + PM - 1) / PM;
  p.num_n = p.mode == GEMM_SWIGLU ? p.N / (BN / 2) : (p.N + BN - 1) / BN;
  p.num_tiles = p.num_m * p.num_n;
  p.num_k = p.K / BK;
  // as many row blocks per group as keep about 48 MiB of A in L2
  const size_t a_block_bytes = (size_t)PM * p.K * 2;
  p.group_m = (int)std::max<size_t>(1, std::min<size_t>((size_t)p.num_m,
                                                        (48ull << 20) / a_block_bytes));
  if (p.num_tiles == 0) return cudaSuccess;
  const size_t smem = gemm_tc_smem_bytes();
  cudaError_t e = smem_attr(gemm_tc_kernel, smem);
  if (e != cudaSuccess) return e;
  int pairs = num_sms / 2;
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
  cfg.numAttrs = 1;  // occupancy query with the cluster shape only
  int max_clusters = 0;
  const bool occ_ok =
      cudaOccupancyMaxActiveClusters(&max_clusters, gemm_tc_kernel, &cfg) == cudaSuccess;
  cfg.numAttrs = 2;
  if (occ_ok && max_clusters > 0 && max_clusters < pairs) {
    pairs = max_clusters;
    cfg.gridDim = dim3(2 * pairs, 1, 1);
  }
  cudaGetLastError();
  e = cudaLaunchKernelEx(&cfg, gemm_tc_kernel, tm_a, tm_b0, tm_b1, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace fc
