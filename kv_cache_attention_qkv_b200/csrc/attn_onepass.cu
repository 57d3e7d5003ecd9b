// Bidirectional variable-length attention in ONE scan of the KV cache, on the
// tensor cores: the path of a step that does not ask for attention importance.
//
// Flash-dLLM (paper-digest page, Fig. 2 caption): the fixed-size query of a
// sequence attends bidirectionally to its full KV cache.  Queries of
// different lengths share one launch through block scheduling (infernews post
// "Flash-dLLM: IO-aware KV caching and parallel decoding", Flash-Cache
// paragraph).
//
// For any per-row reference M_r,
//   o_r = sum_j 2^(s_rj - M_r) V_j / l_r,   l_r = sum_j 2^(s_rj - M_r).
// Here M_r is fixed for the whole work item: the row's maximum over the item's
// first 128-key tile.  The unnormalised probabilities u_rj = 2^(s_rj - M_r) of
// every tile are then final as soon as they are computed: O accumulates u V on
// the tensor cores without any rescaling, l_r accumulates in registers, and O
// is divided by l_r once at the end.  K and V are each read once, Q K^T and
// the exponentials computed once.
//
// Safe band: u is held in fp32 and bf16, whose exponent range holds 2^x for x
// up to 127.  An item in which some row has a score more than kBand above its
// reference is not finished here: its output is dropped and the item is
// appended to the hand-over list, which the two-pass kernel (attn_tc.cu)
// computes after this kernel.
//
// (A step that asks for importance uses the two-pass kernel for every item:
// the importance of a key needs each row's final normaliser, and keeping this
// kernel's probability tiles until it is known costs more L2 traffic than a
// second scan over K.)
//
// Work item = (sequence b, head h, 128-row query tile), from the part of the
// work list after its first sched[2] items, longest caches first.
//
// Roles (one CTA per SM, persistent over the work list):
//   warp 0      TMA producer: Q tile, then K_0, K_1, V_0, K_2, V_1, ... into a
//               ring of 32 KiB slots (the order the MMA warp consumes them);
//   warp 1      TMEM allocation, Q copy into TMEM, tcgen05.mma issue: S_j =
//               Q K_j^T into TMEM buffer j % 2 (Q read from TMEM), then after
//               the softmax warps have written P_j over S_j, O += P_j V_j
//               (P read from TMEM) and S_{j+2} into the same buffer;
//   warps 2-17  softmax: two groups of eight take the S buffers alternately.
//               In a group, warp w owns TMEM lane quadrant w % 4 (32 query
//               rows, one per thread) and one 64-key half of the tile.  At the
//               end of an item they merge l and write O / l.
//
// TMEM columns: S/P buffer 0 [0,128), S/P buffer 1 [128,256), O [256,384),
// Q [384,448).
#include <cuda_bf16.h>

#include "fc_internal.h"
#include "ptx.cuh"

namespace fc {
namespace {

constexpr int QT = 128, KT = 128, HD = 128;
constexpr int SLOTS = 5;
constexpr int SOFTMAX_WARPS = 16;
constexpr int PARTS = 4;     // (group, column half) partial row sums
constexpr int CPW = KT / 2;  // columns per softmax warp and tile
constexpr int THREADS = 64 + 32 * SOFTMAX_WARPS;
constexpr float kBand = 64.f;  // largest score above the reference (log2 units)
constexpr uint32_t HALF_BYTES = 128 * 128;       // 128 rows x 64 bf16
constexpr uint32_t TILE_BYTES = 2 * HALF_BYTES;  // 128 rows x 128 bf16
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_SLOT = TILE_BYTES;
constexpr uint32_t OFF_REF = OFF_SLOT + SLOTS * TILE_BYTES;  // float [parity][half][128]
constexpr uint32_t OFF_LSUM = OFF_REF + 2 * 2 * 128 * 4;     // float [parity][part][128]
constexpr uint32_t OFF_FLAG = OFF_LSUM + 2 * PARTS * 128 * 4;  // int [4]: band flag per item
constexpr uint32_t OFF_BARS = OFF_FLAG + 64;
constexpr uint32_t TM_S0 = 0, TM_O = 256, TM_Q = 384;

constexpr uint32_t IDESC_S = ptx::idesc_bf16_f32(128, 128, 0, 0);   // Q K^T, K K-major
constexpr uint32_t IDESC_PV = ptx::idesc_bf16_f32(128, 128, 0, 1);  // P V, V MN-major

struct OnePassParams {
  int H, max_T;
  const WorkItem* items;  // the whole work list; this kernel takes items[sched[2] ..]
  const int32_t* cu_q;
  const int32_t* cu_k;
  __nv_bfloat16* out;
  int32_t* sched;  // [0] items, [2] items for the two-pass kernel, [3] hand-over count
  WorkItem* items_fb;
  int max_fb;
  int32_t* err;
};

struct __align__(8) Bars {
  unsigned long long qfull, qfree;
  unsigned long long full[SLOTS], empty[SLOTS];
  unsigned long long sfull[2], pready[2];
  unsigned long long refbar, statbar;
  unsigned long long ofull, ofree;
  unsigned long long drain;
  uint32_t tmem_base;
  int abort_flag;
};

struct Item {
  int b, qt, h, q0, nrows, k0, L, ntiles;
};

__device__ __forceinline__ Item to_item(const WorkItem& w) {
  Item r;
  r.b = w.seq;
  r.qt = w.tile_head >> 8;
  r.h = w.tile_head & 0xFF;
  r.q0 = w.q0;
  r.nrows = w.nrows;
  r.k0 = w.k0;
  r.L = w.L;
  r.ntiles = (r.L + KT - 1) / KT;
  return r;
}

// Item idx of this kernel's part of the list (a zero item past the end).
__device__ __forceinline__ WorkItem fetch_item(const OnePassParams& p, int first, int n, int idx) {
  WorkItem w = {};
  if (idx < n) w = p.items[first + idx];
  return w;
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* tm, int x, int y,
                                            int z, uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(z), "r"(bar), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

__global__ void __launch_bounds__(THREADS, 1)
    attn_onepass_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, OnePassParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = ptx::smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  Bars* bars = reinterpret_cast<Bars*>(smem + OFF_BARS);
  volatile int* abort_flag = &bars->abort_flag;
  auto bar = [](unsigned long long& b) { return ptx::smem_u32(&b); };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  ptx::griddep_launch_dependents();

  if (tid < 4) reinterpret_cast<int*>(smem + OFF_FLAG)[tid] = 0;
  if (tid == 0) {
    ptx::mbar_init(bar(bars->qfull), 1);
    ptx::mbar_init(bar(bars->qfree), 1);
    for (int s = 0; s < SLOTS; ++s) {
      ptx::mbar_init(bar(bars->full[s]), 1);
      ptx::mbar_init(bar(bars->empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(bar(bars->sfull[s]), 1);
      ptx::mbar_init(bar(bars->pready[s]), SOFTMAX_WARPS / 2);
    }
    ptx::mbar_init(bar(bars->refbar), SOFTMAX_WARPS / 2);  // the first tile's group
    ptx::mbar_init(bar(bars->statbar), SOFTMAX_WARPS);
    ptx::mbar_init(bar(bars->ofull), 1);
    ptx::mbar_init(bar(bars->ofree), SOFTMAX_WARPS);
    ptx::mbar_init(bar(bars->drain), 1);
    bars->abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tm_q);
    ptx::prefetch_tmap(&tm_k);
    ptx::prefetch_tmap(&tm_v);
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_u32(&bars->tmem_base), 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  bool failed = false;
  // the work list, Q and the refreshed cache come from the preceding kernels
  ptx::griddep_wait();
  const int first = p.sched[2];
  const int n_items = p.sched[0] - first;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------- producer
      uint32_t prod = 0;
      int issued_phase[SLOTS];
      for (int s = 0; s < SLOTS; ++s) issued_phase[s] = -1;
      int q_issued_phase = -1;
      uint32_t ic = 0;
      const uint64_t pol = policy_evict_first();  // K and V are read once
      auto load_tile = [&](const CUtensorMap* tm, int h, int row) -> bool {
        const uint32_t s = prod % SLOTS, ph = (prod / SLOTS) & 1u;
        if (!ptx::mbar_wait(bar(bars->empty[s]), ph ^ 1u, abort_flag)) return false;
        const uint32_t dst = base + OFF_SLOT + s * TILE_BYTES;
        ptx::mbar_arrive_expect_tx(bar(bars->full[s]), TILE_BYTES);
        tma_load_3d(dst, tm, 0, h, row, bar(bars->full[s]), pol);
        tma_load_3d(dst + HALF_BYTES, tm, 64, h, row, bar(bars->full[s]), pol);
        issued_phase[s] = (int)ph;
        ++prod;
        return true;
      };
      // the next item's record is fetched while this one runs
      WorkItem wnext = fetch_item(p, first, n_items, snake_item(0, blockIdx.x, gridDim.x));
      for (int r = 0, it = snake_item(0, blockIdx.x, gridDim.x); it < n_items && !failed;
         ++r, it = snake_item(r, blockIdx.x, gridDim.x), ++ic) {
        const Item t = to_item(wnext);
        wnext = fetch_item(p, first, n_items, snake_item(r + 1, blockIdx.x, gridDim.x));
        if (!ptx::mbar_wait(bar(bars->qfree), (ic & 1u) ^ 1u, abort_flag)) {
          failed = true;
          break;
        }
        ptx::mbar_arrive_expect_tx(bar(bars->qfull), TILE_BYTES);
        const int qrow = t.h * p.max_T + t.q0 + t.qt * QT;
        ptx::tma_load_2d(base + OFF_Q, &tm_q, 0, qrow, bar(bars->qfull));
        ptx::tma_load_2d(base + OFF_Q + HALF_BYTES, &tm_q, 64, qrow, bar(bars->qfull));
        q_issued_phase = (int)(ic & 1u);
        // K_0, K_1, then V_j followed by K_{j+2}: the MMA warp's order
        if (!load_tile(&tm_k, t.h, t.k0)) failed = true;
        if (!failed && t.ntiles > 1 && !load_tile(&tm_k, t.h, t.k0 + KT)) failed = true;
        for (int j = 0; j < t.ntiles && !failed; ++j) {
          if (!load_tile(&tm_v, t.h, t.k0 + j * KT)) failed = true;
          if (!failed && j + 2 < t.ntiles && !load_tile(&tm_k, t.h, t.k0 + (j + 2) * KT))
            failed = true;
        }
      }
      if (failed) {
        *abort_flag = 1;
        const unsigned long long t0 = ptx::globaltimer();
        for (int s = 0; s < SLOTS; ++s)
          if (issued_phase[s] >= 0)
            while (!ptx::mbar_try_wait(bar(bars->full[s]), (uint32_t)issued_phase[s]) &&
                   ptx::globaltimer() - t0 < ptx::kWaitLimitNs) {
            }
        if (q_issued_phase >= 0)
          while (!ptx::mbar_try_wait(bar(bars->qfull), (uint32_t)q_issued_phase) &&
                 ptx::globaltimer() - t0 < ptx::kWaitLimitNs) {
          }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      uint32_t cons = 0;            // ring slots consumed (production order)
      uint32_t scnt = 0;            // S tiles issued (buffer = scnt & 1)
      uint32_t pcnt[2] = {0u, 0u};  // pready completions consumed, per buffer
      uint32_t ic = 0;
      const uint32_t q_addr = base + OFF_Q;
      auto slot_wait = [&](uint32_t idx) -> bool {
        return ptx::mbar_wait(bar(bars->full[idx % SLOTS]), (idx / SLOTS) & 1u, abort_flag);
      };
      auto slot_addr = [&](uint32_t idx) { return base + OFF_SLOT + (idx % SLOTS) * TILE_BYTES; };
      // S[scnt & 1] = Q K^T, K in the next ring slot.  The buffer's previous
      // P was read by a P V issued earlier by this thread (in-order execution).
      auto issue_s = [&]() -> bool {
        const uint32_t idx = cons++;
        const uint32_t sb = scnt & 1u;
        if (!slot_wait(idx)) return false;
        ptx::tc_fence_after();
        const uint32_t k_addr = slot_addr(idx);
#pragma unroll
        for (int k = 0; k < HD / 16; ++k) {
          const uint32_t off = (uint32_t)(k >> 2) * HALF_BYTES + (uint32_t)(k & 3) * 32;
          ptx::mma_bf16_ts(tmem + TM_S0 + sb * 128, tmem + TM_Q + (uint32_t)(8 * k),
                           ptx::smem_desc(k_addr + off, 16, 1024), IDESC_S, k > 0 ? 1u : 0u);
        }
        ptx::mma_commit(bar(bars->sfull[sb]));
        ptx::mma_commit(bar(bars->empty[idx % SLOTS]));
        ++scnt;
        return true;
      };
      // O += P V: P (bf16) of the tile in buffer sb, keys 0-63 in columns 0-31
      // and keys 64-127 in columns 64-95; V in the next ring slot
      auto issue_pv = [&](uint32_t sb, bool first_tile) -> bool {
        if (!ptx::mbar_wait(bar(bars->pready[sb]), pcnt[sb] & 1u, abort_flag)) return false;
        ++pcnt[sb];
        const uint32_t idx = cons++;
        if (!slot_wait(idx)) return false;
        ptx::tc_fence_after();
        const uint32_t v_addr = slot_addr(idx);
#pragma unroll
        for (int k = 0; k < KT / 16; ++k) {
          ptx::mma_bf16_ts(tmem + TM_O,
                           tmem + TM_S0 + sb * 128 + (uint32_t)(64 * (k >> 2) + 8 * (k & 3)),
                           ptx::smem_desc(v_addr + (uint32_t)k * 2048, HALF_BYTES, 1024), IDESC_PV,
                           (first_tile && k == 0) ? 0u : 1u);
        }
        ptx::mma_commit(bar(bars->empty[idx % SLOTS]));
        return true;
      };
      // the next item's record is fetched while this one runs
      WorkItem wnext = fetch_item(p, first, n_items, snake_item(0, blockIdx.x, gridDim.x));
      for (int r = 0, it = snake_item(0, blockIdx.x, gridDim.x); it < n_items && !failed;
         ++r, it = snake_item(r, blockIdx.x, gridDim.x), ++ic) {
        const Item t = to_item(wnext);
        wnext = fetch_item(p, first, n_items, snake_item(r + 1, blockIdx.x, gridDim.x));
        if (!ptx::mbar_wait(bar(bars->qfull), ic & 1u, abort_flag)) {
          failed = true;
          break;
        }
        ptx::tc_fence_after();
        // Q: shared memory -> TMEM, one 16-column K slice per copy (in order
        // after the previous item's last S, before this item's first)
#pragma unroll
        for (int k = 0; k < HD / 16; ++k) {
          const uint32_t off = (uint32_t)(k >> 2) * HALF_BYTES + (uint32_t)(k & 3) * 32;
          ptx::tmem_cp_128x256b(tmem + TM_Q + (uint32_t)(8 * k),
                                ptx::smem_desc(q_addr + off, 16, 1024));
        }
        ptx::mma_commit(bar(bars->qfree));
        const uint32_t sb0 = scnt & 1u;
        if (!issue_s()) failed = true;
        if (!failed && t.ntiles > 1 && !issue_s()) failed = true;
        // the previous item's O must have been read out before P V overwrites it
        if (!failed && !ptx::mbar_wait(bar(bars->ofree), (ic & 1u) ^ 1u, abort_flag)) failed = true;
        for (int j = 0; j < t.ntiles && !failed; ++j) {
          if (!issue_pv((sb0 + (uint32_t)j) & 1u, j == 0)) failed = true;
          if (!failed && j + 2 < t.ntiles && !issue_s()) failed = true;
        }
        if (failed) break;
        ptx::mma_commit(bar(bars->ofull));
      }
      if (failed) {
        *abort_flag = 1;
        ptx::mma_commit(bar(bars->drain));
        const unsigned long long t0 = ptx::globaltimer();
        while (!ptx::mbar_try_wait(bar(bars->drain), 0u) &&
               ptx::globaltimer() - t0 < ptx::kWaitLimitNs) {
        }
      }
    }
  } else {
    // ---------------------------------------------------------- softmax warps
    const int sw = warp - 2;
    const int grp = sw >> 3;       // owns the S tiles in TMEM buffer grp
    const int hf = (sw >> 2) & 1;  // 64-column half of every tile
    const int quad = warp & 3;
    const int part = grp * 2 + hf;
    const int rl = quad * 32 + lane;  // query row inside the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const int col0 = CPW * hf;
    const uint32_t sbuf = tmem + TM_S0 + (uint32_t)grp * 128;
    float* ref = reinterpret_cast<float*>(smem + OFF_REF);    // [parity][half][128]
    float* lsum = reinterpret_cast<float*>(smem + OFF_LSUM);  // [parity][part][128]
    int* flags = reinterpret_cast<int*>(smem + OFF_FLAG);     // [item % 4]
    uint32_t gs = 0, ic = 0;  // global S tile index (the MMA warp's scnt)

    // the next item's record, field `lane` in lane `lane` (one register)
    auto fetch_field = [&](int idx) -> int {
      return (lane < 6 && idx < n_items)
                 ? __ldg(reinterpret_cast<const int*>(p.items + first + idx) + lane)
                 : 0;
    };
    int fnext = fetch_field(snake_item(0, blockIdx.x, gridDim.x));
    for (int r = 0, it = snake_item(0, blockIdx.x, gridDim.x); it < n_items && !failed;
         ++r, it = snake_item(r, blockIdx.x, gridDim.x), ++ic) {
      WorkItem wcur;
      wcur.seq = __shfl_sync(0xffffffffu, fnext, 0);
      wcur.tile_head = __shfl_sync(0xffffffffu, fnext, 1);
      wcur.q0 = __shfl_sync(0xffffffffu, fnext, 2);
      wcur.nrows = __shfl_sync(0xffffffffu, fnext, 3);
      wcur.k0 = __shfl_sync(0xffffffffu, fnext, 4);
      wcur.L = __shfl_sync(0xffffffffu, fnext, 5);
      const Item t = to_item(wcur);
      fnext = fetch_field(snake_item(r + 1, blockIdx.x, gridDim.x));
      const int par = (int)(ic & 1u);
      const bool row_ok = rl < t.nrows;
      float M = 0.f, l = 0.f, smax = -INFINITY;
      bool have_ref = false;
      for (int j = 0; j < t.ntiles; ++j) {
        const uint32_t s = gs + (uint32_t)j;
        if ((int)(s & 1u) != grp) continue;
        if (!ptx::mbar_wait(bar(bars->sfull[grp]), (s >> 1) & 1u, abort_flag)) {
          failed = true;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t scol = sbuf + lane_off + (uint32_t)col0;
        uint32_t sv[64];
        ptx::tmem_ld32(scol, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
        ptx::tmem_ld32(scol + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
        ptx::tmem_wait_ld();
        const int kmax = t.L - j * KT - col0;  // columns >= kmax are outside the sequence
        if (kmax < 64) {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (c >= kmax) sv[c] = __float_as_uint(-INFINITY);
        }
        float mx[4] = {__uint_as_float(sv[0]), __uint_as_float(sv[1]), __uint_as_float(sv[2]),
                       __uint_as_float(sv[3])};
#pragma unroll
        for (int c = 4; c < 64; ++c) mx[c & 3] = fmaxf(mx[c & 3], __uint_as_float(sv[c]));
        const float tmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
        smax = fmaxf(smax, tmax);
        if (j == 0) {  // the reference: the row's maximum over the first tile
          ref[(par * 2 + hf) * 128 + rl] = tmax;
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(bar(bars->refbar));
        }
        if (!have_ref) {
          if (!ptx::mbar_wait(bar(bars->refbar), ic & 1u, abort_flag)) {
            failed = true;
            break;
          }
          M = fmaxf(ref[(par * 2) * 128 + rl], ref[(par * 2 + 1) * 128 + rl]);
          have_ref = true;
        }
        // u = 2^(s - M) for keys inside the sequence and rows inside the tile,
        // 32 keys at a time, as bf16 pairs over the S columns already read (P
        // for the P V MMA)
        float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const float u0 = row_ok ? ex2(__uint_as_float(sv[32 * h2 + 2 * c]) - M) : 0.f;
            const float u1 = row_ok ? ex2(__uint_as_float(sv[32 * h2 + 2 * c + 1]) - M) : 0.f;
            ls[c & 3] += u0 + u1;
            pk[c] = pack_bf16(u0, u1);
          }
          ptx::tmem_st16(scol + 16 * h2, pk);
        }
        l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(bars->pready[grp]));
      }
      if (failed) break;
      gs += (uint32_t)t.ntiles;
      // ---- merge the row sums of the four (group, half) parts; any row out
      // of the safe band sends the whole item to the fallback
      if (have_ref && row_ok && smax - M > kBand) atomicOr(&flags[ic & 3u], 1);
      lsum[(par * PARTS + part) * 128 + rl] = l;
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(bars->statbar));
      if (!ptx::mbar_wait(bar(bars->statbar), ic & 1u, abort_flag)) {
        failed = true;
        break;
      }
      const bool bad = flags[ic & 3u] != 0;
      // the flag of item ic + 2 is written only after every warp has passed
      // the statbar of item ic + 1, i.e. after this clear
      if (sw == 0 && lane == 0) flags[(ic + 2) & 3u] = 0;
      const float* ls_par = lsum + par * PARTS * 128;
      const float Ls = ((ls_par[rl] + ls_par[128 + rl]) + ls_par[256 + rl]) + ls_par[384 + rl];
      // ---- O / l -> out: warp sw takes columns 32*(sw/4)..+31 of its rows
      if (!ptx::mbar_wait(bar(bars->ofull), ic & 1u, abort_flag)) {
        failed = true;
        break;
      }
      ptx::tc_fence_after();
      {
        const int ocol = 32 * (sw >> 2);
        uint32_t ov[32];
        ptx::tmem_ld32(tmem + lane_off + TM_O + (uint32_t)ocol, ov);
        ptx::tmem_wait_ld();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(bars->ofree));
        if (!bad && row_ok) {
          const float inv = 1.f / Ls;
          uint4* dst = reinterpret_cast<uint4*>(
              p.out + ((size_t)(t.q0 + t.qt * QT + rl) * p.H + t.h) * HD + ocol);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 w;
            w.x = pack_bf16(__uint_as_float(ov[8 * q + 0]) * inv, __uint_as_float(ov[8 * q + 1]) * inv);
            w.y = pack_bf16(__uint_as_float(ov[8 * q + 2]) * inv, __uint_as_float(ov[8 * q + 3]) * inv);
            w.z = pack_bf16(__uint_as_float(ov[8 * q + 4]) * inv, __uint_as_float(ov[8 * q + 5]) * inv);
            w.w = pack_bf16(__uint_as_float(ov[8 * q + 6]) * inv, __uint_as_float(ov[8 * q + 7]) * inv);
            dst[q] = w;
          }
        }
      }
      if (bad && sw == 0 && lane == 0) {
        const int slot = atomicAdd(&p.sched[3], 1);
        if (slot < p.max_fb) p.items_fb[slot] = p.items[first + it];
      }
    }
    if (failed) *abort_flag = 1;
  }

  __syncwarp();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (tid == 0 && bars->abort_flag) atomicOr(p.err, FC_DEVERR_TIMEOUT);
  if (warp == 1) ptx::tmem_dealloc(tmem, 512);
}

}  // namespace

size_t attn_onepass_smem_bytes() { return OFF_BARS + sizeof(Bars) + 1024; }

cudaError_t launch_attn_onepass(const fc_handle* h, cudaStream_t st, const CUtensorMap& tm_k,
                                const CUtensorMap& tm_v, const int32_t* cu_q, const int32_t* cu_k,
                                void* out) {
  OnePassParams p;
  p.H = h->cfg.n_heads;
  p.max_T = h->cfg.max_total_q;
  p.items = h->ws.items;
  p.cu_q = cu_q;
  p.cu_k = cu_k;
  p.out = (__nv_bfloat16*)out;
  p.sched = h->ws.sched;
  p.items_fb = h->ws.items_fb;
  p.max_fb = h->ws.max_items;
  p.err = h->ws.err;
  const size_t smem = attn_onepass_smem_bytes();
  cudaError_t e = smem_attr(attn_onepass_kernel, smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl_if(h->pdl, attn_onepass_kernel, dim3(h->num_sms), dim3(THREADS), smem, st, h->tm_q, tm_k,
                 tm_v, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace fc
