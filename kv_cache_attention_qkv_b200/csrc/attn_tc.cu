// Bidirectional variable-length attention over the whole per-sequence KV
// cache on the tensor cores, with the per-key column sums of the attention
// probabilities ("attention importance") as a side output.
//
// Flash-dLLM (paper-digest page, Fig. 2 caption): the fixed-size query of a
// sequence attends bidirectionally to its full KV cache; the tracked positions
// are reselected by attention importance.  Queries of different lengths share
// one launch through block scheduling (infernews post "Flash-dLLM: IO-aware KV
// caching and parallel decoding", Flash-Cache paragraph).
//
// One work item = (sequence b, head h, 128-row query tile).  This kernel takes
// every item of a step that asks for importance, and in a step that does not,
// the items the one-pass kernel (attn_onepass.cu) handed over because a score
// left its safe exponent band.  The importance needs the final softmax
// normalisation of every row before columns are summed, so the cache is
// scanned twice:
//   pass 1: S = Q K^T per 128-key tile, row max m and sum l;
//   pass 2: S = Q K^T again, P = 2^(S - m - log2 l) (final probabilities),
//           O += P V on the tensor cores, column sums of P in registers.
// Q arrives pre-scaled by log2(e)/sqrt(d) from the projection epilogue, so
// scores are already in the exp2 domain.
//
// Operand placement: the tensor cores read their A operand from TMEM and only
// K and V (the B operands) from shared memory.  Q is copied once per item from
// shared memory into TMEM (tcgen05.cp); each tile's P is written (bf16) over the
// S tile it came from (tcgen05.st), so P V of tile j and S of tile j+1 use
// different buffers and the softmax never waits for the previous P V.  Keys
// 64h..64h+63 of a tile go, packed, to columns 64h..64h+31 of its buffer: every
// softmax warp overwrites only columns it has already read itself.
//
// Small batches (too few items to fill the SMs) split each item's cache
// across several work entries of the list (key tiles [j0, j1) each) and run
// the two passes as two launches of this kernel: mode 1 stores every entry's
// per-row (max, normaliser) over its key tiles; mode 2 combines the entries'
// statistics of the item into the row's log-sum-exp, runs pass 2 over its
// own tiles (column sums are complete, every key belongs to one entry) and
// stores its part of O (already normalised, fp32); the entry that finishes
// last sums the parts in entry order and writes the output, so the result
// does not depend on which CTA finishes first.  Mode 0 is the fused kernel.
//
// TMEM columns: S/P buffer 0 [0,128), S/P buffer 1 [128,256), O [256,384),
// Q [384,448).
//
// Roles (one CTA per SM, persistent over the work list):
//   warp 0      TMA producer: Q tile, then K tiles (pass 1), then K and V
//               tiles (pass 2) into a ring of four 32 KiB slots;
//   warp 1      TMEM allocation, Q copy and tcgen05.mma issue (S runs two
//               tiles ahead of P V);
//   warps 2-17  softmax, two groups of eight that take S tiles alternately
//               (group g owns the tiles in TMEM buffer g), so one group's
//               exp2 work overlaps the other's hand-off to the tensor cores.
//               In a group, warp w owns TMEM lane quadrant w % 4 (32 query
//               rows, one per thread) and one 64-column half of the tile.
//               Row statistics of the four (group, half) parts are merged once
//               per item through shared memory; column sums are reduced across
//               the warp with shuffles, across the four row quadrants in
//               shared memory (2^-40 fixed point), and added to the global
//               importance accumulator.
#include <cuda_bf16.h>

#include "fc_internal.h"
#include "ptx.cuh"

namespace fc {
namespace {

constexpr int QT = 128, KT = 128, HD = 128;
constexpr int SLOTS = 4;
constexpr int SOFTMAX_WARPS = 16;  // two groups of 8
constexpr int PARTS = 4;           // (group, column half) partial row statistics
constexpr int CPW = KT / 2;        // columns per softmax warp and tile
constexpr int THREADS = 64 + 32 * SOFTMAX_WARPS;
constexpr uint32_t HALF_BYTES = 128 * 128;       // 128 rows x 64 bf16
constexpr uint32_t TILE_BYTES = 2 * HALF_BYTES;  // 128 rows x 128 bf16
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_SLOT = TILE_BYTES;
// column sums, int64 [group][tile parity within the group][128]: a warp can
// reach its group's next tile before the quadrant that flushes this one has
// finished, but not the tile after (that S waits for this warp's own P).
constexpr uint32_t OFF_CSACC = OFF_SLOT + SLOTS * TILE_BYTES;
constexpr uint32_t OFF_CSCNT = OFF_CSACC + 4 * 128 * 8;  // [group][parity][half] arrival counts
constexpr uint32_t OFF_STAT = OFF_CSCNT + 64;
constexpr uint32_t STAT_BYTES = 2 * PARTS * 2 * 128 * 4;  // [parity][part][m, l][row]
constexpr uint32_t OFF_BARS = OFF_STAT + STAT_BYTES;
// TMEM columns
constexpr uint32_t TM_S0 = 0, TM_O = 256, TM_Q = 384;

constexpr uint32_t IDESC_S = ptx::idesc_bf16_f32(128, 128, 0, 0);   // Q K^T, K K-major
constexpr uint32_t IDESC_PV = ptx::idesc_bf16_f32(128, 128, 0, 1);  // P V, V MN-major

struct AttnParams {
  int H, max_T;
  const WorkItem* items;     // the work list: its first sched[2] items come here
  const WorkItem* items_fb;  // then the sched[3] items the one-pass kernel handed over
  int max_fb;
  const int32_t* sched;
  const int32_t* cu_q;
  const int32_t* cu_k;
  __nv_bfloat16* out;
  unsigned long long* imp_acc;
  int want_imp;
  float* stats;  // [entry][m, l][128] row statistics of the entries (modes 1, 2)
  float* opart;  // [entry][128 columns][128 rows] fp32 parts of O of split items (mode 2)
  int32_t* gcnt; // [first entry of an item] entries of the item done (mode 2)
  int max_entries;
  int32_t* err;
};

struct __align__(8) AttnBars {
  unsigned long long qfull, qfree;
  unsigned long long full[SLOTS], empty[SLOTS];
  unsigned long long sfull[2], sfree[2];
  unsigned long long pready[2];
  unsigned long long ofull, ofree;
  unsigned long long statbar;
  unsigned long long obar, obar2;  // split items: parts of O stored / last-entry flag set
  unsigned long long drain;
  uint32_t tmem_base;
  int abort_flag;
};

struct Item {
  int b, qt, h, q0, nrows, k0, L;
  int j0, j1;     // this entry's key tiles
  int first, ns;  // the item's first entry in the list and its entry count
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
  r.j0 = (int)((unsigned)w.pad[0] & 0xFFFFu);
  r.j1 = (int)((unsigned)w.pad[0] >> 16);
  r.first = (int)((unsigned)w.pad[1] & 0x0FFFFFFFu);
  r.ns = (int)((unsigned)w.pad[1] >> 28);
  return r;
}

// Address of item `it` of this kernel's list: the long items, then the
// handed-over ones.
__device__ __forceinline__ const WorkItem* item_ptr(const AttnParams& p, int n_long, int it) {
  return it < n_long ? p.items + it : p.items_fb + (it - n_long);
}

__device__ __forceinline__ WorkItem fetch_item(const AttnParams& p, int n_long, int n, int it) {
  WorkItem w = {};
  if (it < n) w = *item_ptr(p, n_long, it);
  return w;
}

// Tiled 3-D TMA load with an L2 eviction-priority policy (createpolicy).
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* tm, int x, int y,
                                            int z, uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(z), "r"(bar), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
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

template <int MODE>
__global__ void __launch_bounds__(THREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = ptx::smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  AttnBars* bars = reinterpret_cast<AttnBars*>(smem + OFF_BARS);
  volatile int* abort_flag = &bars->abort_flag;
  auto bar = [](unsigned long long& b) { return ptx::smem_u32(&b); };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  ptx::griddep_launch_dependents();

  for (int i = tid; i < 4 * 128; i += THREADS)
    reinterpret_cast<unsigned long long*>(smem + OFF_CSACC)[i] = 0ull;
  if (tid < 8) reinterpret_cast<int*>(smem + OFF_CSCNT)[tid] = 0;
  if (tid == 0) {
    ptx::mbar_init(bar(bars->qfull), 1);
    ptx::mbar_init(bar(bars->qfree), 1);
    for (int s = 0; s < SLOTS; ++s) {
      ptx::mbar_init(bar(bars->full[s]), 1);
      ptx::mbar_init(bar(bars->empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(bar(bars->sfull[s]), 1);
      ptx::mbar_init(bar(bars->sfree[s]), SOFTMAX_WARPS / 2);  // the owning group
      ptx::mbar_init(bar(bars->pready[s]), SOFTMAX_WARPS / 2);
    }
    ptx::mbar_init(bar(bars->ofull), 1);
    ptx::mbar_init(bar(bars->ofree), SOFTMAX_WARPS);
    ptx::mbar_init(bar(bars->statbar), SOFTMAX_WARPS);
    ptx::mbar_init(bar(bars->obar), SOFTMAX_WARPS);
    ptx::mbar_init(bar(bars->obar2), 1);
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
  const int n_long = p.sched[2];
  const int n_items = n_long + min(p.sched[3], p.max_fb);

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------- producer
      uint32_t prod = 0;  // slot production counter
      int issued_phase[SLOTS];
      for (int s = 0; s < SLOTS; ++s) issued_phase[s] = -1;
      int q_issued_phase = -1;
      uint32_t ic = 0;
      // K is read again by pass 2 of the same item: keep it in L2 over V,
      // which (like the second read of K) is read once and streams through.
      const uint64_t pol_keep = policy_evict_last(), pol_stream = policy_evict_first();
      auto load_tile = [&](const CUtensorMap* tm, int h, int row, uint64_t pol) -> bool {
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
      WorkItem wnext = fetch_item(p, n_long, n_items, snake_item(0, blockIdx.x, gridDim.x));
      for (int r = 0, it = snake_item(0, blockIdx.x, gridDim.x); it < n_items && !failed;
         ++r, it = snake_item(r, blockIdx.x, gridDim.x), ++ic) {
        const Item t = to_item(wnext);
        wnext = fetch_item(p, n_long, n_items, snake_item(r + 1, blockIdx.x, gridDim.x));
        if (!ptx::mbar_wait(bar(bars->qfree), (ic & 1u) ^ 1u, abort_flag)) {
          failed = true;
          break;
        }
        ptx::mbar_arrive_expect_tx(bar(bars->qfull), TILE_BYTES);
        const int qrow = t.h * p.max_T + t.q0 + t.qt * QT;
        ptx::tma_load_2d(base + OFF_Q, &tm_q, 0, qrow, bar(bars->qfull));
        ptx::tma_load_2d(base + OFF_Q + HALF_BYTES, &tm_q, 64, qrow, bar(bars->qfull));
        q_issued_phase = (int)(ic & 1u);
        if (MODE != 2)
          for (int j = t.j0; j < t.j1 && !failed; ++j) {
            if (!load_tile(&tm_k, t.h, t.k0 + j * KT, pol_keep)) failed = true;
          }
        if (MODE != 1)
          for (int j = t.j0; j < t.j1 && !failed; ++j) {
            if (!load_tile(&tm_k, t.h, t.k0 + j * KT, pol_stream) ||
                !load_tile(&tm_v, t.h, t.k0 + j * KT, pol_stream))
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
      uint32_t cons = 0;  // slot consumption index base (production order)
      uint32_t scnt = 0;  // S tiles issued
      uint32_t pcnt[2] = {0u, 0u};  // pready completions consumed, per buffer
      uint32_t ic = 0;
      const uint32_t q_addr = base + OFF_Q;
      auto slot_wait = [&](uint32_t idx) -> bool {
        return ptx::mbar_wait(bar(bars->full[idx % SLOTS]), (idx / SLOTS) & 1u, abort_flag);
      };
      auto slot_addr = [&](uint32_t idx) { return base + OFF_SLOT + (idx % SLOTS) * TILE_BYTES; };
      // S[buffer] = Q K^T for the K tile in production slot idx (Q from TMEM)
      auto issue_s = [&](uint32_t idx) -> bool {
        const uint32_t sb = scnt & 1u;
        if (!ptx::mbar_wait(bar(bars->sfree[sb]), ((scnt >> 1) & 1u) ^ 1u, abort_flag)) return false;
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
      // O += P V: P (bf16) of pass-2 tile j sits in columns 0-31 (keys 0-63)
      // and 64-95 (keys 64-127) of its S buffer, V in production slot idx
      auto issue_pv = [&](uint32_t idx, uint32_t sb, bool first) -> bool {
        if (!ptx::mbar_wait(bar(bars->pready[sb]), pcnt[sb] & 1u, abort_flag)) return false;
        ++pcnt[sb];
        if (!slot_wait(idx)) return false;
        ptx::tc_fence_after();
        const uint32_t v_addr = slot_addr(idx);
#pragma unroll
        for (int k = 0; k < KT / 16; ++k) {
          // A = P from TMEM (keys are K); B = V (MN-major: d contiguous)
          ptx::mma_bf16_ts(tmem + TM_O, tmem + TM_S0 + sb * 128 + (uint32_t)(64 * (k >> 2) + 8 * (k & 3)),
                           ptx::smem_desc(v_addr + (uint32_t)k * 2048, HALF_BYTES, 1024), IDESC_PV,
                           (first && k == 0) ? 0u : 1u);
        }
        ptx::mma_commit(bar(bars->empty[idx % SLOTS]));
        return true;
      };
      // the next item's record is fetched while this one runs
      WorkItem wnext = fetch_item(p, n_long, n_items, snake_item(0, blockIdx.x, gridDim.x));
      for (int r = 0, it = snake_item(0, blockIdx.x, gridDim.x); it < n_items && !failed;
         ++r, it = snake_item(r, blockIdx.x, gridDim.x), ++ic) {
        const Item t = to_item(wnext);
        wnext = fetch_item(p, n_long, n_items, snake_item(r + 1, blockIdx.x, gridDim.x));
        if (!ptx::mbar_wait(bar(bars->qfull), ic & 1u, abort_flag)) {
          failed = true;
          break;
        }
        ptx::tc_fence_after();
        // Q: shared memory -> TMEM, one 16-column K slice per copy.  Copies and
        // MMAs issued by this thread execute in order, so the copy cannot
        // overtake the previous item's last S, and this item's S follows it.
#pragma unroll
        for (int k = 0; k < HD / 16; ++k) {
          const uint32_t off = (uint32_t)(k >> 2) * HALF_BYTES + (uint32_t)(k & 3) * 32;
          ptx::tmem_cp_128x256b(tmem + TM_Q + (uint32_t)(8 * k),
                                ptx::smem_desc(q_addr + off, 16, 1024));
        }
        ptx::mma_commit(bar(bars->qfree));  // the shared-memory copy of Q is free again
        const int nt = t.j1 - t.j0;
        // pass 1: S tiles only
        if (MODE != 2)
          for (int j = 0; j < nt && !failed; ++j)
            if (!issue_s(cons + (uint32_t)j)) failed = true;
        if (failed) break;
        const uint32_t base2 = cons + (MODE != 2 ? (uint32_t)nt : 0u);
        if (MODE == 1) {
          cons = base2;
          continue;
        }
        const uint32_t sb0 = scnt & 1u;  // buffer of pass-2 tile 0
        // the previous item's O must have been read out before P V overwrites it
        if (!ptx::mbar_wait(bar(bars->ofree), (ic & 1u) ^ 1u, abort_flag)) {
          failed = true;
          break;
        }
        // S runs two tiles ahead of P V; S[j+2] reuses tile j's buffer and is
        // queued right after P V [j], which reads P[j] from that buffer
        const int lead = nt < 2 ? nt : 2;
        for (int j = 0; j < lead && !failed; ++j)
          if (!issue_s(base2 + 2u * (uint32_t)j)) failed = true;
        for (int j = 0; j < nt && !failed; ++j) {
          if (!issue_pv(base2 + 2u * (uint32_t)j + 1u, (sb0 + (uint32_t)j) & 1u, j == 0)) {
            failed = true;
            break;
          }
          if (j + 2 < nt && !issue_s(base2 + 2u * (uint32_t)(j + 2))) failed = true;
        }
        if (failed) break;
        ptx::mma_commit(bar(bars->ofull));
        cons = base2 + 2u * (uint32_t)nt;
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
    const int grp = sw >> 3;            // owns the S tiles in TMEM buffer grp
    const int hf = (sw >> 2) & 1;       // 64-column half of every tile
    const int quad = warp & 3;
    const int part = grp * 2 + hf;      // index of this warp's partial statistics
    const int rl = quad * 32 + lane;    // query row inside the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const int col0 = CPW * hf;
    const uint32_t sbuf = tmem + TM_S0 + (uint32_t)grp * 128;
    float* stat = reinterpret_cast<float*>(smem + OFF_STAT);  // [parity][part][m, l][row]
    unsigned long long* cs_base =
        reinterpret_cast<unsigned long long*>(smem + OFF_CSACC) + grp * 256 + col0;
    int* cnt_base = reinterpret_cast<int*>(smem + OFF_CSCNT) + grp * 4 + hf;
    uint32_t gs = 0, ic = 0;  // global S tile index (same sequence as the MMA warp)
    uint32_t oc = 0;          // split items finished (obar / obar2 phases)

    // This thread's 64 columns of S tile `s` (buffer grp); the buffer is
    // released to the MMA warp at once.
    auto load_s = [&](uint32_t s, uint32_t (&sv)[64]) -> bool {
      if (!ptx::mbar_wait(bar(bars->sfull[grp]), (s >> 1) & 1u, abort_flag)) return false;
      ptx::tc_fence_after();
      ptx::tmem_ld32(sbuf + lane_off + (uint32_t)col0, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
      ptx::tmem_ld32(sbuf + lane_off + (uint32_t)col0 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
      ptx::tmem_wait_ld();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(bars->sfree[grp]));
      return true;
    };
    // Column sums of 32 rows x 32 columns held one row per lane: recursive
    // halving (stages 0-4, run here from st0 to st1 - 1) leaves column `lane`
    // in v[0].
    auto warp_colsum = [&](float* v, int st0, int st1) -> float {
#pragma unroll
      for (int st = st0; st < st1; ++st) {
        const int o = 16 >> st;
        const int hn = 16 >> st;
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < hn; ++i) {
          const float send = upper ? v[i] : v[i + hn];
          const float keep = upper ? v[i + hn] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
      }
      return v[0];
    };

    // the next item's record, field `lane` in lane `lane` (one register)
    auto fetch_field = [&](int it) -> int {
      return (lane < 8 && it < n_items)
                 ? __ldg(reinterpret_cast<const int*>(item_ptr(p, n_long, it)) + lane)
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
      wcur.pad[0] = __shfl_sync(0xffffffffu, fnext, 6);
      wcur.pad[1] = __shfl_sync(0xffffffffu, fnext, 7);
      const Item t = to_item(wcur);
      fnext = fetch_field(snake_item(r + 1, blockIdx.x, gridDim.x));
      uint32_t sv[64];
      const int nt = t.j1 - t.j0;
      float M = -INFINITY, Ls = 0.f;  // the row's maximum and normaliser (all its keys)
      if (MODE != 2) {
      // ---- pass 1: max and normaliser over this warp's tiles and column half
      float m = -INFINITY, l = 0.f;
      for (int jj = 0; jj < nt; ++jj) {
        const uint32_t s = gs + (uint32_t)jj;
        if ((int)(s & 1u) != grp) continue;
        if (!load_s(s, sv)) {
          failed = true;
          break;
        }
        const int j = t.j0 + jj;
        const int kmax = t.L - j * KT - col0;  // columns >= kmax are outside the sequence
        if (kmax <= 0) continue;
        float x[64];
#pragma unroll
        for (int c = 0; c < 64; ++c) x[c] = __uint_as_float(sv[c]);
        if (kmax < 64) {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (c >= kmax) x[c] = -INFINITY;
        }
        float mx[4] = {x[0], x[1], x[2], x[3]};
#pragma unroll
        for (int c = 4; c < 64; ++c) mx[c & 3] = fmaxf(mx[c & 3], x[c]);
        const float mn = fmaxf(m, fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])));
        float sm[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < 64; ++c) sm[c & 3] += ex2(x[c] - mn);
        l = (m == -INFINITY ? 0.f : l * ex2(m - mn)) + ((sm[0] + sm[1]) + (sm[2] + sm[3]));
        m = mn;
      }
      if (failed) break;
      gs += (uint32_t)nt;
      // merge the four (group, half) parts of every row once per item
      float* st_par = stat + (ic & 1u) * (PARTS * 256);
      st_par[part * 256 + rl] = m;
      st_par[part * 256 + 128 + rl] = l;
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(bars->statbar));
      if (!ptx::mbar_wait(bar(bars->statbar), ic & 1u, abort_flag)) {
        failed = true;
        break;
      }
#pragma unroll
      for (int q = 0; q < PARTS; ++q) M = fmaxf(M, st_par[q * 256 + rl]);
#pragma unroll
      for (int q = 0; q < PARTS; ++q) {
        const float mq = st_par[q * 256 + rl];
        if (mq != -INFINITY) Ls += st_par[q * 256 + 128 + rl] * ex2(mq - M);
      }
      if (MODE == 1) {  // this entry's statistics for the pass-2 launch
        const int entry = it;
        if (part == 0 && entry < p.max_entries) {
          p.stats[(size_t)entry * 256 + rl] = M;
          p.stats[(size_t)entry * 256 + 128 + rl] = Ls;
        }
        continue;
      }
      } else {
        // the statistics of the item's entries (stored by the mode-1 launch),
        // all loaded before they are combined in entry order
        float me[8], le[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int entry = t.first + e;
          const bool ok = e < t.ns && entry < p.max_entries;
          me[e] = ok ? __ldcg(p.stats + (size_t)entry * 256 + rl) : -INFINITY;
          le[e] = ok ? __ldcg(p.stats + (size_t)entry * 256 + 128 + rl) : 0.f;
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) M = fmaxf(M, me[e]);
#pragma unroll
        for (int e = 0; e < 8; ++e)
          if (me[e] != -INFINITY) Ls += le[e] * ex2(me[e] - M);
      }
      // rows past the query tile's end get lse = +inf, i.e. P = 0
      const float lse = rl < t.nrows ? M + __log2f(Ls) : INFINITY;
      // ---- pass 2: final probabilities -> P (TMEM, over its S tile); column sums
      for (int jj = 0; jj < nt; ++jj) {
        const uint32_t s = gs + (uint32_t)jj;
        if ((int)(s & 1u) != grp) continue;
        const uint32_t scol = sbuf + lane_off + (uint32_t)col0;
        const int j = t.j0 + jj;
        const int kmax = t.L - j * KT - col0;  // columns >= kmax are outside the sequence
        if (!ptx::mbar_wait(bar(bars->sfull[grp]), (s >> 1) & 1u, abort_flag)) {
          failed = true;
          break;
        }
        ptx::tc_fence_after();
        uint32_t* sa = &sv[0];
        uint32_t* sb = &sv[32];
        ptx::tmem_ld32(scol, *reinterpret_cast<uint32_t(*)[32]>(sa));
        ptx::tmem_wait_ld();
        // keys col0..col0+31 -> packed columns col0..col0+15 (already read)
        float pv[32];
        auto probs = [&](const uint32_t* x, int lim) {
          if (lim >= 32) {
#pragma unroll
            for (int c = 0; c < 32; ++c) pv[c] = ex2(__uint_as_float(x[c]) - lse);
          } else {
#pragma unroll
            for (int c = 0; c < 32; ++c) pv[c] = c < lim ? ex2(__uint_as_float(x[c]) - lse) : 0.f;
          }
        };
        auto store_p = [&](uint32_t col) {
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) pk[c] = pack_bf16(pv[2 * c], pv[2 * c + 1]);
          ptx::tmem_st16(col, pk);
        };
        probs(sa, kmax);
        store_p(scol);
        // column sums of this warp's first 32 keys: the first halving step
        // frees half of the registers, the rest overlaps the second load
        if (p.want_imp) warp_colsum(pv, 0, 1);
        ptx::tmem_ld32(scol + 32, *reinterpret_cast<uint32_t(*)[32]>(sb));
        const int par = (int)((s >> 1) & 1u);
        unsigned long long* cs_acc = cs_base + par * 128;
        if (p.want_imp) {
          const float c0 = warp_colsum(pv, 1, 5);
          atomicAdd(&cs_acc[lane], (unsigned long long)__double2ll_rn((double)c0 * kImpScale));
        }
        ptx::tmem_wait_ld();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(bars->sfree[grp]));  // S tile fully read
        // keys col0+32..col0+63 -> packed columns col0+16..col0+31
        probs(sb, kmax - 32);
        store_p(scol + 16);
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(bars->pready[grp]));
        if (p.want_imp) {
          const float c1 = warp_colsum(pv, 0, 5);
          atomicAdd(&cs_acc[32 + lane], (unsigned long long)__double2ll_rn((double)c1 * kImpScale));
          // the last of the four row quadrants adds the tile's sums to the keys
          int* cs_cnt = cnt_base + par * 2;
          __threadfence_block();
          __syncwarp();
          int last = 0;
          if (lane == 0) last = atomicAdd(cs_cnt, 1) == 3;
          last = __shfl_sync(0xffffffffu, last, 0);
          if (last) {
            __threadfence_block();
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const unsigned long long fx = atomicExch(&cs_acc[32 * e + lane], 0ull);
              const int key = j * KT + col0 + 32 * e + lane;
              if (key < t.L && fx != 0ull) atomicAdd(&p.imp_acc[t.k0 + key], fx);
            }
            if (lane == 0) *cs_cnt = 0;
          }
        }
      }
      if (failed) break;
      gs += (uint32_t)nt;
      // ---- O (already normalised) -> out: warp sw takes columns 32*(sw/4)..+31
      if (!ptx::mbar_wait(bar(bars->ofull), ic & 1u, abort_flag)) {
        failed = true;
        break;
      }
      ptx::tc_fence_after();
      const int ocol = 32 * (sw >> 2);
      ptx::tmem_ld32(tmem + lane_off + TM_O + (uint32_t)ocol, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
      ptx::tmem_wait_ld();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(bars->ofree));
      if (MODE == 2 && t.ns > 1) {
        // a split item: store this entry's part; the item's last entry to
        // finish adds the parts in entry order and writes the output
        // layout [entry][column][row]: a warp's 32 rows of one column are
        // 128 contiguous bytes
        const int entry = it;
        const bool in_ws = entry < p.max_entries && t.first + t.ns <= p.max_entries;
        auto part_at = [&](int e) { return p.opart + ((size_t)e * HD + ocol) * QT + rl; };
        if (rl < t.nrows && in_ws) {
          float* op = part_at(entry);
#pragma unroll
          for (int c = 0; c < 32; ++c) __stcg(op + c * QT, __uint_as_float(sv[c]));
        }
        __threadfence();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(bars->obar));
        volatile int* last_flag = reinterpret_cast<volatile int*>(smem + OFF_CSCNT) + 8;
        if (sw == 0 && lane == 0) {
          int last = 0;
          if (ptx::mbar_wait(bar(bars->obar), oc & 1u, abort_flag)) {
            __threadfence();
            if (in_ws) last = atomicAdd(&p.gcnt[t.first], 1) == t.ns - 1;
            __threadfence();
          } else {
            *abort_flag = 1;
          }
          *last_flag = last;
          ptx::mbar_arrive(bar(bars->obar2));
        }
        if (!ptx::mbar_wait(bar(bars->obar2), oc & 1u, abort_flag)) {
          failed = true;
          break;
        }
        ++oc;
        if (*last_flag) {
          __threadfence();
          if (rl < t.nrows) {
            // parts in entry order; this entry's own part from its registers
            float acc[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) acc[c] = 0.f;
            for (int e = t.first; e < t.first + t.ns; ++e) {
              if (e == entry) {
#pragma unroll
                for (int c = 0; c < 32; ++c) acc[c] += __uint_as_float(sv[c]);
              } else {
                const float* src = part_at(e);
#pragma unroll
                for (int c = 0; c < 32; ++c) acc[c] += __ldcg(src + c * QT);
              }
            }
#pragma unroll
            for (int c = 0; c < 32; ++c) sv[c] = __float_as_uint(acc[c]);
          }
          if (sw == 0 && lane == 0) p.gcnt[t.first] = 0;  // for the next launch
        } else {
          continue;
        }
      }
      if (rl < t.nrows) {
        uint4* dst = reinterpret_cast<uint4*>(
            p.out + ((size_t)(t.q0 + t.qt * QT + rl) * p.H + t.h) * HD + ocol);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 w;
          w.x = pack_bf16(__uint_as_float(sv[8 * q + 0]), __uint_as_float(sv[8 * q + 1]));
          w.y = pack_bf16(__uint_as_float(sv[8 * q + 2]), __uint_as_float(sv[8 * q + 3]));
          w.z = pack_bf16(__uint_as_float(sv[8 * q + 4]), __uint_as_float(sv[8 * q + 5]));
          w.w = pack_bf16(__uint_as_float(sv[8 * q + 6]), __uint_as_float(sv[8 * q + 7]));
          dst[q] = w;
        }
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

size_t attn_tc_smem_bytes() { return OFF_BARS + sizeof(AttnBars) + 1024; }

cudaError_t launch_attn_tc(const fc_handle* h, cudaStream_t st, const StepShape& s,
                           const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                           const int32_t* cu_q, const int32_t* cu_k, void* out,
                           bool want_importance, int mode) {
  AttnParams p;
  p.H = s.H;
  p.max_T = h->cfg.max_total_q;
  p.items = h->ws.items;
  p.items_fb = h->ws.items_fb;
  p.max_fb = h->ws.max_items;
  p.sched = h->ws.sched;
  p.cu_q = cu_q;
  p.cu_k = cu_k;
  p.out = (__nv_bfloat16*)out;
  p.imp_acc = h->ws.imp_acc;
  p.want_imp = want_importance ? 1 : 0;
  p.stats = h->ws.split_stats;
  p.opart = h->ws.split_o;
  p.gcnt = h->ws.split_cnt;
  p.max_entries = h->ws.split_entries;
  p.err = h->ws.err;
  // mode 0 both passes, 1 pass 1 only (row statistics), 2 pass 2 only
  auto kernel = mode == 1 ? attn_tc_kernel<1> : mode == 2 ? attn_tc_kernel<2> : attn_tc_kernel<0>;
  const size_t smem = attn_tc_smem_bytes();
  cudaError_t e = smem_attr(kernel, smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl_if(h->pdl, kernel, dim3(h->num_sms), dim3(THREADS), smem, st, h->tm_q, tm_k, tm_v, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace fc
