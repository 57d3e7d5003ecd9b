// Importance finalisation and tracked-set reselection.
//
// Flash-Cache keeps tracking the top-k decoded tokens ranked by attention
// importance (Flash-dLLM paper-digest page, Fig. 2 caption; infernews post
// "Flash-dLLM: IO-aware KV caching and parallel decoding", Flash-Cache
// paragraph: only newly decoded tokens and a few key positions chosen by
// attention importance are refreshed).
//
// topk_tracked: one CTA per sequence; up to 8192 candidates are staged in
// shared memory as keys.  An exact radix select (four 8-bit
// digits of an order-preserving 32-bit key) finds the k-th largest score; all
// larger scores are kept, equal ones in position order until k are kept, and
// the kept set is sorted by (score desc, position asc).  The result does not
// depend on thread timing.
//
// Small selections (k <= 64 from at most 8192 candidates, the usual case) take
// a path with five block barriers instead of about forty: each of the 16 warps
// takes a run of up to 512 candidates in blocks of 64 and keeps the 64 largest
// seen so far, in registers, as composite keys score << 32 | ~position (so
// ties go to the lower position).  The first block is sorted by a bitonic
// network as wide as the run needs (32 or 64 keys); of each later block only
// the keys above the current 64th largest can enter, and when there are at
// most 32 of them (the usual case once the running list has filled) they are
// packed into one register and sorted alone.  Lists longer than 128 per warp
// first merge every warp's first 64 keys: the 64th largest of those bounds
// the answer from below, and only later keys above it are gathered and
// sorted.  The warps' lists are then merged pairwise in four rounds.  Merging two sorted
// lists of 64: their elementwise maxima against the other list reversed are
// the 64 largest and form a bitonic sequence, sorted by one half-cleaner
// network.
#include "fc_internal.h"
#include "ptx.cuh"

namespace fc {
namespace {

__global__ void importance_finalize(int S, unsigned long long* __restrict__ acc,
                                    float* __restrict__ imp, int accumulate) {
  ptx::griddep_launch_dependents();
  ptx::griddep_wait();
  for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < S; j += gridDim.x * blockDim.x) {
    const double v = (double)(long long)acc[j] * kImpInvScale;
    const float f = (float)v;
    imp[j] = accumulate ? imp[j] + f : f;
    acc[j] = 0ull;
  }
}

// Order-preserving map float -> uint32 (larger float, larger key).
__device__ __forceinline__ uint32_t fkey(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ unsigned long long shfl_idx_u64(unsigned long long v, int src) {
  const uint32_t lo = __shfl_sync(0xffffffffu, (uint32_t)v, src);
  const uint32_t hi = __shfl_sync(0xffffffffu, (uint32_t)(v >> 32), src);
  return ((unsigned long long)hi << 32) | lo;
}

__device__ __forceinline__ unsigned long long shfl_xor_u64(unsigned long long v, int m) {
  const uint32_t lo = __shfl_xor_sync(0xffffffffu, (uint32_t)v, m);
  const uint32_t hi = __shfl_xor_sync(0xffffffffu, (uint32_t)(v >> 32), m);
  return ((unsigned long long)hi << 32) | lo;
}

// Sort the bitonic sequence of 64 keys m[0] (element lane), m[1] (element
// 32 + lane) descending: half-cleaner stages 32, 16, ..., 1.
__device__ __forceinline__ void warp_bitonic_merge64_desc(unsigned long long (&m)[2], int lane) {
  {
    const unsigned long long a = m[0], b = m[1];
    m[0] = a > b ? a : b;
    m[1] = a > b ? b : a;
  }
#pragma unroll
  for (int j = 16; j > 0; j >>= 1) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const unsigned long long o = shfl_xor_u64(m[r], j);
      const bool lower = (lane & j) == 0;
      m[r] = lower ? (m[r] > o ? m[r] : o) : (m[r] < o ? m[r] : o);
    }
  }
}

// Sort the warp's 32 * R keys descending; element e = 32 * r + lane is v[r].
template <int R>
__device__ __forceinline__ void warp_bitonic_desc(unsigned long long (&v)[R], int lane) {
#pragma unroll
  for (int size = 2; size <= 32 * R; size <<= 1) {
#pragma unroll
    for (int j = size >> 1; j > 0; j >>= 1) {
      if (j >= 32) {
        const int rj = j >> 5;
#pragma unroll
        for (int r = 0; r < R; ++r) {
          if (r & rj) continue;
          const bool desc = ((32 * r + lane) & size) == 0;
          const unsigned long long a = v[r], b = v[r | rj];
          const bool sw = desc ? (a < b) : (a > b);
          v[r] = sw ? b : a;
          v[r | rj] = sw ? a : b;
        }
      } else {
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const int e = 32 * r + lane;
          const bool desc = (e & size) == 0;
          const unsigned long long o = shfl_xor_u64(v[r], j);
          const bool lower = (lane & j) == 0;  // e is the lower index of the pair
          const bool keep_max = lower == desc;
          v[r] = keep_max ? (v[r] > o ? v[r] : o) : (v[r] < o ? v[r] : o);
        }
      }
    }
  }
}

constexpr int TK_THREADS = 512;
constexpr int TK_MAXK = 1024;
constexpr int TK_STAGE = 8192;  // candidate keys staged in shared memory (32 KiB)

__global__ void __launch_bounds__(TK_THREADS) topk_kernel(
    int B, const float* __restrict__ imp, const int32_t* __restrict__ cu_k,
    const int32_t* __restrict__ cand_lo, const int32_t* __restrict__ cand_hi,
    const int32_t* __restrict__ k_per_seq, int k, int32_t* __restrict__ tracked,
    int32_t* __restrict__ err, int S, int max_pos) {
  __shared__ uint32_t hist[256];
  __shared__ unsigned long long sel[TK_MAXK];
  __shared__ int sh_digit, sh_remaining, sh_nsel, sh_run;
  __shared__ int warp_cnt[TK_THREADS / 32];
  __shared__ uint32_t skey[TK_STAGE];

  const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int32_t* row = tracked + (size_t)b * k;
  ptx::griddep_wait();  // importance comes from the preceding step

  const int k0 = cu_k[b], k1 = cu_k[b + 1];
  const int lo = cand_lo[b], hi = cand_hi[b];
  const int kb = k_per_seq ? k_per_seq[b] : k;
  const int L = k1 - k0;
  const bool ok = k0 >= 0 && k0 <= k1 && k1 <= S && L <= max_pos && lo >= 0 && lo <= hi &&
                  hi <= L && kb >= 0 && kb <= k;
  if (!ok) {
    if (tid == 0) atomicOr(err, FC_DEVERR_CAND);
    for (int i = tid; i < k; i += TK_THREADS) row[i] = -1;
    return;
  }
  const int n = hi - lo;
  const int want = min(kb, n);
  const float* sc = imp + k0 + lo;
  // up to TK_STAGE candidates are read from global memory once, as keys
  const bool staged = n <= TK_STAGE;
  if (staged && want > 0) {
    // eight independent loads in flight per thread (the stage is read once)
    for (int base = 0; base < n; base += 8 * TK_THREADS) {
      float f[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = base + u * TK_THREADS + tid;
        f[u] = i < n ? __ldcg(sc + i) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = base + u * TK_THREADS + tid;
        if (i < n) skey[i] = fkey(f[u]);
      }
    }
    __syncthreads();
  }
  auto key_of = [&](int i) { return staged ? skey[i] : fkey(sc[i]); };

  if (staged && want > 0 && want <= 64) {
    // ---- small selection: per-warp register sorts, then a pairwise merge
    const int per = (n + TK_THREADS / 32 - 1) / (TK_THREADS / 32);  // candidates per warp, <= 512
    const int c0 = warp * per;
    unsigned long long run[2] = {0ull, 0ull};  // the warp's 64 largest so far, descending
    auto ckey = [&](int idx) -> unsigned long long {
      const int i = c0 + idx;
      return (idx < per && i < n)
                 ? ((unsigned long long)skey[i] << 32) | (0xFFFFFFFFu - (uint32_t)(lo + i))
                 : 0ull;  // below every candidate's composite key
    };
    // run = the 64 largest of run and the sorted list l0 (elements 0-31),
    // l1 (32-63): element 63 - e of the list sits in lane 31 - lane of the
    // other register
    auto merge_into_run = [&](unsigned long long l0, unsigned long long l1) {
      const unsigned long long r1 = shfl_xor_u64(l1, 31), r0 = shfl_xor_u64(l0, 31);
      unsigned long long m[2];
      m[0] = run[0] > r1 ? run[0] : r1;
      m[1] = run[1] > r0 ? run[1] : r0;
      warp_bitonic_merge64_desc(m, lane);
      run[0] = m[0];
      run[1] = m[1];
    };
    // first block of 64: a network only as wide as the warp's run needs
    if (per <= 32) {
      unsigned long long v[1] = {ckey(lane)};
      warp_bitonic_desc<1>(v, lane);
      run[0] = v[0];
    } else {
      unsigned long long v[2] = {ckey(lane), ckey(32 + lane)};
      warp_bitonic_desc<2>(v, lane);
      run[0] = v[0];
      run[1] = v[1];
    }
    unsigned long long* pack = sel + warp * 64;
    // the 64 largest of the 16 lists in sel (list w at w * 64), merged
    // pairwise in four rounds into list 0, in place: in round r, warp w merges
    // lists 2^(r+1) w and 2^(r+1) w + 2^r into the first of them (each list is
    // read by one warp, and each lane reads the elements it writes first)
    auto merge_lists = [&]() {
      for (int stride = 1; stride < TK_THREADS / 32; stride <<= 1) {
        if (2 * stride * warp < TK_THREADS / 32) {
          unsigned long long* A = sel + (2 * stride * warp) * 64;
          const unsigned long long* B = A + stride * 64;
          unsigned long long m[2];
          m[0] = A[lane] > B[63 - lane] ? A[lane] : B[63 - lane];
          m[1] = A[32 + lane] > B[31 - lane] ? A[32 + lane] : B[31 - lane];
          warp_bitonic_merge64_desc(m, lane);
          A[lane] = m[0];
          A[32 + lane] = m[1];
        }
        __syncthreads();
      }
    };
    if (per > 128) {
      // Long lists: the 64 largest of all warps' first blocks (G) bound the
      // answer from below: a later key at or below G's 64th cannot be
      // selected.  Each warp gathers its later keys above that (and above its
      // own running 64th largest) and sorts them 64 at a time; warp 0 adds G.
      pack[lane] = run[0];
      pack[32 + lane] = run[1];
      __syncthreads();
      merge_lists();
      const unsigned long long tau_g = sel[63];
      unsigned long long g[2] = {0ull, 0ull};
      if (warp == 0) {
        g[0] = sel[lane];
        g[1] = sel[32 + lane];
      }
      __syncthreads();  // G is read before the lists are reused as packs
      run[0] = run[1] = 0ull;
      int pcount = 0;
      auto flush = [&]() {
        unsigned long long x[2] = {lane < pcount ? pack[lane] : 0ull,
                                   32 + lane < pcount ? pack[32 + lane] : 0ull};
        __syncwarp();
        warp_bitonic_desc<2>(x, lane);
        merge_into_run(x[0], x[1]);
        pcount = 0;
      };
      for (int b0 = 64; b0 < per; b0 += 64) {
        unsigned long long thr = shfl_idx_u64(run[1], 31);
        if (thr < tau_g) thr = tau_g;
        unsigned long long v[2];
        uint32_t bal[2];
        int cnt = 0;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          v[r] = ckey(b0 + 32 * r + lane);
          bal[r] = __ballot_sync(0xffffffffu, v[r] > thr);
          cnt += __popc(bal[r]);
        }
        if (cnt == 0) continue;
        if (pcount + cnt > 64) flush();
        int off = pcount;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          if (v[r] > thr) pack[off + __popc(bal[r] & ((1u << lane) - 1u))] = v[r];
          off += __popc(bal[r]);
        }
        pcount = off;
        __syncwarp();
      }
      if (pcount > 0) flush();
      if (warp == 0) merge_into_run(g[0], g[1]);
    }
    // later blocks of 64 (lists of at most 128 per warp): only keys above the
    // current 64th largest can enter; up to 32 of them are packed into one
    // register (through this warp's slice of sel) and sorted alone, more are
    // sorted as the block of 64
    for (int b0 = 64; b0 < per && per <= 128; b0 += 64) {
      const unsigned long long tau = shfl_idx_u64(run[1], 31);  // the 64th largest so far
      unsigned long long v[2];
      uint32_t bal[2];
      int cnt = 0;
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        v[r] = ckey(b0 + 32 * r + lane);
        bal[r] = __ballot_sync(0xffffffffu, v[r] > tau);
        cnt += __popc(bal[r]);
      }
      if (cnt == 0) continue;
      if (cnt <= 32) {
        int off = 0;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          if (v[r] > tau) pack[off + __popc(bal[r] & ((1u << lane) - 1u))] = v[r];
          off += __popc(bal[r]);
        }
        __syncwarp();
        unsigned long long x[1] = {lane < cnt ? pack[lane] : 0ull};
        __syncwarp();
        warp_bitonic_desc<1>(x, lane);
        merge_into_run(x[0], 0ull);
      } else {
        warp_bitonic_desc<2>(v, lane);
        merge_into_run(v[0], v[1]);
      }
    }
    __syncwarp();
    pack[lane] = run[0];
    pack[32 + lane] = run[1];
    __syncthreads();
    merge_lists();
    for (int i = tid; i < k; i += TK_THREADS)
      row[i] = i < want ? (int32_t)(0xFFFFFFFFu - (uint32_t)(sel[i] & 0xFFFFFFFFull)) : -1;
    return;
  }

  // ---- radix select of the want-th largest key
  uint32_t prefix = 0u, mask = 0u;
  int remaining = want;  // how many still to take at or below the current prefix
  if (want > 0) {
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = tid; i < 256; i += TK_THREADS) hist[i] = 0u;
      __syncthreads();
      for (int i = tid; i < n; i += TK_THREADS) {
        const uint32_t key = key_of(i);
        if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 0xFFu], 1u);
      }
      __syncthreads();
      if (warp == 0) {
        // lane l scans digits 255-8l .. 248-8l (descending)
        uint32_t c[8], tot = 0;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          c[t] = hist[255 - 8 * lane - t];
          tot += c[t];
        }
        uint32_t incl = tot;
        for (int o = 1; o < 32; o <<= 1) {
          uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        const uint32_t excl = incl - tot;
        if ((int)excl < remaining && remaining <= (int)incl) {
          uint32_t run = excl;
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            if ((int)run < remaining && remaining <= (int)(run + c[t])) {
              sh_digit = 255 - 8 * lane - t;
              sh_remaining = remaining - (int)run;
            }
            run += c[t];
          }
        }
      }
      __syncthreads();
      prefix |= (uint32_t)sh_digit << shift;
      mask |= 0xFFu << shift;
      remaining = sh_remaining;
      __syncthreads();
    }
  }
  const uint32_t thr = prefix;  // key of the want-th largest score
  // `remaining` equal-to-thr candidates are kept, lowest positions first.

  if (tid == 0) {
    sh_nsel = 0;
    sh_run = 0;
  }
  __syncthreads();
  if (want > 0) {
    for (int base = 0; base < n; base += TK_THREADS) {
      const int i = base + tid;
      uint32_t key = 0u;
      bool gt = false, eq = false;
      if (i < n) {
        key = key_of(i);
        gt = key > thr;
        eq = key == thr;
      }
      const unsigned bal = __ballot_sync(0xffffffffu, eq);
      if (lane == 0) warp_cnt[warp] = __popc(bal);
      __syncthreads();
      int before = sh_run;
      for (int w = 0; w < warp; ++w) before += warp_cnt[w];
      before += __popc(bal & ((1u << lane) - 1u));
      const bool take = gt || (eq && before < remaining);
      if (take) {
        const int slot = atomicAdd(&sh_nsel, 1);
        if (slot < TK_MAXK)
          sel[slot] = ((unsigned long long)key << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)(lo + i));
      }
      __syncthreads();
      if (tid == 0) {
        int tot = 0;
        for (int w = 0; w < TK_THREADS / 32; ++w) tot += warp_cnt[w];
        sh_run += tot;
      }
      __syncthreads();
    }
  }
  // ---- sort the kept set: key desc, position asc (composite descending)
  int m2 = 1;
  while (m2 < want) m2 <<= 1;
  for (int i = want + tid; i < m2; i += TK_THREADS) sel[i] = 0ull;
  __syncthreads();
  for (int size = 2; size <= m2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < m2; i += TK_THREADS) {
        const int j = i ^ stride;
        if (j > i) {
          const bool desc = (i & size) == 0;
          const unsigned long long a = sel[i], c = sel[j];
          if (desc ? (a < c) : (a > c)) {
            sel[i] = c;
            sel[j] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int i = tid; i < k; i += TK_THREADS)
    row[i] = i < want ? (int32_t)(0xFFFFFFFFu - (uint32_t)(sel[i] & 0xFFFFFFFFull)) : -1;
}

}  // namespace

cudaError_t launch_importance_finalize(const fc_handle* h, cudaStream_t st, int S,
                                       float* importance, int accumulate) {
  if (S <= 0) return cudaSuccess;
  int blocks = (S + 255) / 256;
  if (blocks > h->num_sms * 8) blocks = h->num_sms * 8;
  cudaError_t e = launch_pdl_if(h->pdl, importance_finalize, dim3(blocks), dim3(256), 0, st, S, h->ws.imp_acc,
                             importance, accumulate);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_topk(const fc_handle* h, cudaStream_t st, int B, int S, const float* importance,
                        const int32_t* cu_k, const int32_t* cand_lo, const int32_t* cand_hi,
                        const int32_t* k_per_seq, int k, int32_t* tracked) {
  cudaError_t e = launch_pdl_if(h->pdl, topk_kernel, dim3(B), dim3(TK_THREADS), 0, st, B, importance, cu_k,
                             cand_lo, cand_hi, k_per_seq, k, tracked, h->ws.err, S, h->cfg.max_pos);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace fc
