// Step preparation: validate the packed layout on the device, map every query
// row to its cache row, and build the attention work list.
//
// The cache row of query row r of sequence b is cu_seqlens_k[b] + q_pos[r]
// (Flash-Cache writes the refreshed K/V at the rows' absolute positions:
// infernews post "Flash-dLLM: IO-aware KV caching and parallel decoding",
// Flash-Cache paragraph).  Rows whose position is outside the sequence, or
// shared with another row of the same sequence, get -1 and are never written.
#include "fc_internal.h"
#include "ptx.cuh"

namespace fc {
namespace {

__device__ __forceinline__ void set_err(int32_t* err, int bits) { atomicOr(err, bits); }

// Sanity of sequence b's ranges; the same test is applied by every kernel
// that trusts cu_seqlens, so that a bad sequence is skipped consistently.
__device__ __forceinline__ bool seq_ok(const int32_t* cu_q, const int32_t* cu_k, int b, int B,
                                       int T, int S, int max_pos, int max_n) {
  int q0 = cu_q[b], q1 = cu_q[b + 1], k0 = cu_k[b], k1 = cu_k[b + 1];
  bool ok = q0 >= 0 && q0 <= q1 && q1 <= T && k0 >= 0 && k0 <= k1 && k1 <= S &&
            (k1 - k0) <= max_pos && (q1 - q0) <= max_n;
  if (b == 0) ok = ok && q0 == 0 && k0 == 0;
  if (b == B - 1) ok = ok && q1 == T && k1 == S;
  return ok;
}

// Blocks 0..B-1: one sequence each.  Block B: the work list.  Items of
// sequences whose cache spans more than long_tiles 128-key tiles come first
// (the list is ordered by cache length); sched[2] counts them: the two-pass
// attention kernel takes those, the one-pass kernel the rest.
//
// With split_sms > 0 (a small batch), every item is cut into
// ns = max(1, min(split_sms / items, 8, its key tiles / split_min_tiles))
// entries over nearly equal runs of key tiles, so that the entries fill up to
// split_sms CTAs and each keeps at least split_min_tiles tiles.  An entry
// records its key tiles [j0, j1) in pad[0] (j0 | j1 << 16) and its item's
// first entry and entry count in pad[1] (first | ns << 28); without a split,
// ns = 1 and [j0, j1) covers the whole cache.
__global__ void __launch_bounds__(512) prep_kernel(StepShape s, const int32_t* __restrict__ q_pos,
                                                   const int32_t* __restrict__ cu_q,
                                                   const int32_t* __restrict__ cu_k,
                                                   int32_t* __restrict__ row_dst,
                                                   WorkItem* __restrict__ items, int max_items,
                                                   int32_t* __restrict__ sched,
                                                   int32_t* __restrict__ err, int qtile,
                                                   int long_tiles, int split_sms,
                                                   int split_min_tiles) {
  extern __shared__ uint32_t smem[];
  const int b = blockIdx.x;
  const int tid = threadIdx.x, nt = blockDim.x;
  // the projection may start its main loop now; it waits for this grid before
  // its epilogue reads the row map
  ptx::griddep_launch_dependents();

  if (b < s.B) {
    const bool ok = seq_ok(cu_q, cu_k, b, s.B, s.T, s.S, s.max_pos, s.max_seqlen_q);
    int q0 = min(max(cu_q[b], 0), s.T), q1 = min(max(cu_q[b + 1], q0), s.T);
    if (!ok) {
      if (tid == 0) set_err(err, FC_DEVERR_SEQLENS);
      for (int r = q0 + tid; r < q1; r += nt) row_dst[r] = -1;
      return;
    }
    const int k0 = cu_k[b], L = cu_k[b + 1] - k0;
    const int words = (L + 31) >> 5;
    uint32_t* seen = smem;
    uint32_t* dup = smem + words;
    for (int i = tid; i < 2 * words; i += nt) smem[i] = 0u;
    __syncthreads();
    bool bad_range = false;
    for (int r = q0 + tid; r < q1; r += nt) {
      int p = q_pos[r];
      if (p < 0 || p >= L) {
        bad_range = true;
        continue;
      }
      uint32_t bit = 1u << (p & 31);
      if (atomicOr(&seen[p >> 5], bit) & bit) atomicOr(&dup[p >> 5], bit);
    }
    if (bad_range) set_err(err, FC_DEVERR_POS_RANGE);
    __syncthreads();
    bool any_dup = false;
    for (int r = q0 + tid; r < q1; r += nt) {
      int p = q_pos[r];
      int dst = -1;
      if (p >= 0 && p < L) {
        if (dup[p >> 5] & (1u << (p & 31)))
          any_dup = true;
        else
          dst = k0 + p;
      }
      row_dst[r] = dst;
    }
    if (any_dup) set_err(err, FC_DEVERR_POS_DUP);
    return;
  }

  // ---- work list: sequences by cache length descending (longest first), then
  // for each sequence its items ordered (head, query tile) so that the tiles
  // of one (sequence, head) that read the same K/V run close together.
  int n2 = 1;
  while (n2 < s.B) n2 <<= 1;
  unsigned long long* key = reinterpret_cast<unsigned long long*>(smem);
  int* cnt = reinterpret_cast<int*>(key + n2);  // [n2] items per sorted sequence, then offsets
  for (int i = tid; i < n2; i += nt) {
    unsigned long long k = 0ull;
    if (i < s.B) {
      bool ok = seq_ok(cu_q, cu_k, i, s.B, s.T, s.S, s.max_pos, s.max_seqlen_q);
      int n = ok ? cu_q[i + 1] - cu_q[i] : 0;
      int L = ok ? cu_k[i + 1] - cu_k[i] : 0;
      // valid sequences with rows sort before everything else, then by L desc, b asc
      unsigned long long live = (n > 0 && L > 0) ? 1ull : 0ull;
      k = (live << 63) | ((unsigned long long)(unsigned)L << 32) |
          (unsigned long long)(0xFFFFFFFFu - (unsigned)i);
    }
    key[i] = k;
  }
  __syncthreads();
  // bitonic sort, descending
  for (int size = 2; size <= n2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < n2; i += nt) {
        int j = i ^ stride;
        if (j > i) {
          bool desc = ((i & size) == 0);
          unsigned long long a = key[i], c = key[j];
          if (desc ? (a < c) : (a > c)) {
            key[i] = c;
            key[j] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  int* sseq = cnt + n2;   // [n2] sequence of each sorted slot
  int* snq = sseq + n2;   // [n2] query tiles of each sorted slot
  int* sns = snq + n2;    // [n2] entries per item of each sorted slot
  for (int i = tid; i < n2; i += nt) {
    int c = 0, bq = 0, nqt = 0;
    if (i < s.B && (key[i] >> 63)) {
      bq = (int)(0xFFFFFFFFu - (unsigned)(key[i] & 0xFFFFFFFFull));
      const int n = cu_q[bq + 1] - cu_q[bq];
      nqt = (n + qtile - 1) / qtile;
      c = s.H * nqt;
    }
    cnt[i] = c;
    sseq[i] = bq;
    snq[i] = nqt;
  }
  __syncthreads();
  if (tid < 32) {
    // entries per item: split the items of a small batch over the SMs
    int groups = 0;
    for (int i = tid; i < s.B; i += 32) groups += cnt[i];
    for (int o = 16; o > 0; o >>= 1) groups += __shfl_xor_sync(0xffffffffu, groups, o);
    int target = 1;
    if (split_sms > 0 && groups > 0) target = max(1, min(8, split_sms / groups));
    for (int i = tid; i < s.B; i += 32) {
      int ns = 1;
      if (cnt[i] > 0) {
        const int L = (int)((key[i] >> 32) & 0x7FFFFFFFull);
        ns = max(1, min(target, (L + 127) / 128 / max(split_min_tiles, 1)));
      }
      sns[i] = ns;
      cnt[i] *= ns;
    }
    __syncwarp();
    // exclusive scan of cnt[0 .. B) by one warp
    int carry = 0;
    for (int base = 0; base < s.B; base += 32) {
      const int i = base + tid;
      const int v = i < s.B ? cnt[i] : 0;
      int incl = v;
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (tid >= o) incl += u;
      }
      if (i < s.B) cnt[i] = carry + incl - v;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    __syncwarp();  // every lane's offsets are read below
    if (tid == 0) {
      int n_long = carry;  // offset of the first sequence within long_tiles
      for (int i = 0; i < s.B; ++i) {
        if (!(key[i] >> 63)) break;
        const int L = (int)((key[i] >> 32) & 0x7FFFFFFFull);
        if ((L + 127) / 128 <= long_tiles) {
          n_long = cnt[i];
          break;
        }
      }
      sched[0] = min(carry, max_items);
      sched[1] = 0;
      sched[2] = min(n_long, max_items);
      sched[3] = 0;
    }
  }
  __syncthreads();
  for (int i = 0; i < s.B; ++i) {
    if (!(key[i] >> 63)) break;
    const int bq = sseq[i], nqt = snq[i], ns = sns[i];
    const int c = s.H * nqt * ns;
    const int off = cnt[i];
    const int q0 = cu_q[bq], n = cu_q[bq + 1] - q0, k0 = cu_k[bq], L = cu_k[bq + 1] - k0;
    const int ntiles = (L + 127) / 128;
    for (int t = tid; t < c; t += nt) {
      const int g = t / ns, sp = t - g * ns;
      const int hh = g / nqt, qt = g - hh * nqt;
      const int j0 = sp * ntiles / ns, j1 = (sp + 1) * ntiles / ns;
      const int first = off + g * ns;
      if (off + t < max_items)
        items[off + t] = WorkItem{bq, (qt << 8) | hh, q0, min(qtile, n - qt * qtile), k0, L,
                                  {(int)((unsigned)j0 | ((unsigned)j1 << 16)),
                                   (int)((unsigned)first | ((unsigned)ns << 28))}};
    }
  }
}

}  // namespace

size_t prep_smem_bytes(int max_pos, int max_batch) {
  size_t bitmap = 2u * (size_t)((max_pos + 31) / 32) * sizeof(uint32_t);
  int n2 = 1;
  while (n2 < max_batch) n2 <<= 1;
  size_t sortb = (size_t)n2 * (sizeof(unsigned long long) + 4 * sizeof(int));
  return bitmap > sortb ? bitmap : sortb;
}

cudaError_t launch_prep(const fc_handle* h, cudaStream_t st, const StepShape& s,
                        const int32_t* q_pos, const int32_t* cu_q, const int32_t* cu_k,
                        int qtile, int long_tiles, int split_sms, int split_min_tiles) {
  size_t smem = prep_smem_bytes(h->cfg.max_pos, h->cfg.max_batch);
  if (smem > 48 * 1024) {
    cudaError_t e = smem_attr(prep_kernel, smem);
    if (e != cudaSuccess) return e;
  }
  prep_kernel<<<s.B + 1, 512, smem, st>>>(s, q_pos, cu_q, cu_k, h->ws.row_dst, h->ws.items,
                                           h->ws.max_items, h->ws.sched, h->ws.err, qtile,
                                           long_tiles, split_sms, split_min_tiles);
  return cudaGetLastError();
}

}  // namespace fc
