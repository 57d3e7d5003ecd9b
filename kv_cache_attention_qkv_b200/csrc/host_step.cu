// fc_step_host / fc_host_sync: a step whose per-step inputs and outputs live
// in host memory, double-buffered so that copies overlap the kernels.
//
// Call n uses staging set n % 2.  Its input copy (copy stream s_h2d) waits for
// the kernels of call n-2 (the last reader of that set); the kernels on the
// caller's stream wait for the input copy and for the output copy of call n-2
// (the last reader of that set's out / tracked); the output copy (s_d2h) waits
// for the kernels.  So the input copy of call n+1 and the output copy of call
// n-1 run while the kernels of call n run.
#include <string.h>

#include "fc_internal.h"

namespace {

size_t align16(size_t n) { return (n + 15) & ~(size_t)15; }

// input + output bytes of a call from which its kernels are fenced by timed
// events (see fc_step_host)
constexpr size_t kFenceCopyBytes = 16u << 20;

// int32 offsets of the small arrays inside one staging block
struct SmallLayout {
  size_t q_pos, cu_q, cu_k, lo, hi, kps, total;  // in int32 elements
};

SmallLayout small_layout(const fc_config& c) {
  SmallLayout L;
  size_t off = 0;
  auto take = [&](size_t n) {
    const size_t at = off;
    off += align16(n * sizeof(int32_t)) / sizeof(int32_t);
    return at;
  };
  L.q_pos = take((size_t)c.max_total_q);
  L.cu_q = take((size_t)c.max_batch + 1);
  L.cu_k = take((size_t)c.max_batch + 1);
  L.lo = take((size_t)c.max_batch);
  L.hi = take((size_t)c.max_batch);
  L.kps = take((size_t)c.max_batch);
  L.total = off;
  return L;
}

size_t elem_bytes(int dtype) { return dtype == FC_DTYPE_FP32 ? 4 : 2; }

fc_status init_pipe(fc_handle* h) {
  fc::HostPipe& p = h->hp;
  if (p.ready) return FC_OK;
  const fc_config& c = h->cfg;
  const size_t es = elem_bytes(c.dtype);
  const size_t topk = c.max_topk > 0 ? (size_t)c.max_topk : 1;
  bool ok = cudaStreamCreateWithFlags(&p.s_h2d, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&p.s_d2h, cudaStreamNonBlocking) == cudaSuccess &&
            cudaMalloc(&p.importance, (size_t)c.max_total_k * sizeof(float)) == cudaSuccess;
  for (int s = 0; s < 2 && ok; ++s) {
    ok = cudaMalloc(&p.x[s], (size_t)c.max_total_q * c.hidden * es) == cudaSuccess &&
         cudaMalloc(&p.small[s], small_layout(c).total * sizeof(int32_t)) == cudaSuccess &&
         cudaHostAlloc(&p.small_h[s], small_layout(c).total * sizeof(int32_t),
                       cudaHostAllocDefault) == cudaSuccess &&
         cudaMalloc(&p.out[s], (size_t)c.max_total_q * c.n_heads * c.head_dim * es) ==
             cudaSuccess &&
         cudaMalloc(&p.tracked[s], (size_t)c.max_batch * topk * sizeof(int32_t)) == cudaSuccess &&
         cudaEventCreateWithFlags(&p.h2d_done[s], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&p.comp_done[s], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&p.d2h_done[s], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreate(&p.fence[s]) == cudaSuccess;
  }
  if (!ok) {
    const cudaError_t e = cudaGetLastError();
    fc::free_host_pipe(h);
    return e == cudaErrorMemoryAllocation ? FC_ERR_OOM : FC_ERR_CUDA;
  }
  p.ready = true;
  p.calls = 0;
  return FC_OK;
}

}  // namespace

namespace fc {

void free_host_pipe(fc_handle* h) {
  HostPipe& p = h->hp;
  for (int s = 0; s < 2; ++s) {
    if (p.x[s]) cudaFree(p.x[s]);
    if (p.small[s]) cudaFree(p.small[s]);
    if (p.small_h[s]) cudaFreeHost(p.small_h[s]);
    if (p.out[s]) cudaFree(p.out[s]);
    if (p.tracked[s]) cudaFree(p.tracked[s]);
    if (p.h2d_done[s]) cudaEventDestroy(p.h2d_done[s]);
    if (p.comp_done[s]) cudaEventDestroy(p.comp_done[s]);
    if (p.d2h_done[s]) cudaEventDestroy(p.d2h_done[s]);
    if (p.fence[s]) cudaEventDestroy(p.fence[s]);
  }
  if (p.importance) cudaFree(p.importance);
  if (p.s_h2d) cudaStreamDestroy(p.s_h2d);
  if (p.s_d2h) cudaStreamDestroy(p.s_d2h);
  p = HostPipe{};
}

}  // namespace fc

extern "C" {

fc_status fc_step_host(fc_handle* h, void* stream, int batch, const void* x, const int32_t* q_pos,
                       const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int total_q,
                       int total_k, void* k_cache, void* v_cache, const int32_t* cand_lo,
                       const int32_t* cand_hi, const int32_t* k_per_seq, int k, void* out,
                       int32_t* tracked) {
  if (!h) return FC_ERR_INVALID_ARG;
  const fc_config& c = h->cfg;
  if (batch < 1 || batch > c.max_batch || total_q < 0 || total_q > c.max_total_q || total_k < 0 ||
      total_k > c.max_total_k || k < 0 || k > c.max_topk)
    return FC_ERR_INVALID_ARG;
  if (!cu_seqlens_q || !cu_seqlens_k || !cand_lo || !cand_hi || (k > 0 && !tracked))
    return FC_ERR_INVALID_ARG;
  if (total_q > 0 && (!x || !q_pos || !out || !k_cache || !v_cache)) return FC_ERR_INVALID_ARG;
  if (cudaSetDevice(h->device) != cudaSuccess) return FC_ERR_CUDA;
  fc_status st = init_pipe(h);
  if (st != FC_OK) return st;
  fc::HostPipe& p = h->hp;
  cudaStream_t cs = (cudaStream_t)stream;
  const int s = (int)(p.calls & 1ull);
  const bool reuse = p.calls >= 2;
  const size_t es = elem_bytes(c.dtype);
  const SmallLayout L = small_layout(c);
  int32_t* sm = p.small[s];
  const size_t x_bytes = (size_t)total_q * c.hidden * es;
  const size_t out_bytes = (size_t)total_q * c.n_heads * c.head_dim * es;
  const size_t tr_bytes = (size_t)batch * k * sizeof(int32_t);

  // ---- inputs: host -> staging set s, once call n-2's kernels are done with it
  cudaError_t e = cudaSuccess;
  if (reuse) e = cudaStreamWaitEvent(p.s_h2d, p.comp_done[s], 0);
  const int rec_in = fc::prof_begin(h, p.s_h2d, 6);
  auto h2d = [&](void* dst, const void* src, size_t bytes) {
    if (e == cudaSuccess && bytes > 0)
      e = cudaMemcpyAsync(dst, src, bytes, cudaMemcpyHostToDevice, p.s_h2d);
  };
  h2d(p.x[s], x, x_bytes);
  // the small arrays are gathered on the host into this set's pinned block
  // (read now, at the call) and moved in one copy: one driver call instead of
  // six.  The block's previous copy (call n-2) finished long ago as a rule;
  // the host waits for it if not.
  if (e == cudaSuccess && reuse) e = cudaEventSynchronize(p.h2d_done[s]);
  if (e == cudaSuccess) {
    int32_t* hb = p.small_h[s];
    memcpy(hb + L.q_pos, q_pos, (size_t)total_q * sizeof(int32_t));
    memcpy(hb + L.cu_q, cu_seqlens_q, (size_t)(batch + 1) * sizeof(int32_t));
    memcpy(hb + L.cu_k, cu_seqlens_k, (size_t)(batch + 1) * sizeof(int32_t));
    memcpy(hb + L.lo, cand_lo, (size_t)batch * sizeof(int32_t));
    memcpy(hb + L.hi, cand_hi, (size_t)batch * sizeof(int32_t));
    if (k_per_seq) memcpy(hb + L.kps, k_per_seq, (size_t)batch * sizeof(int32_t));
    h2d(sm, hb, (k_per_seq ? L.kps + (size_t)batch : L.kps) * sizeof(int32_t));
  }
  fc::prof_end(h, p.s_h2d, rec_in);
  if (e == cudaSuccess) e = cudaEventRecord(p.h2d_done[s], p.s_h2d);
  // ---- kernels on the caller's stream
  if (e == cudaSuccess) e = cudaStreamWaitEvent(cs, p.h2d_done[s], 0);
  if (e == cudaSuccess && reuse) e = cudaStreamWaitEvent(cs, p.d2h_done[s], 0);
  if (e != cudaSuccess) return FC_ERR_CUDA;
  // The kernels run here beside the input copy of the next call and the
  // output copy of the previous one.  With large copies (batch 32 x 128 rows:
  // 33.5 MB each way), kernels launched back to back stretched the input copy
  // (1.05 ms at 32 GB/s instead of 0.75 ms at 44 GB/s) and the step to
  // 1.0-1.05 ms; with a timed event recorded on each side of every kernel
  // (which also ends programmatic overlap between them, so the kernels are
  // launched plainly) the step takes 0.77-0.80 ms, near the two copies'
  // concurrent rate.  Timing-disabled events, or timed events around a single
  // kernel, did not help.  Small steps are latency-bound instead (batch 1:
  // 1 MB each way), and there the events cost more than they save, so they
  // keep the device path's launches.
  const bool big_copies = x_bytes + out_bytes >= kFenceCopyBytes;
  if (big_copies) {
    h->pdl = false;
    p.fencing = true;
  }
  st = fc_step(h, stream, batch, p.x[s], sm + L.q_pos, sm + L.cu_q, sm + L.cu_k, total_q, total_k,
               k_cache, v_cache, p.out[s], p.importance, 0);
  const int step_launches = h->last_launches;
  if (st == FC_OK)
    st = fc_topk_tracked(h, stream, batch, total_k, p.importance, sm + L.cu_k, sm + L.lo, sm + L.hi,
                         k_per_seq ? sm + L.kps : nullptr, k, p.tracked[s]);
  h->pdl = true;
  p.fencing = false;
  if (st != FC_OK) return st;
  h->last_launches += step_launches;
  e = cudaEventRecord(p.comp_done[s], cs);
  // ---- outputs: staging set s -> host
  if (e == cudaSuccess) e = cudaStreamWaitEvent(p.s_d2h, p.comp_done[s], 0);
  const int rec_out = fc::prof_begin(h, p.s_d2h, 7);
  if (e == cudaSuccess && out_bytes > 0)
    e = cudaMemcpyAsync(out, p.out[s], out_bytes, cudaMemcpyDeviceToHost, p.s_d2h);
  if (e == cudaSuccess && tr_bytes > 0)
    e = cudaMemcpyAsync(tracked, p.tracked[s], tr_bytes, cudaMemcpyDeviceToHost, p.s_d2h);
  fc::prof_end(h, p.s_d2h, rec_out);
  if (e == cudaSuccess) e = cudaEventRecord(p.d2h_done[s], p.s_d2h);
  if (e != cudaSuccess) return FC_ERR_CUDA;
  ++p.calls;
  return FC_OK;
}

fc_status fc_host_sync(fc_handle* h, void* stream) {
  if (!h) return FC_ERR_INVALID_ARG;
  fc::HostPipe& p = h->hp;
  if (!p.ready || p.calls == 0) return FC_OK;
  if (cudaSetDevice(h->device) != cudaSuccess) return FC_ERR_CUDA;
  cudaStream_t cs = (cudaStream_t)stream;
  for (int s = 0; s < 2; ++s)
    if (p.calls > (unsigned long long)s &&
        cudaStreamWaitEvent(cs, p.d2h_done[s], 0) != cudaSuccess)
      return FC_ERR_CUDA;
  return FC_OK;
}

}  // extern "C"
