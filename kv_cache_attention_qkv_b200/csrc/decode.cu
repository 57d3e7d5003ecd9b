// One draft-and-verify decode iteration on top of the model step (Flash-dLLM:
// the model is its own drafter and verifier; draft tokens and [MASK] tokens
// are checked through two views and every prediction that meets the
// confidence threshold is accepted in the same iteration; the tracked
// positions are reselected by attention importance — infernews post
// "Flash-dLLM: IO-aware KV caching and parallel decoding", Flash-Verify
// paragraph; paper-digest page, Fig. 2 caption).
//
// Everything stays on the device, on the caller's stream:
//   decode_query_kernel    query of each sequence = its K tracked positions and
//                          its W-position window; token ids of both views
//   embed_gather_kernel    input rows = embedding rows of those ids
//   fc_model_step x 2      the [MASK] view, then the draft view (importance)
//   decode_accept_kernel   acceptance, drafts, window advance
//   fc_topk_tracked        new tracked positions from the draft view's importance
#include <new>

#include "fc_internal.h"
#include "ptx.cuh"

// the model's internals this file needs (defined in model_api.cu)
struct fc_model;
namespace fc {
int model_hidden(const fc_model* m);
int model_vocab(const fc_model* m);
int model_max_total_q(const fc_model* m);
int model_max_batch(const fc_model* m);
int model_max_head_rows(const fc_model* m);
int model_max_topk(const fc_model* m);
float model_threshold(const fc_model* m);
fc_handle* model_layer(fc_model* m);
void** model_decode_ws(fc_model* m);
}  // namespace fc

namespace fc {
namespace {

__global__ void decode_query_kernel(int B, int K, int W, int mask_id, const int32_t* __restrict__ cu_k,
                                    const int32_t* __restrict__ tracked,
                                    const int32_t* __restrict__ ws, const int32_t* __restrict__ tokens,
                                    const int32_t* __restrict__ draft, int32_t* __restrict__ q_pos,
                                    int32_t* __restrict__ cu_q, int32_t* __restrict__ head_rows,
                                    int32_t* __restrict__ ids_m, int32_t* __restrict__ ids_d) {
  ptx::griddep_launch_dependents();
  ptx::griddep_wait();
  const int b = blockIdx.x, n = K + W;
  const int k0 = cu_k[b], L = cu_k[b + 1] - k0, w0 = ws[b];
  if (threadIdx.x == 0) {
    cu_q[b] = b * n;
    if (b == B - 1) cu_q[B] = B * n;
  }
  for (int r = threadIdx.x; r < n; r += blockDim.x) {
    const int row = b * n + r;
    const int pos = r < K ? tracked[b * K + r] : w0 + (r - K);
    q_pos[row] = pos;
    int tm = mask_id, td = mask_id;
    if (pos >= 0 && pos < L) {  // anything else is reported by the step's checks
      const int t = tokens[k0 + pos];
      if (t >= 0) {
        tm = td = t;
      } else if (draft[k0 + pos] >= 0) {
        td = draft[k0 + pos];
      }
    }
    ids_m[row] = tm;
    ids_d[row] = td;
    if (r >= K) head_rows[b * W + (r - K)] = row;
  }
}

// x[row] = embed[ids[row]] for both views; ids outside [0, V) give a zero row
// and set FC_DEVERR_CAND.
__global__ void embed_gather_kernel(int D, int V, const __nv_bfloat16* __restrict__ embed,
                                    const int32_t* __restrict__ ids_m,
                                    const int32_t* __restrict__ ids_d, __nv_bfloat16* __restrict__ x_m,
                                    __nv_bfloat16* __restrict__ x_d, int32_t* __restrict__ err) {
  ptx::griddep_launch_dependents();
  ptx::griddep_wait();
  const int row = blockIdx.x;
  const int n8 = D / 8;
  for (int v = 0; v < 2; ++v) {
    const int id = (v == 0 ? ids_m : ids_d)[row];
    const bool ok = id >= 0 && id < V;
    if (!ok && threadIdx.x == 0) atomicOr(err, FC_DEVERR_CAND);
    const uint4* src = reinterpret_cast<const uint4*>(embed + (size_t)(ok ? id : 0) * D);
    uint4* dst = reinterpret_cast<uint4*>((v == 0 ? x_m : x_d) + (size_t)row * D);
    for (int c = threadIdx.x; c < n8; c += blockDim.x) dst[c] = ok ? src[c] : make_uint4(0, 0, 0, 0);
  }
}

// One warp per sequence: acceptance over the window, at least one token,
// drafts of the undecided positions, window advance.
__global__ void decode_accept_kernel(int B, int W, float threshold, const int32_t* __restrict__ cu_k,
                                     int32_t* __restrict__ ws, const int32_t* __restrict__ gen_end,
                                     int32_t* __restrict__ tokens, int32_t* __restrict__ draft,
                                     const int32_t* __restrict__ tok_m, const float* __restrict__ conf_m,
                                     const int32_t* __restrict__ tok_d, const float* __restrict__ conf_d,
                                     int32_t* __restrict__ n_accepted) {
  ptx::griddep_launch_dependents();
  ptx::griddep_wait();
  const int b = blockIdx.x, lane = threadIdx.x;
  const int k0 = cu_k[b], L = cu_k[b + 1] - k0, w0 = ws[b];
  int n_acc = 0, n_und = 0;
  float best = -INFINITY;
  int best_j = 0x7fffffff;
  for (int j = lane; j < W; j += 32) {
    const int pos = w0 + j;
    if (pos < 0 || pos >= L) continue;
    const int e = b * W + j;
    if (tokens[k0 + pos] >= 0) continue;
    const int dr = draft[k0 + pos];
    int t = -1;
    if (conf_m[e] >= threshold) {
      t = tok_m[e];
    } else if (dr >= 0 && tok_d[e] == dr && conf_d[e] >= threshold) {
      t = dr;
    }
    if (t >= 0) {
      tokens[k0 + pos] = t;
      ++n_acc;
    } else {
      ++n_und;
      if (conf_m[e] > best) {  // j increases per lane: the first maximum stays
        best = conf_m[e];
        best_j = j;
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    n_acc += __shfl_xor_sync(0xffffffffu, n_acc, o);
    n_und += __shfl_xor_sync(0xffffffffu, n_und, o);
    const float ob = __shfl_xor_sync(0xffffffffu, best, o);
    const int oj = __shfl_xor_sync(0xffffffffu, best_j, o);
    if (ob > best || (ob == best && oj < best_j)) {
      best = ob;
      best_j = oj;
    }
  }
  if (n_acc == 0 && n_und > 0 && lane == 0) {
    tokens[k0 + w0 + best_j] = tok_m[b * W + best_j];
    n_acc = 1;
    --n_und;
  }
  __syncwarp();
  // drafts: the [MASK] view's predictions where still undecided
  for (int j = lane; j < W; j += 32) {
    const int pos = w0 + j;
    if (pos < 0 || pos >= L) continue;
    draft[k0 + pos] = tokens[k0 + pos] < 0 ? tok_m[b * W + j] : -1;
  }
  __syncwarp();
  if (n_und == 0 && w0 + 2 * W <= gen_end[b]) {  // the next window fits in the span
    const int w1 = w0 + W;
    for (int j = lane; j < W; j += 32)
      if (w1 + j < L) draft[k0 + w1 + j] = -1;
    if (lane == 0) ws[b] = w1;
  }
  if (lane == 0) n_accepted[b] = n_acc;
}

}  // namespace
}  // namespace fc

extern "C" {

fc_status fc_decode_iteration(fc_model* m, void* stream, int batch, const int32_t* cu_seqlens_k,
                              int total_k, void* const* k_caches, void* const* v_caches,
                              const void* embed, int mask_id, int n_tracked, int window,
                              int32_t* tracked, int32_t* window_start, const int32_t* gen_end,
                              int32_t* tokens, int32_t* draft, int32_t* n_accepted,
                              float* importance_out) {
  if (!m || batch < 1 || n_tracked < 0 || window < 1 || !cu_seqlens_k || !embed || !tracked ||
      !window_start || !gen_end || !tokens || !draft || !n_accepted || !k_caches || !v_caches)
    return FC_ERR_INVALID_ARG;
  const int V = fc::model_vocab(m), D = fc::model_hidden(m);
  const int T = batch * (n_tracked + window);
  if (mask_id < 0 || mask_id >= V || batch > fc::model_max_batch(m) ||
      T > fc::model_max_total_q(m) || batch * window > fc::model_max_head_rows(m) ||
      n_tracked > fc::model_max_topk(m) || ((uintptr_t)embed & 15u) ||
      (importance_out && ((uintptr_t)importance_out & 3u)))
    return FC_ERR_INVALID_ARG;
  fc_handle* h = fc::model_layer(m);
  if (cudaSetDevice(h->device) != cudaSuccess) return FC_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  // workspace, allocated on first use: ids and rows of both views, predictions
  void** ws_slots = fc::model_decode_ws(m);
  const size_t Tq = (size_t)fc::model_max_total_q(m), Rh = (size_t)fc::model_max_head_rows(m);
  const size_t Bm = (size_t)fc::model_max_batch(m), Sk = (size_t)h->cfg.max_total_k;
  const size_t sizes[] = {Tq * 4, (Bm + 1) * 4, Rh * 4, Tq * 4, Tq * 4, Tq * D * 2, Tq * D * 2,
                          Rh * 4, Rh * 4, Rh * 4, Rh * 4, Rh, Rh, Sk * 4, Bm * 4};
  constexpr int NWS = sizeof(sizes) / sizeof(sizes[0]);
  if (!ws_slots[0]) {
    for (int i = 0; i < NWS; ++i)
      if (cudaMalloc(&ws_slots[i], sizes[i]) != cudaSuccess) {
        cudaGetLastError();
        for (int j = 0; j < i; ++j) cudaFree(ws_slots[j]), ws_slots[j] = nullptr;
        return FC_ERR_OOM;
      }
    if (cudaMemset(ws_slots[14], 0, sizes[14]) != cudaSuccess) return FC_ERR_CUDA;  // cand_lo = 0
  }
  int32_t *q_pos = (int32_t*)ws_slots[0], *cu_q = (int32_t*)ws_slots[1],
          *head_rows = (int32_t*)ws_slots[2], *ids_m = (int32_t*)ws_slots[3],
          *ids_d = (int32_t*)ws_slots[4];
  __nv_bfloat16 *x_m = (__nv_bfloat16*)ws_slots[5], *x_d = (__nv_bfloat16*)ws_slots[6];
  int32_t *tok_m = (int32_t*)ws_slots[7], *tok_d = (int32_t*)ws_slots[8];
  float *conf_m = (float*)ws_slots[9], *conf_d = (float*)ws_slots[10];
  uint8_t *acc_m = (uint8_t*)ws_slots[11], *acc_d = (uint8_t*)ws_slots[12];
  // the draft view's importance: the caller's buffer when given, else the workspace's
  float* importance = importance_out ? importance_out : (float*)ws_slots[13];
  const int32_t* cand_lo = (const int32_t*)ws_slots[14];
  int launches = 0;
  if (fc::launch_pdl(fc::decode_query_kernel, dim3(batch), dim3(128), 0, st, batch, n_tracked,
                     window, mask_id, cu_seqlens_k, (const int32_t*)tracked,
                     (const int32_t*)window_start, (const int32_t*)tokens, (const int32_t*)draft,
                     q_pos, cu_q, head_rows, ids_m, ids_d) != cudaSuccess ||
      fc::launch_pdl(fc::embed_gather_kernel, dim3(T), dim3(128), 0, st, D, V,
                     (const __nv_bfloat16*)embed, (const int32_t*)ids_m, (const int32_t*)ids_d, x_m,
                     x_d, h->ws.err) != cudaSuccess)
    return FC_ERR_CUDA;
  launches += 2;
  const int R = batch * window;
  fc_status s = fc_model_step(m, stream, batch, x_m, q_pos, cu_q, cu_seqlens_k, T, total_k,
                              k_caches, v_caches, head_rows, R, nullptr, tok_m, conf_m, acc_m,
                              nullptr);
  if (s != FC_OK) return s;
  launches += h->last_launches;
  s = fc_model_step(m, stream, batch, x_d, q_pos, cu_q, cu_seqlens_k, T, total_k, k_caches,
                    v_caches, head_rows, R, importance, tok_d, conf_d, acc_d, nullptr);
  if (s != FC_OK) return s;
  launches += h->last_launches;
  if (fc::launch_pdl(fc::decode_accept_kernel, dim3(batch), dim3(32), 0, st, batch, window,
                     fc::model_threshold(m), cu_seqlens_k, window_start, gen_end, tokens, draft,
                     (const int32_t*)tok_m, (const float*)conf_m, (const int32_t*)tok_d,
                     (const float*)conf_d, n_accepted) != cudaSuccess)
    return FC_ERR_CUDA;
  launches += 1;
  s = fc_topk_tracked(h, stream, batch, total_k, importance, cu_seqlens_k, cand_lo, window_start,
                      nullptr, n_tracked, tracked);
  if (s != FC_OK) return s;
  h->last_launches += launches;
  return FC_OK;
}

}  // extern "C"
