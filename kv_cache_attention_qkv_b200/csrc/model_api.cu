// Host runtime of the model step (fc_model_* in include/flashcache.h): the
// decoder stack of LLaDA-8B (the model the Flash-dLLM pages evaluate) around
// the Flash-Cache layer, then the LM head and the Flash-Verify confidence
// test on the rows the caller names.  Per layer, on the caller's stream:
//   a = rms_norm(h) * g_attn                 rmsnorm_kernel
//   o = FlashCache(a) (cache write, attention, importance summed over layers)
//   h = h + o . Wo^T                         gemm_tc (GEMM_RESID, in place)
//   a = rms_norm(h) * g_mlp                  rmsnorm_kernel
//   s = silu(a . Wg^T) * (a . Wu^T)          gemm_tc (GEMM_SWIGLU)
//   h = h + s . Wd^T                         gemm_tc (GEMM_RESID, in place)
// then hr = rms_norm(h[head_rows]) * g_final, the LM head's per-tile softmax
// statistics (gemm_tc, GEMM_LMHEAD) and their merge (lmhead_reduce_kernel).
#include <new>
#include <vector>

#include "fc_internal.h"

struct fc_model {
  fc_model_config cfg;
  fc_handle* layer = nullptr;  // attention workspace shared by every layer
  std::vector<fc_layer_weights> w;
  const void* final_norm = nullptr;
  const void* lm_head = nullptr;
  std::vector<CUtensorMap> tm_qkv, tm_o, tm_gate, tm_up, tm_down;
  CUtensorMap tm_lm;
  // activations (bf16) and LM-head statistics
  __nv_bfloat16 *h = nullptr, *a = nullptr, *o = nullptr, *s = nullptr, *hr = nullptr;
  float* partials = nullptr;
  int num_vn = 0;  // 256-column vocabulary tiles
  CUtensorMap tm_a, tm_oa, tm_s, tm_hr;
  void* decode_ws[16] = {};  // fc_decode_iteration's workspace (allocated on first use)
};

namespace fc {
int model_hidden(const fc_model* m) { return m->cfg.layer.hidden; }
int model_vocab(const fc_model* m) { return m->cfg.vocab; }
int model_max_total_q(const fc_model* m) { return m->cfg.layer.max_total_q; }
int model_max_batch(const fc_model* m) { return m->cfg.layer.max_batch; }
int model_max_head_rows(const fc_model* m) { return m->cfg.max_head_rows; }
int model_max_topk(const fc_model* m) { return m->cfg.layer.max_topk; }
float model_threshold(const fc_model* m) { return m->cfg.threshold; }
fc_handle* model_layer(fc_model* m) { return m->layer; }
void** model_decode_ws(fc_model* m) { return m->decode_ws; }
}  // namespace fc

namespace {

bool al16(const void* p) { return p && ((uintptr_t)p & 15u) == 0; }

void free_model(fc_model* m) {
  void* bufs[] = {m->h, m->a, m->o, m->s, m->hr, m->partials};
  for (void* b : bufs)
    if (b) cudaFree(b);
  for (void* b : m->decode_ws)
    if (b) cudaFree(b);
  if (m->layer) fc_destroy(m->layer);
  delete m;
}

bool enc(CUtensorMap* tm, const void* p, uint64_t rows, uint64_t cols) {
  return fc::encode_bf16_2d(tm, p, rows, cols, cols * 2, fc::kGemmBoxRows, 64);
}

}  // namespace

extern "C" {

fc_status fc_model_create(const fc_model_config* cfg, const fc_layer_weights* layers,
                          const void* final_norm, const void* lm_head, fc_model** out) {
  if (!out) return FC_ERR_INVALID_ARG;
  *out = nullptr;
  if (!cfg || !layers || cfg->n_layers < 1 || cfg->intermediate < 1 || cfg->vocab < 1 ||
      cfg->max_head_rows < 1 || !(cfg->rms_eps >= 0.f) || !(cfg->threshold >= 0.f))
    return FC_ERR_INVALID_ARG;
  const fc_config& c = cfg->layer;
  const int D = c.hidden, HD = c.n_heads * c.head_dim, I = cfg->intermediate;
  // the tensor-core path only: bf16, head_dim 128, even H, 256-wide residual tiles
  if (c.dtype != FC_DTYPE_BF16 || c.head_dim != 128 || (c.n_heads & 1) || D % 256 != 0 ||
      I % 128 != 0 || HD % 64 != 0)
    return FC_ERR_UNSUPPORTED;
  if (!al16(final_norm) || !al16(lm_head)) return FC_ERR_INVALID_ARG;
  for (int l = 0; l < cfg->n_layers; ++l) {
    const fc_layer_weights& w = layers[l];
    if (!al16(w.attn_norm) || !al16(w.w_qkv) || !al16(w.w_o) || !al16(w.mlp_norm) ||
        !al16(w.w_gate) || !al16(w.w_up) || !al16(w.w_down))
      return FC_ERR_INVALID_ARG;
  }
  fc_model* m = new (std::nothrow) fc_model();
  if (!m) return FC_ERR_OOM;
  m->cfg = *cfg;
  fc_status st = fc_create(&c, layers[0].w_qkv, &m->layer);
  if (st != FC_OK) {
    free_model(m);
    return st;
  }
  m->w.assign(layers, layers + cfg->n_layers);
  m->final_norm = final_norm;
  m->lm_head = lm_head;
  const int L = cfg->n_layers;
  m->tm_qkv.resize(L);
  m->tm_o.resize(L);
  m->tm_gate.resize(L);
  m->tm_up.resize(L);
  m->tm_down.resize(L);
  bool ok = true;
  for (int l = 0; l < L && ok; ++l) {
    const fc_layer_weights& w = layers[l];
    ok = fc::encode_bf16_2d(&m->tm_qkv[l], w.w_qkv, (uint64_t)3 * HD, (uint64_t)D, (uint64_t)D * 2,
                            fc::kQkvWBoxRows, 64) &&
         enc(&m->tm_o[l], w.w_o, D, HD) && enc(&m->tm_gate[l], w.w_gate, I, D) &&
         enc(&m->tm_up[l], w.w_up, I, D) && enc(&m->tm_down[l], w.w_down, D, I);
  }
  ok = ok && enc(&m->tm_lm, lm_head, (uint64_t)cfg->vocab, D);
  const size_t T = (size_t)c.max_total_q, R = (size_t)cfg->max_head_rows;
  m->num_vn = (cfg->vocab + 255) / 256;
  ok = ok && cudaMalloc(&m->h, T * D * 2) == cudaSuccess &&
       cudaMalloc(&m->a, T * D * 2) == cudaSuccess &&
       cudaMalloc(&m->o, T * HD * 2) == cudaSuccess &&
       cudaMalloc(&m->s, T * I * 2) == cudaSuccess &&
       cudaMalloc(&m->hr, R * D * 2) == cudaSuccess &&
       cudaMalloc(&m->partials, R * m->num_vn * 3 * sizeof(float)) == cudaSuccess;
  ok = ok && enc(&m->tm_a, m->a, T, D) && enc(&m->tm_oa, m->o, T, HD) && enc(&m->tm_s, m->s, T, I) &&
       enc(&m->tm_hr, m->hr, R, D);
  if (!ok) {
    const cudaError_t e = cudaGetLastError();
    free_model(m);
    return e == cudaErrorMemoryAllocation ? FC_ERR_OOM : FC_ERR_CUDA;
  }
  *out = m;
  return FC_OK;
}

fc_handle* fc_model_layer_handle(fc_model* m) { return m ? m->layer : nullptr; }

fc_status fc_model_step(fc_model* m, void* stream, int batch, const void* x, const int32_t* q_pos,
                        const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int total_q,
                        int total_k, void* const* k_caches, void* const* v_caches,
                        const int32_t* head_rows, int n_head_rows, float* importance,
                        int32_t* token, float* confidence, uint8_t* accept, void* h_out) {
  if (!m) return FC_ERR_INVALID_ARG;
  const fc_model_config& mc = m->cfg;
  const fc_config& c = mc.layer;
  if (total_q < 1 || total_q > c.max_total_q || n_head_rows < 0 ||
      n_head_rows > mc.max_head_rows || !al16(x) || !k_caches || !v_caches)
    return FC_ERR_INVALID_ARG;
  if (n_head_rows > 0 && (!head_rows || !token || !confidence || !accept))
    return FC_ERR_INVALID_ARG;
  if (h_out && !al16(h_out)) return FC_ERR_INVALID_ARG;
  for (int l = 0; l < mc.n_layers; ++l)
    if (!al16(k_caches[l]) || !al16(v_caches[l])) return FC_ERR_INVALID_ARG;
  if (cudaSetDevice(m->layer->device) != cudaSuccess) return FC_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  const int D = c.hidden, HD = c.n_heads * c.head_dim, I = mc.intermediate;
  const int nsm = m->layer->num_sms;
  int launches = 0;
  if (cudaMemcpyAsync(m->h, x, (size_t)total_q * D * 2, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return FC_ERR_CUDA;
  fc::GemmParams gp = {};
  gp.err = m->layer->ws.err;
  auto gemm = [&](int mode, const CUtensorMap& ta, const CUtensorMap& tb0, const CUtensorMap& tb1,
                  int M, int N, int K, __nv_bfloat16* outp, size_t ldo) {
    fc::GemmParams p = gp;
    p.mode = mode;
    p.M = M;
    p.N = N;
    p.K = K;
    p.resid = outp;
    p.out = outp;
    p.ldo = ldo;
    p.partials = m->partials;
    ++launches;
    return fc::launch_gemm_tc(nsm, st, ta, tb0, tb1, p);
  };
  for (int l = 0; l < mc.n_layers; ++l) {
    const fc_layer_weights& w = m->w[l];
    if (fc::launch_rmsnorm(st, m->h, nullptr, total_q, D, (const __nv_bfloat16*)w.attn_norm,
                           mc.rms_eps, m->a) != cudaSuccess)
      return FC_ERR_CUDA;
    fc_status s = fc::step_impl(m->layer, &m->tm_qkv[l], stream, batch, m->a, q_pos, cu_seqlens_q,
                                cu_seqlens_k, total_q, total_k, k_caches[l], v_caches[l], m->o,
                                importance, l > 0 ? 1 : 0);
    if (s != FC_OK) return s;
    launches += 1 + m->layer->last_launches;
    if (gemm(fc::GEMM_RESID, m->tm_oa, m->tm_o[l], m->tm_o[l], total_q, D, HD, m->h, D) != cudaSuccess ||
        fc::launch_rmsnorm(st, m->h, nullptr, total_q, D, (const __nv_bfloat16*)w.mlp_norm,
                           mc.rms_eps, m->a) != cudaSuccess ||
        gemm(fc::GEMM_SWIGLU, m->tm_a, m->tm_gate[l], m->tm_up[l], total_q, I, D, m->s, I) != cudaSuccess ||
        gemm(fc::GEMM_RESID, m->tm_s, m->tm_down[l], m->tm_down[l], total_q, D, I, m->h, D) != cudaSuccess)
      return FC_ERR_CUDA;
    launches += 1;
  }
  if (n_head_rows > 0) {
    if (fc::launch_rmsnorm(st, m->h, head_rows, n_head_rows, D, (const __nv_bfloat16*)m->final_norm,
                           mc.rms_eps, m->hr) != cudaSuccess ||
        gemm(fc::GEMM_LMHEAD, m->tm_hr, m->tm_lm, m->tm_lm, n_head_rows, mc.vocab, D, nullptr, 0) !=
            cudaSuccess ||
        fc::launch_lmhead_reduce(st, m->partials, n_head_rows, m->num_vn, mc.threshold, token,
                                 confidence, accept) != cudaSuccess)
      return FC_ERR_CUDA;
    launches += 2;
  }
  if (h_out && cudaMemcpyAsync(h_out, m->h, (size_t)total_q * D * 2, cudaMemcpyDeviceToDevice, st) !=
                   cudaSuccess)
    return FC_ERR_CUDA;
  m->layer->last_stream = st;
  m->layer->last_launches = launches;
  return FC_OK;
}

fc_status fc_model_lm_head(fc_model* m, void* stream, const void* rows, int n_rows,
                           int32_t* token, float* confidence, uint8_t* accept) {
  if (!m || !al16(rows) || n_rows < 1 || n_rows > m->cfg.max_head_rows || !token || !confidence ||
      !accept)
    return FC_ERR_INVALID_ARG;
  if (cudaSetDevice(m->layer->device) != cudaSuccess) return FC_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  const int D = m->cfg.layer.hidden;
  CUtensorMap tm_rows;
  if (!enc(&tm_rows, rows, (uint64_t)n_rows, (uint64_t)D)) return FC_ERR_CUDA;
  fc::GemmParams p = {};
  p.mode = fc::GEMM_LMHEAD;
  p.M = n_rows;
  p.N = m->cfg.vocab;
  p.K = D;
  p.partials = m->partials;
  p.err = m->layer->ws.err;
  if (fc::launch_gemm_tc(m->layer->num_sms, st, tm_rows, m->tm_lm, m->tm_lm, p) != cudaSuccess ||
      fc::launch_lmhead_reduce(st, m->partials, n_rows, m->num_vn, m->cfg.threshold, token,
                               confidence, accept) != cudaSuccess)
    return FC_ERR_CUDA;
  m->layer->last_stream = st;
  m->layer->last_launches = 2;
  return FC_OK;
}

void fc_model_destroy(fc_model* m) {
  if (!m) return;
  cudaSetDevice(m->layer->device);
  cudaDeviceSynchronize();
  free_model(m);
}

}  // extern "C"
