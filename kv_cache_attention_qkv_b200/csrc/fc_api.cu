// Host runtime of libflashcache.so: the C ABI declared in include/flashcache.h.
//
// It validates arguments, owns the workspace (Q buffer, row map, work list,
// fixed-point importance accumulator, RoPE table, error word), encodes the TMA
// tensor maps of the tensor-core path and enqueues the kernels on the caller's
// stream.  It never synchronises except in fc_get_error / fc_destroy.
#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>
#include <new>
#include <vector>

#include "fc_internal.h"

namespace {

using fc::StepShape;

constexpr int kMaxBatch = 4096;
constexpr int kMaxPos = 262144;
constexpr int kMaxTopk = 1024;
constexpr int kMaxHeadDim = 256;

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

size_t elem_size(int dtype) { return dtype == FC_DTYPE_FP32 ? 4 : 2; }

// ---- TMA tensor-map encoding through the driver entry point (no -lcuda) ----
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
  }
  return fn;
}

// Record-before / record-after around one launch when profiling is on; in a
// pipelined host-buffer step, also a timed event on each side of the launch.
struct ProfScope {
  fc_handle* h;
  cudaStream_t st;
  int idx = -1;
  ProfScope(fc_handle* h_, cudaStream_t st_, int slot) : h(h_), st(st_) {
    fence();
    if (h->profiling && h->prof_n < 4096) {
      idx = h->prof_n++;
      h->prof_slot[idx] = slot;
      cudaEventRecord(h->prof_ev[2 * idx], st);
    }
  }
  ~ProfScope() {
    if (idx >= 0) cudaEventRecord(h->prof_ev[2 * idx + 1], st);
    fence();
  }
  void fence() {
    if (h->hp.fencing) cudaEventRecord(h->hp.fence[h->hp.fence_i++ & 1u], st);
  }
};

// Kernels whose shared-memory attribute is set, per device and size.
struct SmemAttrDone {
  const void* fn;
  int device;
  size_t bytes;
};
std::mutex g_smem_attr_mu;
std::vector<SmemAttrDone> g_smem_attr_done;

// Record a failed CUDA call of a step (slot: the kernel being launched, or -1)
// and return FC_ERR_CUDA.
fc_status cuda_fail(fc_handle* h, int slot, cudaError_t e) {
  h->last_cuda_err = e;
  h->last_cuda_slot = slot;
  return FC_ERR_CUDA;
}

}  // namespace

namespace fc {

cudaError_t smem_attr_once(const void* fn, size_t bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  {
    std::lock_guard<std::mutex> lk(g_smem_attr_mu);
    for (const SmemAttrDone& d : g_smem_attr_done)
      if (d.fn == fn && d.device == dev && d.bytes >= bytes) return cudaSuccess;
  }
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(g_smem_attr_mu);
  g_smem_attr_done.push_back({fn, dev, bytes});
  return cudaSuccess;
}

// 2-D bf16 tensor map over a row-major [rows, cols] array, box [box_rows,
// box_cols], 128-byte swizzle (box_cols * 2 must be 128).
bool encode_bf16_2d(CUtensorMap* tm, const void* base, uint64_t rows, uint64_t cols,
                    uint64_t row_stride_bytes, uint32_t box_rows, uint32_t box_cols) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D bf16 tensor map over a KV cache [S, H, 128]: box = 128 rows of one head,
// 64 columns (one 128-byte swizzle row), so one (sequence, head) key tile is
// two boxes.
bool encode_kv_3d(CUtensorMap* tm, const void* cache, int S, int H) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {128, (cuuint64_t)H, (cuuint64_t)S};
  cuuint64_t strides[2] = {256, (cuuint64_t)H * 256};
  cuuint32_t box[3] = {64, 1, 128};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(cache), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace fc

extern "C" {

const char* fc_status_str(fc_status s) {
  switch (s) {
    case FC_OK: return "ok";
    case FC_ERR_INVALID_ARG: return "invalid argument";
    case FC_ERR_UNSUPPORTED: return "unsupported";
    case FC_ERR_CUDA: return "CUDA error";
    case FC_ERR_OOM: return "out of device memory";
    case FC_ERR_DEVICE_CHECK: return "device-side check failed";
    case FC_ERR_TIMEOUT: return "device barrier wait timed out";
  }
  return "unknown status";
}

static fc_status validate_config(const fc_config* c) {
  if (!c) return FC_ERR_INVALID_ARG;
  if (c->hidden < 1 || c->n_heads < 1 || c->n_heads > 255 || c->head_dim < 2 ||
      (c->head_dim & 1) || !(c->rope_theta > 0.0) || !isfinite(c->rope_theta))
    return FC_ERR_INVALID_ARG;
  if (c->dtype != FC_DTYPE_BF16 && c->dtype != FC_DTYPE_FP32) return FC_ERR_INVALID_ARG;
  if (c->max_batch < 1 || c->max_total_q < 1 || c->max_total_k < 1 || c->max_seqlen_q < 1 ||
      c->max_pos < 1 || c->max_topk < 0)
    return FC_ERR_INVALID_ARG;
  if (c->max_seqlen_q > c->max_total_q) return FC_ERR_INVALID_ARG;
  if (c->max_batch > kMaxBatch || c->max_pos > kMaxPos || c->max_topk > kMaxTopk ||
      c->head_dim > kMaxHeadDim)
    return FC_ERR_UNSUPPORTED;
  // every element index must fit comfortably in 63 bits and every row count in 31
  if ((double)c->max_total_k * c->n_heads * c->head_dim > 9.0e15) return FC_ERR_UNSUPPORTED;
  return FC_OK;
}

static void free_workspace(fc_handle* h) {
  fc::Workspace& w = h->ws;
  void* ptrs[] = {w.q_buf,    w.row_dst,  w.imp_acc,     w.items,   w.sched,
                  w.err,      w.rope_cos, w.rope_sin,    w.items_fb, w.split_stats,
                  w.split_o,  w.split_cnt};
  for (void* p : ptrs)
    if (p) cudaFree(p);
  w = fc::Workspace{};
}

fc_status fc_create(const fc_config* cfg, const void* w_qkv, fc_handle** out) {
  if (!out) return FC_ERR_INVALID_ARG;
  *out = nullptr;
  fc_status st = validate_config(cfg);
  if (st != FC_OK) return st;
  if (!w_qkv || !aligned16(w_qkv)) return FC_ERR_INVALID_ARG;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FC_ERR_CUDA;
  int nsm = 0, cc_major = 0, cc_minor = 0;
  if (cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&cc_major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&cc_minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return FC_ERR_CUDA;
  if (cc_major != 10 || cc_minor != 0) return FC_ERR_UNSUPPORTED;  // built for sm_100a only

  fc_handle* h = new (std::nothrow) fc_handle();
  if (!h) return FC_ERR_OOM;
  h->cfg = *cfg;
  h->device = dev;
  h->num_sms = nsm;
  h->w_qkv = w_qkv;
  const int H = cfg->n_heads, d = cfg->head_dim, half = d / 2;
  const bool tc_shape = cfg->dtype == FC_DTYPE_BF16 && d == 128 && cfg->hidden % 64 == 0 &&
                        (H % 2) == 0;
  h->tc_gemm = tc_shape;
  h->tc_attn = tc_shape;
  if (tc_shape)
    for (int sp = 2; sp <= 8; ++sp) h->splitk_clusters[sp] = fc::qkv_splitk_max_clusters(sp);

  const int qtile = h->tc_attn ? fc::kTcQTile : fc::kSimtQTile;
  h->ws.max_items = H * (cfg->max_total_q / qtile + cfg->max_batch + 1);
  // a split small batch has at most one entry per SM
  if (h->tc_attn) {
    h->ws.split_entries = nsm;
    if (h->ws.max_items < nsm) h->ws.max_items = nsm;
  }

  fc::Workspace& w = h->ws;
  size_t es = elem_size(cfg->dtype);
  bool ok = cudaMalloc(&w.q_buf, (size_t)cfg->max_total_q * H * d * es) == cudaSuccess &&
            cudaMalloc(&w.row_dst, (size_t)cfg->max_total_q * sizeof(int32_t)) == cudaSuccess &&
            cudaMalloc(&w.imp_acc, (size_t)cfg->max_total_k * sizeof(unsigned long long)) ==
                cudaSuccess &&
            cudaMalloc(&w.items, (size_t)w.max_items * sizeof(fc::WorkItem)) == cudaSuccess &&
            cudaMalloc(&w.sched, 4 * sizeof(int32_t)) == cudaSuccess &&
            cudaMalloc(&w.err, sizeof(int32_t)) == cudaSuccess &&
            cudaMalloc(&w.rope_cos, (size_t)cfg->max_pos * half * sizeof(float)) == cudaSuccess &&
            cudaMalloc(&w.rope_sin, (size_t)cfg->max_pos * half * sizeof(float)) == cudaSuccess;
  if (ok && h->tc_attn)
    ok = cudaMalloc(&w.items_fb, (size_t)w.max_items * sizeof(fc::WorkItem)) == cudaSuccess &&
         cudaMalloc(&w.split_stats, (size_t)w.split_entries * 256 * sizeof(float)) == cudaSuccess &&
         cudaMalloc(&w.split_o, (size_t)w.split_entries * 128 * 128 * sizeof(float)) ==
             cudaSuccess &&
         cudaMalloc(&w.split_cnt, (size_t)w.split_entries * sizeof(int32_t)) == cudaSuccess &&
         cudaMemset(w.split_cnt, 0, (size_t)w.split_entries * sizeof(int32_t)) == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    free_workspace(h);
    delete h;
    return FC_ERR_OOM;
  }
  // RoPE table: angle pos * theta^(-2i/d), evaluated in double on the host and
  // stored as float (rotate-half pairing (i, i + d/2)).
  std::vector<float> tc((size_t)cfg->max_pos * half), ts((size_t)cfg->max_pos * half);
  for (int i = 0; i < half; ++i) {
    const double inv_freq = pow(cfg->rope_theta, -2.0 * (double)i / (double)d);
    for (int p = 0; p < cfg->max_pos; ++p) {
      const double a = (double)p * inv_freq;
      tc[(size_t)p * half + i] = (float)cos(a);
      ts[(size_t)p * half + i] = (float)sin(a);
    }
  }
  ok = cudaMemcpy(w.rope_cos, tc.data(), tc.size() * sizeof(float), cudaMemcpyHostToDevice) ==
           cudaSuccess &&
       cudaMemcpy(w.rope_sin, ts.data(), ts.size() * sizeof(float), cudaMemcpyHostToDevice) ==
           cudaSuccess &&
       cudaMemset(w.imp_acc, 0, (size_t)cfg->max_total_k * sizeof(unsigned long long)) ==
           cudaSuccess &&
       cudaMemset(w.err, 0, sizeof(int32_t)) == cudaSuccess &&
       cudaMemset(w.sched, 0, 4 * sizeof(int32_t)) == cudaSuccess &&
       cudaMemset(w.row_dst, 0xFF, (size_t)cfg->max_total_q * sizeof(int32_t)) == cudaSuccess;
  if (ok && h->tc_gemm)
    ok = fc::encode_bf16_2d(&h->tm_w, w_qkv, (uint64_t)3 * H * d, (uint64_t)cfg->hidden,
                            (uint64_t)cfg->hidden * 2, fc::kQkvWBoxRows, 64);
  if (ok && h->tc_attn)
    ok = fc::encode_bf16_2d(&h->tm_q, w.q_buf, (uint64_t)cfg->max_total_q * H, (uint64_t)d,
                            (uint64_t)d * 2, 128, 64) &&
         cudaMemset(w.q_buf, 0, (size_t)cfg->max_total_q * H * d * es) == cudaSuccess;
  if (!ok || cudaDeviceSynchronize() != cudaSuccess) {
    cudaGetLastError();
    free_workspace(h);
    delete h;
    return FC_ERR_CUDA;
  }
  *out = h;
  return FC_OK;
}

fc_status fc_step(fc_handle* h, void* stream, int batch, const void* x, const int32_t* q_pos,
                  const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int total_q,
                  int total_k, void* k_cache, void* v_cache, void* out, float* importance,
                  int accumulate) {
  if (!h) return FC_ERR_INVALID_ARG;
  return fc::step_impl(h, &h->tm_w, stream, batch, x, q_pos, cu_seqlens_q, cu_seqlens_k, total_q,
                       total_k, k_cache, v_cache, out, importance, accumulate);
}

}  // extern "C"

// Projection kernel of the tensor-core path for total_q query rows: the
// CTA-pair kernel unless the split-K kernel is forced (FC_OPT_QKV_KERNEL).
// The split-K kernel spreads each 128-row tile's reduction over a cluster of
// `split` CTAs; measured on one B200 it was never faster than the pair kernel
// (a 128 x 4096 query: 42.5 us at split 2 against 41.3 us, and 66-146 us at
// splits 3-8, whose clusters no longer fit the GPU at once; hidden 256:
// 27 against 19 us), so the default keeps the pair kernel.  With a split
// forced, the largest split whose clusters all fit at once is the default
// cluster size (at most 8 and one CTA per 64-wide K step).
struct QkvPlan {
  int kernel;  // 0 CUDA-core path, 1 CTA pair, 2 split-K
  int split;
};
static QkvPlan plan_qkv(const fc_handle* h, int total_q) {
  if (!h->tc_gemm) return {0, 0};
  const fc_config& c = h->cfg;
  const int n_tiles = 3 * c.n_heads * c.head_dim / 256;
  const int tiles = (total_q + 127) / 128 * n_tiles;
  const int smax = c.hidden / 64 < 8 ? c.hidden / 64 : 8;
  if (h->qkv_kernel != 2) return {1, 0};
  if (h->qkv_split > 0) return {2, h->qkv_split};
  for (int sp = smax; sp >= 2; --sp)
    if (tiles <= h->splitk_clusters[sp]) return {2, sp};
  return {2, 1};
}

fc_status fc::step_impl(fc_handle* h, const CUtensorMap* tm_w, void* stream, int batch,
                        const void* x, const int32_t* q_pos,
                        const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int total_q,
                        int total_k, void* k_cache, void* v_cache, void* out, float* importance,
                        int accumulate) {
  const fc_config& c = h->cfg;
  if (batch < 1 || batch > c.max_batch || total_q < 0 || total_q > c.max_total_q || total_k < 0 ||
      total_k > c.max_total_k || (accumulate != 0 && accumulate != 1))
    return FC_ERR_INVALID_ARG;
  if (!cu_seqlens_q || !cu_seqlens_k) return FC_ERR_INVALID_ARG;
  if (total_q > 0 && (!x || !q_pos || !k_cache || !v_cache || !out)) return FC_ERR_INVALID_ARG;
  if (total_q > 0 && (!aligned16(x) || !aligned16(k_cache) || !aligned16(v_cache) ||
                      !aligned16(out)))
    return FC_ERR_INVALID_ARG;
  if (importance && ((uintptr_t)importance & 3u)) return FC_ERR_INVALID_ARG;
  if (cudaSetDevice(h->device) != cudaSuccess) return FC_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  h->last_stream = st;
  h->last_launches = 0;

  if (total_q == 0) {
    if (importance && !accumulate && total_k > 0) {
      if (cudaMemsetAsync(importance, 0, (size_t)total_k * sizeof(float), st) != cudaSuccess)
        return FC_ERR_CUDA;
    }
    return FC_OK;
  }
  StepShape s{batch, total_q, total_k, c.hidden, c.n_heads, c.head_dim, c.max_pos, c.max_seqlen_q};
  const bool want_imp = importance != nullptr;
  // A small batch (at most one 128-row item per SM even if every sequence
  // ends in a partial query tile) splits its items' caches over the SMs and
  // runs the two attention passes as two launches when its caches hold 1280
  // rows or more on average, or when the step has no importance (its unsplit
  // path is two launches as well: the one-pass kernel and the hand-over
  // kernel).  With importance and shorter caches the single two-pass launch
  // is as fast or faster (each launch costs several microseconds of fixed
  // latency; measured at B = 1: 768 rows 67.8 us unsplit vs 71.2 split, 1024
  // rows 71.7 vs 72.7, 1536 rows 80.1 vs 75.5).
  const bool split_attn =
      h->tc_attn && h->attn_split != 1 &&
      (long long)c.n_heads * ((total_q + fc::kTcQTile - 1) / fc::kTcQTile + batch - 1) <=
          h->ws.split_entries &&
      (h->attn_split == 2 || !want_imp || (long long)total_k >= 1280LL * batch);
  cudaError_t e;
  {
    ProfScope ps(h, st, 0);
    // tensor-core path: with importance (or split) every item goes to the
    // two-pass kernel (long_tiles 0), without it to the one-pass kernel
    e = fc::launch_prep(h, st, s, q_pos, cu_seqlens_q, cu_seqlens_k,
                        h->tc_attn ? fc::kTcQTile : fc::kSimtQTile,
                        (h->tc_attn && (want_imp || split_attn)) ? 0 : 0x7fffffff,
                        split_attn ? h->ws.split_entries : 0, 1);
  }
  if (e != cudaSuccess) return cuda_fail(h, 0, e);
  h->last_launches++;
  if (h->tc_gemm) {
    CUtensorMap tm_x;
    if (!fc::encode_bf16_2d(&tm_x, x, (uint64_t)total_q, (uint64_t)c.hidden,
                            (uint64_t)c.hidden * 2, fc::kQkvXBoxRows, 64))
      return cuda_fail(h, -1, cudaErrorInvalidValue);
    const QkvPlan plan = plan_qkv(h, total_q);
    if (plan.kernel == 2 && plan.split > c.hidden / 64) return FC_ERR_INVALID_ARG;
    ProfScope ps(h, st, 1);
    e = plan.kernel == 2
            ? fc::launch_qkv_splitk(h, st, s, tm_x, *tm_w, q_pos, k_cache, v_cache, plan.split)
            : fc::launch_qkv_tc(h, st, s, tm_x, *tm_w, q_pos, k_cache, v_cache);
  } else {
    ProfScope ps(h, st, 1);
    e = fc::launch_qkv_simt(h, st, s, x, q_pos, k_cache, v_cache);
  }
  if (e != cudaSuccess) return cuda_fail(h, 1, e);
  h->last_launches++;
  if (h->tc_attn) {
    CUtensorMap tm_k, tm_v;
    if (!fc::encode_kv_3d(&tm_k, k_cache, total_k, c.n_heads) ||
        !fc::encode_kv_3d(&tm_v, v_cache, total_k, c.n_heads))
      return cuda_fail(h, -1, cudaErrorInvalidValue);
    if (split_attn) {
      // pass 1 of every entry (row statistics), then pass 2 and the combine
      {
        ProfScope ps(h, st, 8);
        e = fc::launch_attn_tc(h, st, s, tm_k, tm_v, cu_seqlens_q, cu_seqlens_k, out, want_imp, 1);
      }
      if (e != cudaSuccess) return cuda_fail(h, 8, e);
      h->last_launches++;
      ProfScope ps(h, st, 2);
      e = fc::launch_attn_tc(h, st, s, tm_k, tm_v, cu_seqlens_q, cu_seqlens_k, out, want_imp, 2);
      if (e != cudaSuccess) return cuda_fail(h, 2, e);
    } else if (want_imp) {
      // the importance needs every row's final normaliser: two scans of K
      ProfScope ps(h, st, 2);
      e = fc::launch_attn_tc(h, st, s, tm_k, tm_v, cu_seqlens_q, cu_seqlens_k, out, true, 0);
      if (e != cudaSuccess) return cuda_fail(h, 2, e);
    } else {
      {
        ProfScope ps(h, st, 5);
        e = fc::launch_attn_onepass(h, st, tm_k, tm_v, cu_seqlens_q, cu_seqlens_k, out);
      }
      if (e != cudaSuccess) return cuda_fail(h, 5, e);
      h->last_launches++;
      // the items the one-pass kernel handed over (usually none)
      ProfScope ps(h, st, 2);
      e = fc::launch_attn_tc(h, st, s, tm_k, tm_v, cu_seqlens_q, cu_seqlens_k, out, false, 0);
      if (e != cudaSuccess) return cuda_fail(h, 2, e);
    }
  } else {
    ProfScope ps(h, st, 2);
    e = fc::launch_attn_simt(h, st, s, cu_seqlens_q, cu_seqlens_k, k_cache, v_cache, out,
                             want_imp);
    if (e != cudaSuccess) return cuda_fail(h, 2, e);
  }
  h->last_launches++;
  if (want_imp) {
    {
      ProfScope ps(h, st, 3);
      e = fc::launch_importance_finalize(h, st, total_k, importance, accumulate);
    }
    if (e != cudaSuccess) return cuda_fail(h, 3, e);
    h->last_launches++;
  }
  return FC_OK;
}

extern "C" {

fc_status fc_topk_tracked(fc_handle* h, void* stream, int batch, int total_k,
                          const float* importance, const int32_t* cu_seqlens_k,
                          const int32_t* cand_lo, const int32_t* cand_hi,
                          const int32_t* k_per_seq, int k, int32_t* tracked) {
  if (!h) return FC_ERR_INVALID_ARG;
  if (batch < 1 || batch > h->cfg.max_batch || k < 0 || k > h->cfg.max_topk || total_k < 0 ||
      total_k > h->cfg.max_total_k)
    return FC_ERR_INVALID_ARG;
  if (!importance || !cu_seqlens_k || !cand_lo || !cand_hi || (k > 0 && !tracked))
    return FC_ERR_INVALID_ARG;
  if (cudaSetDevice(h->device) != cudaSuccess) return FC_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  h->last_stream = st;
  h->last_launches = 0;
  if (k == 0) return FC_OK;
  cudaError_t e;
  {
    ProfScope ps(h, st, 4);
    e = fc::launch_topk(h, st, batch, total_k, importance, cu_seqlens_k, cand_lo, cand_hi,
                        k_per_seq, k, tracked);
  }
  if (e != cudaSuccess) return FC_ERR_CUDA;
  h->last_launches = 1;
  return FC_OK;
}

fc_status fc_last_step_work(fc_handle* h, int32_t* items, int32_t* two_pass_items,
                            int32_t* handed_over) {
  if (!h || !items || !two_pass_items || !handed_over) return FC_ERR_INVALID_ARG;
  if (cudaSetDevice(h->device) != cudaSuccess) return FC_ERR_CUDA;
  if (cudaStreamSynchronize(h->last_stream) != cudaSuccess) return FC_ERR_CUDA;
  int32_t sc[4] = {0, 0, 0, 0};
  if (cudaMemcpy(sc, h->ws.sched, sizeof(sc), cudaMemcpyDeviceToHost) != cudaSuccess)
    return FC_ERR_CUDA;
  *items = sc[0];
  *two_pass_items = h->tc_attn ? sc[2] : 0;
  *handed_over = h->tc_attn ? sc[3] : 0;
  return FC_OK;
}

fc_status fc_get_error(fc_handle* h, int32_t* device_error_word) {
  if (!h || !device_error_word) return FC_ERR_INVALID_ARG;
  if (cudaSetDevice(h->device) != cudaSuccess) return FC_ERR_CUDA;
  if (cudaStreamSynchronize(h->last_stream) != cudaSuccess) return FC_ERR_CUDA;
  int32_t word = 0;
  if (cudaMemcpy(&word, h->ws.err, sizeof(int32_t), cudaMemcpyDeviceToHost) != cudaSuccess)
    return FC_ERR_CUDA;
  if (cudaMemset(h->ws.err, 0, sizeof(int32_t)) != cudaSuccess) return FC_ERR_CUDA;
  *device_error_word = word;
  if (word == 0) return FC_OK;
  return (word & FC_DEVERR_TIMEOUT) ? FC_ERR_TIMEOUT : FC_ERR_DEVICE_CHECK;
}

int fc_last_launch_count(const fc_handle* h) { return h ? h->last_launches : 0; }

fc_status fc_qkv_plan(const fc_handle* h, int total_q, int* kernel, int* split,
                      int* max_clusters) {
  if (!h || total_q < 0 || !kernel || !split) return FC_ERR_INVALID_ARG;
  const QkvPlan p = plan_qkv(h, total_q);
  *kernel = p.kernel;
  *split = p.split;
  if (max_clusters) {
    const int smax = h->cfg.hidden / 64 < 8 ? h->cfg.hidden / 64 : 8;
    const int sp = p.split >= 2 ? p.split : smax;
    *max_clusters = (h->tc_gemm && sp >= 2) ? h->splitk_clusters[sp] : 0;
  }
  return FC_OK;
}

fc_status fc_set_option(fc_handle* h, int option, int value) {
  if (!h) return FC_ERR_INVALID_ARG;
  if (option == FC_OPT_QKV_KERNEL) {
    if (value < 0 || value > 2) return FC_ERR_INVALID_ARG;
    h->qkv_kernel = value;
    return FC_OK;
  }
  if (option == FC_OPT_QKV_SPLIT) {
    if (value < 0 || value > 8) return FC_ERR_INVALID_ARG;
    h->qkv_split = value;
    return FC_OK;
  }
  if (option == FC_OPT_ATTN_SPLIT) {
    if (value < 0 || value > 2) return FC_ERR_INVALID_ARG;
    h->attn_split = value;
    return FC_OK;
  }
  return FC_ERR_INVALID_ARG;
}

const char* fc_last_cuda_error(const fc_handle* h) {
  static const char* const kSlot[] = {"prep", "qkv_rope_scatter", "attention",
                                      "importance_finalize", "topk", "attention_one_pass",
                                      "h2d_copy", "d2h_copy", "attention_split_pass1"};
  static thread_local char buf[256];
  if (!h || h->last_cuda_err == cudaSuccess) return "no CUDA error recorded";
  snprintf(buf, sizeof(buf), "%s: %s (%s)",
           h->last_cuda_slot >= 0 && h->last_cuda_slot < 8 ? kSlot[h->last_cuda_slot]
                                                           : "host call",
           cudaGetErrorName(h->last_cuda_err), cudaGetErrorString(h->last_cuda_err));
  return buf;
}

fc_status fc_selftest_wait_timeout(fc_handle* h, void* stream, int limit_us) {
  if (!h || limit_us < 1 || limit_us > 2000000) return FC_ERR_INVALID_ARG;
  if (cudaSetDevice(h->device) != cudaSuccess) return FC_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  h->last_stream = st;
  h->last_launches = 0;
  if (fc::launch_selftest_wait_timeout(h, st, limit_us) != cudaSuccess) return FC_ERR_CUDA;
  h->last_launches = 1;
  return FC_OK;
}

fc_status fc_profile(fc_handle* h, int enable) {
  if (!h || (enable != 0 && enable != 1)) return FC_ERR_INVALID_ARG;
  if (cudaSetDevice(h->device) != cudaSuccess) return FC_ERR_CUDA;
  if (enable && !h->prof_ev) {
    h->prof_ev = new (std::nothrow) cudaEvent_t[2 * 4096];
    if (!h->prof_ev) return FC_ERR_OOM;
    for (int i = 0; i < 2 * 4096; ++i)
      if (cudaEventCreate(&h->prof_ev[i]) != cudaSuccess) return FC_ERR_CUDA;
  }
  h->profiling = enable != 0;
  return FC_OK;
}

fc_status fc_profile_timeline(fc_handle* h, int max_records, int32_t* slot, float* start_ms,
                              float* end_ms, int* n) {
  if (!h || max_records < 0 || !n || (max_records > 0 && (!slot || !start_ms || !end_ms)))
    return FC_ERR_INVALID_ARG;
  *n = 0;
  if (!h->prof_ev || h->prof_n == 0) return FC_OK;
  if (cudaSetDevice(h->device) != cudaSuccess) return FC_ERR_CUDA;
  const int m = h->prof_n < max_records ? h->prof_n : max_records;
  for (int i = 0; i < h->prof_n; ++i)
    if (cudaEventSynchronize(h->prof_ev[2 * i + 1]) != cudaSuccess) return FC_ERR_CUDA;
  for (int i = 0; i < m; ++i) {
    float a = 0.f, b = 0.f;
    if (cudaEventElapsedTime(&a, h->prof_ev[0], h->prof_ev[2 * i]) != cudaSuccess ||
        cudaEventElapsedTime(&b, h->prof_ev[0], h->prof_ev[2 * i + 1]) != cudaSuccess)
      return FC_ERR_CUDA;
    slot[i] = h->prof_slot[i];
    start_ms[i] = a;
    end_ms[i] = b;
  }
  *n = m;
  return FC_OK;
}

fc_status fc_profile_read(fc_handle* h, float* ms, int* launches) {
  if (!h || !ms || !launches) return FC_ERR_INVALID_ARG;
  for (int s = 0; s < FC_PROFILE_SLOTS; ++s) {
    ms[s] = 0.f;
    launches[s] = 0;
  }
  if (!h->prof_ev || h->prof_n == 0) return FC_OK;
  if (cudaSetDevice(h->device) != cudaSuccess) return FC_ERR_CUDA;
  for (int i = 0; i < h->prof_n; ++i) {
    if (cudaEventSynchronize(h->prof_ev[2 * i + 1]) != cudaSuccess) return FC_ERR_CUDA;
    float t = 0.f;
    if (cudaEventElapsedTime(&t, h->prof_ev[2 * i], h->prof_ev[2 * i + 1]) != cudaSuccess)
      return FC_ERR_CUDA;
    ms[h->prof_slot[i]] += t;
    launches[h->prof_slot[i]] += 1;
  }
  h->prof_n = 0;
  return FC_OK;
}

void fc_destroy(fc_handle* h) {
  if (!h) return;
  cudaSetDevice(h->device);
  cudaDeviceSynchronize();
  free_workspace(h);
  fc::free_host_pipe(h);
  if (h->prof_ev) {
    for (int i = 0; i < 2 * 4096; ++i) cudaEventDestroy(h->prof_ev[i]);
    delete[] h->prof_ev;
  }
  delete h;
}

}  // extern "C"
