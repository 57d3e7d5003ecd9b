// Internal declarations shared by the host runtime and the kernels of
// libflashcache.so.  Not part of the public ABI (include/flashcache.h).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/flashcache.h"

namespace fc {

// Query rows per attention work item of the tensor-core path and of the SIMT
// path.  A work item is one (sequence, head, query tile).
constexpr int kTcQTile = 128;
constexpr int kSimtQTile = 16;

// TMA boxes of the tensor-core projection (rows x 64 bf16 columns): each CTA
// of a pair loads 128 rows of X and 128 rows (half the 256-row tile) of W.
constexpr int kQkvXBoxRows = 128;
constexpr int kQkvWBoxRows = 128;
// TMA boxes of the model's other projections (gemm_tc): 128 rows x 64 columns
// for both operands.
constexpr int kGemmBoxRows = 128;

// Epilogues of the generic tensor-core GEMM (gemm_tc.cu).
enum GemmMode { GEMM_RESID = 0, GEMM_SWIGLU = 1, GEMM_LMHEAD = 2 };

struct GemmParams {
  int mode;
  int M, N, K;     // rows of A, output columns (SwiGLU: features), reduction length
  int num_m, num_n, num_tiles, num_k;  // filled by the launcher
  int group_m;                         // tile raster (launcher): row blocks per group
  const __nv_bfloat16* resid;  // GEMM_RESID: [M, ldo] added to the product (may equal out)
  __nv_bfloat16* out;          // GEMM_RESID / GEMM_SWIGLU: [M, ldo]
  size_t ldo;                  // row stride of resid / out in elements
  float* partials;             // GEMM_LMHEAD: [M, num_n, 3] (max, sum exp, argmax bits)
  int32_t* err;
};

// Importance is accumulated in fixed point (int64, 2^-40 units) so that the
// sum over heads and query tiles is exact and independent of the order in
// which work items finish.  One column sum is at most kSimtQTile..128 and a
// key receives at most H * n_b contributions, far inside 2^23.
constexpr double kImpScale = 1099511627776.0;  // 2^40
constexpr double kImpInvScale = 1.0 / 1099511627776.0;

// Work-list item: sequence, query tile, head, and the item's ranges (written
// by the prep kernel, so a kernel starts an item with one 32-byte load).
struct __align__(16) WorkItem {
  int32_t seq;
  int32_t tile_head;  // (qtile << 8) | head
  int32_t q0;         // first query row of the sequence
  int32_t nrows;      // query rows of this tile
  int32_t k0;         // first cache row of the sequence
  int32_t L;          // cache rows of the sequence
  int32_t pad[2];
};

// Item index of CTA `cta` in round `round` of a persistent schedule over a
// work list ordered by decreasing cost: the rounds alternate direction (CTA c
// takes position c, then position ctas - 1 - c), which spreads the costly
// items more evenly than plain round-robin.
__device__ __forceinline__ int snake_item(int round, int cta, int ctas) {
  return round * ctas + ((round & 1) ? ctas - 1 - cta : cta);
}

struct Workspace {
  void* q_buf = nullptr;                  // [max_total_q, H, d] dtype; rotated, pre-scaled q
  int32_t* row_dst = nullptr;             // [max_total_q] cache row of query row, or -1
  unsigned long long* imp_acc = nullptr;  // [max_total_k] fixed-point importance
  WorkItem* items = nullptr;              // attention work list
  // [0] = item count, [1] = dynamic item counter (CUDA-core path),
  // [2] = items for the two-pass kernel (the first ones of the list),
  // [3] = items the one-pass kernel handed to the two-pass kernel
  int32_t* sched = nullptr;
  WorkItem* items_fb = nullptr;           // [max_items] those handed-over items
  int32_t* err = nullptr;                 // device error word
  float* rope_cos = nullptr;              // [max_pos, d/2]
  float* rope_sin = nullptr;              // [max_pos, d/2]
  int max_items = 0;
  // small batches, items split over several CTAs (tensor-core attention):
  float* split_stats = nullptr;           // [split_entries][m, l][128]
  float* split_o = nullptr;               // [split_entries][128 cols][128 rows] fp32 parts of O
  int32_t* split_cnt = nullptr;           // [split_entries] finished entries per item
  int split_entries = 0;
};

// Shapes of one step, as the kernels see them.
struct StepShape {
  int B, T, S, D, H, d;
  int max_pos, max_seqlen_q;
};

}  // namespace fc

namespace fc {
// Device staging and copy streams of fc_step_host (allocated on first use).
struct HostPipe {
  bool ready = false;
  cudaStream_t s_h2d = nullptr, s_d2h = nullptr;
  void* x[2] = {nullptr, nullptr};        // [max_total_q, hidden] dtype
  int32_t* small[2] = {nullptr, nullptr}; // q_pos | cu_q | cu_k | lo | hi | k_per_seq
  int32_t* small_h[2] = {nullptr, nullptr};  // pinned host copy of that block (one DMA per call)
  void* out[2] = {nullptr, nullptr};      // [max_total_q, H, d] dtype
  int32_t* tracked[2] = {nullptr, nullptr};  // [max_batch, max_topk]
  float* importance = nullptr;            // [max_total_k]
  cudaEvent_t h2d_done[2] = {}, comp_done[2] = {}, d2h_done[2] = {};
  // timed events recorded around each kernel of a pipelined step (never
  // queried; see fc_step_host)
  cudaEvent_t fence[2] = {};
  unsigned fence_i = 0;
  bool fencing = false;
  unsigned long long calls = 0;
};
}  // namespace fc

struct fc_handle {
  fc_config cfg;
  int device = 0;
  int num_sms = 0;
  // tensor-core kernels: bf16, head_dim 128, hidden % 64 == 0, H even
  bool tc_gemm = false;
  bool tc_attn = false;
  const void* w_qkv = nullptr;
  fc::Workspace ws;
  cudaStream_t last_stream = nullptr;
  int last_launches = 0;
  // launch the step's kernels with programmatic dependent launch (off while
  // fc_step_host runs: between the copies of neighbouring steps it lengthened
  // the pipelined step by a quarter)
  bool pdl = true;
  // projection kernel on the tensor-core path: 0 chooses by shape, 1 the CTA
  // pair kernel, 2 the split-K cluster kernel (fc_set_option)
  int qkv_kernel = 0;
  int qkv_split = 0;  // split-K cluster size: 0 chosen by shape, else forced
  int attn_split = 0;  // small-batch attention split: 0 by shape, 1 never
  // resident clusters of the split-K projection kernel per cluster size 2..8
  int splitk_clusters[9] = {};
  // the last CUDA call of fc_step that failed: its error and the profile slot
  // of the kernel being launched (-1: not a launch)
  cudaError_t last_cuda_err = cudaSuccess;
  int last_cuda_slot = -1;
  // optional per-kernel event timing (fc_profile)
  bool profiling = false;
  int prof_n = 0;
  int prof_slot[4096];
  cudaEvent_t* prof_ev = nullptr;  // 2 * 4096 events, created on first fc_profile(1)
  CUtensorMap tm_w;  // W_qkv, bf16 tensor-core path
  CUtensorMap tm_q;  // Q buffer, bf16 tensor-core path
  fc::HostPipe hp;   // fc_step_host
};

namespace fc {
void free_host_pipe(fc_handle* h);

// Begin / end one profiling record (slot, event pair) on a stream; no-op
// unless fc_profile is on.  Returns the record index or -1.
inline int prof_begin(fc_handle* h, cudaStream_t st, int slot) {
  if (!h->profiling || h->prof_n >= 4096) return -1;
  const int idx = h->prof_n++;
  h->prof_slot[idx] = slot;
  cudaEventRecord(h->prof_ev[2 * idx], st);
  return idx;
}
inline void prof_end(fc_handle* h, cudaStream_t st, int idx) {
  if (idx >= 0) cudaEventRecord(h->prof_ev[2 * idx + 1], st);
}
}

namespace fc {

// Launch with programmatic stream serialisation (when `pdl`): the kernel may
// be scheduled while the previous kernel of the stream is still running; it
// must call griddepcontrol.wait before touching that kernel's outputs (a
// no-op when it was launched without the attribute).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_if(bool pdl, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args... args) {
  return launch_pdl_if(true, kernel, grid, block, smem, st, args...);
}

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize, bytes) for `fn`, once per
// kernel, device and size: the runtime call costs host time at every launch.
cudaError_t smem_attr_once(const void* fn, size_t bytes);
template <typename... A>
inline cudaError_t smem_attr(void (*fn)(A...), size_t bytes) {
  return smem_attr_once(reinterpret_cast<const void*>(fn), bytes);
}

// ---- launchers (each returns the CUDA error of its launch) -----------------
cudaError_t launch_prep(const fc_handle* h, cudaStream_t st, const StepShape& s,
                        const int32_t* q_pos, const int32_t* cu_q, const int32_t* cu_k,
                        int qtile, int long_tiles, int split_sms, int split_min_tiles);
cudaError_t launch_qkv_simt(const fc_handle* h, cudaStream_t st, const StepShape& s,
                            const void* x, const int32_t* q_pos, void* k_cache, void* v_cache);
cudaError_t launch_attn_simt(const fc_handle* h, cudaStream_t st, const StepShape& s,
                             const int32_t* cu_q, const int32_t* cu_k, const void* k_cache,
                             const void* v_cache, void* out, bool want_importance);
cudaError_t launch_qkv_tc(const fc_handle* h, cudaStream_t st, const StepShape& s,
                          const CUtensorMap& tm_x, const CUtensorMap& tm_w, const int32_t* q_pos,
                          void* k_cache, void* v_cache);
cudaError_t launch_qkv_splitk(const fc_handle* h, cudaStream_t st, const StepShape& s,
                              const CUtensorMap& tm_x, const CUtensorMap& tm_w,
                              const int32_t* q_pos, void* k_cache, void* v_cache, int split);
size_t qkv_splitk_smem_bytes();
// thread-block clusters of `split` CTAs of the split-K kernel that can be
// resident at once (cudaOccupancyMaxActiveClusters); minus the CUDA error
// code when the query fails
int qkv_splitk_max_clusters(int split);
cudaError_t launch_gemm_tc(int num_sms, cudaStream_t st, const CUtensorMap& tm_a,
                           const CUtensorMap& tm_b0, const CUtensorMap& tm_b1, GemmParams p);
size_t gemm_tc_smem_bytes();
// model_kernels.cu
cudaError_t launch_rmsnorm(cudaStream_t st, const __nv_bfloat16* x, const int32_t* rows, int n_rows,
                           int D, const __nv_bfloat16* g, float eps, __nv_bfloat16* y);
cudaError_t launch_lmhead_reduce(cudaStream_t st, const float* partials, int R, int num_n,
                                 float threshold, int32_t* token, float* confidence,
                                 uint8_t* accept);
// The body of fc_step with the projection weights' tensor map given (the
// model runs every layer through one handle's workspace).
fc_status step_impl(fc_handle* h, const CUtensorMap* tm_w, void* stream, int batch, const void* x, const int32_t* q_pos, const int32_t* cu_seqlens_q,
                    const int32_t* cu_seqlens_k, int total_q, int total_k, void* k_cache,
                    void* v_cache, void* out, float* importance, int accumulate);
cudaError_t launch_attn_tc(const fc_handle* h, cudaStream_t st, const StepShape& s,
                           const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                           const int32_t* cu_q, const int32_t* cu_k, void* out,
                           bool want_importance, int mode);
cudaError_t launch_attn_onepass(const fc_handle* h, cudaStream_t st, const CUtensorMap& tm_k,
                                const CUtensorMap& tm_v, const int32_t* cu_q, const int32_t* cu_k,
                                void* out);
size_t attn_onepass_smem_bytes();
cudaError_t launch_importance_finalize(const fc_handle* h, cudaStream_t st, int S,
                                       float* importance, int accumulate);
cudaError_t launch_topk(const fc_handle* h, cudaStream_t st, int B, int S, const float* importance,
                        const int32_t* cu_k, const int32_t* cand_lo, const int32_t* cand_hi,
                        const int32_t* k_per_seq, int k, int32_t* tracked);

cudaError_t launch_selftest_wait_timeout(const fc_handle* h, cudaStream_t st, int limit_us);
size_t qkv_tc_smem_bytes();
size_t attn_tc_smem_bytes();
bool encode_kv_3d(CUtensorMap* tm, const void* cache, int S, int H);
bool encode_bf16_2d(CUtensorMap* tm, const void* base, uint64_t rows, uint64_t cols,
                    uint64_t row_stride_bytes, uint32_t box_rows, uint32_t box_cols);

// Dynamic shared memory the prep kernel needs for a given max_pos.
size_t prep_smem_bytes(int max_pos, int max_batch);

}  // namespace fc
