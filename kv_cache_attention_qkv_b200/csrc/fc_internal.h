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
  void* out[2] = {nullptr, nullptr};      // [max_total_q, H, d] dtype
  int32_t* tracked[2] = {nullptr, nullptr};  // [max_batch, max_topk]
  float* importance = nullptr;            // [max_total_k]
  cudaEvent_t h2d_done[2] = {}, comp_done[2] = {}, d2h_done[2] = {};
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
}

namespace fc {

// Launch with programmatic stream serialisation: the kernel may be scheduled
// while the previous kernel of the stream is still running; it must call
// griddepcontrol.wait before touching that kernel's outputs.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
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
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// ---- launchers (each returns the CUDA error of its launch) -----------------
cudaError_t launch_prep(const fc_handle* h, cudaStream_t st, const StepShape& s,
                        const int32_t* q_pos, const int32_t* cu_q, const int32_t* cu_k,
                        int qtile, int long_tiles);
cudaError_t launch_qkv_simt(const fc_handle* h, cudaStream_t st, const StepShape& s,
                            const void* x, const int32_t* q_pos, void* k_cache, void* v_cache);
cudaError_t launch_attn_simt(const fc_handle* h, cudaStream_t st, const StepShape& s,
                             const int32_t* cu_q, const int32_t* cu_k, const void* k_cache,
                             const void* v_cache, void* out, bool want_importance);
cudaError_t launch_qkv_tc(const fc_handle* h, cudaStream_t st, const StepShape& s,
                          const CUtensorMap& tm_x, const CUtensorMap& tm_w, const int32_t* q_pos,
                          void* k_cache, void* v_cache);
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
                           bool want_importance);
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
