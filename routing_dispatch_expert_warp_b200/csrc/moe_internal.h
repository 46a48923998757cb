// Host-side declarations shared by the translation units of the MoE library: the checked
// layer shape, the workspace layout and the kernel launchers.  Not part of the C ABI.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "moe.h"
#include "moe_device.cuh"

namespace moe {

constexpr int kDispatchBlockTokens = 256;   // tokens per block of the ranking kernels
constexpr int kMaxDevices = 64;
constexpr size_t kWsAlign = 256;

// A validated moe_config_t with the derived sizes.
struct Shape {
  int64_t T, d, f;
  int E, k, gating, layout, dtype;
  int n_groups, topk_groups, bias_mode, drop_policy;
  int64_t C;         // capacity, -1 when dropless
  int64_t max_rows;  // rows of x_perm / h / y_perm / token_of_row
  int64_t elem;      // bytes per element of x, weights and activations
};

// Offsets (bytes) of the workspace sections.
struct WsLayout {
  size_t status;        // DevStatus, 256 B
  size_t hist;          // [n_dispatch_blocks, planes, E] int32 per-block counts
  size_t hist_bytes;
  size_t logits;        // [T, E] fp32 logits when the caller passes none
  size_t logits_bytes;
  size_t partials;      // split-K router partial sums (E > 32) / lane-ordered W_r (E <= 32)
  size_t partials_bytes;
  size_t router_tc;     // bf16 split of W_r for the tensor-core router
  size_t router_tc_bytes;
  size_t ep_base;       // [E] int32: first row of this rank's rows per expert at the owner
  size_t arrive;        // [T, ceil(d/256)] int32 counters of the combine fused into the FFN
  size_t score;         // score-priority dispatch scratch (dispatch_score_scratch_bytes)
  size_t total;
};

inline int64_t dispatch_blocks(int64_t T) {
  return (T + kDispatchBlockTokens - 1) / kDispatchBlockTokens;
}
// Count planes of dispatch: one per pick rank when drops go by pick rank, else one.
inline int dispatch_planes(const Shape& s) {
  return s.drop_policy == MOE_DROP_PICK_RANK ? s.k : 1;
}
// Bytes of per-block expert counts dispatch needs.
inline size_t dispatch_hist_bytes(const Shape& s) {
  return static_cast<size_t>(dispatch_blocks(s.T)) * dispatch_planes(s) * s.E * sizeof(int32_t);
}
WsLayout workspace_layout(const Shape& s);

// Kernel launchers (return the CUDA error of the launch).
// Router on CUDA cores: fused top-k for E <= 32; for E > 32 a tiled fp32 GEMM, split along
// d into router_splits(s) pieces (partials: that many [T, E] fp32 buffers) when the token
// count alone cannot fill the GPU.
constexpr int kMaxRouterSplits = 64;
int router_splits(const Shape& s);
cudaError_t launch_router(const Shape& s, const void* x, const float* w_router,
                          const float* bias, int64_t bias_stride, float* logits,
                          int32_t* topk_idx, float* topk_w, float* partials, cudaStream_t st);
// Router on tensor cores (bf16 layers, E > 32, d % 64 == 0): W_r split into two bf16 terms,
// W' = [E, 2 d] (hi | lo along K).
bool router_uses_tensor_cores(const Shape& s);
// pieces each 128-token tile's K steps are split into (1: none) and K steps per piece
int router_tc_splits(const Shape& s, int* kb_per_split);
bool router_split_applies(const Shape& s);   // the layer shape admits the split (any T)
size_t router_split_bytes(const Shape& s);   // bytes of W' (0 when the split does not apply)
cudaError_t launch_router_split(const Shape& s, const float* w_router, void* w_split,
                                cudaStream_t st);
// w_split: W' made earlier by launch_router_split, or nullptr (then W_r is split into
// split_ws for this call).  logits: the caller's [T, E] buffer, or nullptr (then z goes to
// logits_scratch, the workspace copy).  partials: router_tc_splits(s) x [T, E] fp32 (used
// only when K is split).
cudaError_t launch_router_tc(const Shape& s, const void* x, const float* w_router,
                             const void* w_split, const float* bias, int64_t bias_stride,
                             float* logits, float* logits_scratch, int32_t* topk_idx,
                             float* topk_w, void* split_ws, float* partials, DevStatus* status,
                             uint64_t wait_ns, cudaStream_t st, const char** why);
size_t router_tc_workspace_bytes(const Shape& s);
cudaError_t launch_topk_from_logits(const Shape& s, const float* logits, const float* bias,
                                    int64_t bias_stride, int32_t* topk_idx, float* topk_w,
                                    cudaStream_t st);
// top-k over nsplit [T, E] fp32 partial sums (added in split order, then the bias unless it
// only steers selection), writing the finished logits to `logits`
cudaError_t launch_topk_from_partials(const Shape& s, const float* partials, int nsplit,
                                      const float* bias, int64_t bias_stride, float* logits,
                                      int32_t* topk_idx, float* topk_w, cudaStream_t st);
// Selection scores for dispatch with drop_policy == MOE_DROP_SCORE: score of (t, e) =
// logits[t, e] (+ bias[t * bias_stride + e] when the bias is selection-only), and the
// scratch (dispatch_score_scratch_bytes, 256-byte aligned) the ranking by score needs.
struct DispatchScores {
  const float* logits;
  const float* bias;
  int64_t bias_stride;
  void* scratch;
};
size_t dispatch_score_scratch_bytes(const Shape& s);
cudaError_t launch_dispatch(const Shape& s, const void* x, const int32_t* topk_idx,
                            int32_t* routed, int32_t* kept, int32_t* offsets,
                            int32_t* assign_row, int32_t* token_of_row, void* x_perm,
                            int32_t* hist, DevStatus* status, uint64_t wait_ns,
                            cudaStream_t st, const DispatchScores* scores = nullptr);
// Second-choice counters: per pick rank j and expert e the assignments (routed) and the
// kept ones, and per j the tokens whose pick j lies in another group than pick 0.
cudaError_t launch_pick_rank_counts(const Shape& s, const int32_t* topk_idx,
                                    const int32_t* assign_row, const int32_t* group_of_expert,
                                    int32_t* routed, int32_t* kept, int32_t* differs,
                                    DevStatus* status, cudaStream_t st);
// Expert FFN.  `a` holds the gate/up GEMM's A rows: x_perm (a_rows == nullptr) or x itself,
// bucket row r reading row a_rows[r] of x (token_of_row: dispatch without the permute copy).
cudaError_t launch_ffn_simt(const Shape& s, const float* a, const int32_t* a_rows,
                            const int32_t* offsets, const int32_t* kept, const float* wg,
                            const float* wu, const float* wd, float* h, float* y,
                            cudaStream_t st);
// Combine fused into the bf16 down launch (bitwise the combine kernel's result).
struct FusedCombine {
  const int32_t* token_of_row;
  const int32_t* assign_row;
  const float* topk_w;
  int32_t* arrive;  // workspace counters [T, ceil(d / 256)]
  void* out;        // [T, d]
};
cudaError_t launch_ffn_tc(const Shape& s, const void* a, const int32_t* a_rows,
                          const int32_t* offsets, const int32_t* kept, const void* wg,
                          const void* wu, const void* wd, void* h, void* y, DevStatus* status,
                          uint64_t wait_ns, cudaStream_t st, const char** why,
                          const FusedCombine* comb = nullptr);
cudaError_t launch_combine(const Shape& s, const void* y_perm, const int32_t* assign_row,
                           const float* topk_w, void* out, cudaStream_t st);
cudaError_t launch_stats(const Shape& s, const int32_t* routed, const int32_t* kept,
                         const int32_t* assign_row, moe_load_stats_t* out, cudaStream_t st);
// The job record of data-parallel replicas from their summed counts and their records.
cudaError_t launch_stats_merge(const Shape& s, const int32_t* routed_sum,
                               const int32_t* kept_sum, const moe_load_stats_t* parts,
                               int n_parts, moe_load_stats_t* out, cudaStream_t st);
cudaError_t launch_wait_selftest(DevStatus* status, uint64_t wait_ns, cudaStream_t st);

int sm_count();

// Expert parallelism over peer (or shared-device) memory.
cudaError_t launch_ep_put_counts(const Shape& s, const int32_t* kept, int rank, int world,
                                 int32_t* const* mats, cudaStream_t st);
cudaError_t launch_ep_plan(const Shape& s, const int32_t* mat, const int32_t* expert_rank,
                           int world, int rank, int n_local, int64_t recv_rows,
                           const int32_t* topk_idx,
                           const int32_t* assign_row, const int32_t* expert_offsets,
                           int32_t* base, int32_t* send_row, int32_t* recv_offsets,
                           int32_t* recv_counts, DevStatus* status, cudaStream_t st);
cudaError_t launch_ep_dispatch(const Shape& s, const void* x, const int32_t* topk_idx,
                               const int32_t* send_row, const int32_t* expert_rank, int world,
                               void* const* recv, int64_t recv_rows, DevStatus* status,
                               cudaStream_t st);
cudaError_t launch_ep_combine(const Shape& s, const void* const* ybuf, const int32_t* topk_idx,
                              const int32_t* send_row, const int32_t* expert_rank, int world,
                              int64_t recv_rows, const float* topk_w, void* out,
                              cudaStream_t st);
cudaError_t launch_ep_stats(const Shape& s, const int32_t* mat, const int32_t* expert_rank,
                            int world, int ranks_per_node, moe_ep_stats_t* out,
                            cudaStream_t st);

// Which kernel runs the expert FFN of the plain (permuted-copy) path, process-wide: a
// moe_ffn_kernel_t value (include/moe.h).
void set_ffn_kernel(int kind);
int ffn_kernel();

// Process-wide count of this library's kernel launches (every launch site calls it once).
void note_launch();

// Allocation-free dispatch: scratch lives in a fixed device array (moe_dispatch.cu).
constexpr size_t kStaticDispatchHistBytes = size_t(1) << 20;  // 1 MiB of block histograms
cudaError_t dispatch_static_scratch(const Shape& s, const void* x, const int32_t* topk_idx,
                                    int32_t* routed, int32_t* kept, int32_t* offsets,
                                    int32_t* assign_row, int32_t* token_of_row, void* x_perm,
                                    uint64_t wait_ns, cudaStream_t st);
// Synchronise `st`, copy the fixed scratch's status record to *out and clear it if it holds
// an error.  Allocates nothing.
cudaError_t static_scratch_status(DevStatus* out, cudaStream_t st);

}  // namespace moe
