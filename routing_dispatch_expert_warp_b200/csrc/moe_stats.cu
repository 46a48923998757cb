// Per-layer load statistics.
//
// "MoE expert parallelism needs measurements before launch" (airouter.kz), "Mean expert
// load proves almost nothing": with n_e the tokens assigned to expert e, mu = sum n_e / E;
// every layer reports tokens_per_expert, p50, p95, max, max/mean, the share of the top 5%
// of experts and dropped tokens.  "Capacity factor changes quality, memory and the latency
// tail": drop rate per layer and per route (first pick, second pick, ...).
//
// The drops per pick rank and per token are counted over assign_row -- above 32768 picks by
// a kernel spread over the GPU (one thread per token) into the output record, else by the
// record kernel itself -- and one block sorts the E kept counts in shared memory (bitonic
// network over the next power of two of E) and one thread evaluates the fp64 formulas.  The job record of data-parallel replicas runs the same kernel on the
// replicas' summed counts, taking the token count, capacity and drop counters from the
// replicas' own records instead of an assign_row.  Percentiles interpolate linearly between order statistics:
// h = (E - 1) p, v = s[floor h] + (h - floor h) (s[floor h + 1] - s[floor h]).
#include <limits.h>

#include "moe_internal.h"

namespace moe {
namespace {

__device__ double percentile_linear(const int32_t* s, int n, double p) {
  const double h = __dmul_rn(static_cast<double>(n - 1), p);
  const double fl = floor(h);
  const int lo = static_cast<int>(fl);
  const int hi = lo + 1 < n ? lo + 1 : n - 1;
  const double diff = __dadd_rn(static_cast<double>(s[hi]), -static_cast<double>(s[lo]));
  return __dadd_rn(static_cast<double>(s[lo]), __dmul_rn(__dadd_rn(h, -fl), diff));
}

constexpr int kStatsThreads = 1024;

__device__ __forceinline__ int warp_sum(int v) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

// Counters are reduced within each warp first and then added with 32-bit shared atomics
// (one per warp), so the block never serialises on a contended 64-bit atomic.
// The drop counters over assign_row, spread over the GPU: a thread per token, its k picks
// loaded at once; each block adds its counts to out (zeroed before the launch) with one
// 64-bit atomic per counter.  Integer sums, so the order of the additions does not matter.
constexpr int kDropThreads = 256;
// up to this many picks one block counts the drops faster than a memset, a spread kernel
// and the record kernel: 14 against 17 us at 8192 picks, 43 against 25 us at 131072
constexpr int64_t kStatsOneBlockPicks = 32768;
__global__ void __launch_bounds__(kDropThreads) drop_count_kernel(
    const int32_t* __restrict__ assign_row, int64_t T, int k,
    moe_load_stats_t* __restrict__ out) {
  __shared__ int s_rank[MOE_MAX_TOPK];
  __shared__ int s_td, s_tf;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  if (tid < MOE_MAX_TOPK) s_rank[tid] = 0;
  if (tid == 0) s_td = s_tf = 0;
  __syncthreads();
  int rank_local[MOE_MAX_TOPK];
#pragma unroll
  for (int j = 0; j < MOE_MAX_TOPK; ++j) rank_local[j] = 0;
  int td = 0, tf = 0;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * kDropThreads + tid; t < T;
       t += static_cast<int64_t>(gridDim.x) * kDropThreads) {
    int32_t a[MOE_MAX_TOPK];
#pragma unroll
    for (int j = 0; j < MOE_MAX_TOPK; ++j) a[j] = j < k ? __ldg(assign_row + t * k + j) : 0;
    int nd = 0;
#pragma unroll
    for (int j = 0; j < MOE_MAX_TOPK; ++j)
      if (j < k && a[j] < 0) {
        ++rank_local[j];
        ++nd;
      }
    td += nd > 0;
    tf += nd == k;
  }
#pragma unroll
  for (int j = 0; j < MOE_MAX_TOPK; ++j) {
    const int v = warp_sum(rank_local[j]);
    if (lane == 0 && v) atomicAdd(&s_rank[j], v);
  }
  td = warp_sum(td);
  tf = warp_sum(tf);
  if (lane == 0) {
    if (td) atomicAdd(&s_td, td);
    if (tf) atomicAdd(&s_tf, tf);
  }
  __syncthreads();
  if (tid < MOE_MAX_TOPK && tid < k && s_rank[tid])
    atomicAdd(reinterpret_cast<unsigned long long*>(&out->dropped_by_rank[tid]),
              static_cast<unsigned long long>(s_rank[tid]));
  if (tid == 0 && s_td)
    atomicAdd(reinterpret_cast<unsigned long long*>(&out->tokens_with_drop),
              static_cast<unsigned long long>(s_td));
  if (tid == 0 && s_tf)
    atomicAdd(reinterpret_cast<unsigned long long*>(&out->tokens_fully_dropped),
              static_cast<unsigned long long>(s_tf));
}

// counted: the drop counters are already in out (drop_count_kernel); assign_row unused.
__global__ void __launch_bounds__(kStatsThreads) stats_kernel(
    const int32_t* __restrict__ routed, const int32_t* __restrict__ kept,
    const int32_t* __restrict__ assign_row, int64_t T, int k, int E, int64_t C,
    const moe_load_stats_t* __restrict__ parts, int n_parts, bool counted,
    moe_load_stats_t* __restrict__ out) {
  __shared__ int32_t sorted[MOE_MAX_EXPERTS];
  __shared__ unsigned long long sum_kept, sum_routed;
  __shared__ int max_routed;
  __shared__ int drop_rank[MOE_MAX_TOPK];
  __shared__ int tok_drop, tok_full;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  if (tid < MOE_MAX_EXPERTS) sorted[tid] = tid < E ? kept[tid] : INT_MAX;
  if (tid == 0) {
    sum_kept = 0ull;
    sum_routed = 0ull;
    max_routed = 0;
    tok_drop = 0;
    tok_full = 0;
  }
  if (tid < MOE_MAX_TOPK) drop_rank[tid] = 0;
  __syncthreads();
  if (tid < MOE_MAX_EXPERTS) {  // warps 0..7 cover the experts
    const int kv = tid < E ? kept[tid] : 0;
    const int rv = tid < E ? routed[tid] : 0;
    int mx = rv;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    unsigned long long sk = static_cast<unsigned int>(kv), sr = static_cast<unsigned int>(rv);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
      sk += __shfl_xor_sync(0xffffffffu, sk, off);
      sr += __shfl_xor_sync(0xffffffffu, sr, off);
    }
    if (lane == 0) {
      atomicAdd(&sum_kept, sk);
      atomicAdd(&sum_routed, sr);
      atomicMax(&max_routed, mx);
    }
  }
  // bitonic sort, ascending, of the smallest power-of-two number of slots holding E (the
  // slots past E hold INT_MAX and stay at the end)
  int n2 = 2;
  while (n2 < E) n2 <<= 1;
  for (int size = 2; size <= n2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const int partner = tid ^ stride;
      if (tid < n2 && partner > tid) {
        const bool asc = (tid & size) == 0;
        const int32_t a = sorted[tid], b = sorted[partner];
        if ((a > b) == asc) {
          sorted[tid] = b;
          sorted[partner] = a;
        }
      }
      __syncthreads();
    }
  }
  // drops per pick rank and per token (thread per token, counters in registers); four
  // tokens' picks are loaded before any is counted, so each thread keeps 4 k loads in flight
  int rank_local[MOE_MAX_TOPK];
#pragma unroll
  for (int j = 0; j < MOE_MAX_TOPK; ++j) rank_local[j] = 0;
  int td = 0, tf = 0;
  constexpr int kTokUnroll = 4;
  const int64_t step = static_cast<int64_t>(blockDim.x);
  for (int64_t t0 = tid; assign_row != nullptr && t0 < T; t0 += step * kTokUnroll) {
    int32_t a[kTokUnroll][MOE_MAX_TOPK];
#pragma unroll
    for (int u = 0; u < kTokUnroll; ++u) {
      const int64_t t = t0 + u * step;
#pragma unroll
      for (int j = 0; j < MOE_MAX_TOPK; ++j)
        a[u][j] = (j < k && t < T) ? __ldg(assign_row + t * k + j) : 0;
    }
#pragma unroll
    for (int u = 0; u < kTokUnroll; ++u) {
      if (t0 + u * step >= T) break;
      int nd = 0;
#pragma unroll
      for (int j = 0; j < MOE_MAX_TOPK; ++j) {
        if (j < k && a[u][j] < 0) {
          ++rank_local[j];
          ++nd;
        }
      }
      td += nd > 0;
      tf += nd == k;
    }
  }
#pragma unroll
  for (int j = 0; j < MOE_MAX_TOPK; ++j) {
    const int v = warp_sum(rank_local[j]);
    if (lane == 0 && v) atomicAdd(&drop_rank[j], v);
  }
  td = warp_sum(td);
  tf = warp_sum(tf);
  if (lane == 0) {
    if (td) atomicAdd(&tok_drop, td);
    if (tf) atomicAdd(&tok_full, tf);
  }
  __syncthreads();

  if (tid == 0) {
    moe_load_stats_t st;
    int64_t drops[MOE_MAX_TOPK];
    int64_t with_drop = tok_drop, fully = tok_full;
    for (int j = 0; j < MOE_MAX_TOPK; ++j) drops[j] = j < k ? drop_rank[j] : 0;
    if (counted) {
      with_drop = out->tokens_with_drop;
      fully = out->tokens_fully_dropped;
      for (int j = 0; j < MOE_MAX_TOPK; ++j) drops[j] = j < k ? out->dropped_by_rank[j] : 0;
    }
    if (parts != nullptr) {  // job record: tokens, capacity and drop counters of the replicas
      T = 0;
      C = 0;
      with_drop = fully = 0;
      for (int j = 0; j < MOE_MAX_TOPK; ++j) drops[j] = 0;
      for (int p = 0; p < n_parts; ++p) {
        T += parts[p].active_tokens;
        C = (C < 0 || parts[p].capacity < 0) ? -1 : C + parts[p].capacity;
        with_drop += parts[p].tokens_with_drop;
        fully += parts[p].tokens_fully_dropped;
        for (int j = 0; j < k; ++j) drops[j] += parts[p].dropped_by_rank[j];
      }
    }
    st.E = E;
    st.k = k;
    st.active_tokens = T;
    st.capacity = C;
    st.routed_total = static_cast<int64_t>(sum_routed);
    st.kept_total = static_cast<int64_t>(sum_kept);
    st.dropped = T * k - static_cast<int64_t>(sum_kept);
    st.tokens_with_drop = with_drop;
    st.tokens_fully_dropped = fully;
    st.p50 = percentile_linear(sorted, E, 0.50);
    st.p95 = percentile_linear(sorted, E, 0.95);
    st.p99 = percentile_linear(sorted, E, 0.99);
    st.max = static_cast<double>(sorted[E - 1]);
    const double mean = static_cast<double>(sum_kept) / static_cast<double>(E);
    st.mean = mean;
    st.max_to_mean = mean > 0.0 ? st.max / mean : 0.0;
    st.routed_max = static_cast<double>(max_routed);
    const double rmean = static_cast<double>(sum_routed) / static_cast<double>(E);
    st.routed_max_to_mean = rmean > 0.0 ? st.routed_max / rmean : 0.0;
    const int n_top = (E + 19) / 20;  // ceil(0.05 E)
    long long top = 0;
    for (int i = 0; i < n_top; ++i) top += sorted[E - 1 - i];
    st.top5pct_share =
        sum_kept > 0 ? static_cast<double>(top) / static_cast<double>(sum_kept) : 0.0;
    for (int j = 0; j < MOE_MAX_TOPK; ++j) st.dropped_by_rank[j] = drops[j];
    *out = st;
  }
}

}  // namespace

cudaError_t launch_stats(const Shape& s, const int32_t* routed, const int32_t* kept,
                         const int32_t* assign_row, moe_load_stats_t* out, cudaStream_t st) {
  if (s.T * s.k <= kStatsOneBlockPicks) {  // few picks: one block scans them itself
    stats_kernel<<<1, kStatsThreads, 0, st>>>(routed, kept, assign_row, s.T, s.k, s.E, s.C,
                                              nullptr, 0, false, out);
    note_launch();
    return cudaGetLastError();
  }
  // the drop counters of assign_row over many blocks into out, then the one-block rest
  cudaError_t err = cudaMemsetAsync(out, 0, sizeof(moe_load_stats_t), st);
  if (err != cudaSuccess) return err;
  int64_t blocks = (s.T + kDropThreads - 1) / kDropThreads;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 4;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  drop_count_kernel<<<static_cast<unsigned>(blocks), kDropThreads, 0, st>>>(assign_row, s.T,
                                                                          s.k, out);
  note_launch();
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  stats_kernel<<<1, kStatsThreads, 0, st>>>(routed, kept, nullptr, s.T, s.k, s.E, s.C,
                                            nullptr, 0, true, out);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_stats_merge(const Shape& s, const int32_t* routed_sum,
                               const int32_t* kept_sum, const moe_load_stats_t* parts,
                               int n_parts, moe_load_stats_t* out, cudaStream_t st) {
  stats_kernel<<<1, kStatsThreads, 0, st>>>(routed_sum, kept_sum, nullptr, 0, s.k, s.E, 0,
                                            parts, n_parts, false, out);
  note_launch();
  return cudaGetLastError();
}

}  // namespace moe
