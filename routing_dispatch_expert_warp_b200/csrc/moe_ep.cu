// Expert parallelism across ranks (one GPU each) over peer memory.
//
// "Expert Parallelism for MoE Serving" (aiunderstanding.org), "Deep dive" / "Technical
// insight": experts live on different GPUs and every MoE layer runs two all-to-alls,
// dispatch (tokens to their experts' owners) and combine (results back).  "MoE expert
// parallelism needs measurements before launch" (airouter.kz): tokens past the capacity
// are dropped before the exchange; "Expert and GPU can be balanced differently" gives the
// per-layer rank / node / pair-traffic record computed by ep_stats_kernel.
//
// No collective library moves data here.  Every rank can address every rank's receive
// buffer, result buffer and count matrix (peer pointers through NVLink, or plain device
// pointers when all ranks share one GPU), and the exchange is folded into the kernels
// around it:
//   put_counts  each rank writes its kept counts [E] into row `rank` of every rank's count
//               matrix [world, E];
//   plan        from the full matrix: where this rank's rows land in each owner's buffer
//               (owner's experts ascending, then source ranks ascending, then the source's
//               slot order), the row of every kept pick there (send_row), and this rank's
//               own bucket offsets / counts for its local grouped GEMM;
//   dispatch    a warp per token reads the token's row of x once and stores it straight
//               into the owners' receive buffers (the dispatch all-to-all fused with the
//               permutation);
//   combine     out[t] = sum over kept picks, in pick order, of w[t, j] * the result row in
//               its owner's buffer (the combine all-to-all fused with the weighted sum).
// Ordering between ranks (counts written before plan, rows before the FFN, results before
// combine) is the caller's: a stream-ordered barrier on multi-GPU runs, stream order when
// the ranks share one GPU.  Stores and loads are plain 16-byte global accesses (no TMA, no
// copies shared across a cluster), so the same kernels run on peer and local memory.
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kPlanThreads = 256;  // >= MOE_MAX_EXPERTS

__global__ void ep_put_counts_kernel(const int32_t* __restrict__ kept, int E, int rank,
                                     int world, int32_t* const* __restrict__ mats) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < world * E; i += gridDim.x * blockDim.x) {
    const int g = i / E, e = i - g * E;
    mats[g][static_cast<int64_t>(rank) * E + e] = kept[e];
  }
}

// One block.  Thread e: column total and the rows of ranks before this one for expert e;
// then the bucket start of e in its owner's buffer (sum of the column totals of the
// owner's lower experts), base[e] = bucket start + rows of lower source ranks, and, for
// this rank's own experts, the local bucket table.
__global__ void __launch_bounds__(kPlanThreads) ep_plan_base_kernel(
    const int32_t* __restrict__ mat, const int32_t* __restrict__ expert_rank, int world, int E,
    int rank, int n_local, int64_t recv_rows, int32_t* __restrict__ base,
    int32_t* __restrict__ recv_offsets, int32_t* __restrict__ recv_counts, DevStatus* status) {
  __shared__ int32_t col_s[MOE_MAX_EXPERTS];
  __shared__ int32_t owner_s[MOE_MAX_EXPERTS];
  const int e = threadIdx.x;
  int col = 0, before = 0, owner = -1;
  if (e < E) {
    owner = expert_rank[e];
    if (owner < 0 || owner >= world) {
      record_error(status, DEV_BAD_EXPERT, 30, static_cast<unsigned long long>(e));
      owner = -1;
    }
    for (int s = 0; s < world; ++s) {
      const int c = mat[static_cast<int64_t>(s) * E + e];
      col += c;
      if (s < rank) before += c;
    }
    col_s[e] = col;
    owner_s[e] = owner;
  }
  __syncthreads();
  if (e < E && owner >= 0) {
    int start = 0, local = 0;
    for (int q = 0; q < e; ++q)
      if (owner_s[q] == owner) {
        start += col_s[q];
        ++local;
      }
    base[e] = start + before;
    if (owner == rank && local < n_local) {
      // the local GEMM never reaches past the buffer: a bucket is cut at recv_rows (the
      // rows past it were never stored; dispatch reports them)
      const int64_t room = recv_rows - start;
      recv_offsets[local] = start;
      recv_counts[local] = static_cast<int32_t>(room <= 0 ? 0 : (col < room ? col : room));
      if (start + col > recv_rows)
        record_error(status, DEV_RECV_OVERFLOW, 32, static_cast<unsigned long long>(e));
    }
  } else if (e < E) {
    base[e] = -1;
  }
  if (e == 0) {  // rows this rank receives (at most recv_rows)
    int64_t tot = 0;
    for (int q = 0; q < E; ++q)
      if (owner_s[q] == rank) tot += col_s[q];
    recv_offsets[n_local] = static_cast<int32_t>(tot < recv_rows ? tot : recv_rows);
  }
}

// send_row[t, j] = base[e] + (assign_row[t, j] - expert_offsets[e]), -1 for a dropped pick.
__global__ void ep_send_rows_kernel(const int32_t* __restrict__ topk_idx,
                                    const int32_t* __restrict__ assign_row,
                                    const int32_t* __restrict__ expert_offsets,
                                    const int32_t* __restrict__ base, int64_t n, int E,
                                    int32_t* __restrict__ send_row) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int32_t r = assign_row[i];
    const int32_t e = topk_idx[i];
    int32_t out = -1;
    if (r >= 0 && e >= 0 && e < E && base[e] >= 0) out = base[e] + (r - expert_offsets[e]);
    send_row[i] = out;
  }
}

// A warp per token: lane j < k holds pick j's destination; the row of x is read 16 bytes
// per lane, UNR vectors at a time, and stored to every kept pick's row in its owner's
// receive buffer.  A destination row at or past recv_rows is an overflow: recorded, skipped.
template <int UNR>
__global__ void __launch_bounds__(256) ep_dispatch_kernel(
    const uint4* __restrict__ x, int64_t T, int k, int64_t vec_per_row,
    const int32_t* __restrict__ topk_idx, const int32_t* __restrict__ send_row,
    const int32_t* __restrict__ expert_rank, int E, int world, uint4* const* __restrict__ recv,
    int64_t recv_rows, DevStatus* status) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t t = warp; t < T; t += nwarps) {
    uint4* dst = nullptr;  // lane j < k: row of pick j in its owner's buffer, or nullptr
    if (lane < k) {
      const int32_t r = send_row[t * k + lane];
      const int32_t e = topk_idx[t * k + lane];
      if (r >= 0) {
        const int32_t g = (e >= 0 && e < E) ? expert_rank[e] : -1;
        if (r >= recv_rows || g < 0 || g >= world) {
          record_error(status, DEV_RECV_OVERFLOW, 31, static_cast<unsigned long long>(t * k + lane));
        } else {
          dst = recv[g] + static_cast<int64_t>(r) * vec_per_row;
        }
      }
    }
    const uint4* src = x + t * vec_per_row;
    for (int64_t v0 = 0; v0 < vec_per_row; v0 += 32 * UNR) {
      uint4 buf[UNR];
#pragma unroll
      for (int u = 0; u < UNR; ++u) {
        const int64_t v = v0 + u * 32 + lane;
        if (v < vec_per_row) buf[u] = __ldg(src + v);
      }
      for (int j = 0; j < k; ++j) {
        uint4* d = reinterpret_cast<uint4*>(
            __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(dst), j));
        if (d == nullptr) continue;
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
          const int64_t v = v0 + u * 32 + lane;
          if (v < vec_per_row) d[v] = buf[u];
        }
      }
    }
  }
}

// combine over the owners' result buffers: a thread makes NV 16-byte vectors of one output
// row, from k x NV loads issued together, summed in pick order in fp32.
template <bool BF16, int NV>
__global__ void __launch_bounds__(256) ep_combine_kernel(
    const uint4* const* __restrict__ ybuf, const int32_t* __restrict__ topk_idx,
    const int32_t* __restrict__ send_row, const int32_t* __restrict__ expert_rank, int E,
    int world, int64_t recv_rows, const float* __restrict__ topk_w, int64_t T, int k,
    int64_t vec_per_row, uint4* __restrict__ out) {
  constexpr int NE = BF16 ? 8 : 4;
  const int64_t groups_per_row = vec_per_row / NV;
  const int64_t total = T * groups_per_row;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / groups_per_row;
    const int64_t v0 = (i - t * groups_per_row) * NV;
    float acc[NV][NE];
#pragma unroll
    for (int u = 0; u < NV; ++u)
#pragma unroll
      for (int q = 0; q < NE; ++q) acc[u][q] = 0.f;
    for (int j = 0; j < k; ++j) {
      const int32_t r = __ldg(send_row + t * k + j);
      if (r < 0 || r >= recv_rows) continue;
      const int32_t e = __ldg(topk_idx + t * k + j);
      if (e < 0 || e >= E) continue;
      const int32_t g = __ldg(expert_rank + e);
      if (g < 0 || g >= world) continue;
      const float w = __ldg(topk_w + t * k + j);
      const uint4* row = ybuf[g] + static_cast<int64_t>(r) * vec_per_row + v0;
      uint4 src[NV];
#pragma unroll
      for (int u = 0; u < NV; ++u) src[u] = row[u];
#pragma unroll
      for (int u = 0; u < NV; ++u) {
        const uint32_t uu[4] = {src[u].x, src[u].y, src[u].z, src[u].w};
        if (BF16) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            acc[u][2 * q] = fmaf(w, bf16_lo(uu[q]), acc[u][2 * q]);
            acc[u][2 * q + 1] = fmaf(w, bf16_hi(uu[q]), acc[u][2 * q + 1]);
          }
        } else {
#pragma unroll
          for (int q = 0; q < 4; ++q) acc[u][q] = fmaf(w, __uint_as_float(uu[q]), acc[u][q]);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < NV; ++u) {
      uint4 o;
      if (BF16) {
        o = make_uint4(pack_bf16x2(acc[u][0], acc[u][1]), pack_bf16x2(acc[u][2], acc[u][3]),
                       pack_bf16x2(acc[u][4], acc[u][5]), pack_bf16x2(acc[u][6], acc[u][7]));
      } else {
        o = make_uint4(__float_as_uint(acc[u][0]), __float_as_uint(acc[u][1]),
                       __float_as_uint(acc[u][2]), __float_as_uint(acc[u][3]));
      }
      out[t * vec_per_row + v0 + u] = o;
    }
  }
}

// ------------------------------------------------------------------ EP record
constexpr int kStatThreads = 1024;
constexpr int kPairSort = 4096;  // >= kMaxDevices * (kMaxDevices - 1) ordered pairs

// Type-7 percentile of the pair sizes in bytes (sorted holds rows; bytes = rows x row_bytes,
// exact in double below 2^53).
__device__ double pct_linear(const uint32_t* sorted, int n, double p, int64_t row_bytes) {
  const double h = __dmul_rn(static_cast<double>(n - 1), p);
  const int lo = static_cast<int>(floor(h));
  const int hi = lo + 1 < n ? lo + 1 : n - 1;
  const double a = static_cast<double>(static_cast<int64_t>(sorted[lo]) * row_bytes);
  const double b = static_cast<double>(static_cast<int64_t>(sorted[hi]) * row_bytes);
  return __dadd_rn(a, __dmul_rn(__dadd_rn(h, -static_cast<double>(lo)), __dadd_rn(b, -a)));
}

// One block: pair rows [source][owner] from the count matrix, then loads, bytes and the
// pair-size percentiles (all ordered pairs s != g, empty ones included; bitonic sort).
__global__ void __launch_bounds__(kStatThreads) ep_stats_kernel(
    const int32_t* __restrict__ mat, const int32_t* __restrict__ expert_rank, int world, int E,
    int ranks_per_node, int64_t row_bytes, moe_ep_stats_t* __restrict__ out) {
  __shared__ uint32_t pair_s[kMaxDevices * kMaxDevices];  // rows, [s][g]
  __shared__ uint32_t sorted_s[kPairSort];                 // off-diagonal pair rows
  const int tid = threadIdx.x;
  const int G = world;
  for (int i = tid; i < G * G; i += blockDim.x) pair_s[i] = 0;
  __syncthreads();
  for (int i = tid; i < G * E; i += blockDim.x) {
    const int s = i / E, e = i - s * E;
    const int g = expert_rank[e];
    if (g >= 0 && g < G) atomicAdd(&pair_s[s * G + g], static_cast<uint32_t>(mat[i]));
  }
  __syncthreads();
  const int n_pairs = G * (G - 1);
  for (int i = tid; i < kPairSort; i += blockDim.x) {
    uint32_t v = 0xffffffffu;  // padding sorts last
    if (i < n_pairs) {
      const int s = i / (G - 1);
      int g = i - s * (G - 1);
      if (g >= s) ++g;
      v = pair_s[s * G + g];
    }
    sorted_s[i] = v;
  }
  __syncthreads();
  int n2 = 2;  // sort the smallest power of two that holds the pairs (padding sorts last)
  while (n2 < n_pairs) n2 <<= 1;
  for (int size = 2; size <= n2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < n2; i += blockDim.x) {
        const int j = i ^ stride;
        if (j > i) {
          const bool up = (i & size) == 0;
          const uint32_t a = sorted_s[i], b = sorted_s[j];
          if ((a > b) == up) {
            sorted_s[i] = b;
            sorted_s[j] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  const int nodes = (G + ranks_per_node - 1) / ranks_per_node;
  // per-rank and per-node columns, one thread each
  if (tid < kMaxDevices) {
    long long load = 0, sent = 0, recvd = 0, nload = 0;
    if (tid < G) {
      for (int s = 0; s < G; ++s) {
        load += pair_s[s * G + tid];
        if (s != tid) {
          sent += static_cast<long long>(pair_s[tid * G + s]) * row_bytes;
          recvd += static_cast<long long>(pair_s[s * G + tid]) * row_bytes;
        }
      }
    }
    if (tid < nodes)
      for (int g = tid * ranks_per_node; g < G && g < (tid + 1) * ranks_per_node; ++g)
        for (int s = 0; s < G; ++s) nload += pair_s[s * G + g];
    out->rank_load[tid] = load;
    out->bytes_sent[tid] = sent;
    out->bytes_recv[tid] = recvd;
    out->node_load[tid] = nload;
  }
  if (tid == 0) {
    long long total = 0, local = 0, remote = 0, cross = 0, rmax = 0, nmax = 0;
    for (int s = 0; s < G; ++s)
      for (int g = 0; g < G; ++g) {
        const long long rows = pair_s[s * G + g];
        total += rows;
        if (s == g) {
          local += rows;
        } else {
          remote += rows * row_bytes;
          if (s / ranks_per_node != g / ranks_per_node) cross += rows * row_bytes;
        }
      }
    for (int g = 0; g < G; ++g) {
      long long l = 0;
      for (int s = 0; s < G; ++s) l += pair_s[s * G + g];
      rmax = l > rmax ? l : rmax;
    }
    for (int n = 0; n < nodes; ++n) {
      long long l = 0;
      for (int g = n * ranks_per_node; g < G && g < (n + 1) * ranks_per_node; ++g)
        for (int s = 0; s < G; ++s) l += pair_s[s * G + g];
      nmax = l > nmax ? l : nmax;
    }
    out->world = G;
    out->ranks_per_node = ranks_per_node;
    out->nodes = nodes;
    out->reserved = 0;
    out->total_assignments = total;
    out->local_assignments = local;
    out->remote_bytes = remote;
    out->cross_node_bytes = cross;
    out->local_fraction =
        total > 0 ? static_cast<double>(local) / static_cast<double>(total) : 0.0;
    out->cross_node_fraction =
        remote > 0 ? static_cast<double>(cross) / static_cast<double>(remote) : 0.0;
    out->pair_bytes_p50 = n_pairs > 0 ? pct_linear(sorted_s, n_pairs, 0.50, row_bytes) : 0.0;
    out->pair_bytes_p99 = n_pairs > 0 ? pct_linear(sorted_s, n_pairs, 0.99, row_bytes) : 0.0;
    out->pair_bytes_max =
        n_pairs > 0 ? static_cast<double>(static_cast<int64_t>(sorted_s[n_pairs - 1]) * row_bytes)
                    : 0.0;
    const double mean = static_cast<double>(total) / G;
    const double nmean = static_cast<double>(total) / nodes;
    out->rank_load_max = static_cast<double>(rmax);
    out->rank_load_mean = mean;
    out->rank_load_max_minus_mean = static_cast<double>(rmax) - mean;
    out->rank_load_max_to_mean = mean > 0 ? static_cast<double>(rmax) / mean : 0.0;
    out->node_load_max_to_mean = nmean > 0 ? static_cast<double>(nmax) / nmean : 0.0;
  }
}

template <bool BF16>
cudaError_t launch_ep_combine_typed(const Shape& s, const void* const* ybuf,
                                    const int32_t* topk_idx, const int32_t* send_row,
                                    const int32_t* expert_rank, int world, int64_t recv_rows,
                                    const float* topk_w, void* out, cudaStream_t st) {
  const int64_t vec_per_row = s.d * s.elem / 16;
  const bool wide = vec_per_row % 4 == 0;
  const int64_t total = s.T * (wide ? vec_per_row / 4 : vec_per_row);
  int64_t blocks = (total + 255) / 256;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  const uint4* const* y = reinterpret_cast<const uint4* const*>(ybuf);
  uint4* o = static_cast<uint4*>(out);
  if (wide)
    ep_combine_kernel<BF16, 4><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        y, topk_idx, send_row, expert_rank, s.E, world, recv_rows, topk_w, s.T, s.k, vec_per_row,
        o);
  else
    ep_combine_kernel<BF16, 1><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        y, topk_idx, send_row, expert_rank, s.E, world, recv_rows, topk_w, s.T, s.k, vec_per_row,
        o);
  note_launch();
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_ep_put_counts(const Shape& s, const int32_t* kept, int rank, int world,
                                 int32_t* const* mats, cudaStream_t st) {
  const int n = world * s.E;
  const int blocks = (n + 255) / 256;
  ep_put_counts_kernel<<<blocks, 256, 0, st>>>(kept, s.E, rank, world, mats);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_ep_plan(const Shape& s, const int32_t* mat, const int32_t* expert_rank,
                           int world, int rank, int n_local, int64_t recv_rows,
                           const int32_t* topk_idx,
                           const int32_t* assign_row, const int32_t* expert_offsets,
                           int32_t* base, int32_t* send_row, int32_t* recv_offsets,
                           int32_t* recv_counts, DevStatus* status, cudaStream_t st) {
  ep_plan_base_kernel<<<1, kPlanThreads, 0, st>>>(mat, expert_rank, world, s.E, rank, n_local,
                                                  recv_rows, base, recv_offsets, recv_counts,
                                                  status);
  note_launch();
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const int64_t n = s.T * s.k;
  int64_t blocks = (n + 255) / 256;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 4;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  ep_send_rows_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(
      topk_idx, assign_row, expert_offsets, base, n, s.E, send_row);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_ep_dispatch(const Shape& s, const void* x, const int32_t* topk_idx,
                               const int32_t* send_row, const int32_t* expert_rank, int world,
                               void* const* recv, int64_t recv_rows, DevStatus* status,
                               cudaStream_t st) {
  const int64_t vec_per_row = s.d * s.elem / 16;
  int64_t blocks = (s.T + 7) / 8;  // 8 warps (tokens) per block
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  ep_dispatch_kernel<4><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
      static_cast<const uint4*>(x), s.T, s.k, vec_per_row, topk_idx, send_row, expert_rank,
      s.E, world, reinterpret_cast<uint4* const*>(recv), recv_rows, status);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_ep_combine(const Shape& s, const void* const* ybuf, const int32_t* topk_idx,
                              const int32_t* send_row, const int32_t* expert_rank, int world,
                              int64_t recv_rows, const float* topk_w, void* out,
                              cudaStream_t st) {
  if (s.dtype == MOE_BF16)
    return launch_ep_combine_typed<true>(s, ybuf, topk_idx, send_row, expert_rank, world,
                                         recv_rows, topk_w, out, st);
  return launch_ep_combine_typed<false>(s, ybuf, topk_idx, send_row, expert_rank, world,
                                        recv_rows, topk_w, out, st);
}

cudaError_t launch_ep_stats(const Shape& s, const int32_t* mat, const int32_t* expert_rank,
                            int world, int ranks_per_node, moe_ep_stats_t* out,
                            cudaStream_t st) {
  ep_stats_kernel<<<1, kStatThreads, 0, st>>>(mat, expert_rank, world, s.E, ranks_per_node,
                                              s.d * s.elem, out);
  note_launch();
  return cudaGetLastError();
}

}  // namespace moe
