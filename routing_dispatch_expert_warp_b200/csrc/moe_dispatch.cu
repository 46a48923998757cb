// Dispatch on one GPU: per-expert histogram, prefix scan with the capacity limit, stable
// ranking of every (token, pick) assignment inside its expert, and the row permutation of
// x into expert-major buckets.
//
// "Expert Parallelism for MoE Serving" (aiunderstanding.org), "Technical insight": the
// dispatch all-to-all sends every token to its experts; capacity factors and expert
// buffers bound the rows per expert, and tokens past the capacity are dropped or the
// bucket is padded.  "MoE expert parallelism needs measurements before launch"
// (airouter.kz), "Profile all-to-all separately from compute": pack/permute comes before
// the exchange, and with EP=1 the exchange itself disappears -- what remains is this
// local permutation.
//
// Assignment order: within expert e, assignments are ranked by token index (a token picks
// an expert at most once, so its pick slot j does not matter).  slot < C is kept.  With
// pick-rank drops the ranking goes pick rank by pick rank.  With score drops ("MoE expert
// parallelism needs measurements before launch", "Top-2 does not insure against hot
// experts": the second route has its own capacity and drops) an overflowing expert keeps
// its C picks of highest selection score (equal scores: lower token), found by a radix
// selection over each expert's picks; the kept picks are then ranked by token index.
//
// Kernels (no host synchronisation anywhere):
//   1. count:  block b of 256 tokens builds, per warp w and expert e, the 32-bit mask of
//              lanes (tokens) that picked e; per-block counts = sum of popcounts.
//   2. rank:   block b rebuilds its masks and, from all blocks' counts, its base slot per
//              expert, routed = total, kept = min(routed, C) and the bucket offsets; then
//              slot = block base + earlier warps' counts + popcount(mask & lanes below me).
//              Writes assign_row and token_of_row (-1 for rows no assignment uses).
//   3. permute: token-major row copy with bulk (TMA) copies: each row of x is read from HBM
//              once into shared memory and written to each of its kept rows of x_perm.
#include <mutex>

#include "moe_internal.h"
#include "moe_keys.cuh"

namespace moe {
namespace {

constexpr int kWarps = kDispatchBlockTokens / 32;

// Which picks the ranking kernels count.  thr == nullptr: all of them.  Otherwise pick
// (t, e) counts (is kept) iff pick_priority(score of (t, e), t) >= thr[e], the score being
// the fp32 logit plus, when the bias only steers selection, the fp32 bias: the same single
// addition the top-k takes its decision on.
struct ScoreFilter {
  const uint64_t* thr;
  const float* logits;
  const float* bias;
  int64_t bias_stride;
};

__device__ __forceinline__ float selection_score(const ScoreFilter& f, int64_t t, int E, int e) {
  float v = f.logits[t * E + e];
  if (f.bias != nullptr) v = v + f.bias[t * f.bias_stride + e];
  return v;
}

__device__ __forceinline__ bool filter_keeps(const ScoreFilter& f, int64_t t, int E, int e) {
  return f.thr == nullptr || pick_priority(selection_score(f, t, E, e), t) >= f.thr[e];
}

// Fill masks[w][e] for the block's tokens, counting the picks of `plane` only when the
// assignments are ranked pick rank by pick rank (planes == k), all picks otherwise
// (planes == 1), and only the picks the filter keeps.  Invalid experts are recorded and
// skipped.
__device__ __forceinline__ void build_masks(const int32_t* __restrict__ topk_idx, int64_t T,
                                            int k, int E, uint32_t (*masks)[MOE_MAX_EXPERTS],
                                            DevStatus* status, int plane, int planes,
                                            const ScoreFilter& flt) {
  for (int i = threadIdx.x; i < kWarps * MOE_MAX_EXPERTS; i += blockDim.x)
    (&masks[0][0])[i] = 0u;
  __syncthreads();
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kDispatchBlockTokens + threadIdx.x;
  const int w = threadIdx.x >> 5;
  const uint32_t bit = 1u << (threadIdx.x & 31);
  if (t < T) {
    int ev[MOE_MAX_TOPK];  // the token's picks, all loads in flight before any is used
#pragma unroll
    for (int j = 0; j < MOE_MAX_TOPK; ++j) ev[j] = j < k ? __ldg(topk_idx + t * k + j) : 0;
#pragma unroll
    for (int j = 0; j < MOE_MAX_TOPK; ++j) {
      if (j >= k) break;
      if (planes > 1 && j != plane) continue;
      const int e = ev[j];
      if (e < 0 || e >= E) {
        record_error(status, DEV_BAD_EXPERT, 1, static_cast<unsigned long long>(t * k + j));
        continue;
      }
      if (!filter_keeps(flt, t, E, e)) continue;
      atomicOr(&masks[w][e], bit);
    }
  }
  __syncthreads();
}

// hist[b][p][e]: assignments of plane p (a pick rank, or all picks) from block b to expert e.
__global__ void __launch_bounds__(kDispatchBlockTokens) dispatch_count_kernel(
    const int32_t* __restrict__ topk_idx, int64_t T, int k, int E, int planes,
    int32_t* __restrict__ hist, DevStatus* status, ScoreFilter flt) {
  __shared__ uint32_t masks[kWarps][MOE_MAX_EXPERTS];
  for (int p = 0; p < planes; ++p) {
    build_masks(topk_idx, T, k, E, masks, p == 0 ? status : nullptr, p, planes, flt);
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
      int c = 0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) c += __popc(masks[w][e]);
      hist[(static_cast<int64_t>(blockIdx.x) * planes + p) * E + e] = c;
    }
    __syncthreads();  // masks are rebuilt for the next plane
  }
}

// Ranking.  Every block first derives what it needs from the per-block counts of all
// blocks: thread e adds up expert e's counts per plane over the blocks (plane totals, and
// the part that comes from blocks before this one), caps the routed total at C (kept), and
// the block scans kept over the experts (bucket offsets).  Block 0 publishes routed / kept /
// offsets; the others only use them.  A plane is all picks (token-order drops) or one pick
// rank (pick-rank drops: plane p starts after the totals of planes < p).  Then, plane by
// plane, slot = plane start + base from earlier blocks + earlier warps of this block +
// popcount(mask & lanes below me), kept iff slot < C, row = offset + slot.  Finally the
// rows no assignment uses are marked -1 in token_of_row.  With a filter, hist counts the
// kept picks only, the others get row -1, and routed (the demand, counted by an earlier
// unfiltered pass) is left as it is.
__global__ void __launch_bounds__(kDispatchBlockTokens) dispatch_rank_kernel(
    const int32_t* __restrict__ topk_idx, int64_t T, int k, int E, int64_t C, int layout,
    int planes, int64_t nblk, const int32_t* __restrict__ hist, int32_t* __restrict__ routed,
    int32_t* __restrict__ kept, int32_t* __restrict__ offsets, int32_t* __restrict__ assign_row,
    int32_t* __restrict__ token_of_row, int64_t max_rows, ScoreFilter flt) {
  static_assert(kDispatchBlockTokens == MOE_MAX_EXPERTS, "one thread per expert");
  __shared__ uint32_t masks[kWarps][MOE_MAX_EXPERTS];
  __shared__ int32_t wbase[kWarps][MOE_MAX_EXPERTS];
  __shared__ int32_t pbase[MOE_MAX_TOPK][MOE_MAX_EXPERTS];  // plane start + earlier blocks
  __shared__ int32_t off_s[MOE_MAX_EXPERTS];
  __shared__ int32_t kept_s[MOE_MAX_EXPERTS];
  __shared__ int64_t scan[MOE_MAX_EXPERTS];

  const int e = threadIdx.x;
  int64_t run = 0;  // routed total over all planes
  if (e < E) {
    for (int p = 0; p < planes; ++p) {
      int64_t tot = 0, before = 0;
      for (int64_t b = 0; b < nblk; b += 32) {  // loads issued 32 at a time, sums in block order
        int32_t c[32];
#pragma unroll
        for (int u = 0; u < 32; ++u)
          c[u] = b + u < nblk ? __ldg(hist + ((b + u) * planes + p) * E + e) : 0;
#pragma unroll
        for (int u = 0; u < 32; ++u) {
          if (b + u == blockIdx.x) before = tot;
          tot += c[u];
        }
      }
      pbase[p][e] = static_cast<int32_t>(run + before);
      run += tot;
    }
  }
  const int64_t kp = (e < E) ? ((C >= 0 && run > C) ? C : run) : 0;
  scan[e] = kp;
  __syncthreads();
  for (int off = 1; off < MOE_MAX_EXPERTS; off <<= 1) {  // inclusive scan over experts
    const int64_t add = e >= off ? scan[e - off] : 0;
    __syncthreads();
    scan[e] += add;
    __syncthreads();
  }
  const int64_t total_kept = scan[MOE_MAX_EXPERTS - 1];
  if (e < E) {
    const int64_t off =
        layout == MOE_LAYOUT_PADDED ? static_cast<int64_t>(e) * C : scan[e] - kp;
    off_s[e] = static_cast<int32_t>(off);
    kept_s[e] = static_cast<int32_t>(kp);
    if (blockIdx.x == 0) {
      if (flt.thr == nullptr) routed[e] = static_cast<int32_t>(run);
      kept[e] = static_cast<int32_t>(kp);
      offsets[e] = static_cast<int32_t>(off);
      if (e == E - 1)
        offsets[E] = static_cast<int32_t>(layout == MOE_LAYOUT_PADDED
                                              ? static_cast<int64_t>(E) * C
                                              : total_kept);
    }
  }

  const int64_t t = static_cast<int64_t>(blockIdx.x) * kDispatchBlockTokens + threadIdx.x;
  const int w = threadIdx.x >> 5;
  const uint32_t below = (1u << (threadIdx.x & 31)) - 1u;
  for (int p = 0; p < planes; ++p) {
    __syncthreads();  // pbase / off_s ready; masks of the previous plane no longer read
    build_masks(topk_idx, T, k, E, masks, nullptr, p, planes, flt);
    if (e < E) {
      int32_t wb = pbase[p][e];
#pragma unroll
      for (int ww = 0; ww < kWarps; ++ww) {
        wbase[ww][e] = wb;
        wb += __popc(masks[ww][e]);
      }
    }
    __syncthreads();
    if (t < T) {
      int ev[MOE_MAX_TOPK];
#pragma unroll
      for (int j = 0; j < MOE_MAX_TOPK; ++j) ev[j] = j < k ? __ldg(topk_idx + t * k + j) : 0;
#pragma unroll
      for (int j = 0; j < MOE_MAX_TOPK; ++j) {
        if (j >= k) break;
        if (planes > 1 && j != p) continue;
        const int ee = ev[j];
        int32_t row = -1;
        if (ee >= 0 && ee < E && filter_keeps(flt, t, E, ee)) {
          const int64_t slot = wbase[w][ee] + __popc(masks[w][ee] & below);
          if (C < 0 || slot < C) {
            row = off_s[ee] + static_cast<int32_t>(slot);
            token_of_row[row] = static_cast<int32_t>(t);
          }
        }
        assign_row[t * k + j] = row;
      }
    }
  }

  // unused rows: COMPACT [total_kept, max_rows); PADDED the slots past kept in each bucket
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t first = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (layout == MOE_LAYOUT_PADDED) {
    for (int64_t r = first; r < max_rows; r += stride) {
      const int64_t eb = r / C;
      if (eb < E && r - eb * C >= kept_s[eb]) token_of_row[r] = -1;
    }
  } else {
    for (int64_t r = total_kept + first; r < max_rows; r += stride) token_of_row[r] = -1;
  }
}

// Score-priority threshold of expert e (block e).  Its picks sit in rows
// [offsets[e], offsets[e] + routed[e]) of the dropless token-order layout, token_of_row
// giving each row's token.  When routed[e] > C the block writes every pick's priority to
// its own rows of prio, then finds the C-th largest by most-significant-digit radix
// selection, 8 bits a pass: a pass counts the candidates (priorities whose higher digits
// equal the prefix found so far) per digit value, and the digit at which the running count
// from the top reaches the rank still needed joins the prefix.  Priorities are unique per
// expert, so after 8 passes the prefix is the C-th largest and the kept picks are exactly
// those at or above it.  thr[e] = 0 keeps every pick (no overflow); C == 0 keeps none.
constexpr int kSelectThreads = 512;

__global__ void __launch_bounds__(kSelectThreads) score_select_kernel(
    const int32_t* __restrict__ routed, const int32_t* __restrict__ offsets,
    const int32_t* __restrict__ token_of_row, ScoreFilter flt, int E, int64_t C,
    uint64_t* __restrict__ prio, uint64_t* __restrict__ thr) {
  __shared__ uint32_t hist[256];
  __shared__ uint64_t s_prefix;
  __shared__ uint32_t s_need;
  const int e = blockIdx.x;
  const int64_t n = routed[e];
  if (C < 0 || n <= C) {
    if (threadIdx.x == 0) thr[e] = 0;
    return;
  }
  if (C == 0) {
    if (threadIdx.x == 0) thr[e] = ~0ull;
    return;
  }
  const int64_t start = offsets[e];
  uint64_t* seg = prio + start;
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) {
    const int64_t t = token_of_row[start + i];
    seg[i] = pick_priority(selection_score(flt, t, E, e), t);
  }
  const int lane = threadIdx.x & 31;
  uint64_t prefix = 0, mask = 0;
  uint32_t need = static_cast<uint32_t>(C);  // 1-based rank among the candidates
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0u;
    __syncthreads();  // seg written (first pass); s_prefix read by all (later passes)
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x) {
      const uint64_t v = seg[i];
      if ((v & mask) == prefix) atomicAdd(&hist[(v >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      // lane l holds digit values 255 - 8l down to 248 - 8l; counts run from the top
      uint32_t c[8], sum = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        c[i] = hist[255 - 8 * lane - i];
        sum += c[i];
      }
      uint32_t incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
      }
      uint32_t acc = incl - sum;
      if (acc < need && incl >= need) {  // exactly one lane
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (acc < need && acc + c[i] >= need) {
            s_prefix = prefix | (static_cast<uint64_t>(255 - 8 * lane - i) << shift);
            s_need = need - acc;
          }
          acc += c[i];
        }
      }
    }
    __syncthreads();
    prefix = s_prefix;
    need = s_need;
    mask |= 0xFFull << shift;
  }
  if (threadIdx.x == 0) thr[e] = prefix;
}

// Second-choice counters ("MoE expert parallelism needs measurements before launch", "Top-2
// does not insure against hot experts").  Block j takes pick rank j over all tokens:
// shared counts per expert of the picks and of the kept picks, and of the tokens whose
// pick j lies in another group than their pick 0; then it writes its row of each output.
// Integer sums: the result does not depend on the order of the additions.
constexpr int kCountThreads = 1024;

__global__ void __launch_bounds__(kCountThreads) pick_rank_counts_kernel(
    const int32_t* __restrict__ topk_idx, const int32_t* __restrict__ assign_row,
    const int32_t* __restrict__ group_of_expert, int64_t T, int k, int E,
    int32_t* __restrict__ routed, int32_t* __restrict__ kept, int32_t* __restrict__ differs,
    DevStatus* status) {
  __shared__ uint32_t r_s[MOE_MAX_EXPERTS];
  __shared__ uint32_t k_s[MOE_MAX_EXPERTS];
  __shared__ uint32_t d_s;
  const int j = blockIdx.x;
  for (int e = threadIdx.x; e < MOE_MAX_EXPERTS; e += blockDim.x) {
    r_s[e] = 0u;
    k_s[e] = 0u;
  }
  if (threadIdx.x == 0) d_s = 0u;
  __syncthreads();
  uint32_t dif = 0;
  for (int64_t t = threadIdx.x; t < T; t += blockDim.x) {
    const int e = topk_idx[t * k + j];
    const int e0 = topk_idx[t * k];
    if (e < 0 || e >= E || e0 < 0 || e0 >= E) {
      record_error(status, DEV_BAD_EXPERT, 4, static_cast<unsigned long long>(t * k + j));
      continue;
    }
    atomicAdd(&r_s[e], 1u);
    if (assign_row[t * k + j] >= 0) atomicAdd(&k_s[e], 1u);
    const bool other = group_of_expert != nullptr ? group_of_expert[e] != group_of_expert[e0]
                                                  : e != e0;
    dif += other ? 1u : 0u;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) dif += __shfl_xor_sync(0xffffffffu, dif, o);
  if ((threadIdx.x & 31) == 0 && dif != 0u) atomicAdd(&d_s, dif);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    routed[static_cast<int64_t>(j) * E + e] = static_cast<int32_t>(r_s[e]);
    kept[static_cast<int64_t>(j) * E + e] = static_cast<int32_t>(k_s[e]);
  }
  if (threadIdx.x == 0) differs[j] = static_cast<int32_t>(d_s);
}

// Token-major bulk copy.  One lane per block issues every copy: a ring of NBUF shared
// buffers, LOOKAHEAD loads in flight, stores of the rows already loaded in flight behind
// them.  A work item is one segment (<= 16 KB) of one token's row.  The whole warp fetches
// the rows each item goes to, 32 items (a chunk) per lane-parallel load: while lane 0 copies
// chunk c, the loads for chunk c + 2 are in flight in registers and chunk c + 1 (which the
// lookahead reaches) already sits in shared memory, so the issuing lane never waits on a
// global load after the first chunk.
constexpr uint32_t kPermMaxSeg = 16384;
constexpr int kPermMaxNBuf = 16;

template <int kPermNBuf, int kPermLookahead>
__global__ void __launch_bounds__(32) permute_rows_kernel(
    const uint8_t* __restrict__ x, const int32_t* __restrict__ assign_row, int64_t T, int k,
    int64_t row_bytes, uint32_t seg_bytes, int64_t segs_per_row, uint8_t* __restrict__ x_perm,
    DevStatus* status, uint64_t wait_ns) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t full[kPermNBuf];
  __shared__ int32_t meta_rows[3][32][MOE_MAX_TOPK];  // rows of the items of three chunks
  __shared__ uint32_t meta_any[3];                    // bit l: item l has a kept row
  static_assert(kPermNBuf <= kPermMaxNBuf && kPermLookahead < kPermNBuf &&
                    kPermLookahead <= 32,
                "ring shape; the lookahead stays inside the next chunk");
  const int lane = threadIdx.x;
  if (lane == 0) {
    for (int b = 0; b < kPermNBuf; ++b) mbar_init(&full[b], 1);
    fence_barrier_init();
  }

  const int64_t items = T * segs_per_row;
  const int64_t first = blockIdx.x, step = gridDim.x;
  const int64_t n = first < items ? (items - first + step - 1) / step : 0;
  uint32_t phase_bits = 0;  // parity of the next completion per buffer
  uint32_t armed = 0;       // buffers with a load in flight

  int32_t mr[MOE_MAX_TOPK];  // this lane's item of the chunk in flight
  auto fetch = [&](int64_t c) {  // issue the loads of chunk c's rows (item c * 32 + lane)
    const int64_t i = c * 32 + lane;
    const int64_t t = i < n ? (first + i * step) / segs_per_row : -1;
#pragma unroll
    for (int j = 0; j < MOE_MAX_TOPK; ++j)
      mr[j] = (t >= 0 && j < k) ? __ldg(assign_row + t * k + j) : -1;
  };
  auto publish = [&](int64_t c) {  // the fetched rows into buffer c % 3 (whole warp)
    bool any = false;
#pragma unroll
    for (int j = 0; j < MOE_MAX_TOPK; ++j) {
      meta_rows[c % 3][lane][j] = mr[j];
      any = any || mr[j] >= 0;
    }
    const uint32_t bits = __ballot_sync(0xffffffffu, any);
    if (lane == 0) meta_any[c % 3] = bits;
  };
  auto has_rows = [&](int64_t i) { return ((meta_any[(i >> 5) % 3] >> (i & 31)) & 1u) != 0u; };
  auto seg_of = [&](int64_t i, int64_t& t, int64_t& off) {
    const int64_t it = first + i * step;
    t = it / segs_per_row;
    off = (it - t * segs_per_row) * seg_bytes;
    return static_cast<uint32_t>(row_bytes - off < static_cast<int64_t>(seg_bytes)
                                     ? row_bytes - off
                                     : seg_bytes);
  };
  auto issue_load = [&](int64_t i) {
    int64_t t, off;
    const uint32_t bytes = seg_of(i, t, off);
    const int b = static_cast<int>(i % kPermNBuf);
    armed |= 1u << b;
    mbar_arrive_expect_tx(&full[b], bytes);
    bulk_load(smem + static_cast<size_t>(b) * seg_bytes, x + t * row_bytes + off, bytes,
              &full[b]);
  };

  fetch(0);
  publish(0);
  if (n > 32) fetch(1);
  __syncwarp();
  // Tokens whose picks were all dropped are skipped: their buffer is never filled and
  // their barrier never armed, so skipping must be decided identically at issue and use.
  if (lane == 0)
    for (int64_t i = 0; i < n && i < kPermLookahead; ++i)
      if (has_rows(i)) issue_load(i);

  for (int64_t c = 0; c * 32 < n; ++c) {
    // chunk c + 1 into the buffer chunk c - 2 used (the lookahead reads it from here on),
    // then the loads of chunk c + 2 go out and land while lane 0 copies chunk c
    if ((c + 1) * 32 < n) publish(c + 1);
    if ((c + 2) * 32 < n) fetch(c + 2);
    __syncwarp();
    int failed = 0;
    if (lane == 0) {
      const int64_t end = (c + 1) * 32 < n ? (c + 1) * 32 : n;
      for (int64_t i = c * 32; i < end; ++i) {
        const int b = static_cast<int>(i % kPermNBuf);
        if (has_rows(i)) {
          int64_t t, off;
          const uint32_t bytes = seg_of(i, t, off);
          if (!mbar_wait(&full[b], (phase_bits >> b) & 1u, wait_ns, nullptr)) {
            record_error(status, DEV_TIMEOUT, 10,
                         static_cast<unsigned long long>(first + i * step));
            // drain: let every load still in flight land before the block exits
            for (int q = 0; q < kPermNBuf; ++q)
              if ((armed >> q) & 1u) mbar_wait(&full[q], (phase_bits >> q) & 1u, wait_ns, nullptr);
            bulk_wait_all();
            failed = 1;
            break;
          }
          phase_bits ^= (1u << b);
          armed &= ~(1u << b);
          const int32_t* rows = meta_rows[(i >> 5) % 3][i & 31];
          for (int j = 0; j < k; ++j) {
            const int32_t r = rows[j];
            if (r >= 0)
              bulk_store(x_perm + static_cast<int64_t>(r) * row_bytes + off,
                         smem + static_cast<size_t>(b) * seg_bytes, bytes);
          }
        }
        bulk_commit();  // one group per item (possibly empty) keeps the group count regular
        const int64_t nxt = i + kPermLookahead;
        if (nxt < n) {
          // buffer nxt % NBUF was last read by the stores of item nxt - NBUF; at most
          // NBUF - LOOKAHEAD groups committed after it may still be reading
          bulk_wait_read<kPermNBuf - kPermLookahead>();
          if (has_rows(nxt)) issue_load(nxt);
        }
      }
    }
    failed = __shfl_sync(0xffffffffu, failed, 0);
    if (failed) return;
  }
  if (lane == 0) bulk_wait_all();
}

}  // namespace

namespace {
inline size_t round256(size_t b) { return (b + 255) / 256 * 256; }

// Scratch of the score-priority dispatch: the dropless token-order layout of all picks
// (row of each pick, token of each row, kept and offsets of that layout), the threshold
// of each expert, and each pick's priority in its dropless row.
struct ScoreScratch {
  int32_t* assign_row;    // [T * k]
  int32_t* token_of_row;  // [T * k]
  int32_t* kept;          // [E]
  int32_t* offsets;       // [E + 1]
  uint64_t* thr;          // [E]
  uint64_t* prio;         // [T * k]
};

ScoreScratch score_scratch(const Shape& s, void* base) {
  const size_t a = static_cast<size_t>(s.T) * s.k;
  uint8_t* p = static_cast<uint8_t*>(base);
  ScoreScratch sc;
  sc.assign_row = reinterpret_cast<int32_t*>(p);
  p += round256(a * sizeof(int32_t));
  sc.token_of_row = reinterpret_cast<int32_t*>(p);
  p += round256(a * sizeof(int32_t));
  sc.kept = reinterpret_cast<int32_t*>(p);
  p += round256(static_cast<size_t>(s.E) * sizeof(int32_t));
  sc.offsets = reinterpret_cast<int32_t*>(p);
  p += round256(static_cast<size_t>(s.E + 1) * sizeof(int32_t));
  sc.thr = reinterpret_cast<uint64_t*>(p);
  p += round256(static_cast<size_t>(s.E) * sizeof(uint64_t));
  sc.prio = reinterpret_cast<uint64_t*>(p);
  return sc;
}
}  // namespace

size_t dispatch_score_scratch_bytes(const Shape& s) {
  if (s.drop_policy != MOE_DROP_SCORE) return 0;
  const size_t a = static_cast<size_t>(s.T) * s.k;
  return 2 * round256(a * sizeof(int32_t)) + round256(static_cast<size_t>(s.E) * 4) +
         round256(static_cast<size_t>(s.E + 1) * 4) + round256(static_cast<size_t>(s.E) * 8) +
         round256(a * sizeof(uint64_t));
}

cudaError_t launch_dispatch(const Shape& s, const void* x, const int32_t* topk_idx,
                            int32_t* routed, int32_t* kept, int32_t* offsets,
                            int32_t* assign_row, int32_t* token_of_row, void* x_perm,
                            int32_t* hist, DevStatus* status, uint64_t wait_ns,
                            cudaStream_t st, const DispatchScores* scores) {
  const int64_t nblk = dispatch_blocks(s.T);
  cudaError_t err;
  const int planes = dispatch_planes(s);
  const ScoreFilter all{nullptr, nullptr, nullptr, 0};
  if (s.drop_policy == MOE_DROP_SCORE) {
    if (scores == nullptr || scores->logits == nullptr || scores->scratch == nullptr)
      return cudaErrorInvalidValue;
    const ScoreScratch sc = score_scratch(s, scores->scratch);
    ScoreFilter flt{nullptr, scores->logits, scores->bias, scores->bias_stride};
    // 1. every pick, dropless, in token order: routed, and each expert's picks grouped
    dispatch_count_kernel<<<static_cast<unsigned>(nblk), kDispatchBlockTokens, 0, st>>>(
        topk_idx, s.T, s.k, s.E, 1, hist, status, all);
    note_launch();
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    dispatch_rank_kernel<<<static_cast<unsigned>(nblk), kDispatchBlockTokens, 0, st>>>(
        topk_idx, s.T, s.k, s.E, -1, MOE_LAYOUT_COMPACT, 1, nblk, hist, routed, sc.kept,
        sc.offsets, sc.assign_row, sc.token_of_row, s.T * s.k, all);
    note_launch();
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    // 2. per expert, the priority of its C-th best pick
    score_select_kernel<<<static_cast<unsigned>(s.E), kSelectThreads, 0, st>>>(
        routed, sc.offsets, sc.token_of_row, flt, s.E, s.C, sc.prio, sc.thr);
    note_launch();
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    // 3. the kept picks, ranked in token order inside their buckets
    flt.thr = sc.thr;
    dispatch_count_kernel<<<static_cast<unsigned>(nblk), kDispatchBlockTokens, 0, st>>>(
        topk_idx, s.T, s.k, s.E, 1, hist, nullptr, flt);
    note_launch();
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    dispatch_rank_kernel<<<static_cast<unsigned>(nblk), kDispatchBlockTokens, 0, st>>>(
        topk_idx, s.T, s.k, s.E, s.C, s.layout, 1, nblk, hist, routed, kept, offsets,
        assign_row, token_of_row, s.max_rows, flt);
    note_launch();
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  } else {
    dispatch_count_kernel<<<static_cast<unsigned>(nblk), kDispatchBlockTokens, 0, st>>>(
        topk_idx, s.T, s.k, s.E, planes, hist, status, all);
    note_launch();
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    dispatch_rank_kernel<<<static_cast<unsigned>(nblk), kDispatchBlockTokens, 0, st>>>(
        topk_idx, s.T, s.k, s.E, s.C, s.layout, planes, nblk, hist, routed, kept, offsets,
        assign_row, token_of_row, s.max_rows, all);
    note_launch();
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  }
  if (x_perm == nullptr) return cudaSuccess;  // bookkeeping only: the FFN gathers rows of x

  const int64_t row_bytes = s.d * s.elem;
  const int64_t segs = (row_bytes + kPermMaxSeg - 1) / kPermMaxSeg;
  // equal segments, each a multiple of 16 bytes
  int64_t seg = (row_bytes + segs - 1) / segs;
  seg = (seg + 15) / 16 * 16;
  // about 96 KB of ring per block, two blocks per SM; half the ring is loads in flight.  A
  // short run (at most 8 items per block of 4 per SM, e.g. 4096 tokens) takes 6-segment rings
  // in 4 blocks per SM instead: more copies start at once, fewer wait behind each other
  const int64_t items = s.T * segs;
  int64_t grid = static_cast<int64_t>(sm_count()) * 2;
  const bool short_run = items <= static_cast<int64_t>(sm_count()) * 4 * 8;
  if (short_run) grid = static_cast<int64_t>(sm_count()) * 4;
  if (grid > items) grid = items;
  if (grid < 1) grid = 1;
  const uint8_t* xb = static_cast<const uint8_t*>(x);
  uint8_t* xp = static_cast<uint8_t*>(x_perm);
  const uint32_t sg = static_cast<uint32_t>(seg);
  if (short_run || seg > 8 * 1024) {
    const size_t smem = 6 * static_cast<size_t>(seg);
    err = cudaFuncSetAttribute(permute_rows_kernel<6, 3>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    permute_rows_kernel<6, 3><<<static_cast<unsigned>(grid), 32, smem, st>>>(
        xb, assign_row, s.T, s.k, row_bytes, sg, segs, xp, status, wait_ns);
    note_launch();
  } else if (seg <= 6 * 1024) {
    const size_t smem = 16 * static_cast<size_t>(seg);
    err = cudaFuncSetAttribute(permute_rows_kernel<16, 8>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    permute_rows_kernel<16, 8><<<static_cast<unsigned>(grid), 32, smem, st>>>(
        xb, assign_row, s.T, s.k, row_bytes, sg, segs, xp, status, wait_ns);
    note_launch();
  } else {
    const size_t smem = 12 * static_cast<size_t>(seg);
    err = cudaFuncSetAttribute(permute_rows_kernel<12, 6>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    permute_rows_kernel<12, 6><<<static_cast<unsigned>(grid), 32, smem, st>>>(
        xb, assign_row, s.T, s.k, row_bytes, sg, segs, xp, status, wait_ns);
    note_launch();
  }
  return cudaGetLastError();
}

cudaError_t launch_pick_rank_counts(const Shape& s, const int32_t* topk_idx,
                                    const int32_t* assign_row, const int32_t* group_of_expert,
                                    int32_t* routed, int32_t* kept, int32_t* differs,
                                    DevStatus* status, cudaStream_t st) {
  pick_rank_counts_kernel<<<static_cast<unsigned>(s.k), kCountThreads, 0, st>>>(
      topk_idx, assign_row, group_of_expert, s.T, s.k, s.E, routed, kept, differs, status);
  note_launch();
  return cudaGetLastError();
}

// ------------------------------------------------------------------ allocation-free variant
// Scratch for moe_dispatch_static_scratch(): a status record followed by the per-block
// expert histogram, in a fixed array that every GPU loading this library keeps until the
// process exits.  All calls share it, so calls that run on the GPU at the same time race.
constexpr size_t kStaticStatusBytes = 256;
static __device__ __align__(256) uint8_t g_dispatch_scratch[kStaticStatusBytes +
                                                            kStaticDispatchHistBytes];

namespace {
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// The fixed array's device address on the current device.  Set-up, once per device with
// that device current: the host-side name of the array is not a device address, so the
// runtime is asked for the device address, which is kept.
cudaError_t static_scratch_base(void** base) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_dispatch_scratch);
    if (err != cudaSuccess) return err;
    g_scratch_ptr[dev] = p;
  }
  *base = g_scratch_ptr[dev];
  return cudaSuccess;
}
}  // namespace

cudaError_t dispatch_static_scratch(const Shape& s, const void* x, const int32_t* topk_idx,
                                    int32_t* routed, int32_t* kept, int32_t* offsets,
                                    int32_t* assign_row, int32_t* token_of_row, void* x_perm,
                                    uint64_t wait_ns, cudaStream_t st) {
  void* base = nullptr;
  cudaError_t err = static_scratch_base(&base);
  if (err != cudaSuccess) return err;
  // The status record starts at zero (static storage) and holds the first error since the
  // last static_scratch_status() read, which clears it; the histogram is fully rewritten
  // by every call.
  DevStatus* status = static_cast<DevStatus*>(base);
  int32_t* hist = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(base) + kStaticStatusBytes);
  return launch_dispatch(s, x, topk_idx, routed, kept, offsets, assign_row, token_of_row,
                         x_perm, hist, status, wait_ns, st);
}

cudaError_t static_scratch_status(DevStatus* out, cudaStream_t st) {
  void* base = nullptr;
  cudaError_t err = static_scratch_base(&base);
  if (err != cudaSuccess) return err;
  err = cudaStreamSynchronize(st);
  if (err != cudaSuccess) return err;
  err = cudaMemcpy(out, base, sizeof(DevStatus), cudaMemcpyDeviceToHost);
  if (err != cudaSuccess || out->code == DEV_OK) return err;
  return cudaMemset(base, 0, sizeof(DevStatus));
}

}  // namespace moe
