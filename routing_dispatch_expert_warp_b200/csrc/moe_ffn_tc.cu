// Expert SwiGLU FFN for bf16 layers: a grouped GEMM on the 5th-generation tensor cores
// (tcgen05 MMA with accumulators in tensor memory), fed by TMA, over the variable-sized
// expert buckets that dispatch produced.
//
// "MoE expert parallelism needs measurements before launch" (airouter.kz), "Profile
// all-to-all separately from compute": expert compute runs as grouped GEMMs over many
// experts; "Expert Parallelism for MoE Serving" (aiunderstanding.org), "Technical
// insight": capacity and padding exist to keep those GEMMs regular -- here the kernel
// takes the ragged buckets as they are and masks the tails.
//
// Two launches of one persistent kernel template:
//   gate/up (GATED): for a 128-row x 128-column tile of h, the B operand is the 128 rows of
//     W_g[e] stacked on the same 128 rows of W_u[e] (256 rows), so one 128x256x16 MMA per
//     K step produces the gate tile in TMEM columns [0,128) and the up tile in [128,256);
//     the epilogue writes h = silu(gate) * up as bf16.
//   down: a 128 x 256 tile of y_perm = h . W_d[e]^T; the epilogue stages each 32-column
//     chunk in shared memory and stores whole 32-row groups with tensor stores.
//   router (E > 32, bf16 x): z = x . W_r with W_r split into two bf16 terms, W' = [E, 2d] =
//     [hi | lo] along K: all E <= 256 experts of 128 tokens in one accumulator, each 64-wide
//     chunk of x taken against hi and then lo, each tile starting its K loop at its own chunk;
//     the epilogue (8 warps, two halves of the experts) writes z + bias in fp32 and, without
//     a group limit, the top-k and gate weights.
//
// Block = 6 warps (10 for the router), one block per SM, persistent over tiles:
//   warp 0 (one lane)   TMA producer: A = 128 x 64 bf16 slice of x_perm/h rows, B = 256 x 64
//                       slice of the expert's weights, 128-byte swizzle, 4-stage ring.
//                       With gathered A (dispatch without x_perm) the whole warp copies the
//                       128 rows of x with cp.async into the same swizzled layout.
//   warp 1 (one lane)   MMA issuer: 4 MMAs (K = 16 each) per stage into one of two TMEM
//                       accumulators (256 fp32 columns each); commits free the smem stage
//                       and, at the end of a tile, hand the accumulator to the epilogue.
//   warps 2-5           epilogue: each thread owns one accumulator row (TMEM lane), reads
//                       it 32 columns at a time, converts and stores; the accumulator is
//                       returned while the MMA warp already fills the other one.
// Tiles are numbered expert by expert, n-block by n-block, with the m-blocks of one
// (expert, n-block) consecutive, so the blocks running at the same time share weight tiles
// through L2.  The tile table is built on the device from the bucket counts: no host read.
// Every barrier wait is bounded; a wait that runs out records MOE_ERR_TIMEOUT, makes the
// other roles stop, drains the copies and MMAs in flight, frees TMEM and returns.
#include <atomic>
#include <mutex>

#include "moe_internal.h"
#include "moe_keys.cuh"

namespace moe {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr int MMA_N = 256;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = MMA_N * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int THREADS = 192;
// the router mode runs 8 epilogue warps: two per TMEM lane quarter, each taking half of the
// 256 expert columns of its 32 tokens, their two top-k lists merged through shared memory
constexpr int ROUTER_THREADS = 320;
constexpr int ACC_COLS = 256;
constexpr int TMEM_COLS = 512;
// per epilogue warp: two buffers of 32 rows x 64 bytes (one 32-column chunk of bf16) in the
// layout of a 64-byte-swizzled tensor tile (16-byte piece c of row r at r * 64 +
// ((c ^ ((r >> 1) & 3)) * 16)), 2 KB apart from a 1 KB-aligned base
constexpr int XBUF_BYTES = 32 * 64;
constexpr int XSTAGE_BYTES = 2 * XBUF_BYTES;
constexpr int DYN_SMEM = STAGES * STAGE_BYTES + 4 * XSTAGE_BYTES + 1024;  // + alignment slack

enum TcMode { MODE_DOWN = 0, MODE_SWIGLU = 1, MODE_ROUTER = 2 };

struct TcParams {
  const int32_t* seg_start;  // [E] first row of each bucket
  const int32_t* seg_count;  // [E] rows of each bucket
  int E;
  int K;         // reduction length (multiple of 64)
  int n_blocks;  // output column blocks
  int N_out;     // output columns
  int mb_outer;  // 1: tiles of one m-block consecutive (all n-blocks share the A rows)
  __nv_bfloat16* out;
  float* out_f32;            // MODE_ROUTER output
  const float* bias;         // MODE_ROUTER logit bias (or nullptr)
  int64_t bias_stride;
  DevStatus* status;
  uint64_t wait_ns;
  // Gathered A (gate/up only): A row i of a bucket is row a_rows[seg_start[e] + i] of the
  // tensor behind tm_a (x itself, [a_rows_limit, K]); nullptr: A rows are the bucket rows.
  const int32_t* a_rows;
  int32_t a_rows_limit;
  const void* a_src;  // x itself, [a_rows_limit, K] bf16, when a_rows is set
  // Combine fused into the down launch (comb_out != nullptr): after a row's 256-column
  // block of y_perm is stored, the row's token counter for that block is bumped; the
  // thread that completes it sums the token's kept rows in pick order into comb_out.
  const int32_t* row_token;   // token_of_row
  const int32_t* assign_row;  // [T, k]
  const float* topk_w;        // [T, k]
  int32_t* arrive;            // [T, n_blocks] counters, zero before the launch
  __nv_bfloat16* comb_out;    // [T, N_out]
  int k;
  int32_t T;
  // MODE_ROUTER: the A rows (x) are a_k wide; the K = 2 a_k reduction takes each 64-wide
  // chunk of x against the hi and then the lo half of the split router weight ([E, 2 a_k]:
  // hi in columns [0, a_k), lo in [a_k, 2 a_k)).
  int a_k;
  int fuse_topk;              // 1: the epilogue selects the top-k and writes the gate weights
  int gating;                 // MOE_GATE_SOFTMAX / MOE_GATE_SIGMOID
  const float* sel_bias;      // bias added to the selection score only (or nullptr)
  int32_t* route_idx;         // [T, k] picks (fused top-k)
  float* route_w;             // [T, k] gate weights (fused top-k)
  int32_t router_rows;        // MODE_ROUTER: its one bucket is rows [0, router_rows) of x
  // MODE_ROUTER split along K (few tiles): work item i is K steps
  // [s kb_per_split, (s + 1) kb_per_split) of tile i / ksplit, s = i % ksplit; the epilogue
  // writes that piece's fp32 sums to out_f32 + s router_rows N_out (no bias, no top-k)
  int ksplit;
  int kb_per_split;
};

// The last of a token's kept picks to finish column block nb has its warp sum the token's
// rows of that block in pick order (fp32 FMA, then bf16: the arithmetic of the combine
// kernel).  Lane l owns columns [8 l, 8 l + 8) of the 256-column block and loads its 16
// bytes of every pick's row at once.  The other picks' rows were stored by other threads,
// possibly of other blocks: their stores precede their counter increments (fence), the
// increment seen here precedes these loads (fence), and the loads bypass L1.
__device__ __forceinline__ void combine_token_block(const TcParams& p, int t, int nb, int lane) {
  const int64_t col = static_cast<int64_t>(nb) * 256 + lane * 8;
  if (col >= p.N_out) return;
  const int32_t* ar = p.assign_row + static_cast<int64_t>(t) * p.k;
  const float* tw = p.topk_w + static_cast<int64_t>(t) * p.k;
  uint4 v[MOE_MAX_TOPK];
  int32_t rr[MOE_MAX_TOPK];
#pragma unroll
  for (int j = 0; j < MOE_MAX_TOPK; ++j) {
    rr[j] = j < p.k ? ar[j] : -1;
    if (rr[j] >= 0)
      v[j] = __ldcg(reinterpret_cast<const uint4*>(p.out + static_cast<int64_t>(rr[j]) * p.N_out +
                                                   col));
  }
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll
  for (int j = 0; j < MOE_MAX_TOPK; ++j) {
    if (rr[j] < 0) continue;
    const float w = tw[j];
    const uint32_t uu[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      acc[2 * q] = fmaf(w, bf16_lo(uu[q]), acc[2 * q]);
      acc[2 * q + 1] = fmaf(w, bf16_hi(uu[q]), acc[2 * q + 1]);
    }
  }
  *reinterpret_cast<uint4*>(p.comb_out + static_cast<int64_t>(t) * p.N_out + col) =
      make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                 pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
}

__device__ __forceinline__ void decode_tile(int tile, const int* tile_base, const int* mblocks,
                                            int E, int n_blocks, int mb_outer, int& e, int& mb,
                                            int& nb) {
  int lo = 0, hi = E - 1;  // largest e with tile_base[e] <= tile
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tile_base[mid] <= tile) lo = mid;
    else hi = mid - 1;
  }
  e = lo;
  const int local = tile - tile_base[e];
  if (mb_outer) {
    mb = local / n_blocks;
    nb = local - mb * n_blocks;
  } else {
    const int mbs = mblocks[e];
    nb = local / mbs;
    mb = local - nb * mbs;
  }
}

__device__ __forceinline__ float silu_mul(float g, float u) {
  return g / (1.0f + __expf(-g)) * u;
}

// One 32-column chunk of a 128-row tile, bf16, from the warp that holds TMEM lane quarter q.
// Each lane writes its row (16 packed words) into the warp's staging buffer `buf` in the
// 64-byte-swizzled layout.  When all 32 rows of the quarter are bucket rows (`tma_rows`),
// lane 0 stores the 32 x 32 block with one tensor store; otherwise every 4 lanes store one
// row's 64 bytes, 8 rows per instruction, skipping rows at or past `valid` (with M = 64
// tiles TMEM lane i < 16 of quarter q holds tile row 16 q + i).  The caller has made sure
// that no earlier tensor store still reads `buf`; lane 0 commits one bulk group per call.
__device__ __forceinline__ void store_chunk_staged(uint8_t* buf, const uint32_t (&pk)[16],
                                                   const CUtensorMap* tm_out,
                                                   __nv_bfloat16* out, int64_t n_out, int row0,
                                                   int64_t col, int q, int valid, bool m64,
                                                   bool cols_ok, bool tma_rows, int lane) {
  const int sw = (lane >> 1) & 3;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    *reinterpret_cast<uint4*>(buf + lane * 64 + ((i ^ sw) << 4)) =
        make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
  if (tma_rows) {
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0 && cols_ok)
      tma_store_2d(tm_out, buf, static_cast<int32_t>(col), row0 + 32 * q);
  } else {
    __syncwarp();
    if (cols_ok) {
      const int seg = lane & 3;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int sr = 8 * i + (lane >> 2);  // staging row = TMEM lane within the quarter
        const int tr = m64 ? (sr < 16 ? 16 * q + sr : BM) : 32 * q + sr;
        if (tr < valid) {
          const uint4 v =
              *reinterpret_cast<const uint4*>(buf + sr * 64 + ((seg ^ ((sr >> 1) & 3)) << 4));
          *reinterpret_cast<uint4*>(out + static_cast<int64_t>(row0 + tr) * n_out + col +
                                    seg * 8) = v;
        }
      }
    }
  }
  if (lane == 0) bulk_commit();  // one group per chunk, empty or not
}

// tm_out (MODE_DOWN): the output y_perm [rows, N_out], 32 x 32 boxes, 64-byte swizzle, for
// the epilogue's tensor stores; the other modes do not read it.
template <int MODE>
__global__ void __launch_bounds__(MODE == 2 ? ROUTER_THREADS : THREADS, 1) grouped_gemm_tc_kernel(
    const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b0,
    const __grid_constant__ CUtensorMap tm_b1, const __grid_constant__ CUtensorMap tm_out,
    const TcParams p) {
  constexpr bool GATED = MODE == MODE_SWIGLU;  // B tile = two stacked 128-row halves
  constexpr int BN_OUT = GATED ? 128 : 256;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[STAGES];
  __shared__ __align__(8) uint64_t empty_bar[STAGES];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ __align__(8) uint64_t mfull_bar;   // router: the upper-half lists are written
  __shared__ __align__(8) uint64_t mempty_bar;  // router: ... and read
  __shared__ uint32_t tmem_base_s;
  __shared__ volatile int abort_s;
  __shared__ int tile_base[MOE_MAX_EXPERTS + 1];
  __shared__ int mblocks[MOE_MAX_EXPERTS];
  constexpr unsigned EPI_THREADS = MODE == MODE_ROUTER ? ROUTER_THREADS - 64 : THREADS - 64;

  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // the router's one bucket is rows [0, router_rows) of x; the FFN's buckets are the
  // dispatch's offsets and kept counts
  auto seg_start = [&](int e) { return MODE == MODE_ROUTER ? 0 : p.seg_start[e]; };
  auto seg_count = [&](int e) { return MODE == MODE_ROUTER ? p.router_rows : p.seg_count[e]; };

  if (warp == 0) {  // tile table: m-blocks per expert and their prefix (x n_blocks)
    int carry = 0;
    for (int e0 = 0; e0 < p.E; e0 += 32) {
      const int e = e0 + lane;
      const int mb = e < p.E ? (seg_count(e) + BM - 1) / BM : 0;
      int v = mb;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += o;
      }
      if (e < p.E) {
        mblocks[e] = mb;
        tile_base[e] = (carry + v - mb) * p.n_blocks;
      }
      carry += __shfl_sync(0xffffffffu, v, 31);
    }
    if (lane == 0) tile_base[p.E] = carry * p.n_blocks;
    if (lane == 0) {
      prefetch_tensormap(&tm_a);
      prefetch_tensormap(&tm_b0);
      if (GATED) prefetch_tensormap(&tm_b1);
    }
  } else if (warp == 1) {
    tmem_alloc(&tmem_base_s, TMEM_COLS);
    tmem_relinquish();
  } else if (threadIdx.x == 64) {
    // full: the producer's arm (+ TMA bytes), plus one arrival per lane of the producer warp
    // when those lanes copy the A rows themselves (gathered A)
    const unsigned full_count = p.a_rows != nullptr ? 33u : 1u;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], full_count);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], EPI_THREADS);
    }
    mbar_init(&drain_bar, 1);
    mbar_init(&mfull_bar, 128);
    mbar_init(&mempty_bar, 128);
    abort_s = 0;
    fence_barrier_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem_base = tmem_base_s;
  const int total_tiles = tile_base[p.E];
  const int KB = p.K / BK;
  // work items: tiles, or (router split along K) tile x K piece, strided over the grid
  const int ksplit = MODE == MODE_ROUTER && p.ksplit > 1 ? p.ksplit : 1;
  const int total_items = total_tiles * ksplit;
  auto item_range = [&](int item, int& tile, int& piece, int& kb0, int& kb1) {
    tile = item / ksplit;
    piece = item - tile * ksplit;
    kb0 = ksplit > 1 ? piece * p.kb_per_split : 0;
    kb1 = ksplit > 1 && kb0 + p.kb_per_split < KB ? kb0 + p.kb_per_split : KB;
  };

  if (warp == 0 && p.a_rows == nullptr) {
    // ---------------------------------------------------------------- TMA producer
    // One lane: waits for a free stage, arms it, loads the A tile (128 bucket rows) and B.
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      uint32_t armed = 0, armed_parity = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < total_items; item += gridDim.x) {
        int tile, piece, kb0, kb1;
        item_range(item, tile, piece, kb0, kb1);
        int e, mb, nb;
        decode_tile(tile, tile_base, mblocks, p.E, p.n_blocks, p.mb_outer, e, mb, nb);
        const int row0 = seg_start(e) + mb * BM;
        // The router's tiles all read the same split weight: tile t starts its K loop at
        // chunk pair t * pairs / tiles and wraps, so the blocks in flight read different parts
        // of it at any moment instead of all the same lines at once.  (The fp32 sum then runs
        // in a per-tile order: deterministic, a rounding-level difference per tile.)
        const int pairs = KB >> 1;
        const int rot = MODE == MODE_ROUTER && ksplit == 1
                            ? static_cast<int>(static_cast<int64_t>(tile) * pairs / total_tiles)
                            : 0;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty_bar[s], ph ^ 1u, p.wait_ns, &abort_s)) {
            if (!abort_s)
              record_error(p.status, DEV_TIMEOUT, 20, static_cast<unsigned long long>(tile));
            abort_s = 1;
            ok = false;
            break;
          }
          uint8_t* sa = smem + s * STAGE_BYTES;
          uint8_t* sb = sa + A_BYTES;
          mbar_arrive_expect_tx(&full_bar[s], STAGE_BYTES);
          armed |= 1u << s;
          armed_parity = (armed_parity & ~(1u << s)) | (ph << s);
          // the router takes each 64-wide chunk of its x rows twice in a row, against the hi
          // and then the lo half of the split weight (the second read hits L2)
          int pr = (kb >> 1) + rot;
          if (pr >= pairs) pr -= pairs;
          const int a_col = MODE == MODE_ROUTER ? pr * BK : kb * BK;
          const int b_col = MODE == MODE_ROUTER ? (kb & 1) * p.a_k + pr * BK : kb * BK;
          tma_load_2d(sa, &tm_a, &full_bar[s], a_col, row0);
          if (GATED) {
            tma_load_3d(sb, &tm_b0, &full_bar[s], b_col, nb * 128, e);
            tma_load_3d(sb + B_BYTES / 2, &tm_b1, &full_bar[s], b_col, nb * 128, e);
          } else {
            tma_load_3d(sb, &tm_b0, &full_bar[s], b_col, nb * 256, e);
          }
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      // every fill this thread armed must land before the block can exit
      for (int q = 0; q < STAGES; ++q)
        if ((armed >> q) & 1u)
          mbar_wait(&full_bar[q], (armed_parity >> q) & 1u, p.wait_ns, nullptr);
    }
  } else if (warp == 0) {
    // ---------------------------------------------------------------- producer, gathered A
    // Lane 0 waits for free stages, arms them for the B bytes and loads B with TMA.  The A
    // tile is 128 rows of x picked through a_rows: lane l copies rows l, l+32, l+64, l+96,
    // eight 16-byte chunks each, with cp.async into the 128-byte-swizzled K-major layout a
    // TMA tile load would produce (chunk c of row r at r * 128 + ((c ^ (r % 8)) * 16)), then
    // has the hardware arrive on the stage's full barrier once its copies have landed; the
    // full barrier expects 1 + 32 arrivals.  (Copying whole 128-byte row pieces per
    // instruction, 8 lanes a row, measured slower: one warp then spends more instructions
    // per copy than the copies save.)
    int s = 0;
    uint32_t ph = 0;
    uint32_t armed = 0, armed_parity = 0;
    bool ok = true;
    const int64_t row_bytes = static_cast<int64_t>(p.K) * 2;
    const uint8_t* xa = reinterpret_cast<const uint8_t*>(p.a_src);
    for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
      int e, mb, nb;
      decode_tile(tile, tile_base, mblocks, p.E, p.n_blocks, p.mb_outer, e, mb, nb);
      const int row0 = seg_start(e) + mb * BM;
      // rows past the bucket read token 0; the epilogue never stores them
      const uint8_t* src[4];
      const int valid = seg_count(e) - mb * BM;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = lane + 32 * i;
        int t = 0;
        if (r < valid) {
          t = __ldg(p.a_rows + row0 + r);
          if (t < 0 || t >= p.a_rows_limit) t = 0;
        }
        src[i] = xa + static_cast<int64_t>(t) * row_bytes;
      }
      for (int kb = 0; kb < KB; ++kb) {
        int got = 1;
        if (lane == 0) got = mbar_wait(&empty_bar[s], ph ^ 1u, p.wait_ns, &abort_s) ? 1 : 0;
        got = __shfl_sync(0xffffffffu, got, 0);
        if (!got) {
          if (lane == 0 && !abort_s)
            record_error(p.status, DEV_TIMEOUT, 20, static_cast<unsigned long long>(tile));
          abort_s = 1;
          ok = false;
          break;
        }
        __syncwarp();  // the stage lane 0 saw released is released for every lane's copies
        uint8_t* sa = smem + s * STAGE_BYTES;
        uint8_t* sb = sa + A_BYTES;
        if (lane == 0) {
          mbar_arrive_expect_tx(&full_bar[s], B_BYTES);
          if (GATED) {
            tma_load_3d(sb, &tm_b0, &full_bar[s], kb * BK, nb * 128, e);
            tma_load_3d(sb + B_BYTES / 2, &tm_b1, &full_bar[s], kb * BK, nb * 128, e);
          } else {
            tma_load_3d(sb, &tm_b0, &full_bar[s], kb * BK, nb * 256, e);
          }
        }
        armed |= 1u << s;
        armed_parity = (armed_parity & ~(1u << s)) | (ph << s);
        const uint32_t sa_addr = smem_addr(sa);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = lane + 32 * i;
          const uint8_t* g = src[i] + static_cast<int64_t>(kb) * (BK * 2);
#pragma unroll
          for (int c = 0; c < 8; ++c)
            cp_async16(sa_addr + r * 128 + ((c ^ (r & 7)) << 4), g + c * 16);
        }
        cp_async_arrive_noinc(&full_bar[s]);
        if (++s == STAGES) {
          s = 0;
          ph ^= 1u;
        }
      }
    }
    cp_async_wait_all();  // every copy this lane issued lands before it exits
    // every stage armed (its B bytes in flight) must complete before the block can exit
    if (lane == 0)
      for (int q = 0; q < STAGES; ++q)
        if ((armed >> q) & 1u)
          mbar_wait(&full_bar[q], (armed_parity >> q) & 1u, p.wait_ns, nullptr);
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------------- MMA issuer
    // a bucket's last tile with at most 64 rows runs as M = 64 MMAs (half the tensor work)
    constexpr uint32_t idesc_full = idesc_bf16_f32(BM, MMA_N);
    constexpr uint32_t idesc_half = idesc_bf16_f32(BM / 2, MMA_N);
    int s = 0;
    uint32_t ph = 0;
    int acc = 0;
    uint32_t aph = 0;
    bool ok = true;
    bool issued = false;
    for (int item = blockIdx.x; ok && item < total_items; item += gridDim.x) {
      int tile, piece, kb0, kb1;
      item_range(item, tile, piece, kb0, kb1);
      int e, mb, nb;
      decode_tile(tile, tile_base, mblocks, p.E, p.n_blocks, p.mb_outer, e, mb, nb);
      const uint32_t idesc =
          seg_count(e) - mb * BM <= BM / 2 ? idesc_half : idesc_full;
      if (!mbar_wait(&tempty_bar[acc], aph ^ 1u, p.wait_ns, &abort_s)) {
        if (!abort_s) record_error(p.status, DEV_TIMEOUT, 21, static_cast<unsigned long long>(tile));
        abort_s = 1;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * ACC_COLS);
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(&full_bar[s], ph, p.wait_ns, &abort_s)) {
          if (!abort_s) record_error(p.status, DEV_TIMEOUT, 22, static_cast<unsigned long long>(tile));
          abort_s = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = smem_addr(smem + s * STAGE_BYTES);
        const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          tc_mma_f16(d_tmem, sw128_kmajor_desc(a_addr + kk * 32),
                     sw128_kmajor_desc(b_addr + kk * 32), idesc,
                     (kb != kb0 || kk != 0) ? 1u : 0u);
        }
        issued = true;
        tc_commit(&empty_bar[s]);
        if (++s == STAGES) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (!ok) break;
      tc_commit(&tfull_bar[acc]);
      acc ^= 1;
      if (acc == 0) aph ^= 1u;
    }
    if (!ok && issued) {  // MMAs still reading smem / writing TMEM must finish first
      tc_commit(&drain_bar);
      mbar_wait(&drain_bar, 0, p.wait_ns, nullptr);
    }
  } else if (warp >= 2) {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;             // TMEM lane quarter this warp may access
    const int r = q * 32 + lane;        // accumulator row owned by this thread
    uint8_t* xstage = smem + STAGES * STAGE_BYTES + (warp - 2) * XSTAGE_BYTES;
    // router: warps 2-5 take expert columns [0, 128), warps 6-9 [128, 256)
    const int half = MODE == MODE_ROUTER ? (warp - 2) >> 2 : 0;
    int acc = 0;
    uint32_t aph = 0;
    uint32_t mph = 0;  // router: phase of the list handoff
    for (int item = blockIdx.x; item < total_items; item += gridDim.x) {
      int tile, piece, kb0, kb1;
      item_range(item, tile, piece, kb0, kb1);
      int e, mb, nb;
      decode_tile(tile, tile_base, mblocks, p.E, p.n_blocks, p.mb_outer, e, mb, nb);
      const int row0 = seg_start(e) + mb * BM;
      const int valid = seg_count(e) - mb * BM;
      int ok = 1;
      if (lane == 0) ok = mbar_wait(&tfull_bar[acc], aph, p.wait_ns, &abort_s) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) {
        if (lane == 0 && !abort_s) record_error(p.status, DEV_TIMEOUT, 23, static_cast<unsigned long long>(tile));
        abort_s = 1;
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(acc * ACC_COLS);
      // M = 64 tiles (valid <= 64) hold row 16 q + i in lane i < 16 of TMEM quarter q
      const int rt = valid <= BM / 2 ? (lane < 16 ? q * 16 + lane : BM) : r;
      const bool row_ok = rt < valid;
      __nv_bfloat16* orow =
          p.out + static_cast<int64_t>(row0 + rt) * p.N_out + static_cast<int64_t>(nb) * BN_OUT;
      const int cols_left = p.N_out - nb * BN_OUT;
      if (MODE == MODE_ROUTER && ksplit > 1) {
        // one K piece of the tile: this thread's row of its half of the experts, as summed
        float* prow = p.out_f32 +
                      (static_cast<int64_t>(piece) * p.router_rows + row0 + rt) * p.N_out;
#pragma unroll 1
        for (int c = 4 * half; c < 4 * half + 4; ++c) {
          uint32_t v[32];
          tmem_ld32(taddr + c * 32, v);
          tmem_ld_wait();
          if (row_ok && c * 32 < cols_left) {
            if (c * 32 + 32 <= cols_left && (p.N_out & 3) == 0) {
              float4* dst = reinterpret_cast<float4*>(prow + c * 32);
#pragma unroll
              for (int i = 0; i < 8; ++i)
                dst[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                     __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (c * 32 + i < cols_left) prow[c * 32 + i] = __uint_as_float(v[i]);
            }
          }
        }
      } else if (MODE == MODE_ROUTER) {
        // one token per thread, all experts of the tile (up to 256) in its accumulator row
        const int64_t grow = static_cast<int64_t>(row0 + rt);
        float* zrow = p.out_f32 != nullptr ? p.out_f32 + grow * p.N_out : nullptr;
        const float* brow = p.bias != nullptr ? p.bias + grow * p.bias_stride : nullptr;
        const float* srow = p.sel_bias != nullptr ? p.sel_bias + grow * p.bias_stride : nullptr;
        // the k best (key, expert, logit) so far, best first; equal keys keep the expert seen
        // first, i.e. the lower index
        uint32_t tk[MOE_MAX_TOPK];
        int ti[MOE_MAX_TOPK];
        float tz[MOE_MAX_TOPK];
#pragma unroll
        for (int j = 0; j < MOE_MAX_TOPK; ++j) {
          tk[j] = 0u;
          ti[j] = 0;
          tz[j] = 0.f;
        }
        uint32_t thr = 0u;  // key of the k-th best so far
        const uint32_t kth_mask = 1u << (p.k - 1);
        // (key, expert, logit) into the list behind the equal keys it holds; static indices
        auto insert = [&](uint32_t key, int col, float zv) {
#pragma unroll
          for (int j = MOE_MAX_TOPK - 1; j > 0; --j) {
            if (key > tk[j - 1]) {
              tk[j] = tk[j - 1];
              ti[j] = ti[j - 1];
              tz[j] = tz[j - 1];
            } else if (key > tk[j]) {
              tk[j] = key;
              ti[j] = col;
              tz[j] = zv;
            }
          }
          if (key > tk[0]) {
            tk[0] = key;
            ti[0] = col;
            tz[0] = zv;
          }
        };
#pragma unroll 1
        for (int c = 4 * half; c < 4 * half + 4; ++c) {
          uint32_t v[32];
          tmem_ld32(taddr + c * 32, v);
          tmem_ld_wait();
          if (row_ok && c * 32 < cols_left) {
            float z[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int col = c * 32 + i;
              z[i] = __uint_as_float(v[i]);
              if (brow != nullptr && col < cols_left) z[i] += brow[col];
            }
            if (zrow != nullptr) {
              if (c * 32 + 32 <= cols_left && (p.N_out & 3) == 0) {
                float4* dst = reinterpret_cast<float4*>(zrow + c * 32);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                  dst[i] = make_float4(z[4 * i], z[4 * i + 1], z[4 * i + 2], z[4 * i + 3]);
              } else {
#pragma unroll
                for (int i = 0; i < 32; ++i)
                  if (c * 32 + i < cols_left) zrow[c * 32 + i] = z[i];
              }
            }
            if (p.fuse_topk) {
              // the chunk's selection keys (0 past the last expert), then its keys above the
              // k-th best so far, largest first -- equal keys lowest expert first -- inserted
              // behind the equal keys already held (lower experts); every index is static
              uint32_t key[32];
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const int col = c * 32 + i;
                key[i] = col < cols_left ? order_key(srow != nullptr ? z[i] + srow[col] : z[i])
                                         : 0u;
              }
#pragma unroll 1
              while (true) {
                uint32_t best = 0u;
                int bi = 0;
#pragma unroll
                for (int i = 0; i < 32; ++i)
                  if (key[i] > best) {
                    best = key[i];
                    bi = i;
                  }
                if (best <= thr) break;
                float bz = 0.f;
#pragma unroll
                for (int i = 0; i < 32; ++i)
                  if (i == bi) {
                    bz = z[i];
                    key[i] = 0u;
                  }
                insert(best, c * 32 + bi, bz);
                // thr = tk[k - 1], as arithmetic on a one-hot mask (no indexed access)
                thr = 0u;
#pragma unroll
                for (int j = 0; j < MOE_MAX_TOPK; ++j)
                  thr |= tk[j] & (0u - ((kth_mask >> j) & 1u));
              }
            }
          }
        }
        if (p.fuse_topk) {
          // the upper half hands its list to the lower half's thread of the same token, which
          // inserts it behind its own (the upper experts lose ties); both waits are bounded
          uint32_t* mk = reinterpret_cast<uint32_t*>(smem + STAGES * STAGE_BYTES);
          int32_t* mi = reinterpret_cast<int32_t*>(mk + BM * MOE_MAX_TOPK);
          float* mz = reinterpret_cast<float*>(mi + BM * MOE_MAX_TOPK);
          const int slot = r * MOE_MAX_TOPK;
          int mok = 1;
          if (lane == 0)
            mok = mbar_wait(half ? &mempty_bar : &mfull_bar, half ? mph ^ 1u : mph, p.wait_ns,
                            &abort_s) ? 1 : 0;
          mok = __shfl_sync(0xffffffffu, mok, 0);
          if (!mok) {
            if (lane == 0 && !abort_s)
              record_error(p.status, DEV_TIMEOUT, 24, static_cast<unsigned long long>(tile));
            abort_s = 1;
            break;
          }
          if (half) {
#pragma unroll
            for (int j = 0; j < MOE_MAX_TOPK; ++j) {
              mk[slot + j] = tk[j];
              mi[slot + j] = ti[j];
              mz[slot + j] = tz[j];
            }
            mbar_arrive(&mfull_bar);
          } else {
            uint32_t ok2[MOE_MAX_TOPK];
            int oi[MOE_MAX_TOPK];
            float oz[MOE_MAX_TOPK];
#pragma unroll
            for (int j = 0; j < MOE_MAX_TOPK; ++j) {
              ok2[j] = mk[slot + j];
              oi[j] = mi[slot + j];
              oz[j] = mz[slot + j];
            }
            mbar_arrive(&mempty_bar);
#pragma unroll
            for (int j = 0; j < MOE_MAX_TOPK; ++j)
              if (j < p.k) insert(ok2[j], oi[j], oz[j]);
          }
          mph ^= 1u;
        }
        if (p.fuse_topk && row_ok && half == 0) {
          // gate weights over the k picks, the normaliser summed in pick order
          float w[MOE_MAX_TOPK];
          float m = tz[0];
#pragma unroll
          for (int j = 1; j < MOE_MAX_TOPK; ++j)
            if (j < p.k) m = fmaxf(m, tz[j]);
          float ssum = 0.f;
#pragma unroll
          for (int j = 0; j < MOE_MAX_TOPK; ++j) {
            w[j] = p.gating == MOE_GATE_SOFTMAX ? expf(tz[j] - m) : 1.0f / (1.0f + expf(-tz[j]));
            if (j < p.k) ssum += w[j];
          }
          const float inv = 1.0f / ssum;
#pragma unroll
          for (int j = 0; j < MOE_MAX_TOPK; ++j)
            if (j < p.k) {
              p.route_idx[grow * p.k + j] = ti[j];
              p.route_w[grow * p.k + j] = w[j] * inv;
            }
        }
      } else if (GATED) {
#pragma unroll 1
        for (int c = 0; c < BN_OUT / 32; ++c) {
          uint32_t g[32], u[32];
          tmem_ld32(taddr + c * 32, g);
          tmem_ld32(taddr + 128 + c * 32, u);
          tmem_ld_wait();
          // gate/up tiles are long (K = d_model) next to their 32 KB of output: each thread
          // stores its own row (staging these stores measured no faster)
          if (row_ok && c * 32 < cols_left) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[i] = pack_bf16x2(silu_mul(__uint_as_float(g[2 * i]), __uint_as_float(u[2 * i])),
                                  silu_mul(__uint_as_float(g[2 * i + 1]),
                                           __uint_as_float(u[2 * i + 1])));
            uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
          }
        }
      } else {
        // down tiles (K = d_ff) end every few K steps with 64 KB of output: stores go through
        // the staging buffers, a 32 x 32 tensor store per chunk where the quarter's 32 rows
        // are all bucket rows, else 8 rows of 64 bytes per instruction; the fused combine
        // needs each row stored by its owner
        const bool staged = p.comb_out == nullptr;
        const bool tma_rows = valid > BM / 2 && valid >= 32 * (q + 1);
#pragma unroll 1
        for (int c = 0; c < BN_OUT / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(taddr + c * 32, v);
          tmem_ld_wait();
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
          if (staged) {
            // buffer c & 1 was last read by the store of two chunks ago (one group may stay)
            if (lane == 0) bulk_wait_read<1>();
            __syncwarp();
            store_chunk_staged(xstage + (c & 1) * XBUF_BYTES, pk, &tm_out, p.out, p.N_out, row0,
                               static_cast<int64_t>(nb) * BN_OUT + c * 32, q, valid,
                               valid <= BM / 2, c * 32 < cols_left, tma_rows, lane);
          } else if (row_ok && c * 32 < cols_left) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty_bar[acc]);
      acc ^= 1;
      if (acc == 0) aph ^= 1u;
      if (MODE == MODE_DOWN && p.comb_out != nullptr) {
        // the accumulator is already handed back: this overlaps the next tile's MMAs
        int t = -1;
        bool last = false;
        if (row_ok) {
          t = p.row_token[row0 + rt];
          if (t >= 0 && t < p.T) {
            int picks = 0;
            for (int j = 0; j < p.k; ++j)
              picks += p.assign_row[static_cast<int64_t>(t) * p.k + j] >= 0 ? 1 : 0;
            __threadfence();
            const int before =
                atomicAdd(&p.arrive[static_cast<int64_t>(t) * p.n_blocks + nb], 1);
            last = before == picks - 1;
          }
        }
        unsigned todo = __ballot_sync(0xffffffffu, last);
        if (todo != 0u) {  // acquire by the last arrivers, then shared with the whole warp
          __threadfence();
          __syncwarp();
        }
        while (todo != 0u) {
          const int src = __ffs(todo) - 1;
          todo &= todo - 1u;
          combine_token_block(p, __shfl_sync(0xffffffffu, t, src), nb, lane);
        }
      }
    }
    if (lane == 0) bulk_wait_all();  // this warp's tensor stores have written y_perm
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ------------------------------------------------------------------ CTA-pair variant
// The same grouped GEMM with each 256 x 256 tile shared by the two CTAs of a cluster, which
// sit on the two SMs of a TPC and issue one tcgen05 MMA together (cta_group::2, 256x256x16):
// CTA r loads rows [128 r, 128 r + 128) of the tile's A and rows [128 r, 128 r + 128) of its
// 256 B rows (gate/up: rank 0 the W_g rows, rank 1 the same W_u rows), so each SM moves
// 32 KB per 64-deep K step instead of 48 KB for the same MMA work, and a 6-stage ring fits
// where the single-CTA kernel holds 4.  Rank 0's producer arms its stage barrier for both
// CTAs' bytes, both CTAs' copies complete on it, rank 0's MMA warp waits on it alone and its
// commits arrive on the stage-free and accumulator-full barriers of both CTAs.  Each CTA's
// epilogue drains its own 128 accumulator rows (TMEM lane r = tile row 128 rank + r) and
// arrives on rank 0's accumulator-free barrier.  Tiles: (expert, n-block, 256-row m-block),
// m-blocks innermost, one cluster per tile.
constexpr int PBM = 256;                               // rows of a pair tile
constexpr int P_STAGES = 6;
constexpr int P_A_BYTES = 128 * BK * 2;                // this CTA's 128 rows of A
constexpr int P_B_BYTES = 128 * BK * 2;                // this CTA's 128 of the 256 B rows
constexpr int P_STAGE_BYTES = P_A_BYTES + P_B_BYTES;   // 32 KB
constexpr int P_DYN_SMEM = P_STAGES * P_STAGE_BYTES + 1024;
constexpr uint32_t P_EPI_ARRIVALS = 8;                 // 4 epilogue warps x 2 CTAs

template <int MODE>
__global__ void __launch_bounds__(THREADS, 1) grouped_gemm_pair_kernel(
    const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b0,
    const __grid_constant__ CUtensorMap tm_b1, const TcParams p) {
  static_assert(MODE == MODE_DOWN || MODE == MODE_SWIGLU, "expert FFN launches only");
  constexpr bool GATED = MODE == MODE_SWIGLU;
  constexpr int BN_OUT = GATED ? 128 : 256;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[P_STAGES];   // used in rank 0 only
  __shared__ __align__(8) uint64_t empty_bar[P_STAGES];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];        // used in rank 0 only
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t tmem_base_s;
  __shared__ volatile int abort_s;
  __shared__ int tile_base[MOE_MAX_EXPERTS + 1];
  __shared__ int mblocks[MOE_MAX_EXPERTS];

  // the same offsets in both CTAs: the MMA reads the peer's operands at this CTA's offsets
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int cluster = static_cast<int>(blockIdx.x >> 1);
  const int clusters = static_cast<int>(gridDim.x >> 1);

  if (warp == 0) {  // tile table: 256-row m-blocks per expert and their prefix (x n_blocks)
    int carry = 0;
    for (int e0 = 0; e0 < p.E; e0 += 32) {
      const int e = e0 + lane;
      const int mb = e < p.E ? (p.seg_count[e] + PBM - 1) / PBM : 0;
      int v = mb;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += o;
      }
      if (e < p.E) {
        mblocks[e] = mb;
        tile_base[e] = (carry + v - mb) * p.n_blocks;
      }
      carry += __shfl_sync(0xffffffffu, v, 31);
    }
    if (lane == 0) {
      tile_base[p.E] = carry * p.n_blocks;
      prefetch_tensormap(&tm_a);
      prefetch_tensormap(&tm_b0);
      if (GATED) prefetch_tensormap(&tm_b1);
    }
  } else if (warp == 1) {
    tmem_alloc_pair(&tmem_base_s, TMEM_COLS);
    tmem_relinquish_pair();
  } else if (threadIdx.x == 64) {
    for (int s = 0; s < P_STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], P_EPI_ARRIVALS);
    }
    mbar_init(&drain_bar, 1);
    abort_s = 0;
    fence_barrier_init();
  }
  // barriers of both CTAs initialised (the peer signals rank 0's) and the TMEM address known
  tc_fence_before();
  __syncwarp();
  cluster_sync();
  tc_fence_after();

  const uint32_t tmem_base = tmem_base_s;
  const int total_tiles = tile_base[p.E];
  const int KB = p.K / BK;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- TMA producer (both)
    int s = 0;
    uint32_t ph = 0;
    uint32_t armed = 0, armed_parity = 0;
    bool ok = true;
    for (int tile = cluster; ok && tile < total_tiles; tile += clusters) {
      int e, mb, nb;
      decode_tile(tile, tile_base, mblocks, p.E, p.n_blocks, 0, e, mb, nb);
      const int row0 = p.seg_start[e] + mb * PBM + static_cast<int>(rank) * 128;
      for (int kb = 0; kb < KB; ++kb) {
        if (!mbar_wait(&empty_bar[s], ph ^ 1u, p.wait_ns, &abort_s)) {
          if (!abort_s)
            record_error(p.status, DEV_TIMEOUT, 30, static_cast<unsigned long long>(tile));
          abort_s = 1;
          ok = false;
          break;
        }
        uint8_t* sa = smem + s * P_STAGE_BYTES;
        uint8_t* sb = sa + P_A_BYTES;
        const uint32_t full = cluster_addr(smem_addr(&full_bar[s]), 0);
        if (rank == 0) {  // both CTAs' bytes complete on rank 0's barrier
          mbar_arrive_expect_tx(&full_bar[s], 2 * P_STAGE_BYTES);
          armed |= 1u << s;
          armed_parity = (armed_parity & ~(1u << s)) | (ph << s);
        }
        tma_load_2d_pair(sa, &tm_a, full, kb * BK, row0);
        if (GATED)
          tma_load_3d_pair(sb, rank == 0 ? &tm_b0 : &tm_b1, full, kb * BK, nb * 128, e);
        else
          tma_load_3d_pair(sb, &tm_b0, full, kb * BK, nb * 256 + static_cast<int>(rank) * 128, e);
        if (++s == P_STAGES) {
          s = 0;
          ph ^= 1u;
        }
      }
    }
    // every fill rank 0 armed must land before the block can exit (the peer's own fills are
    // counted there too; a peer that gave up waited at least the wait limit first)
    for (int q = 0; q < P_STAGES; ++q)
      if ((armed >> q) & 1u)
        mbar_wait(&full_bar[q], (armed_parity >> q) & 1u, p.wait_ns, nullptr);
  } else if (warp == 1 && lane == 0 && rank == 0) {
    // ---------------------------------------------------------------- MMA issuer (rank 0)
    constexpr uint32_t idesc = idesc_bf16_f32(PBM, MMA_N);
    int s = 0;
    uint32_t ph = 0;
    int acc = 0;
    uint32_t aph = 0;
    bool ok = true;
    bool issued = false;
    for (int tile = cluster; ok && tile < total_tiles; tile += clusters) {
      if (!mbar_wait(&tempty_bar[acc], aph ^ 1u, p.wait_ns, &abort_s)) {
        if (!abort_s) record_error(p.status, DEV_TIMEOUT, 31, static_cast<unsigned long long>(tile));
        abort_s = 1;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * ACC_COLS);
      for (int kb = 0; kb < KB; ++kb) {
        if (!mbar_wait(&full_bar[s], ph, p.wait_ns, &abort_s)) {
          if (!abort_s) record_error(p.status, DEV_TIMEOUT, 32, static_cast<unsigned long long>(tile));
          abort_s = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = smem_addr(smem + s * P_STAGE_BYTES);
        const uint32_t b_addr = a_addr + P_A_BYTES;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          tc_mma_f16_pair(d_tmem, sw128_kmajor_desc(a_addr + kk * 32),
                          sw128_kmajor_desc(b_addr + kk * 32), idesc, (kb | kk) != 0 ? 1u : 0u);
        }
        issued = true;
        tc_commit_pair(&empty_bar[s], 0x3);
        if (++s == P_STAGES) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (!ok) break;
      tc_commit_pair(&tfull_bar[acc], 0x3);
      acc ^= 1;
      if (acc == 0) aph ^= 1u;
    }
    if (!ok && issued) {  // MMAs still reading shared memory / writing TMEM must finish first
      tc_commit_pair(&drain_bar, 0x1);
      mbar_wait(&drain_bar, 0, p.wait_ns, nullptr);
    }
  } else if (warp >= 2) {
    // ---------------------------------------------------------------- epilogue (both)
    const int q = warp & 3;             // TMEM lane quarter this warp may access
    const int r = q * 32 + lane;        // accumulator row owned by this thread
    int acc = 0;
    uint32_t aph = 0;
    for (int tile = cluster; tile < total_tiles; tile += clusters) {
      int e, mb, nb;
      decode_tile(tile, tile_base, mblocks, p.E, p.n_blocks, 0, e, mb, nb);
      const int half0 = mb * PBM + static_cast<int>(rank) * 128;
      const int row0 = p.seg_start[e] + half0;
      const int valid = p.seg_count[e] - half0;
      int ok = 1;
      if (lane == 0) ok = mbar_wait(&tfull_bar[acc], aph, p.wait_ns, &abort_s) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) {
        if (lane == 0 && !abort_s) record_error(p.status, DEV_TIMEOUT, 33, static_cast<unsigned long long>(tile));
        abort_s = 1;
        break;
      }
      tc_fence_after();
      if (valid > q * 32) {  // this warp's 32 rows hold at least one of the bucket's rows
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                               static_cast<uint32_t>(acc * ACC_COLS);
        const bool row_ok = r < valid;
        __nv_bfloat16* orow = p.out + static_cast<int64_t>(row0 + r) * p.N_out +
                              static_cast<int64_t>(nb) * BN_OUT;
        const int cols_left = p.N_out - nb * BN_OUT;
        if (GATED) {
#pragma unroll 1
          for (int c = 0; c < BN_OUT / 32; ++c) {
            uint32_t g[32], u[32];
            tmem_ld32(taddr + c * 32, g);
            tmem_ld32(taddr + 128 + c * 32, u);
            tmem_ld_wait();
            if (row_ok && c * 32 < cols_left) {
              uint32_t pk[16];
#pragma unroll
              for (int i = 0; i < 16; ++i)
                pk[i] = pack_bf16x2(silu_mul(__uint_as_float(g[2 * i]), __uint_as_float(u[2 * i])),
                                    silu_mul(__uint_as_float(g[2 * i + 1]),
                                             __uint_as_float(u[2 * i + 1])));
              uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
            }
          }
        } else {
#pragma unroll 1
          for (int c = 0; c < BN_OUT / 32; ++c) {
            uint32_t v[32];
            tmem_ld32(taddr + c * 32, v);
            tmem_ld_wait();
            if (row_ok && c * 32 < cols_left) {
              uint32_t pk[16];
#pragma unroll
              for (int i = 0; i < 16; ++i)
                pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
              uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(cluster_addr(smem_addr(&tempty_bar[acc]), 0));
      acc ^= 1;
      if (acc == 0) aph ^= 1u;
    }
  }

  // nothing of either CTA may still be signalled, read or written when one of them exits
  tc_fence_before();
  __syncwarp();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

// ------------------------------------------------------------------ token-N variant
// The same grouped GEMM with the operands' roles swapped: the MMA's M = 128 rows are weight
// rows (output features) and its N is the bucket's tokens, up to 256 per tile and, in a
// bucket's last tile, its remaining tokens rounded up to 16 -- so a ragged bucket wastes at
// most 15 rows of tensor work instead of up to 127 with 128-row token tiles.  Per 64-deep
// K step a tile loads 16 KB of weights and up to 32 KB of token rows (128-row boxes), the
// bytes per FLOP of the 128 x 256 token-major tile.
//   gate/up: a tile is 64 features: A rows 0-63 are those rows of W_g, rows 64-127 the
//     same rows of W_u, so TMEM lane quarters 0-1 hold gate and 2-3 hold up.  The epilogue
//     warp of quarter 2 + i hands its up values, 32 tokens at a time, to the warp of
//     quarter i through a double-buffered shared buffer (mbarrier handshake, bounded
//     waits); that warp forms silu(gate) * up.
//   down: a tile is 128 features of y (rows of W_d).
// The storing warp writes each 32-token chunk (one feature per lane) transposed into a
// padded per-warp shared buffer and stores each token's 32 features contiguously.  Tiles:
// (expert, feature block, 256-token block), token blocks innermost.
constexpr int TN_TOK = 256;                              // tokens per tile (max MMA N)
constexpr int TN_BOX = 128;                              // token rows per TMA box
constexpr int TN_STAGES = 4;
constexpr int TN_A_BYTES = 128 * BK * 2;                 // 16 KB of weight rows
constexpr int TN_B_BYTES = TN_TOK * BK * 2;              // up to 32 KB of token rows
constexpr int TN_STAGE_BYTES = TN_A_BYTES + TN_B_BYTES;  // 48 KB
constexpr int TN_XPOSE_STRIDE = 80;                      // bytes per token row in the buffer
constexpr int TN_XPOSE_BYTES = 32 * TN_XPOSE_STRIDE;     // per storing warp
constexpr int TN_XCHG_BYTES = 32 * 32 * 4;               // one chunk of up values (fp32)
// transposition buffers for the 4 storing warps of down (2 of gate/up), then gate/up's two
// warp pairs' double-buffered exchange
constexpr int TN_EPI_BYTES = 4 * TN_XPOSE_BYTES + 2 * 2 * TN_XCHG_BYTES;
constexpr int TN_DYN_SMEM = TN_STAGES * TN_STAGE_BYTES + TN_EPI_BYTES + 1024;

template <int MODE>
__global__ void __launch_bounds__(THREADS, 1) grouped_gemm_tokn_kernel(
    const __grid_constant__ CUtensorMap tm_tok, const __grid_constant__ CUtensorMap tm_w0,
    const __grid_constant__ CUtensorMap tm_w1, const TcParams p) {
  static_assert(MODE == MODE_DOWN || MODE == MODE_SWIGLU, "expert FFN launches only");
  constexpr bool GATED = MODE == MODE_SWIGLU;
  constexpr int FB = GATED ? 64 : 128;  // output features per tile
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[TN_STAGES];
  __shared__ __align__(8) uint64_t empty_bar[TN_STAGES];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ __align__(8) uint64_t xfull_bar[2][2];    // [warp pair][buffer]: up values written
  __shared__ __align__(8) uint64_t xempty_bar[2][2];   // [warp pair][buffer]: up values read
  __shared__ uint32_t tmem_base_s;
  __shared__ volatile int abort_s;
  __shared__ int tile_base[MOE_MAX_EXPERTS + 1];
  __shared__ int tblocks[MOE_MAX_EXPERTS];

  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* epi = smem + TN_STAGES * TN_STAGE_BYTES;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (warp == 0) {  // tile table: 256-token blocks per expert and their prefix (x feature blocks)
    int carry = 0;
    for (int e0 = 0; e0 < p.E; e0 += 32) {
      const int e = e0 + lane;
      const int tb = e < p.E ? (p.seg_count[e] + TN_TOK - 1) / TN_TOK : 0;
      int v = tb;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += o;
      }
      if (e < p.E) {
        tblocks[e] = tb;
        tile_base[e] = (carry + v - tb) * p.n_blocks;
      }
      carry += __shfl_sync(0xffffffffu, v, 31);
    }
    if (lane == 0) {
      tile_base[p.E] = carry * p.n_blocks;
      prefetch_tensormap(&tm_tok);
      prefetch_tensormap(&tm_w0);
      if (GATED) prefetch_tensormap(&tm_w1);
    }
  } else if (warp == 1) {
    tmem_alloc(&tmem_base_s, TMEM_COLS);
    tmem_relinquish();
  } else if (threadIdx.x == 64) {
    for (int s = 0; s < TN_STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], 128);
      for (int b = 0; b < 2; ++b) {
        mbar_init(&xfull_bar[a][b], 1);
        mbar_init(&xempty_bar[a][b], 1);
      }
    }
    mbar_init(&drain_bar, 1);
    abort_s = 0;
    fence_barrier_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem_base = tmem_base_s;
  const int total_tiles = tile_base[p.E];
  const int KB = p.K / BK;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- TMA producer
    int s = 0;
    uint32_t ph = 0;
    uint32_t armed = 0, armed_parity = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
      int e, tb, fb;
      decode_tile(tile, tile_base, tblocks, p.E, p.n_blocks, 0, e, tb, fb);
      const int tok0 = p.seg_start[e] + tb * TN_TOK;
      const int n_valid = min(TN_TOK, p.seg_count[e] - tb * TN_TOK);
      const int nbox = (n_valid + TN_BOX - 1) / TN_BOX;
      const uint32_t bytes = TN_A_BYTES + static_cast<uint32_t>(nbox) * (TN_BOX * BK * 2);
      for (int kb = 0; kb < KB; ++kb) {
        if (!mbar_wait(&empty_bar[s], ph ^ 1u, p.wait_ns, &abort_s)) {
          if (!abort_s)
            record_error(p.status, DEV_TIMEOUT, 40, static_cast<unsigned long long>(tile));
          abort_s = 1;
          ok = false;
          break;
        }
        uint8_t* sa = smem + s * TN_STAGE_BYTES;
        uint8_t* sb = sa + TN_A_BYTES;
        mbar_arrive_expect_tx(&full_bar[s], bytes);
        armed |= 1u << s;
        armed_parity = (armed_parity & ~(1u << s)) | (ph << s);
        if (GATED) {
          tma_load_3d(sa, &tm_w0, &full_bar[s], kb * BK, fb * FB, e);
          tma_load_3d(sa + TN_A_BYTES / 2, &tm_w1, &full_bar[s], kb * BK, fb * FB, e);
        } else {
          tma_load_3d(sa, &tm_w0, &full_bar[s], kb * BK, fb * FB, e);
        }
        for (int j = 0; j < nbox; ++j)
          tma_load_2d(sb + j * (TN_BOX * BK * 2), &tm_tok, &full_bar[s], kb * BK,
                      tok0 + j * TN_BOX);
        if (++s == TN_STAGES) {
          s = 0;
          ph ^= 1u;
        }
      }
    }
    for (int q = 0; q < TN_STAGES; ++q)
      if ((armed >> q) & 1u)
        mbar_wait(&full_bar[q], (armed_parity >> q) & 1u, p.wait_ns, nullptr);
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------------- MMA issuer
    int s = 0;
    uint32_t ph = 0;
    int acc = 0;
    uint32_t aph = 0;
    bool ok = true;
    bool issued = false;
    for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
      int e, tb, fb;
      decode_tile(tile, tile_base, tblocks, p.E, p.n_blocks, 0, e, tb, fb);
      const int n_valid = min(TN_TOK, p.seg_count[e] - tb * TN_TOK);
      const uint32_t idesc = idesc_bf16_f32(128, (n_valid + 15) & ~15);
      if (!mbar_wait(&tempty_bar[acc], aph ^ 1u, p.wait_ns, &abort_s)) {
        if (!abort_s) record_error(p.status, DEV_TIMEOUT, 41, static_cast<unsigned long long>(tile));
        abort_s = 1;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * ACC_COLS);
      for (int kb = 0; kb < KB; ++kb) {
        if (!mbar_wait(&full_bar[s], ph, p.wait_ns, &abort_s)) {
          if (!abort_s) record_error(p.status, DEV_TIMEOUT, 42, static_cast<unsigned long long>(tile));
          abort_s = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = smem_addr(smem + s * TN_STAGE_BYTES);
        const uint32_t b_addr = a_addr + TN_A_BYTES;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          tc_mma_f16(d_tmem, sw128_kmajor_desc(a_addr + kk * 32),
                     sw128_kmajor_desc(b_addr + kk * 32), idesc, (kb | kk) != 0 ? 1u : 0u);
        }
        issued = true;
        tc_commit(&empty_bar[s]);
        if (++s == TN_STAGES) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (!ok) break;
      tc_commit(&tfull_bar[acc]);
      acc ^= 1;
      if (acc == 0) aph ^= 1u;
    }
    if (!ok && issued) {
      tc_commit(&drain_bar);
      mbar_wait(&drain_bar, 0, p.wait_ns, nullptr);
    }
  } else if (warp >= 2) {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;   // TMEM lane quarter this warp may access
    // gate/up: quarters 2-3 (warps 2-3) hand their up values to quarters 0-1 (warps 4-5)
    const bool sender = GATED && q >= 2;
    const int pair = q & 1;
    uint8_t* xb = epi + (GATED ? pair : warp - 2) * TN_XPOSE_BYTES;
    __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(xb);
    float* xchg = reinterpret_cast<float*>(epi + 4 * TN_XPOSE_BYTES + pair * 2 * TN_XCHG_BYTES);
    const int warp_feat0 = GATED ? 32 * pair : 32 * q;   // first feature of this warp's lanes
    uint32_t nchunk = 0;     // chunks exchanged so far (buffer = nchunk & 1)
    int acc = 0;
    uint32_t aph = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
      int e, tb, fb;
      decode_tile(tile, tile_base, tblocks, p.E, p.n_blocks, 0, e, tb, fb);
      const int tok0 = p.seg_start[e] + tb * TN_TOK;
      const int n_valid = min(TN_TOK, p.seg_count[e] - tb * TN_TOK);
      int got = 1;
      if (lane == 0) got = mbar_wait(&tfull_bar[acc], aph, p.wait_ns, &abort_s) ? 1 : 0;
      got = __shfl_sync(0xffffffffu, got, 0);
      if (!got) {
        if (lane == 0 && !abort_s) record_error(p.status, DEV_TIMEOUT, 43, static_cast<unsigned long long>(tile));
        abort_s = 1;
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(acc * ACC_COLS);
      const int col0 = fb * FB + warp_feat0;   // first output feature this warp stores
      const bool feats_ok = col0 < p.N_out;    // N_out is a multiple of 64: all 32 or none
      const int chunks = (n_valid + 31) >> 5;
#pragma unroll 1
      for (int c = 0; c < chunks; ++c, ++nchunk) {
        uint32_t v[32];
        tmem_ld32(taddr + c * 32, v);
        tmem_ld_wait();
        const uint32_t buf = nchunk & 1u, use = (nchunk >> 1) & 1u;
        float* xc = xchg + buf * (32 * 32);
        if (sender) {
          // wait until the partner has read this buffer's previous chunk, then fill it
          int w = 1;
          if (lane == 0) w = mbar_wait(&xempty_bar[pair][buf], use ^ 1u, p.wait_ns, &abort_s) ? 1 : 0;
          w = __shfl_sync(0xffffffffu, w, 0);
          if (!w) {
            if (lane == 0 && !abort_s) record_error(p.status, DEV_TIMEOUT, 44, static_cast<unsigned long long>(tile));
            abort_s = 1;
            ok = false;
            break;
          }
#pragma unroll
          for (int j = 0; j < 32; ++j) xc[j * 32 + lane] = __uint_as_float(v[j]);
          __syncwarp();
          if (lane == 0) mbar_arrive(&xfull_bar[pair][buf]);
          continue;
        }
        if (GATED) {
          int w = 1;
          if (lane == 0) w = mbar_wait(&xfull_bar[pair][buf], use, p.wait_ns, &abort_s) ? 1 : 0;
          w = __shfl_sync(0xffffffffu, w, 0);
          if (!w) {
            if (lane == 0 && !abort_s) record_error(p.status, DEV_TIMEOUT, 45, static_cast<unsigned long long>(tile));
            abort_s = 1;
            ok = false;
            break;
          }
          float u[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) u[j] = xc[j * 32 + lane];
          __syncwarp();
          if (lane == 0) mbar_arrive(&xempty_bar[pair][buf]);
          __syncwarp();  // the previous chunk's reads of the transposition buffer are done
#pragma unroll
          for (int j = 0; j < 32; ++j)
            xs[j * (TN_XPOSE_STRIDE / 2) + lane] =
                __float2bfloat16_rn(silu_mul(__uint_as_float(v[j]), u[j]));
        } else {
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 32; ++j)
            xs[j * (TN_XPOSE_STRIDE / 2) + lane] = __float2bfloat16_rn(__uint_as_float(v[j]));
        }
        __syncwarp();
        const int t = c * 32 + lane;   // this lane stores token t's 32 features
        if (feats_ok && t < n_valid) {
          const uint4* src = reinterpret_cast<const uint4*>(xb + lane * TN_XPOSE_STRIDE);
          uint4* dst = reinterpret_cast<uint4*>(p.out + static_cast<int64_t>(tok0 + t) * p.N_out +
                                                col0);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = src[i];
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty_bar[acc]);
      acc ^= 1;
      if (acc == 0) aph ^= 1u;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// W_r [d, E] fp32 -> W' [E, 2d] bf16, row e = [hi(W[:, e]), lo(W[:, e])] with
// hi = bf16(W), lo = bf16(W - hi), so that x . W = [x, x] . W' up to the rounding of lo (a
// relative 2^-17 of each weight).  32 x 32 tiles transposed through shared memory.
__global__ void __launch_bounds__(256) split_router_weight_kernel(
    const float* __restrict__ w, int d, int E, __nv_bfloat16* __restrict__ wsplit) {
  __shared__ float tile[32][33];
  const int e0 = blockIdx.x * 32, i0 = blockIdx.y * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  for (int r = ty; r < 32; r += 8) {
    const int i = i0 + r, e = e0 + tx;
    tile[r][tx] = (i < d && e < E) ? w[static_cast<int64_t>(i) * E + e] : 0.f;
  }
  __syncthreads();
  for (int r = ty; r < 32; r += 8) {
    const int e = e0 + r, i = i0 + tx;
    if (e < E && i < d) {
      const float v = tile[tx][r];
      const __nv_bfloat16 h = __float2bfloat16_rn(v);
      const __nv_bfloat16 l = __float2bfloat16_rn(v - __bfloat162float(h));
      wsplit[static_cast<int64_t>(e) * 2 * d + i] = h;
      wsplit[static_cast<int64_t>(e) * 2 * d + d + i] = l;
    }
  }
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000,
                                         cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// [rows, K] bf16 row-major, box 128 rows x 64 columns, 128-byte swizzle
bool make_map_rows(CUtensorMap* m, const void* base, int64_t rows, int64_t K) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K * 2)};
  const cuuint32_t box[2] = {BK, BM};
  const cuuint32_t estr[2] = {1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [rows, K] bf16 row-major, box 128 rows x 64 columns, 128-byte swizzle (token-N tiles)
bool make_map_tokens(CUtensorMap* m, const void* base, int64_t rows, int64_t K) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K * 2)};
  const cuuint32_t box[2] = {BK, TN_BOX};
  const cuuint32_t estr[2] = {1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [rows, N] bf16 row-major output, box 32 rows x 32 columns, 64-byte swizzle (epilogue stores)
bool make_map_out(CUtensorMap* m, const void* base, int64_t rows, int64_t N) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(N * 2)};
  const cuuint32_t box[2] = {32, 32};
  const cuuint32_t estr[2] = {1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [E, N, K] bf16 weights, box 1 x box_n x 64, 128-byte swizzle
bool make_map_weights(CUtensorMap* m, const void* base, int E, int64_t N, int64_t K,
                      int box_n) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(E)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(K * 2),
                                 static_cast<cuuint64_t>(N * K * 2)};
  const cuuint32_t box[3] = {BK, static_cast<cuuint32_t>(box_n), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Clusters of two of grouped_gemm_pair_kernel<MODE> that fit on the GPU at once (0: none).
template <int MODE>
int pair_clusters_resident(cudaLaunchConfig_t cfg) {
  static int cached[2] = {-1, -1};
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  int& c = cached[MODE == MODE_SWIGLU ? 1 : 0];
  if (c < 0) {
    int n = 0;
    cfg.gridDim = dim3(2 * static_cast<unsigned>(sm_count() / 2));
    if (cudaOccupancyMaxActiveClusters(&n, grouped_gemm_pair_kernel<MODE>, &cfg) != cudaSuccess) {
      cudaGetLastError();
      n = 0;
    }
    c = n;
  }
  return c;
}

// One launch of the pair kernel over at most `tiles` tiles; *launched = false (nothing
// enqueued) when no cluster of two fits.
template <int MODE>
cudaError_t launch_pair(const CUtensorMap& ta, const CUtensorMap& tb0, const CUtensorMap& tb1,
                        const TcParams& p, int64_t tiles, cudaStream_t st, bool* launched) {
  *launched = false;
  cudaError_t err = cudaFuncSetAttribute(grouped_gemm_pair_kernel<MODE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, P_DYN_SMEM);
  if (err != cudaSuccess) return err;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = P_DYN_SMEM;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int64_t clusters = pair_clusters_resident<MODE>(cfg);
  if (clusters <= 0) return cudaSuccess;
  if (clusters > tiles) clusters = tiles;
  if (clusters < 1) clusters = 1;
  cfg.gridDim = dim3(static_cast<unsigned>(2 * clusters));
  err = cudaLaunchKernelEx(&cfg, grouped_gemm_pair_kernel<MODE>, ta, tb0, tb1, p);
  if (err != cudaSuccess) return err;
  note_launch();
  *launched = true;
  return cudaSuccess;
}

// One launch of the token-N kernel over at most `tiles` tiles, one CTA per SM.
template <int MODE>
cudaError_t launch_tokn(const CUtensorMap& tt, const CUtensorMap& tw0, const CUtensorMap& tw1,
                        const TcParams& p, int64_t tiles, cudaStream_t st) {
  cudaError_t err = cudaFuncSetAttribute(grouped_gemm_tokn_kernel<MODE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, TN_DYN_SMEM);
  if (err != cudaSuccess) return err;
  int64_t g = tiles;
  if (g > sm_count()) g = sm_count();
  if (g < 1) g = 1;
  grouped_gemm_tokn_kernel<MODE><<<static_cast<unsigned>(g), THREADS, TN_DYN_SMEM, st>>>(tt, tw0,
                                                                                         tw1, p);
  note_launch();
  return cudaGetLastError();
}

std::atomic<int> g_ffn_kernel{MOE_FFN_TOKEN_MAJOR};

}  // namespace

void set_ffn_kernel(int kind) { g_ffn_kernel.store(kind); }
int ffn_kernel() { return g_ffn_kernel.load(); }

// Before a down launch with the combine fused in: zero the arrival counters and the output
// rows of tokens none of whose picks was kept (no thread of the launch ever writes those).
__global__ void combine_prep_kernel(int32_t* __restrict__ arrive, int64_t n_counters,
                                    const int32_t* __restrict__ assign_row, int64_t T, int k,
                                    uint4* __restrict__ out, int64_t vec_per_row) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t i0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (int64_t i = i0; i < n_counters; i += stride) arrive[i] = 0;
  // a warp per token: lanes < k look at the picks; a token with none gets a zero row
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = stride >> 5;
  for (int64_t t = i0 >> 5; t < T; t += nwarps) {
    const bool kept = lane < k && assign_row[t * k + lane] >= 0;
    if (__ballot_sync(0xffffffffu, kept) != 0u) continue;
    for (int64_t v = lane; v < vec_per_row; v += 32) out[t * vec_per_row + v] = make_uint4(0u, 0u, 0u, 0u);
  }
}

cudaError_t launch_ffn_tc(const Shape& s, const void* a, const int32_t* a_rows,
                          const int32_t* offsets, const int32_t* kept, const void* wg,
                          const void* wu, const void* wd, void* h, void* y, DevStatus* status,
                          uint64_t wait_ns, cudaStream_t st, const char** why,
                          const FusedCombine* comb) {
  if (encode_fn() == nullptr) {
    *why = "cuTensorMapEncodeTiled is not available from the driver";
    return cudaErrorNotSupported;
  }
  CUtensorMap ta1, tg, tu, ta2, td, ty;
  // gathered A is copied by the producer warp itself; the A map then only stays valid
  const bool a_ok = make_map_rows(&ta1, a, a_rows != nullptr ? s.T : s.max_rows, s.d);
  if (!a_ok ||
      !make_map_weights(&tg, wg, s.E, s.f, s.d, 128) ||
      !make_map_weights(&tu, wu, s.E, s.f, s.d, 128) ||
      !make_map_rows(&ta2, h, s.max_rows, s.f) ||
      !make_map_weights(&td, wd, s.E, s.d, s.f, 256) ||
      !make_map_out(&ty, y, s.max_rows, s.d)) {
    *why = "tensor map encoding failed (pointer alignment or sizes)";
    return cudaErrorInvalidValue;
  }
  cudaError_t err;
  err = cudaFuncSetAttribute(grouped_gemm_tc_kernel<MODE_SWIGLU>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, DYN_SMEM);
  if (err != cudaSuccess) return err;
  err = cudaFuncSetAttribute(grouped_gemm_tc_kernel<MODE_DOWN>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, DYN_SMEM);
  if (err != cudaSuccess) return err;

  const int64_t row_blocks_bound = (s.max_rows + BM - 1) / BM + s.E;
  const int sms = sm_count();

  const int kind = g_ffn_kernel.load();
  if (a_rows == nullptr && comb == nullptr && kind == MOE_FFN_TOKEN_N) {
    // token-N kernel: weight maps with 64-row (W_g, W_u) and 128-row (W_d) boxes, token
    // maps with 128-row boxes
    CUtensorMap tx, tg64, tu64, th, td128;
    if (!make_map_tokens(&tx, a, s.max_rows, s.d) || !make_map_weights(&tg64, wg, s.E, s.f, s.d, 64) ||
        !make_map_weights(&tu64, wu, s.E, s.f, s.d, 64) || !make_map_tokens(&th, h, s.max_rows, s.f) ||
        !make_map_weights(&td128, wd, s.E, s.d, s.f, 128)) {
      *why = "tensor map encoding failed (pointer alignment or sizes)";
      return cudaErrorInvalidValue;
    }
    const int64_t tok_blocks_bound = (s.max_rows + TN_TOK - 1) / TN_TOK + s.E;
    TcParams q1 = {};
    q1.seg_start = offsets;
    q1.seg_count = kept;
    q1.E = s.E;
    q1.K = static_cast<int>(s.d);
    q1.n_blocks = static_cast<int>((s.f + 63) / 64);
    q1.N_out = static_cast<int>(s.f);
    q1.out = static_cast<__nv_bfloat16*>(h);
    q1.status = status;
    q1.wait_ns = wait_ns;
    err = launch_tokn<MODE_SWIGLU>(tx, tg64, tu64, q1, tok_blocks_bound * q1.n_blocks, st);
    if (err != cudaSuccess) return err;
    TcParams q2 = q1;
    q2.K = static_cast<int>(s.f);
    q2.n_blocks = static_cast<int>((s.d + 127) / 128);
    q2.N_out = static_cast<int>(s.d);
    q2.out = static_cast<__nv_bfloat16*>(y);
    return launch_tokn<MODE_DOWN>(th, td128, td128, q2, tok_blocks_bound * q2.n_blocks, st);
  }

  if (a_rows == nullptr && comb == nullptr && kind == MOE_FFN_CTA_PAIRS) {
    // the CTA-pair kernel: B maps with 128-row boxes (each CTA loads half of the 256 rows)
    CUtensorMap td128;
    if (!make_map_weights(&td128, wd, s.E, s.d, s.f, 128)) {
      *why = "tensor map encoding failed (pointer alignment or sizes)";
      return cudaErrorInvalidValue;
    }
    const int64_t pair_blocks_bound = (s.max_rows + PBM - 1) / PBM + s.E;
    TcParams q1 = {};
    q1.seg_start = offsets;
    q1.seg_count = kept;
    q1.E = s.E;
    q1.K = static_cast<int>(s.d);
    q1.n_blocks = static_cast<int>((s.f + 127) / 128);
    q1.N_out = static_cast<int>(s.f);
    q1.out = static_cast<__nv_bfloat16*>(h);
    q1.status = status;
    q1.wait_ns = wait_ns;
    bool launched = false;
    err = launch_pair<MODE_SWIGLU>(ta1, tg, tu, q1, pair_blocks_bound * q1.n_blocks, st, &launched);
    if (err != cudaSuccess) return err;
    if (launched) {
      TcParams q2 = q1;
      q2.K = static_cast<int>(s.f);
      q2.n_blocks = static_cast<int>((s.d + 255) / 256);
      q2.N_out = static_cast<int>(s.d);
      q2.out = static_cast<__nv_bfloat16*>(y);
      err = launch_pair<MODE_DOWN>(ta2, td128, td128, q2, pair_blocks_bound * q2.n_blocks, st,
                                   &launched);
      if (err != cudaSuccess) return err;
      if (!launched) {
        *why = "the down launch found no room for a cluster of two";
        return cudaErrorLaunchOutOfResources;
      }
      return cudaSuccess;
    }
    // no cluster of two fits: the single-CTA kernel below
  }

  TcParams p1 = {};
  p1.seg_start = offsets;
  p1.seg_count = kept;
  p1.E = s.E;
  p1.K = static_cast<int>(s.d);
  p1.n_blocks = static_cast<int>((s.f + 127) / 128);
  p1.N_out = static_cast<int>(s.f);
  p1.out = static_cast<__nv_bfloat16*>(h);
  p1.status = status;
  p1.wait_ns = wait_ns;
  p1.a_rows = a_rows;
  p1.a_rows_limit = static_cast<int32_t>(s.T);
  p1.a_src = a;
  int64_t g1 = row_blocks_bound * p1.n_blocks;
  if (g1 > sms) g1 = sms;
  grouped_gemm_tc_kernel<MODE_SWIGLU><<<static_cast<unsigned>(g1), THREADS, DYN_SMEM, st>>>(
      ta1, tg, tu, ty, p1);
  note_launch();
  if ((err = cudaGetLastError()) != cudaSuccess) return err;

  TcParams p2 = p1;
  p2.a_rows = nullptr;
  p2.K = static_cast<int>(s.f);
  p2.n_blocks = static_cast<int>((s.d + 255) / 256);
  p2.N_out = static_cast<int>(s.d);
  p2.out = static_cast<__nv_bfloat16*>(y);
  if (comb != nullptr) {
    const int64_t vec_per_row = s.d * 2 / 16;
    const int64_t n_counters = s.T * p2.n_blocks;
    int64_t pb = (s.T * 32 + 255) / 256;  // a warp per token
    if (pb > static_cast<int64_t>(sms) * 4) pb = static_cast<int64_t>(sms) * 4;
    if (pb < 1) pb = 1;
    combine_prep_kernel<<<static_cast<unsigned>(pb), 256, 0, st>>>(
        comb->arrive, n_counters, comb->assign_row, s.T, s.k, static_cast<uint4*>(comb->out),
        vec_per_row);
    note_launch();
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    p2.row_token = comb->token_of_row;
    p2.assign_row = comb->assign_row;
    p2.topk_w = comb->topk_w;
    p2.arrive = comb->arrive;
    p2.comb_out = static_cast<__nv_bfloat16*>(comb->out);
    p2.k = s.k;
    p2.T = static_cast<int32_t>(s.T);
  }
  int64_t g2 = row_blocks_bound * p2.n_blocks;
  if (g2 > sms) g2 = sms;
  grouped_gemm_tc_kernel<MODE_DOWN><<<static_cast<unsigned>(g2), THREADS, DYN_SMEM, st>>>(
      ta2, td, td, ty, p2);
  note_launch();
  return cudaGetLastError();
}

bool router_uses_tensor_cores(const Shape& s) { return router_split_applies(s); }

// With fewer 128-token tiles than half the SMs, each tile's K steps are split over several
// blocks (at least 4 K steps, an even number, per piece; at most 16 pieces), whose fp32 sums
// the top-k kernel adds in piece order.  1: no split.
int router_tc_splits(const Shape& s, int* kb_per_split) {
  const int tiles = static_cast<int>((s.T + BM - 1) / BM);
  const int KB = static_cast<int>(2 * s.d / BK);
  *kb_per_split = KB;
  if (2 * tiles >= sm_count()) return 1;
  int ks = sm_count() / tiles;
  if (ks > KB / 4) ks = KB / 4;
  if (ks > 16) ks = 16;
  if (ks < 2) return 1;
  int per = (KB + ks - 1) / ks;
  per += per & 1;
  *kb_per_split = per;
  return (KB + per - 1) / per;
}

bool router_split_applies(const Shape& s) {
  return s.dtype == MOE_BF16 && s.E > 32 && s.d % 64 == 0;
}

size_t router_split_bytes(const Shape& s) {
  if (!router_split_applies(s)) return 0;
  return 2 * static_cast<size_t>(s.E) * s.d * sizeof(__nv_bfloat16);
}

size_t router_tc_workspace_bytes(const Shape& s) {
  return router_uses_tensor_cores(s) ? router_split_bytes(s) : 0;
}

cudaError_t launch_router_split(const Shape& s, const float* w_router, void* w_split,
                                cudaStream_t st) {
  dim3 sgrid((s.E + 31) / 32, static_cast<unsigned>((s.d + 31) / 32));
  split_router_weight_kernel<<<sgrid, 256, 0, st>>>(w_router, static_cast<int>(s.d), s.E,
                                                    static_cast<__nv_bfloat16*>(w_split));
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_router_tc(const Shape& s, const void* x, const float* w_router,
                             const void* w_split, const float* bias, int64_t bias_stride,
                             float* logits, float* logits_scratch, int32_t* topk_idx,
                             float* topk_w, void* split_ws, float* partials, DevStatus* status,
                             uint64_t wait_ns, cudaStream_t st, const char** why) {
  if (encode_fn() == nullptr) {
    *why = "cuTensorMapEncodeTiled is not available from the driver";
    return cudaErrorNotSupported;
  }
  cudaError_t err;
  if (w_split == nullptr) {  // split W_r into the workspace for this call
    if ((err = launch_router_split(s, w_router, split_ws, st)) != cudaSuccess) return err;
    w_split = split_ws;
  }
  // all E <= 256 experts in one 256-column accumulator: K = 2 d (hi half, then lo half)
  CUtensorMap ta, tw;
  if (!make_map_rows(&ta, x, s.T, s.d) || !make_map_weights(&tw, w_split, 1, s.E, 2 * s.d, 256)) {
    *why = "tensor map encoding failed for the router";
    return cudaErrorInvalidValue;
  }
  err = cudaFuncSetAttribute(grouped_gemm_tc_kernel<MODE_ROUTER>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, DYN_SMEM);
  if (err != cudaSuccess) return err;
  const bool sel_only = s.bias_mode == MOE_BIAS_SELECTION_ONLY;
  int kb_per_split = 0;
  const int ksplit = router_tc_splits(s, &kb_per_split);
  // the top-k rides in the epilogue unless the picks are limited to groups or K is split
  const bool fuse = s.n_groups <= 1 && ksplit == 1;
  TcParams p = {};
  p.router_rows = static_cast<int32_t>(s.T);
  p.E = 1;
  p.K = static_cast<int>(2 * s.d);
  p.a_k = static_cast<int>(s.d);
  p.n_blocks = 1;
  p.N_out = s.E;
  p.mb_outer = 1;
  // z always lands somewhere: in the caller's buffer, or in the workspace copy that the
  // dispatch of score-priority drops and moe_layer_forward read when the caller has none
  p.out_f32 = logits != nullptr ? logits : logits_scratch;
  // logits carry the bias unless it is for selection only (then only the keys add it)
  p.bias = sel_only ? nullptr : bias;
  p.sel_bias = sel_only ? bias : nullptr;
  p.bias_stride = bias_stride;
  p.fuse_topk = fuse ? 1 : 0;
  p.k = s.k;
  p.gating = s.gating;
  p.route_idx = topk_idx;
  p.route_w = topk_w;
  p.status = status;
  p.wait_ns = wait_ns;
  int64_t g = (s.T + BM - 1) / BM;
  if (ksplit > 1) {  // the pieces' sums go to the partials; bias and top-k come after
    p.ksplit = ksplit;
    p.kb_per_split = kb_per_split;
    p.out_f32 = partials;
    p.bias = nullptr;
    p.sel_bias = nullptr;
    g *= ksplit;
  }
  if (g > sm_count()) g = sm_count();
  grouped_gemm_tc_kernel<MODE_ROUTER><<<static_cast<unsigned>(g), ROUTER_THREADS, DYN_SMEM, st>>>(
      ta, tw, tw, tw, p);
  note_launch();
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  if (fuse) return cudaSuccess;
  if (ksplit > 1)
    return launch_topk_from_partials(s, partials, ksplit, bias, bias_stride,
                                     logits != nullptr ? logits : logits_scratch, topk_idx,
                                     topk_w, st);
  return launch_topk_from_logits(s, p.out_f32, bias, bias_stride, topk_idx, topk_w, st);
}

}  // namespace moe
