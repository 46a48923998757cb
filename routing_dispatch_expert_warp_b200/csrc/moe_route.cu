// Router scoring, top-k selection and renormalised gate weights.
//
// "Expert Parallelism for MoE Serving" (aiunderstanding.org), "Deep dive": a router
// scores the experts for every token and picks the top-k of them.  Here:
//   z[t, e]  = sum_i x[t, i] * W_r[i, e] + b[t, e]        (fp32 FMA, fixed order)
//   picks    = the k largest z[t, :], best first; equal z -> lower expert index
//   weights  = softmax or sigmoid of the picked logits, renormalised over the k picks.
//
// Two kernels:
//   * E <= 32: one fused kernel.  A warp scores 32/ET tokens at once (ET = 8, 16 or 32
//     expert slots), every lane walking a strided slice of d with 16-byte loads of x; a
//     transposing butterfly reduction leaves lane l with the logit of (token l / ET,
//     expert l % ET); each group of ET lanes then selects its token's top-k with
//     shuffles.  The pass is bound by reading x once from HBM.
//   * E > 32: a tiled fp32 GEMM writes z (64 tokens x 128 experts per block), then a warp
//     per token selects the top-k from z.
#include <math.h>

#include <type_traits>

#include "moe_internal.h"
#include "moe_keys.cuh"

namespace moe {
namespace {

template <typename TX>
struct XLoad;
template <>
struct XLoad<float> {
  // 8 consecutive fp32 values (two 16-byte loads)
  static __device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
};
template <>
struct XLoad<__nv_bfloat16> {
  // 8 consecutive bf16 values (one 16-byte load), widened exactly to fp32
  static __device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&v)[8]) {
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
    v[0] = bf16_lo(a.x); v[1] = bf16_hi(a.x); v[2] = bf16_lo(a.y); v[3] = bf16_hi(a.y);
    v[4] = bf16_lo(a.z); v[5] = bf16_hi(a.z); v[6] = bf16_lo(a.w); v[7] = bf16_hi(a.w);
  }
};

// (valid, value, index) ordering of the top-k: larger value first, then lower index.
__device__ __forceinline__ bool better(bool va, float a, int ia, bool vb, float b, int ib) {
  if (va != vb) return va;
  if (a != b) return a > b;
  return ia < ib;
}

// One block scores TW = 32 / ET tokens.  The d axis is cut into 256-element chunks dealt
// round-robin to the 8 warps.  Inside a chunk, lane l owns the element pairs
// (64 q + 2 l, 64 q + 2 l + 1), q = 0..3: the warp's loads of x are 128 contiguous bytes per
// token and q, and its loads of the matching W_r rows are contiguous too (lane l reads rows
// 2l and 2l+1), so both streams are coalesced.  Each warp folds its 32 partial values (TW
// tokens x ET experts) with a butterfly transpose-reduction, the 8 warp partials are added
// in warp order through shared memory, and warp 0 finishes: bias, logits, top-k and gate
// weights.
// 8 consecutive elements of x kept in their storage form until used (4 registers for bf16).
template <typename TX>
struct XRaw;
template <>
struct XRaw<__nv_bfloat16> {
  uint4 v;
  __device__ __forceinline__ void load(const __nv_bfloat16* p) {
    v = __ldg(reinterpret_cast<const uint4*>(p));
  }
  __device__ __forceinline__ void zero() { v = make_uint4(0u, 0u, 0u, 0u); }
  template <int I>
  __device__ __forceinline__ float get() const {
    const uint32_t w = I < 2 ? v.x : (I < 4 ? v.y : (I < 6 ? v.z : v.w));
    return (I & 1) ? bf16_hi(w) : bf16_lo(w);
  }
};
template <>
struct XRaw<float> {
  float4 a, b;
  __device__ __forceinline__ void load(const float* p) {
    a = __ldg(reinterpret_cast<const float4*>(p));
    b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  }
  __device__ __forceinline__ void zero() { a = b = make_float4(0.f, 0.f, 0.f, 0.f); }
  template <int I>
  __device__ __forceinline__ float get() const {
    const float4& q = I < 4 ? a : b;
    constexpr int J = I & 3;
    return J == 0 ? q.x : (J == 1 ? q.y : (J == 2 ? q.z : q.w));
  }
};

template <int RR, typename TX, int ET, int TW, int CPW>
__device__ __forceinline__ void router_row_fma(const XRaw<TX> (&xr)[CPW][TW], int j,
                                               const float (&wv)[ET], float (&v)[32]) {
#pragma unroll
  for (int tw = 0; tw < TW; ++tw) {
    const float xval = xr[j][tw].template get<RR>();
#pragma unroll
    for (int e = 0; e < ET; ++e) v[tw * ET + e] = fmaf(xval, wv[e], v[tw * ET + e]);
  }
}

// W_r [d, E] re-laid out for the warp access pattern of the small-E router: in chunk c
// (256 rows of d) lane l owns rows c*256 + 8l .. 8l+7; vector u = rr * (ET/4) + qq holds
// row 8l + rr, experts 4qq .. 4qq+3, and the 32 lanes' vectors u are consecutive (512 B),
// so every W load of the router is one fully used 512-byte span.  Experts past E and rows
// past d are zero.
template <int ET>
__global__ void __launch_bounds__(256) router_weight_lanes_kernel(const float* __restrict__ w,
                                                                  int d, int E,
                                                                  float4* __restrict__ wl) {
  constexpr int U = 8 * ET / 4;
  const int nchunks = (d + 255) / 256;
  const int64_t total = static_cast<int64_t>(nchunks) * U * 32;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int lane = static_cast<int>(i % 32);
    const int u = static_cast<int>((i / 32) % U);
    const int64_t c = i / (32 * U);
    const int rr = u / (ET / 4), qq = u % (ET / 4);
    const int64_t row = c * 256 + 8 * lane + rr;
    const int e0 = qq * 4;
    float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
    if (row < d) {
      const float* src = w + row * E;
      f.x = e0 + 0 < E ? src[e0 + 0] : 0.f;
      f.y = e0 + 1 < E ? src[e0 + 1] : 0.f;
      f.z = e0 + 2 < E ? src[e0 + 2] : 0.f;
      f.w = e0 + 3 < E ? src[e0 + 3] : 0.f;
    }
    wl[i] = f;
  }
}

// Lane l of a warp holds the logit z of (token t0 + l / ET, expert l % ET): add the bias,
// write the logits, pick the top-k of each token (one ET-lane group per token) and write
// the picks and gate weights.
template <int ET>
__device__ __forceinline__ void finish_small_e(float z, int lane, int64_t t0, int64_t T, int E,
                                               int k, int gating, int bias_mode,
                                               const float* __restrict__ bias,
                                               int64_t bias_stride, float* __restrict__ logits,
                                               int32_t* __restrict__ topk_idx,
                                               float* __restrict__ topk_w) {
  const int tw = lane / ET;
  const int e = lane % ET;
  const int64_t t = t0 + tw;
  const bool valid = (e < E) && (t < T);
  float key = z;  // selection score
  if (valid) {
    if (bias != nullptr) {
      const float b = bias[t * bias_stride + e];
      if (bias_mode == MOE_BIAS_SELECTION_ONLY) {
        key = z + b;
      } else {
        z += b;
        key = z;
      }
    }
    if (logits != nullptr) logits[t * E + e] = z;
  }
  // top-k within each group of ET lanes (one token per group); lane j of the group keeps
  // the j-th pick (k <= E <= ET)
  bool taken = false;
  float my_z = 0.f;
  int my_i = 0;
  for (int j = 0; j < k; ++j) {
    bool bv = valid && !taken;
    float bk = key, bz = z;
    int bi = e;
#pragma unroll
    for (int off = ET / 2; off >= 1; off >>= 1) {
      const bool ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const float ok = __shfl_xor_sync(0xffffffffu, bk, off);
      const float oz = __shfl_xor_sync(0xffffffffu, bz, off);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
      if (better(ov, ok, oi, bv, bk, bi)) {
        bv = ov; bk = ok; bz = oz; bi = oi;
      }
    }
    if (bi == e) taken = true;
    if (e == j) {
      my_z = bz;
      my_i = bi;
    }
  }
  // gate weights over the group's k picks; the normaliser is summed in pick order
  const int base = lane - e;
  float wgt;
  if (gating == MOE_GATE_SOFTMAX) {
    float m = __shfl_sync(0xffffffffu, my_z, base);
    for (int j = 1; j < k; ++j) m = fmaxf(m, __shfl_sync(0xffffffffu, my_z, base + j));
    wgt = expf(my_z - m);
  } else {
    wgt = 1.0f / (1.0f + expf(-my_z));
  }
  float ssum = 0.f;
  for (int j = 0; j < k; ++j) ssum += __shfl_sync(0xffffffffu, wgt, base + j);
  if (e < k && t < T) {
    topk_idx[t * k + e] = my_i;
    topk_w[t * k + e] = wgt * (1.0f / ssum);
  }
}

// One block scores TW = 32 / ET tokens.  The d axis is cut into 256-element chunks dealt
// round-robin to the 8 warps; in a chunk lane l owns 8 consecutive elements (one 16-byte
// load of x per token).  A warp first issues the x loads of up to CPW chunks at once, then
// walks the lane-ordered W rows.  Each warp folds its 32 partial values (TW tokens x ET
// experts) with a butterfly transpose-reduction, the 8 warp partials are added in warp
// order through shared memory, and warp 0 finishes: bias, logits, top-k and gate weights.
template <typename TX, int ET>
__global__ void __launch_bounds__(256, ET == 8 ? 2 : 3) router_small_e_kernel(
    const TX* __restrict__ x, const float4* __restrict__ wl, const float* __restrict__ bias,
    int64_t bias_stride, int64_t T, int d, int E, int k, int gating, int bias_mode,
    float* __restrict__ logits, int32_t* __restrict__ topk_idx, float* __restrict__ topk_w) {
  constexpr int TW = 32 / ET;  // tokens per block
  constexpr int NW = 8;        // warps per block
  constexpr int CPW = sizeof(TX) == 2 ? 2 : 1;  // chunks whose x loads are in flight together
  constexpr int U = 8 * ET / 4;
  __shared__ float part[NW][32];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int nchunks = (d + 255) / 256;

  for (int64_t t0 = static_cast<int64_t>(blockIdx.x) * TW; t0 < T;
       t0 += static_cast<int64_t>(gridDim.x) * TW) {
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = 0.f;

    for (int cb = warp; cb < nchunks; cb += NW * CPW) {
      XRaw<TX> xr[CPW][TW];
#pragma unroll
      for (int j = 0; j < CPW; ++j) {
        const int i0 = (cb + NW * j) * 256 + lane * 8;
#pragma unroll
        for (int tw = 0; tw < TW; ++tw) {
          if (i0 < d && t0 + tw < T) xr[j][tw].load(x + (t0 + tw) * d + i0);
          else xr[j][tw].zero();
        }
      }
#pragma unroll
      for (int j = 0; j < CPW; ++j) {
        const int c = cb + NW * j;
        if (c >= nchunks) continue;
        const float4* wq = wl + static_cast<int64_t>(c) * U * 32 + lane;
        auto row = [&](auto rr_const) {
          constexpr int RR = decltype(rr_const)::value;
          float wv[ET];
#pragma unroll
          for (int qq = 0; qq < ET / 4; ++qq) {
            const float4 f = __ldg(wq + (RR * (ET / 4) + qq) * 32);
            wv[4 * qq] = f.x; wv[4 * qq + 1] = f.y; wv[4 * qq + 2] = f.z; wv[4 * qq + 3] = f.w;
          }
          router_row_fma<RR, TX, ET, TW, CPW>(xr, j, wv, v);
        };
        row(std::integral_constant<int, 0>{});
        row(std::integral_constant<int, 1>{});
        row(std::integral_constant<int, 2>{});
        row(std::integral_constant<int, 3>{});
        row(std::integral_constant<int, 4>{});
        row(std::integral_constant<int, 5>{});
        row(std::integral_constant<int, 6>{});
        row(std::integral_constant<int, 7>{});
      }
    }

    // Butterfly transpose-reduction: afterwards lane l holds the warp's sum of value l.
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
      const bool upper = (lane & off) != 0;
#pragma unroll
      for (int i = 0; i < off; ++i) {
        const float send = upper ? v[i] : v[i + off];
        const float keep = upper ? v[i + off] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
      }
    }
    part[warp][lane] = v[0];
    __syncthreads();

    if (warp == 0) {
      float z = part[0][lane];
#pragma unroll
      for (int w = 1; w < NW; ++w) z += part[w][lane];
      finish_small_e<ET>(z, lane, t0, T, E, k, gating, bias_mode, bias, bias_stride, logits,
                         topk_idx, topk_w);
    }
    __syncthreads();
  }
}

// z = x W_r + b as a tiled fp32 GEMM: 64 tokens x 128 experts per block, K steps of 32.
constexpr int RT_M = 64, RT_N = 128, RT_K = 32;

// With gridDim.z = S > 1 the K range is split in S contiguous pieces and block z writes its
// partial sums to z + blockIdx.z * T * E (bias left out); the top-k kernel adds the S
// partials in order, so the result does not depend on scheduling.
template <typename TX>
__global__ void __launch_bounds__(256) router_gemm_kernel(
    const TX* __restrict__ x, const float* __restrict__ w_router, const float* __restrict__ bias,
    int64_t bias_stride, int64_t T, int d, int E, int k_per_split, float* __restrict__ z) {
  __shared__ __align__(16) float xs[RT_K][RT_M];
  __shared__ __align__(16) float ws[RT_K][RT_N];
  const int tid = threadIdx.x;
  const int ty = tid / 16, tx = tid % 16;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * RT_M;
  const int n0 = blockIdx.x * RT_N;
  float acc[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  const int kbeg = blockIdx.z * k_per_split;
  const int kend = kbeg + k_per_split < d ? kbeg + k_per_split : d;
  if (gridDim.z > 1) {
    z += static_cast<int64_t>(blockIdx.z) * T * E;
    bias = nullptr;
  }
  for (int k0 = kbeg; k0 < kend; k0 += RT_K) {
    {  // x tile: 64 rows x 32 columns, 8 consecutive elements per thread, stored transposed
      const int r = tid / 4, c = (tid % 4) * 8;
      float v[8];
      const int64_t t = m0 + r;
      if (t < T && k0 + c + 8 <= kend) {
        XLoad<TX>::load8(x + t * d + k0 + c, v);
      } else {
#pragma unroll
        for (int q = 0; q < 8; ++q)
          v[q] = (t < T && k0 + c + q < kend) ? static_cast<float>(x[t * d + k0 + c + q]) : 0.f;
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) xs[c + q][r] = v[q];
    }
    {  // W tile: 32 rows x 128 experts
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int r = tid / 32 + 8 * q, c = (tid % 32) * 4;
        const int kk = k0 + r;
        float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
        if (kk < kend) {
          const float* src = w_router + static_cast<int64_t>(kk) * E + n0 + c;
          if (n0 + c + 4 <= E && (E % 4) == 0) {
            f = __ldg(reinterpret_cast<const float4*>(src));
          } else {
            f.x = n0 + c + 0 < E ? src[0] : 0.f;
            f.y = n0 + c + 1 < E ? src[1] : 0.f;
            f.z = n0 + c + 2 < E ? src[2] : 0.f;
            f.w = n0 + c + 3 < E ? src[3] : 0.f;
          }
        }
        *reinterpret_cast<float4*>(&ws[r][c]) = f;
      }
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < RT_K; ++kk) {
      const float4 a = *reinterpret_cast<const float4*>(&xs[kk][4 * ty]);
      const float4 b0 = *reinterpret_cast<const float4*>(&ws[kk][4 * tx]);
      const float4 b1 = *reinterpret_cast<const float4*>(&ws[kk][64 + 4 * tx]);
      const float av[4] = {a.x, a.y, a.z, a.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t t = m0 + 4 * ty + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = n0 + (j < 4 ? 4 * tx + j : 64 + 4 * tx + (j - 4));
      if (e >= E) continue;
      float zz = acc[i][j];
      if (bias != nullptr) zz += bias[t * bias_stride + e];
      z[t * E + e] = zz;
    }
  }
}


// Warp-wide argmax over keys held as lane + 32 q: the largest key, equal keys -> the lower
// index.  Two warp reductions (max of the keys, then min of the indices holding it).
template <int Q>
__device__ __forceinline__ int warp_argmax(const uint32_t (&key)[Q], int lane) {
  uint32_t m = key[0];
#pragma unroll
  for (int q = 1; q < Q; ++q) m = max(m, key[q]);
  m = __reduce_max_sync(0xffffffffu, m);
  int bi = 0x7fffffff;
#pragma unroll
  for (int q = Q - 1; q >= 0; --q)
    if (key[q] == m) bi = lane + 32 * q;
  return __reduce_min_sync(0xffffffffu, bi);
}

// A warp per token (E <= 256, lane holds experts lane + 32 q).  z holds nsplit partial sums
// per logit (split-K) that are added in split order; `bias_into_z` adds the bias to them
// (logits with bias), `bias_into_key` adds it to the selection score only.  The summed
// logits are written to `logits` when nsplit > 1.  With n_groups > 1, the token first keeps
// its topk_groups best expert groups (group score = best score in the group, equal scores
// -> lower group index).  Every selection round is one warp_argmax over order keys; lane j
// keeps the j-th pick, and lanes 0..k-1 write the token's picks and gate weights.
__global__ void __launch_bounds__(256) topk_from_logits_kernel(
    const float* __restrict__ z, int nsplit, const float* __restrict__ bias, int64_t bias_stride,
    int bias_into_z, int bias_into_key, float* __restrict__ logits, int64_t T, int E, int k,
    int gating, int n_groups, int topk_groups, int32_t* __restrict__ topk_idx,
    float* __restrict__ topk_w) {
  __shared__ uint32_t gkey_s[8][MOE_MAX_EXPERTS];
  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int gsize = n_groups > 1 ? E / n_groups : E;
  for (int64_t t = warp; t < T; t += nwarps) {
    float zv[8];
    uint32_t key[8];
    // the nsplit partial sums of each of the lane's 8 logits, added strictly in split order;
    // the loads of 8 splits x 8 logits are issued together
    float part[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int e = lane + 32 * q;
      part[q] = e < E ? z[t * E + e] : 0.f;
    }
    if (nsplit > 1) {
      const int64_t stride = T * E;
      int sp = 1;
      for (; sp + 8 <= nsplit; sp += 8) {
        float b[8][8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const int e = lane + 32 * q;
            b[u][q] = e < E ? z[(sp + u) * stride + t * E + e] : 0.f;
          }
#pragma unroll
        for (int u = 0; u < 8; ++u)
#pragma unroll
          for (int q = 0; q < 8; ++q) part[q] += b[u][q];
      }
      for (; sp < nsplit; ++sp)
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int e = lane + 32 * q;
          if (e < E) part[q] += z[sp * stride + t * E + e];
        }
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int e = lane + 32 * q;
      float acc = part[q];
      key[q] = 0u;
      if (e < E) {
        if (bias != nullptr && bias_into_z) acc += bias[t * bias_stride + e];
        if (nsplit > 1 && logits != nullptr) logits[t * E + e] = acc;
        key[q] = order_key((bias != nullptr && bias_into_key) ? acc + bias[t * bias_stride + e]
                                                              : acc);
      }
      zv[q] = acc;
    }
    if (n_groups > 1) {
      uint32_t* ks = gkey_s[wib];
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (lane + 32 * q < E) ks[lane + 32 * q] = key[q];
      __syncwarp();
      // group scores (the largest key of each group), lane g + 32 q holds group g + 32 q
      uint32_t gk[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) gk[q] = 0u;
      if (gsize >= 32) {
        for (int g = 0; g < n_groups; ++g) {
          uint32_t m = 0u;
          for (int i = lane; i < gsize; i += 32) m = max(m, ks[g * gsize + i]);
          m = __reduce_max_sync(0xffffffffu, m);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            if (lane + 32 * q == g) gk[q] = m;
        }
      } else {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int g = lane + 32 * q;
          if (g < n_groups) {
            uint32_t m = 0u;
            for (int i = 0; i < gsize; ++i) m = max(m, ks[g * gsize + i]);
            gk[q] = m;
          }
        }
      }
      __syncwarp();
      // keep the topk_groups best groups; flags[g] != 0 marks a kept group
      uint32_t chosen = 0;  // bit q: group lane + 32 q kept
      for (int r = 0; r < topk_groups; ++r) {
        const int bg = warp_argmax(gk, lane);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          if (lane + 32 * q == bg) {
            chosen |= 1u << q;
            gk[q] = 0u;
          }
      }
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (lane + 32 * q < n_groups) ks[lane + 32 * q] = (chosen >> q) & 1u;
      __syncwarp();
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (lane + 32 * q < E && ks[(lane + 32 * q) / gsize] == 0u) key[q] = 0u;
      __syncwarp();
    }
    int mysel = 0;  // lane j < k: the j-th pick
    for (int j = 0; j < k; ++j) {
      const int bi = warp_argmax(key, lane);
      if (lane == j) mysel = bi;
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (lane + 32 * q == bi) key[q] = 0u;
    }
    // the picked logits, from the lanes that hold them
    float myz = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float v = __shfl_sync(0xffffffffu, zv[q], mysel & 31);
      if ((mysel >> 5) == q) myz = v;
    }
    // gate weights over the k picks; the normaliser is summed in pick order
    float w;
    if (gating == MOE_GATE_SOFTMAX) {
      float m = myz;
      for (int j = 1; j < k; ++j) m = fmaxf(m, __shfl_sync(0xffffffffu, myz, j));
      m = __shfl_sync(0xffffffffu, m, 0);
      w = expf(myz - m);
    } else {
      w = 1.0f / (1.0f + expf(-myz));
    }
    float ssum = 0.f;
    for (int j = 0; j < k; ++j) ssum += __shfl_sync(0xffffffffu, w, j);
    if (lane < k) {
      topk_idx[t * k + lane] = mysel;
      topk_w[t * k + lane] = w * (1.0f / ssum);
    }
  }
}

template <typename TX, int ET>
cudaError_t launch_small_e(const Shape& s, const TX* x, const float* w_router, const float* bias,
                           int64_t bias_stride, float* logits, int32_t* topk_idx, float* topk_w,
                           float4* wl, cudaStream_t st) {
  const int d = static_cast<int>(s.d);
  const int64_t lanes_total = static_cast<int64_t>((d + 255) / 256) * (8 * ET / 4) * 32;
  const int pblocks = static_cast<int>((lanes_total + 255) / 256 < 1024 ? (lanes_total + 255) / 256 : 1024);
  router_weight_lanes_kernel<ET><<<pblocks, 256, 0, st>>>(w_router, d, s.E, wl);
  note_launch();
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  constexpr int TW = 32 / ET;
  const int64_t blocks_needed = (s.T + TW - 1) / TW;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 64;
  const int blocks = static_cast<int>(blocks_needed < cap ? blocks_needed : cap);
  router_small_e_kernel<TX, ET><<<blocks, 256, 0, st>>>(x, wl, bias, bias_stride, s.T, d, s.E,
                                                        s.k, s.gating, s.bias_mode, logits,
                                                        topk_idx, topk_w);
  note_launch();
  return cudaGetLastError();
}

template <typename TX>
cudaError_t launch_router_typed(const Shape& s, const TX* x, const float* w_router,
                                const float* bias, int64_t bias_stride, float* logits,
                                int32_t* topk_idx, float* topk_w, float* partials,
                                cudaStream_t st) {
  const int d = static_cast<int>(s.d);
  if (s.E <= 32 && s.n_groups <= 1) {
    float4* wl = reinterpret_cast<float4*>(partials);  // the workspace's router area
    if (s.E <= 8)
      return launch_small_e<TX, 8>(s, x, w_router, bias, bias_stride, logits, topk_idx, topk_w,
                                   wl, st);
    if (s.E <= 16)
      return launch_small_e<TX, 16>(s, x, w_router, bias, bias_stride, logits, topk_idx, topk_w,
                                    wl, st);
    return launch_small_e<TX, 32>(s, x, w_router, bias, bias_stride, logits, topk_idx, topk_w,
                                  wl, st);
  }
  const int tiles_n = (s.E + RT_N - 1) / RT_N;
  const int64_t tiles_m = (s.T + RT_M - 1) / RT_M;
  const int nsplit = router_splits(s);
  int k_per_split = (d + nsplit - 1) / nsplit;
  k_per_split = (k_per_split + RT_K - 1) / RT_K * RT_K;
  dim3 grid(tiles_n, static_cast<unsigned>(tiles_m), nsplit);
  const bool sel_only = s.bias_mode == MOE_BIAS_SELECTION_ONLY;
  // the GEMM adds the bias itself only when it writes finished logits that carry it
  const float* gemm_bias = (nsplit == 1 && !sel_only) ? bias : nullptr;
  router_gemm_kernel<TX><<<grid, 256, 0, st>>>(x, w_router, gemm_bias, bias_stride, s.T, d, s.E,
                                               k_per_split, nsplit > 1 ? partials : logits);
  note_launch();
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const int64_t blocks_needed = (s.T + 7) / 8;
  const int blocks = static_cast<int>(blocks_needed < 148 * 16 ? blocks_needed : 148 * 16);
  topk_from_logits_kernel<<<blocks, 256, 0, st>>>(
      nsplit > 1 ? partials : logits, nsplit, bias, bias_stride,
      (nsplit > 1 && !sel_only) ? 1 : 0, sel_only ? 1 : 0, logits, s.T, s.E, s.k, s.gating,
      s.n_groups, s.topk_groups, topk_idx, topk_w);
  note_launch();
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_topk_from_logits(const Shape& s, const float* logits, const float* bias,
                                    int64_t bias_stride, int32_t* topk_idx, float* topk_w,
                                    cudaStream_t st) {
  const int64_t blocks_needed = (s.T + 7) / 8;
  const int blocks = static_cast<int>(blocks_needed < 148 * 16 ? blocks_needed : 148 * 16);
  const bool sel_only = s.bias_mode == MOE_BIAS_SELECTION_ONLY;
  topk_from_logits_kernel<<<blocks, 256, 0, st>>>(logits, 1, sel_only ? bias : nullptr,
                                                  bias_stride, 0, sel_only ? 1 : 0, nullptr, s.T,
                                                  s.E, s.k, s.gating, s.n_groups, s.topk_groups,
                                                  topk_idx, topk_w);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_topk_from_partials(const Shape& s, const float* partials, int nsplit,
                                      const float* bias, int64_t bias_stride, float* logits,
                                      int32_t* topk_idx, float* topk_w, cudaStream_t st) {
  const int64_t blocks_needed = (s.T + 7) / 8;
  const int blocks = static_cast<int>(blocks_needed < 148 * 16 ? blocks_needed : 148 * 16);
  const bool sel_only = s.bias_mode == MOE_BIAS_SELECTION_ONLY;
  topk_from_logits_kernel<<<blocks, 256, 0, st>>>(
      partials, nsplit, bias, bias_stride, sel_only ? 0 : 1, sel_only ? 1 : 0, logits, s.T, s.E,
      s.k, s.gating, s.n_groups, s.topk_groups, topk_idx, topk_w);
  note_launch();
  return cudaGetLastError();
}

int router_splits(const Shape& s) {
  if (s.E <= 32) return 1;
  const int64_t tiles = ((s.E + RT_N - 1) / RT_N) * ((s.T + RT_M - 1) / RT_M);
  const int64_t target = 296;  // two waves of blocks on a 148-SM part; device-independent
  if (tiles >= target) return 1;
  int64_t sp = (target + tiles - 1) / tiles;
  const int64_t max_sp = (s.d + 4 * RT_K - 1) / (4 * RT_K);  // at least 4 K steps per split
  if (sp > max_sp) sp = max_sp;
  if (sp > kMaxRouterSplits) sp = kMaxRouterSplits;
  return sp < 1 ? 1 : static_cast<int>(sp);
}

cudaError_t launch_router(const Shape& s, const void* x, const float* w_router,
                          const float* bias, int64_t bias_stride, float* logits,
                          int32_t* topk_idx, float* topk_w, float* partials, cudaStream_t st) {
  if (s.dtype == MOE_F32)
    return launch_router_typed(s, static_cast<const float*>(x), w_router, bias, bias_stride,
                               logits, topk_idx, topk_w, partials, st);
  return launch_router_typed(s, static_cast<const __nv_bfloat16*>(x), w_router, bias,
                             bias_stride, logits, topk_idx, topk_w, partials, st);
}

}  // namespace moe
