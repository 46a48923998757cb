// Combine on one GPU: the inverse permutation with the gate-weighted sum.
//
// "Expert Parallelism for MoE Serving" (aiunderstanding.org), "Deep dive": after the FFN
// the results are shuffled back to their tokens; "MoE expert parallelism needs
// measurements before launch" (airouter.kz), "Profile all-to-all separately from
// compute": combine and unpack close the layer.  With the experts local (EP=1) this is
//   out[t, :] = sum_{j = 0..k-1, assign_row[t, j] >= 0} topk_w[t, j] * y_perm[assign_row[t, j], :]
// A thread produces 16-byte pieces of one output row (8 bf16 or 4 fp32 values each), reads
// the k source rows' matching bytes and accumulates in fp32 in pick order -- one fixed
// order, no atomics, so the result is bitwise reproducible.  Dropped picks contribute
// nothing and the remaining weights are used as they are.
#include "moe_internal.h"

namespace moe {
namespace {

// A thread owns NV 16-byte vectors of one output row.  It first reads the token's k rows and
// weights, then issues all k x NV source loads at once (KMAX x NV <= 8 uint4 in flight per
// thread), and only then adds them up in pick order.  Up to 16 blocks per SM, grid-stride.
template <bool BF16, int KMAX, int NV>
__global__ void __launch_bounds__(256) combine_kernel(const uint4* __restrict__ y_perm,
                                                      const int32_t* __restrict__ assign_row,
                                                      const float* __restrict__ topk_w,
                                                      int64_t T, int k, int64_t vec_per_row,
                                                      uint4* __restrict__ out) {
  constexpr int NE = BF16 ? 8 : 4;  // values per 16-byte vector
  const int64_t groups_per_row = vec_per_row / NV;
  const int64_t total = T * groups_per_row;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / groups_per_row;
    const int64_t v0 = (i - t * groups_per_row) * NV;
    int32_t rows[KMAX];
    float ws[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      rows[j] = -1;
      ws[j] = 0.f;
      if (j < k) {
        rows[j] = __ldg(assign_row + t * k + j);
        ws[j] = __ldg(topk_w + t * k + j);
      }
    }
    uint4 src[KMAX][NV];
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
#pragma unroll
      for (int u = 0; u < NV; ++u)
        src[j][u] = rows[j] >= 0
                        ? __ldg(y_perm + static_cast<int64_t>(rows[j]) * vec_per_row + v0 + u)
                        : make_uint4(0u, 0u, 0u, 0u);
    float acc[NV][NE];
#pragma unroll
    for (int u = 0; u < NV; ++u)
#pragma unroll
      for (int q = 0; q < NE; ++q) acc[u][q] = 0.f;
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      if (rows[j] < 0) continue;  // dropped picks (and j >= k) contribute nothing
      const float w = ws[j];
#pragma unroll
      for (int u = 0; u < NV; ++u) {
        const uint32_t uu[4] = {src[j][u].x, src[j][u].y, src[j][u].z, src[j][u].w};
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

template <bool BF16, int KMAX, int NV>
cudaError_t launch_combine_shaped(const Shape& s, const uint4* y, const int32_t* assign_row,
                                  const float* topk_w, uint4* o, cudaStream_t st) {
  const int64_t vec_per_row = s.d * s.elem / 16;
  const int64_t total = s.T * (vec_per_row / NV);
  int64_t blocks = (total + 255) / 256;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 16;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  combine_kernel<BF16, KMAX, NV><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
      y, assign_row, topk_w, s.T, s.k, vec_per_row, o);
  note_launch();
  return cudaGetLastError();
}

// KMAX = k rounded up to 2, 4 or 8; NV vectors per thread when the row allows it: 2 for
// KMAX = 2 (4 loads in flight; measured faster on 4096 tokens than 4 vectors with half the
// threads), 8 / KMAX otherwise
template <bool BF16, int KMAX>
cudaError_t launch_combine_k(const Shape& s, const uint4* y, const int32_t* assign_row,
                             const float* topk_w, uint4* o, cudaStream_t st) {
  constexpr int NV = KMAX == 2 ? 2 : 8 / KMAX;
  const int64_t vec_per_row = s.d * s.elem / 16;
  if (NV > 1 && vec_per_row % NV == 0)
    return launch_combine_shaped<BF16, KMAX, NV>(s, y, assign_row, topk_w, o, st);
  return launch_combine_shaped<BF16, KMAX, 1>(s, y, assign_row, topk_w, o, st);
}

template <bool BF16>
cudaError_t launch_combine_typed(const Shape& s, const void* y_perm, const int32_t* assign_row,
                                 const float* topk_w, void* out, cudaStream_t st) {
  const uint4* y = static_cast<const uint4*>(y_perm);
  uint4* o = static_cast<uint4*>(out);
  if (s.k <= 2) return launch_combine_k<BF16, 2>(s, y, assign_row, topk_w, o, st);
  if (s.k <= 4) return launch_combine_k<BF16, 4>(s, y, assign_row, topk_w, o, st);
  return launch_combine_k<BF16, 8>(s, y, assign_row, topk_w, o, st);
}

}  // namespace

cudaError_t launch_combine(const Shape& s, const void* y_perm, const int32_t* assign_row,
                           const float* topk_w, void* out, cudaStream_t st) {
  if (s.dtype == MOE_BF16)
    return launch_combine_typed<true>(s, y_perm, assign_row, topk_w, out, st);
  return launch_combine_typed<false>(s, y_perm, assign_row, topk_w, out, st);
}

}  // namespace moe
