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

// A thread owns NV 16-byte vectors of one output row (NV = 4 when the row allows it): its
// k x NV source loads are independent and issued together before the pick-ordered sums.
template <bool BF16, int NV>
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
    float acc[NV][NE];
#pragma unroll
    for (int u = 0; u < NV; ++u)
#pragma unroll
      for (int q = 0; q < NE; ++q) acc[u][q] = 0.f;
    for (int j = 0; j < k; ++j) {
      const int32_t r = __ldg(assign_row + t * k + j);
      if (r < 0) continue;
      const float w = __ldg(topk_w + t * k + j);
      uint4 src[NV];
#pragma unroll
      for (int u = 0; u < NV; ++u) src[u] = __ldg(y_perm + static_cast<int64_t>(r) * vec_per_row + v0 + u);
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

template <bool BF16>
cudaError_t launch_combine_typed(const Shape& s, const void* y_perm, const int32_t* assign_row,
                                 const float* topk_w, void* out, cudaStream_t st) {
  const int64_t vec_per_row = s.d * s.elem / 16;
  const bool wide = vec_per_row % 4 == 0;
  const int64_t total = s.T * (wide ? vec_per_row / 4 : vec_per_row);
  int64_t blocks = (total + 255) / 256;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  const uint4* y = static_cast<const uint4*>(y_perm);
  uint4* o = static_cast<uint4*>(out);
  if (wide)
    combine_kernel<BF16, 4><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        y, assign_row, topk_w, s.T, s.k, vec_per_row, o);
  else
    combine_kernel<BF16, 1><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        y, assign_row, topk_w, s.T, s.k, vec_per_row, o);
  note_launch();
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_combine(const Shape& s, const void* y_perm, const int32_t* assign_row,
                           const float* topk_w, void* out, cudaStream_t st) {
  if (s.dtype == MOE_BF16)
    return launch_combine_typed<true>(s, y_perm, assign_row, topk_w, out, st);
  return launch_combine_typed<false>(s, y_perm, assign_row, topk_w, out, st);
}

}  // namespace moe
