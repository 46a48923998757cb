// Combine on one GPU: the inverse permutation with the gate-weighted sum.
//
// "Expert Parallelism for MoE Serving" (aiunderstanding.org), "Deep dive": after the FFN
// the results are shuffled back to their tokens; "MoE expert parallelism needs
// measurements before launch" (airouter.kz), "Profile all-to-all separately from
// compute": combine and unpack close the layer.  With the experts local (EP=1) this is
//   out[t, :] = sum_{j = 0..k-1, assign_row[t, j] >= 0} topk_w[t, j] * y_perm[assign_row[t, j], :]
// A thread produces 16 bytes of one output row (8 bf16 or 4 fp32 values), reads the k
// source rows' matching 16 bytes and accumulates in fp32 in pick order -- one fixed
// order, no atomics, so the result is bitwise reproducible.  Dropped picks contribute
// nothing and the remaining weights are used as they are.
#include "moe_internal.h"

namespace moe {
namespace {

template <bool BF16>
__global__ void __launch_bounds__(256) combine_kernel(const uint4* __restrict__ y_perm,
                                                      const int32_t* __restrict__ assign_row,
                                                      const float* __restrict__ topk_w,
                                                      int64_t T, int k, int64_t vec_per_row,
                                                      uint4* __restrict__ out) {
  constexpr int NV = BF16 ? 8 : 4;  // values per 16-byte vector
  const int64_t total = T * vec_per_row;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / vec_per_row;
    const int64_t v = i - t * vec_per_row;
    float acc[NV];
#pragma unroll
    for (int q = 0; q < NV; ++q) acc[q] = 0.f;
    for (int j = 0; j < k; ++j) {
      const int32_t r = __ldg(assign_row + t * k + j);
      if (r < 0) continue;
      const float w = __ldg(topk_w + t * k + j);
      const uint4 src = __ldg(y_perm + static_cast<int64_t>(r) * vec_per_row + v);
      const uint32_t u[4] = {src.x, src.y, src.z, src.w};
      if (BF16) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          acc[2 * q] = fmaf(w, bf16_lo(u[q]), acc[2 * q]);
          acc[2 * q + 1] = fmaf(w, bf16_hi(u[q]), acc[2 * q + 1]);
        }
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[q] = fmaf(w, __uint_as_float(u[q]), acc[q]);
      }
    }
    uint4 o;
    if (BF16) {
      o = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                     pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
    } else {
      o = make_uint4(__float_as_uint(acc[0]), __float_as_uint(acc[1]), __float_as_uint(acc[2]),
                     __float_as_uint(acc[3]));
    }
    out[i] = o;
  }
}

}  // namespace

cudaError_t launch_combine(const Shape& s, const void* y_perm, const int32_t* assign_row,
                           const float* topk_w, void* out, cudaStream_t st) {
  const int64_t vec_per_row = s.d * s.elem / 16;
  const int64_t total = s.T * vec_per_row;
  int64_t blocks = (total + 255) / 256;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  if (s.dtype == MOE_BF16)
    combine_kernel<true><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        static_cast<const uint4*>(y_perm), assign_row, topk_w, s.T, s.k, vec_per_row,
        static_cast<uint4*>(out));
  else
    combine_kernel<false><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        static_cast<const uint4*>(y_perm), assign_row, topk_w, s.T, s.k, vec_per_row,
        static_cast<uint4*>(out));
  return cudaGetLastError();
}

}  // namespace moe
