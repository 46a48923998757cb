// Expert SwiGLU FFN in fp32 (CUDA-core FMA) for fp32 layers.
//
// For each expert e and each row r of its bucket [offsets[e], offsets[e] + kept[e]):
//   h[r] = silu(x_perm[r] . W_g[e]^T) * (x_perm[r] . W_u[e]^T),  y[r] = h[r] . W_d[e]^T,
// where x_perm[r] is either a row of the permuted copy or, gathering, x[token_of_row[r]].
// A 32 x 32 output tile per block, 2 x 2 outputs per thread, K in steps of 32 through
// shared memory; every output is one fp32 FMA chain in K order.  Blocks whose rows lie
// past the expert's count exit at once, so the grid covers the largest possible bucket
// without a host read of the counts.
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int ST = 32;

template <bool GATED>
__global__ void __launch_bounds__(256) ffn_simt_kernel(
    const float* __restrict__ A, const int32_t* __restrict__ a_rows, int64_t a_limit,
    const float* __restrict__ B0, const float* __restrict__ B1, int N, int K,
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ kept,
    float* __restrict__ out) {
  const int e = blockIdx.z;
  const int cnt = kept[e];
  const int m0 = blockIdx.y * ST;
  if (m0 >= cnt) return;
  const int n0 = blockIdx.x * ST;
  const int64_t row0 = static_cast<int64_t>(offsets[e]) + m0;
  const float* b0 = B0 + static_cast<int64_t>(e) * N * K;
  const float* b1 = GATED ? B1 + static_cast<int64_t>(e) * N * K : nullptr;

  __shared__ int64_t arow_s[ST];  // source row of A for each tile row
  __shared__ float As[ST][ST + 1];
  __shared__ float Bs0[ST][ST + 1];
  __shared__ float Bs1[GATED ? ST : 1][ST + 1];
  const int tid = threadIdx.x;
  const int ty = tid / 16, tx = tid % 16;
  float acc0[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
  float acc1[2][2] = {{0.f, 0.f}, {0.f, 0.f}};

  if (tid < ST) {
    int64_t src = row0 + tid;
    if (a_rows != nullptr && m0 + tid < cnt) {
      const int32_t t = a_rows[row0 + tid];
      src = (t >= 0 && t < a_limit) ? t : 0;  // a corrupt index reads row 0, never out of range
    }
    arow_s[tid] = src;
  }
  __syncthreads();
  for (int k0 = 0; k0 < K; k0 += ST) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int idx = tid + 256 * i;
      const int r = idx / ST, c = idx % ST;
      const bool kin = k0 + c < K;
      As[r][c] = (m0 + r < cnt && kin) ? A[arow_s[r] * K + k0 + c] : 0.f;
      Bs0[r][c] = (n0 + r < N && kin) ? b0[static_cast<int64_t>(n0 + r) * K + k0 + c] : 0.f;
      if (GATED)
        Bs1[r][c] = (n0 + r < N && kin) ? b1[static_cast<int64_t>(n0 + r) * K + k0 + c] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < ST; ++kk) {
      const float a[2] = {As[2 * ty][kk], As[2 * ty + 1][kk]};
      const float g[2] = {Bs0[2 * tx][kk], Bs0[2 * tx + 1][kk]};
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 2; ++j) acc0[i][j] = fmaf(a[i], g[j], acc0[i][j]);
      if (GATED) {
        const float u[2] = {Bs1[2 * tx][kk], Bs1[2 * tx + 1][kk]};
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
          for (int j = 0; j < 2; ++j) acc1[i][j] = fmaf(a[i], u[j], acc1[i][j]);
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int r = 2 * ty + i;
    if (m0 + r >= cnt) continue;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int c = n0 + 2 * tx + j;
      if (c >= N) continue;
      float v = acc0[i][j];
      if (GATED) v = v / (1.0f + expf(-v)) * acc1[i][j];
      out[(row0 + r) * N + c] = v;
    }
  }
}

}  // namespace

cudaError_t launch_ffn_simt(const Shape& s, const float* a, const int32_t* a_rows,
                            const int32_t* offsets, const int32_t* kept, const float* wg,
                            const float* wu, const float* wd, float* h, float* y,
                            cudaStream_t st) {
  // a token picks an expert at most once, so no bucket holds more than T rows
  int64_t max_bucket = s.T;
  if (s.C >= 0 && s.C < max_bucket) max_bucket = s.C;
  const unsigned gy = static_cast<unsigned>((max_bucket + ST - 1) / ST);
  const int d = static_cast<int>(s.d), f = static_cast<int>(s.f);
  dim3 g1((f + ST - 1) / ST, gy, s.E);
  ffn_simt_kernel<true><<<g1, 256, 0, st>>>(a, a_rows, s.T, wg, wu, f, d, offsets, kept, h);
  note_launch();
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  dim3 g2((d + ST - 1) / ST, gy, s.E);
  ffn_simt_kernel<false><<<g2, 256, 0, st>>>(h, nullptr, 0, wd, nullptr, d, f, offsets, kept,
                                             y);
  note_launch();
  return cudaGetLastError();
}

}  // namespace moe
