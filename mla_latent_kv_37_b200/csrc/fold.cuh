// Offline weight folding for the folded execution mode: the query's W_UK_h absorbed into W_Q
// and W_UV_h into W_O ahead of time instead of at every step ([LP] "MLA: compress the pair, not
// the heads": Q K^T = (Q W_UK^T) c^T by associativity; [IA] "O preço da economia: mais contas":
// the mode that reuses pre-multiplied matrices).  One-time preparation, not part of a step.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

namespace mla {
namespace fold {

constexpr int kTile = 64;     // output tile: 64 x 64
constexpr int kKc = 16;       // K chunk staged in shared memory
constexpr int kThreads = 256; // 16 x 16 threads, 4 x 4 outputs each

// C[g][i][j] = sum_{k < K} A(g, i, k) B(g, k, j) for i < M, j < N: bf16 inputs read through
// element strides, fp32 accumulation in k order, bf16 (round to nearest even) output.
__global__ void __launch_bounds__(kThreads)
    batched_gemm_kernel(const __nv_bfloat16* __restrict__ a, long long a_g, long long a_i,
                        long long a_k, const __nv_bfloat16* __restrict__ b, long long b_g,
                        long long b_k, long long b_j, __nv_bfloat16* __restrict__ c,
                        long long c_g, long long c_i, long long c_j, int M, int N, int K) {
  __shared__ float as[kKc][kTile + 1];  // [k][i]
  __shared__ float bs[kKc][kTile + 1];  // [k][j]
  const long long g = blockIdx.z;
  const int i0 = blockIdx.y * kTile, j0 = blockIdx.x * kTile;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[r][q] = 0.f;
  for (int k0 = 0; k0 < K; k0 += kKc) {
    for (int e = threadIdx.x; e < kKc * kTile; e += kThreads) {
      const int kk = e / kTile, x = e - kk * kTile, k = k0 + kk;
      const int i = i0 + x, j = j0 + x;
      as[kk][x] = (i < M && k < K) ? __bfloat162float(a[g * a_g + i * a_i + k * a_k]) : 0.f;
      bs[kk][x] = (j < N && k < K) ? __bfloat162float(b[g * b_g + k * b_k + j * b_j]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kKc; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) av[r] = as[kk][ty + 16 * r];
#pragma unroll
      for (int q = 0; q < 4; ++q) bv[q] = bs[kk][tx + 16 * q];
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[r][q] = fmaf(av[r], bv[q], acc[r][q]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int i = i0 + ty + 16 * r;
    if (i >= M) continue;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int j = j0 + tx + 16 * q;
      if (j < N) c[g * c_g + i * c_i + j * c_j] = __float2bfloat16_rn(acc[r][q]);
    }
  }
}

// Copy `rows` rows of `cols` bf16 per group from src (group stride src_g, row stride cols) to
// dst (group stride dst_g, row stride cols); cols is a multiple of 8 (16-byte pieces).
__global__ void copy_rows_kernel(const __nv_bfloat16* __restrict__ src, long long src_g,
                                 __nv_bfloat16* __restrict__ dst, long long dst_g, int groups,
                                 int rows, int cols) {
  const long long per_group = static_cast<long long>(rows) * cols / 8;
  const long long n = per_group * groups;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long g = e / per_group, w = e - g * per_group;
    reinterpret_cast<uint4*>(dst + g * dst_g)[w] =
        reinterpret_cast<const uint4*>(src + g * src_g)[w];
  }
}

}  // namespace fold
}  // namespace mla
