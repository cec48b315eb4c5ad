// E4M3 (FP8) storage of weight matrices: one fp32 scale per row, so that the row's largest
// magnitude maps to 448, the largest finite E4M3 value ([IA] "De onde vem o 93%": the pages'
// throughput figure used weights converted to FP8).  One-time preparation, not part of a step.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

namespace mla {
namespace fp8 {

// Row r of w [rows][cols] (bf16): s_r = max_j |w_rj| / 448 (fp32, round to nearest; 1 for a zero
// row), code_rj = w_rj / s_r (fp32) rounded to the nearest E4M3 value, ties to even,
// saturating at +-448.  One block per row; cols is even.
__global__ void __launch_bounds__(256)
    quantize_rows_kernel(const __nv_bfloat16* __restrict__ w, long long cols,
                         uint8_t* __restrict__ q, float* __restrict__ scale) {
  __shared__ float part[8];
  const long long row = blockIdx.x;
  const __nv_bfloat16* wr = w + row * cols;
  float m = 0.f;
  for (long long j = threadIdx.x; j < cols; j += blockDim.x)
    m = fmaxf(m, fabsf(__bfloat162float(wr[j])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = m;
  __syncthreads();
  m = part[0];
  for (int k = 1; k < static_cast<int>(blockDim.x >> 5); ++k) m = fmaxf(m, part[k]);
  const float s = m > 0.f ? __fdiv_rn(m, 448.f) : 1.f;
  if (threadIdx.x == 0) scale[row] = s;
  uint16_t* qr = reinterpret_cast<uint16_t*>(q + row * cols);
  for (long long j = threadIdx.x; j < cols / 2; j += blockDim.x) {
    const float y0 = __fdiv_rn(__bfloat162float(wr[2 * j]), s);
    const float y1 = __fdiv_rn(__bfloat162float(wr[2 * j + 1]), s);
    uint16_t c;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(c) : "f"(y1), "f"(y0));
    qr[j] = c;  // low byte: element 2j
  }
}

}  // namespace fp8
}  // namespace mla
