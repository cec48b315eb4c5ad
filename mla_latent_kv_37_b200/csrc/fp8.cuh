// E4M3 (FP8) storage of weight matrices: one fp32 scale per row, so that the row's largest
// magnitude maps to 448, the largest finite E4M3 value ([IA] "De onde vem o 93%": the pages'
// throughput figure used weights converted to FP8).  One-time preparation, not part of a step.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cfloat>

#include "ptx_sm100.cuh"

namespace mla {
namespace fp8 {

// Row r of w [rows][cols] (bf16): s_r = max_j |w_rj| / 448 (fp32, round to nearest; 1 for a zero
// row), code_rj = w_rj / s_r (fp32) rounded to the nearest E4M3 value, ties to even,
// saturating at +-448.  The codes are stored in tiles of 128 rows x 128 columns, each tile
// contiguous and row-major inside, tiles ordered by row tile then column tile:
// code_rj at ((r / 128) * (cols / 128) + j / 128) * 16384 + (r % 128) * 128 + j % 128.  One block
// per row; cols a multiple of 128.
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
  uint8_t* qt = q + (row / 128) * cols * 128 + (row % 128) * 128;
  for (long long j = threadIdx.x; j < cols / 2; j += blockDim.x) {
    const float y0 = __fdiv_rn(__bfloat162float(wr[2 * j]), s);
    const float y1 = __fdiv_rn(__bfloat162float(wr[2 * j + 1]), s);
    uint16_t c;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(c) : "f"(y1), "f"(y0));
    // low byte: element 2j; a pair never straddles a tile
    *reinterpret_cast<uint16_t*>(qt + (2 * j / 128) * 16384 + (2 * j) % 128) = c;
  }
}

// Two fp32 values -> two E4M3 codes (round to nearest even, saturating), low byte from `lo`.
__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
  uint16_t c;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(c) : "f"(hi), "f"(lo));
  return c;
}
// Two E4M3 codes -> their exact values (every E4M3 value is an f16 value).
__device__ __forceinline__ float2 e4m3x2_value(uint16_t c) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(c));
  return __half22float2(*reinterpret_cast<const __half2*>(&h));
}

// fp32 activation rows x_b (K values each) as a scale and n_planes (2 or 3) E4M3 planes:
// s_b = m_b / 448 (at least FLT_MIN) with m_b = max_k |x_bk| given as fp32 bits in rowmax[b];
// y = x / s_b; p1 = E4M3(y), p2 = E4M3(y - p1), p3 = E4M3(y - p1 - p2), each difference exact
// in fp32.  The planes' sum keeps about 4 significant bits of y per plane (8 with two, 12 with
// three), so s_b (p1 + p2 [+ p3]) stands in for x_b in a product with E4M3 weights.  planes:
// [n_planes][rows_pad][K]; rows in [rows, rows_pad) are written as zeros.  Each thread converts
// 8 consecutive values (grid-stride); K a multiple of 8; x and planes 16- and 8-byte aligned.
__global__ void __launch_bounds__(256)
    split_planes_kernel(const float* __restrict__ x, const unsigned int* __restrict__ rowmax,
                        int rows, long long K, int rows_pad, int n_planes,
                        uint8_t* __restrict__ planes, float* __restrict__ scale) {
  griddep_launch_dependents();
  griddep_wait();
  const long long n8 = K / 8;
  const size_t plane8 = static_cast<size_t>(rows_pad) * n8;  // one plane, in 8-byte groups
  uint2* out = reinterpret_cast<uint2*>(planes);
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
       i < static_cast<long long>(plane8); i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int b = static_cast<int>(i / n8);
    if (b >= rows) {
      for (int pl = 0; pl < n_planes; ++pl) out[pl * plane8 + i] = make_uint2(0u, 0u);
      continue;
    }
    const float s = fmaxf(__fdiv_rn(__uint_as_float(rowmax[b]), 448.f), FLT_MIN);
    if (i - static_cast<long long>(b) * n8 == 0) scale[b] = s;
    const float4 u = reinterpret_cast<const float4*>(x)[2 * i];
    const float4 w = reinterpret_cast<const float4*>(x)[2 * i + 1];
    float y[8] = {u.x, u.y, u.z, u.w, w.x, w.y, w.z, w.w};
#pragma unroll
    for (int k = 0; k < 8; ++k) y[k] = __fdiv_rn(y[k], s);
#pragma unroll
    for (int pl = 0; pl < 3; ++pl) {
      if (pl == n_planes) break;
      uint32_t c[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint16_t q = e4m3x2(y[2 * k], y[2 * k + 1]);
        const float2 d = e4m3x2_value(q);
        y[2 * k] -= d.x;
        y[2 * k + 1] -= d.y;
        c[k] = q;
      }
      out[pl * plane8 + i] = make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
    }
  }
}

// bf16 activation rows x_b (K values each) as a power-of-two scale and two E4M3 planes:
// s_b = the smallest power of two >= max_k |x_bk| / 448 (fp32; 1 for a zero row), y = x / s_b
// (exact), p1 = E4M3(y), p2 = E4M3(y - p1).  A bf16 value has 8 significant bits and y - p1 at
// most the low 4 of them, so p1 + p2 = y exactly unless that remainder falls below E4M3's
// smallest subnormal (elements under about 2^-8 of the row's largest).  planes: [2][rows_pad][K];
// rows in [rows, rows_pad) are zeros.  Grid (rows_pad, slices): every block of row b finds the
// row's maximum itself (K bf16 values, from L2), then converts its slice of K / slices values,
// 8 per thread.  K a multiple of 8 * slices; x 16-byte and planes 8-byte aligned.
__global__ void __launch_bounds__(256)
    split_planes_bf16_kernel(const __nv_bfloat16* __restrict__ x, int rows, long long K,
                             int rows_pad, uint8_t* __restrict__ planes,
                             float* __restrict__ scale) {
  __shared__ float part[8];
  griddep_launch_dependents();
  griddep_wait();
  const int b = blockIdx.x;
  const long long n8 = K / 8, slice8 = n8 / gridDim.y, j0 = slice8 * blockIdx.y;
  const size_t plane8 = static_cast<size_t>(rows_pad) * n8;
  uint2* out = reinterpret_cast<uint2*>(planes) + static_cast<size_t>(b) * n8;
  if (b >= rows) {
    for (long long j = j0 + threadIdx.x; j < j0 + slice8; j += blockDim.x) {
      out[j] = make_uint2(0u, 0u);
      out[plane8 + j] = make_uint2(0u, 0u);
    }
    if (blockIdx.y == 0 && threadIdx.x == 0) scale[b] = 0.f;
    return;
  }
  const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<size_t>(b) * K);
  float m = 0.f;
  for (long long j = threadIdx.x; j < n8; j += blockDim.x) {
    const uint4 u = xr[j];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int k = 0; k < 4; ++k)
      m = fmaxf(m, fmaxf(fabsf(__uint_as_float(w[k] << 16)),
                         fabsf(__uint_as_float(w[k] & 0xffff0000u))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = m;
  __syncthreads();
  m = part[0];
  for (int k = 1; k < static_cast<int>(blockDim.x >> 5); ++k) m = fmaxf(m, part[k]);
  // the smallest power of two >= m / 448 (round the quotient's exponent up unless it is exact)
  float s = 1.f;
  if (m > 0.f) {
    const uint32_t t = __float_as_uint(__fdiv_ru(m, 448.f));
    const uint32_t e = t >> 23;  // biased exponent (t > 0, so the sign bit is clear)
    s = (t & 0x7fffffu) == 0u ? __uint_as_float(t) : __uint_as_float(min(e + 1u, 254u) << 23);
    if (e == 0u) s = 1.17549435e-38f;  // a subnormal quotient: FLT_MIN
  }
  if (blockIdx.y == 0 && threadIdx.x == 0) scale[b] = s;
  for (long long j = j0 + threadIdx.x; j < j0 + slice8; j += blockDim.x) {
    const uint4 u = xr[j];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    float y[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      y[2 * k] = __fdiv_rn(__uint_as_float(w[k] << 16), s);
      y[2 * k + 1] = __fdiv_rn(__uint_as_float(w[k] & 0xffff0000u), s);
    }
#pragma unroll
    for (int pl = 0; pl < 2; ++pl) {
      uint32_t c[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint16_t q = e4m3x2(y[2 * k], y[2 * k + 1]);
        const float2 d = e4m3x2_value(q);
        y[2 * k] -= d.x;
        y[2 * k + 1] -= d.y;
        c[k] = q;
      }
      out[pl * plane8 + j] = make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
    }
  }
}

}  // namespace fp8
}  // namespace mla
