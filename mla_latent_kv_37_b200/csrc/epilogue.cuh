// Epilogues of the projection products: finish the split-K sums (fixed order), apply RoPE,
// round to the storage type and place results (paged cache slot, q_cat, o_heads, out).
// Also the "hi/lo" splits that carry an fp32 value into a bf16 tensor-core product as two
// bf16 rows (hi = bf16(x), lo = bf16(x - hi)); the product's two halves are summed here.
#pragma once
#include "ptx_sm100.cuh"
#include "rope.cuh"

namespace mla {

template <typename T> __device__ __forceinline__ T to_elem(float x);
template <> __device__ __forceinline__ float to_elem<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 to_elem<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

// cos/sin of the RoPE angle of rotary pair `pair` at position `pos` (see rope_cs).
__device__ __forceinline__ void rope_cos_sin(int pos, int pair, float theta, float& c, float& s) {
  const float2 cs = rope_cs(theta, pair, pos);
  c = cs.x;
  s = cs.y;
}

__device__ __forceinline__ float sum_splits(const float* part, int k_splits, size_t split_stride,
                                            size_t idx) {
  float v = 0.f;
  for (int ks = 0; ks < k_splits; ++ks) v += part[ks * split_stride + idx];
  return v;
}

// ---------------------------------------------------------------------------------------------
// cache append: rows 0..511 -> c_KV, rows 512..575 -> RoPE(k_R); scatter into the page slot.
// part: [k_splits][576][n_pad].  rows_in != null: scatter-only mode (rows already formed).
// grid (ceil(288 / 96), B), block 96: one thread per pair of columns.
// ---------------------------------------------------------------------------------------------
template <typename T>
__global__ void append_epilogue_kernel(const float* __restrict__ part, int k_splits, int n_pad,
                                       const T* __restrict__ rows_in,
                                       const int32_t* __restrict__ positions,
                                       const int32_t* __restrict__ page_table, int max_pages,
                                       T* __restrict__ pool, int num_pages, float theta,
                                       unsigned int* status) {
  constexpr int kRow = 576, kDc = 512, kPage = 64;
  const int b = blockIdx.y;
  const int q = blockIdx.x * blockDim.x + threadIdx.x;
  if (2 * q >= kRow) return;
  const int pos = positions[b];
  if (pos < 0 || pos >= max_pages * kPage) {
    if (q == 0) atomicOr(status, MLA_STATUS_BAD_POSITION);
    return;
  }
  const int page = page_table[static_cast<size_t>(b) * max_pages + pos / kPage];
  if (page < 0 || page >= num_pages) {
    if (q == 0) atomicOr(status, MLA_STATUS_BAD_PAGE);
    return;
  }
  T* dst = pool + (static_cast<size_t>(page) * kPage + pos % kPage) * kRow + 2 * q;
  if (rows_in) {
    dst[0] = rows_in[static_cast<size_t>(b) * kRow + 2 * q];
    dst[1] = rows_in[static_cast<size_t>(b) * kRow + 2 * q + 1];
    return;
  }
  const size_t split_stride = static_cast<size_t>(kRow) * n_pad;
  float v0 = sum_splits(part, k_splits, split_stride, static_cast<size_t>(2 * q) * n_pad + b);
  float v1 = sum_splits(part, k_splits, split_stride, static_cast<size_t>(2 * q + 1) * n_pad + b);
  if (2 * q >= kDc) {
    float c, s;
    rope_cos_sin(pos, (2 * q - kDc) / 2, theta, c, s);
    const float r0 = v0 * c - v1 * s, r1 = v0 * s + v1 * c;
    v0 = r0;
    v1 = r1;
  }
  dst[0] = to_elem<T>(v0);
  dst[1] = to_elem<T>(v1);
}

// ---------------------------------------------------------------------------------------------
// W_Q product -> q_nope (for the W_UK product) and RoPE(q_rope) into q_cat[:, :, 512:576].
// part: [k_splits][H*192][n_pad].  grid (H, B), block 96 (one thread per column pair).
// bf16: qn_out = [2][B][H][128] hi/lo planes;  fp32: qn_out = [B][H][128].
// ---------------------------------------------------------------------------------------------
template <typename T>
__global__ void wq_epilogue_kernel(const float* __restrict__ part, int k_splits, int n_pad, int B,
                                   int H, const int32_t* __restrict__ positions, float theta,
                                   T* __restrict__ q_cat, __nv_bfloat16* __restrict__ q_lo,
                                   void* __restrict__ qn_out) {
  constexpr int kDn = 128, kDq = 192, kRow = 576, kDc = 512;
  const int h = blockIdx.x, b = blockIdx.y;
  const int d = 2 * threadIdx.x;
  if (d >= kDq) return;
  const size_t split_stride = static_cast<size_t>(H) * kDq * n_pad;
  const size_t m = static_cast<size_t>(h) * kDq + d;
  float v0 = sum_splits(part, k_splits, split_stride, m * n_pad + b);
  float v1 = sum_splits(part, k_splits, split_stride, (m + 1) * n_pad + b);
  if (d < kDn) {
    const size_t o = (static_cast<size_t>(b) * H + h) * kDn + d;
    if constexpr (sizeof(T) == 2) {
      __nv_bfloat16* qn = static_cast<__nv_bfloat16*>(qn_out);
      const size_t plane = static_cast<size_t>(B) * H * kDn;
      const __nv_bfloat16 h0 = __float2bfloat16_rn(v0), h1 = __float2bfloat16_rn(v1);
      qn[o] = h0;
      qn[o + 1] = h1;
      qn[plane + o] = __float2bfloat16_rn(v0 - __bfloat162float(h0));
      qn[plane + o + 1] = __float2bfloat16_rn(v1 - __bfloat162float(h1));
    } else {
      float* qn = static_cast<float*>(qn_out);
      qn[o] = v0;
      qn[o + 1] = v1;
    }
    return;
  }
  const int pos = positions[b];
  float c, s;
  rope_cos_sin(pos, (d - kDn) / 2, theta, c, s);
  const float r0 = v0 * c - v1 * s, r1 = v0 * s + v1 * c;
  const size_t o = (static_cast<size_t>(b) * H + h) * kRow + kDc + (d - kDn);
  const T e0 = to_elem<T>(r0), e1 = to_elem<T>(r1);
  q_cat[o] = e0;
  q_cat[o + 1] = e1;
  if (q_lo) {
    q_lo[o] = __float2bfloat16_rn(r0 - to_f32(e0));
    q_lo[o + 1] = __float2bfloat16_rn(r1 - to_f32(e1));
  }
}

// ---------------------------------------------------------------------------------------------
// W_UK product -> q_lat into q_cat[:, :, 0:512].  part: [1][H][512][n_pad]; with split input
// the columns [0, B) hold W_UK^T q_hi and [B, 2B) hold W_UK^T q_lo.  grid (H, B), block 128.
// ---------------------------------------------------------------------------------------------
template <typename T, bool kSplitIn>
__global__ void wuk_epilogue_kernel(const float* __restrict__ part, int n_pad, int B, int H,
                                    T* __restrict__ q_cat, __nv_bfloat16* __restrict__ q_lo) {
  constexpr int kDc = 512, kRow = 576;
  const int h = blockIdx.x, b = blockIdx.y;
  for (int m = threadIdx.x; m < kDc; m += blockDim.x) {
    const size_t i = (static_cast<size_t>(h) * kDc + m) * n_pad;
    float v = part[i + b];
    if (kSplitIn) v += part[i + B + b];
    const size_t o = (static_cast<size_t>(b) * H + h) * kRow + m;
    const T e = to_elem<T>(v);
    q_cat[o] = e;
    if (q_lo) q_lo[o] = __float2bfloat16_rn(v - to_f32(e));
  }
}

// o_lat fp32 [n] -> bf16 hi/lo planes: out[i] = hi, out[plane + i] = lo (plane >= n).  n and
// plane are multiples of 8 and x, out 16-byte aligned: each thread converts 8 values with one
// 32-byte load and two 16-byte stores.  Also zeroes zero[0 .. n_zero) (block 0), a buffer the
// next kernel accumulates into.
__global__ void split_hi_lo_kernel(const float* __restrict__ x, size_t n, size_t plane,
                                   __nv_bfloat16* __restrict__ out, unsigned int* zero,
                                   int n_zero) {
  griddep_launch_dependents();
  griddep_wait();
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < n_zero; i += blockDim.x) zero[i] = 0u;
  const size_t n8 = n / 8;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const float4 a = reinterpret_cast<const float4*>(x)[2 * i];
    const float4 b = reinterpret_cast<const float4*>(x)[2 * i + 1];
    const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const __nv_bfloat16 h0 = __float2bfloat16_rn(v[2 * k]);
      const __nv_bfloat16 h1 = __float2bfloat16_rn(v[2 * k + 1]);
      const __nv_bfloat16 l0 = __float2bfloat16_rn(v[2 * k] - __bfloat162float(h0));
      const __nv_bfloat16 l1 = __float2bfloat16_rn(v[2 * k + 1] - __bfloat162float(h1));
      hi[k] = static_cast<uint32_t>(__bfloat16_as_ushort(h0)) |
              (static_cast<uint32_t>(__bfloat16_as_ushort(h1)) << 16);
      lo[k] = static_cast<uint32_t>(__bfloat16_as_ushort(l0)) |
              (static_cast<uint32_t>(__bfloat16_as_ushort(l1)) << 16);
    }
    reinterpret_cast<uint4*>(out)[i] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    reinterpret_cast<uint4*>(out + plane)[i] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
  }
}

// ---------------------------------------------------------------------------------------------
// W_UV product -> o_heads, plus the input of the W_O product.
// part: [k_splits][H][128][n_pad].  grid (H, B), block 128 (one thread per value column).
// bf16: oh_out = [2][B][H*128] hi/lo planes;  fp32: oh_out = [B][H*128].
// ---------------------------------------------------------------------------------------------
template <typename T, bool kSplitIn>
__global__ void wuv_epilogue_kernel(const float* __restrict__ part, int k_splits, int n_pad, int B,
                                    int H, T* __restrict__ o_heads, void* __restrict__ oh_out) {
  constexpr int kDv = 128;
  const int h = blockIdx.x, b = blockIdx.y, v = threadIdx.x;
  const size_t split_stride = static_cast<size_t>(H) * kDv * n_pad;
  const size_t i = (static_cast<size_t>(h) * kDv + v) * n_pad;
  float val = sum_splits(part, k_splits, split_stride, i + b);
  if (kSplitIn) val += sum_splits(part, k_splits, split_stride, i + B + b);
  const size_t o = (static_cast<size_t>(b) * H + h) * kDv + v;
  if (o_heads) o_heads[o] = to_elem<T>(val);
  if (oh_out) {
    if constexpr (sizeof(T) == 2) {
      __nv_bfloat16* oh = static_cast<__nv_bfloat16*>(oh_out);
      const __nv_bfloat16 hi = __float2bfloat16_rn(val);
      oh[o] = hi;
      oh[static_cast<size_t>(B) * H * kDv + o] = __float2bfloat16_rn(val - __bfloat162float(hi));
    } else {
      static_cast<float*>(oh_out)[o] = val;
    }
  }
}

// W_O product -> out [B][D].  part: [k_splits][D][n_pad].  grid (ceil(D/256), B), block 256.
template <typename T, bool kSplitIn>
__global__ void wo_epilogue_kernel(const float* __restrict__ part, int k_splits, int n_pad, int B,
                                   int D, T* __restrict__ out) {
  const int b = blockIdx.y;
  const int d = blockIdx.x * blockDim.x + threadIdx.x;
  if (d >= D) return;
  const size_t split_stride = static_cast<size_t>(D) * n_pad;
  const size_t i = static_cast<size_t>(d) * n_pad;
  float val = sum_splits(part, k_splits, split_stride, i + b);
  if (kSplitIn) val += sum_splits(part, k_splits, split_stride, i + B + b);
  out[static_cast<size_t>(b) * D + d] = to_elem<T>(val);
}

// ---------------------------------------------------------------------------------------------
// fp32 SIMT products for the fp32 path (no tensor-core fp32 mode meets a 1e-5 tolerance).
// P[g][m][n] = sum_k A_g[m][k] X_g[n][k], written in the same [1][G][M][N] partial layout.
// ---------------------------------------------------------------------------------------------
// A_g[m][k] at A[g*a_gs + m*lda + k] (K contiguous).  grid (ceil(M/8), G), block 256.
__global__ void f32_gemm_k_kernel(const float* __restrict__ A, size_t a_gs, int lda,
                                  const float* __restrict__ X, size_t x_ns, size_t x_gs, int M,
                                  int K, int N, float* __restrict__ P) {
  const int g = blockIdx.y;
  const int m = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (m >= M) return;
  const float* a = A + g * a_gs + static_cast<size_t>(m) * lda;
  for (int n0 = 0; n0 < N; n0 += 8) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int k = lane; k < K; k += 32) {
      const float av = a[k];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (n0 + j < N) acc[j] = fmaf(av, X[(n0 + j) * x_ns + g * x_gs + k], acc[j]);
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float v = acc[j];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0 && n0 + j < N) P[(static_cast<size_t>(g) * M + m) * N + n0 + j] = v;
    }
  }
}

// A_g[m][k] at A[g*a_gs + k*lda + m] (M contiguous).  grid (ceil(M/128), G), block 128.
__global__ void f32_gemm_mn_kernel(const float* __restrict__ A, size_t a_gs, int lda,
                                   const float* __restrict__ X, size_t x_ns, size_t x_gs, int M,
                                   int K, int N, float* __restrict__ P) {
  const int g = blockIdx.y;
  const int m = blockIdx.x * 128 + threadIdx.x;
  if (m >= M) return;
  const float* a = A + g * a_gs + m;
  for (int n0 = 0; n0 < N; n0 += 8) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int k = 0; k < K; ++k) {
      const float av = a[static_cast<size_t>(k) * lda];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (n0 + j < N) acc[j] = fmaf(av, X[(n0 + j) * x_ns + g * x_gs + k], acc[j]);
    }
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (n0 + j < N) P[(static_cast<size_t>(g) * M + m) * N + n0 + j] = acc[j];
  }
}

}  // namespace mla
