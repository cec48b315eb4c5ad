// Weight-streaming GEMM on the 5th-generation tensor core (tcgen05), "swap-AB" form:
//
//   P[ks][g][m][n] = sum_{k in split ks} A_g[m][k] * B_g[n][k]
//
// A is a weight matrix (output features m on the MMA's M side, 128 per tile), B holds the few
// activation rows (batch, padded to N = 16..256) on the MMA's N side.  Decode projections
// multiply large weights by a handful of token vectors, so the kernel is bound by how fast
// the weights stream from HBM: TMA brings 128 x 64 weight tiles into a multi-stage shared
// memory ring, one thread issues tcgen05.mma (M=128, N=n_pad, K=16) into a TMEM accumulator,
// and four epilogue warps drain TMEM into fp32 partial sums that a small reduction kernel
// finishes (summing the K splits in a fixed order, so results are deterministic).
//
// Operand layouts (shared memory, 128-byte swizzle, filled by TMA):
//   A K-major : box (64 k, 128 m)        -> [128 rows][128 B],  SBO = 1024 B
//   A MN-major: 2 boxes (64 m, 64 k)     -> [64 k rows][128 B] per 64-m chunk, LBO = 8 KiB
//   B K-major : box (64 k, 1, n_pad)     -> [n_pad rows][128 B], SBO = 1024 B
#pragma once
#include "ptx_sm100.cuh"

namespace mla {

struct GemmParams {
  int m_total;        // output rows per group (partial row count)
  int m_tiles;        // 128-row tiles per group
  int a1_tile_start;  // tiles >= this read tensor map A1 (rows relative to it); > m_tiles: none
  int k_blocks;       // 64-wide K blocks
  int k_splits;       // gridDim.y
  int n_pad;          // MMA N (multiple of 16, <= 256)
  int a_mn_major;     // 0: A is K-major, 1: A is MN-major
  int stages;         // shared-memory ring depth
  int groups;         // gridDim.z (heads for per-head products, else 1)
  float* partial;     // [k_splits][groups][m_total][n_pad]
  unsigned int* status;
  uint64_t wait_ns;
};

constexpr int kGemmThreads = 192;  // warp 0: TMA, warp 1: MMA + TMEM, warps 2..5: epilogue
constexpr uint32_t kGemmATileBytes = 128 * 64 * 2;

__host__ __device__ inline uint32_t gemm_stage_bytes(int n_pad) {
  return kGemmATileBytes + static_cast<uint32_t>(n_pad) * 128u;
}

__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_swapab_kernel(const __grid_constant__ CUtensorMap tmA0,
                       const __grid_constant__ CUtensorMap tmA1,
                       const __grid_constant__ CUtensorMap tmB, const GemmParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the swizzled tiles
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t stage_bytes = gemm_stage_bytes(p.n_pad);
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + p.stages * stage_bytes);
  uint64_t* empty_bar = full_bar + p.stages;
  uint64_t* accum_bar = empty_bar + p.stages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m_tile = blockIdx.x;
  const int ks = blockIdx.y;
  const int g = blockIdx.z;
  const int kpc = (p.k_blocks + p.k_splits - 1) / p.k_splits;
  const int kb0 = ks * kpc;
  const int kb1 = min(p.k_blocks, kb0 + kpc);
  const int nk = max(0, kb1 - kb0);
  uint32_t tmem_cols = 32;
  while (tmem_cols < static_cast<uint32_t>(p.n_pad)) tmem_cols <<= 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(accum_bar, 1);
    *abort_flag = 0;
    fence_mbar_init_cluster();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;
  WaitCtx wc{abort_flag, p.status, p.wait_ns};

  const bool use_a1 = m_tile >= p.a1_tile_start;
  const CUtensorMap* tmA = use_a1 ? &tmA1 : &tmA0;
  const int m_row0 = (use_a1 ? (m_tile - p.a1_tile_start) : m_tile) * 128;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0 && nk > 0) {
      tma_prefetch_desc(tmA);
      tma_prefetch_desc(&tmB);
      const uint64_t pol_w = l2_policy_evict_first();
      const uint64_t pol_x = l2_policy_evict_last();
      int issued = 0;
      for (int i = 0; i < nk; ++i) {
        const int s = i % p.stages;
        const uint32_t ph = (i / p.stages) & 1;
        if (i >= p.stages && !mbar_wait(&empty_bar[s], ph ^ 1, wc)) break;
        uint8_t* a_dst = smem + s * stage_bytes;
        uint8_t* b_dst = a_dst + kGemmATileBytes;
        mbar_arrive_expect_tx(&full_bar[s], stage_bytes);
        const int k0 = (kb0 + i) * 64;
        if (p.a_mn_major) {
          tma_load_3d_hint(a_dst, tmA, &full_bar[s], m_row0, k0, g, pol_w);
          tma_load_3d_hint(a_dst + 8192, tmA, &full_bar[s], m_row0 + 64, k0, g, pol_w);
        } else {
          tma_load_3d_hint(a_dst, tmA, &full_bar[s], k0, m_row0, g, pol_w);
        }
        tma_load_3d_hint(b_dst, &tmB, &full_bar[s], k0, g, 0, pol_x);
        ++issued;
      }
      if (*abort_flag) {
        // wait (bounded, ignoring the abort flag) for every copy still landing in the ring
        volatile int never = 0;
        WaitCtx drain{&never, p.status, p.wait_ns};
        for (int i = max(0, issued - p.stages); i < issued; ++i)
          mbar_wait(&full_bar[i % p.stages], (i / p.stages) & 1, drain);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0 && nk > 0) {
      const uint32_t idesc = idesc_bf16(128, p.n_pad, p.a_mn_major, 0);
      bool ok = true;
      for (int i = 0; i < nk && ok; ++i) {
        const int s = i % p.stages;
        const uint32_t ph = (i / p.stages) & 1;
        if (!mbar_wait(&full_bar[s], ph, wc)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_base = smem_u32(smem + s * stage_bytes);
        const uint32_t b_base = a_base + kGemmATileBytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          uint64_t adesc;
          if (p.a_mn_major)
            adesc = smem_desc(a_base + kk * 2048, 8192, 1024, kSwizzle128B);
          else
            adesc = smem_desc(a_base + kk * 32, 16, 1024, kSwizzle128B);
          const uint64_t bdesc = smem_desc(b_base + kk * 32, 16, 1024, kSwizzle128B);
          mma_ss(tmem_d, adesc, bdesc, idesc, (i > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&empty_bar[s]);
      }
      mma_commit(accum_bar);  // also fires after an abort, once issued MMAs drain
    }
  } else {
    // ---------------- epilogue: TMEM -> fp32 partials ----------------
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int m_local = quarter * 32 + lane;
    const int m = m_tile * 128 + m_local;
    float* dst = p.partial +
                 ((static_cast<size_t>(ks) * p.groups + g) * p.m_total + m) * p.n_pad;
    const bool row_ok = m < p.m_total;
    if (nk == 0) {
      if (row_ok)
        for (int n = 0; n < p.n_pad; ++n) dst[n] = 0.f;
    } else if (mbar_wait(accum_bar, 0, wc)) {
      tc_fence_after();
      for (int c = 0; c < p.n_pad; c += 16) {
        uint32_t r[16];
        tmem_ld16(tmem_d + (static_cast<uint32_t>(quarter * 32) << 16) + c, r);
        tmem_wait_ld();
        if (row_ok) {
          float4* d4 = reinterpret_cast<float4*>(dst + c);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            d4[j] = make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
        }
      }
    }
  }

  // Never release TMEM while issued MMAs may still write it.
  if (warp == 1 && lane == 0 && nk > 0 && *abort_flag) {
    volatile int never = 0;
    WaitCtx drain{&never, p.status, p.wait_ns};
    mbar_wait(accum_bar, 0, drain);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_d, tmem_cols);
  }
}

}  // namespace mla
