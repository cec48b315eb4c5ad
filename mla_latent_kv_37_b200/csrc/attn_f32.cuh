// fp32 split-KV decode attention on the SIMT cores (fp32 configuration; tensor cores have no
// fp32 mode accurate to 1e-5).  Same work division, plan and partial layout as the tcgen05
// kernel: block (part, head) walks the part's segments page by page with an online softmax.
#pragma once
#include "attn_sm100.cuh"

namespace mla {
namespace attn {

__global__ void __launch_bounds__(128)
    f32_split_kernel(const float* __restrict__ q_cat, const float* __restrict__ pool,
                     const int32_t* __restrict__ page_table, int max_pages, int num_pages,
                     const int32_t* __restrict__ seq_lens, const int32_t* __restrict__ plan_words,
                     int B, int C, int H, float scale, float* __restrict__ o_lat,
                     float* __restrict__ lse, float* __restrict__ part_o,
                     float* __restrict__ part_lse, unsigned int* status) {
  __shared__ float q[kRow];
  __shared__ float sc[kPage];
  const PlanView plan(plan_words, B, C);
  const int part = blockIdx.x, h = blockIdx.y;
  if (part >= plan.parts()) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  SegIter it{plan.seq_pages(), plan.seq_prefix(), B, plan.part_start()[part],
             plan.part_start()[part + 1], plan.part_seq()[part]};
  int seq, p0, p1;
  while (it.next(seq, p0, p1)) {
    __syncthreads();
    for (int i = threadIdx.x; i < kRow; i += blockDim.x)
      q[i] = q_cat[(static_cast<size_t>(seq) * H + h) * kRow + i];
    __syncthreads();
    const int len = min(seq_lens[seq], max_pages * kPage);
    float m = -__int_as_float(0x7f800000), l = 0.f;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};  // latent columns 4*tid .. 4*tid+3
    for (int pg = p0; pg < p1; ++pg) {
      int page = page_table[static_cast<size_t>(seq) * max_pages + pg];
      if (page < 0 || page >= num_pages) {
        if (threadIdx.x == 0) atomicOr(status, MLA_STATUS_BAD_PAGE);
        page = 0;
      }
      const float* rows = pool + static_cast<size_t>(page) * kPage * kRow;
      const int valid = min(kPage, len - pg * kPage);
      for (int j = warp; j < kPage; j += 4) {
        float d = 0.f;
        if (j < valid)
          for (int i = lane; i < kRow; i += 32) d = fmaf(q[i], rows[j * kRow + i], d);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
        if (lane == 0) sc[j] = j < valid ? d * scale : -__int_as_float(0x7f800000);
      }
      __syncthreads();
      float tmax = m;
      for (int j = 0; j < valid; ++j) tmax = fmaxf(tmax, sc[j]);
      const float alpha = expf(m - tmax);
      m = tmax;
      l *= alpha;
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[c] *= alpha;
      for (int j = 0; j < valid; ++j) {
        const float pj = expf(sc[j] - m);
        l += pj;
        const float4 r = reinterpret_cast<const float4*>(rows + j * kRow)[threadIdx.x];
        acc[0] = fmaf(pj, r.x, acc[0]);
        acc[1] = fmaf(pj, r.y, acc[1]);
        acc[2] = fmaf(pj, r.z, acc[2]);
        acc[3] = fmaf(pj, r.w, acc[3]);
      }
      __syncthreads();
    }
    const int nparts = plan.seq_nparts()[seq];
    float* dst;
    float* dst_lse;
    if (nparts == 1) {
      dst = o_lat + (static_cast<size_t>(seq) * H + h) * 512;
      dst_lse = lse ? lse + static_cast<size_t>(seq) * H + h : nullptr;
    } else {
      const int slot = plan.seq_slot()[seq] + (part - plan.seq_first_part()[seq]);
      dst = part_o + (static_cast<size_t>(slot) * H + h) * 512;
      dst_lse = part_lse + static_cast<size_t>(slot) * H + h;
    }
    const float inv = 1.f / l;
    reinterpret_cast<float4*>(dst)[threadIdx.x] =
        make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
    if (threadIdx.x == 0 && dst_lse) *dst_lse = m + logf(l);
  }
}

}  // namespace attn
}  // namespace mla
