// Split-KV flash-decode over the paged latent cache, on tcgen05 tensor cores.
//
// What it computes ([LP] "Classic attention and the cost of the KV cache" and "MLA: compress
// the pair, not the heads"): for each sequence b and head h, with the absorbed query
// q = [q_lat | q_rope] (576) and cache rows c_j = [c_KV,j | k_R,j] (576),
//     s_j = scale * <q, c_j>,  p = softmax_j(s),  o_lat = sum_j p_j c_KV,j   (512 wide),
// every cached row j < len_b being visible to the newest token.
//
// Design (B200): all H = 128 heads of a sequence share every cache row, so the per-page work
// is two dense contractions, S = Q C^T ([128 x 576] x [576 x 64]) and O += P C_lat
// ([128 x 64] x [64 x 512]).  O (128 x 512 fp32) alone fills a whole SM's tensor memory, so
// each work unit runs on a CLUSTER OF TWO CTAs that split the 576 columns of every row:
//   CTA r loads latent columns [256r, 256r+256) and RoPE columns [512+32r, 512+32r+32) of
//   q_cat and of each cache page (TMA, 128B/64B swizzle), computes the partial scores of its
//   288 columns, sends them to its peer through distributed shared memory (st.async with
//   byte-counted mbarrier completion) and adds the peer's partial -- both CTAs then hold the
//   same full S and run the same online softmax -- and accumulates its own 256 columns of O.
// Per CTA the tensor memory holds O (256 cols), S double-buffered (2 x 64) and P as bf16
// (2 x 32, the A operand of the PV product read straight from TMEM); shared memory holds the
// Q half (72 KiB), a 3-stage page ring (3 x 36 KiB) and the 32 KiB score-exchange buffer.
// HBM traffic is each cache byte once.
//
// The concatenated page list of all sequences is cut into `num_parts` contiguous ranges of
// (nearly) equal length, one per cluster; a range may end inside a sequence and may span
// several.  A sequence covered by one range gets its final o_lat/lse written directly; one
// split over several ranges gets normalised partials that the combine kernel merges with
// log-sum-exp weights.
//
// Roles in each CTA (192 threads): warps 0-3 softmax (thread i owns head row i = TMEM lane i),
// warp 4 TMA producer, warp 5 MMA issuer.  Online softmax keeps a per-row reference maximum
// and rescales O only when the running maximum grows by more than 2^8.
#pragma once
#include "ptx_sm100.cuh"

namespace mla {
namespace attn {

constexpr int kThreads = 192;
constexpr int kPage = 64;
constexpr int kRow = 576;
constexpr int kStages = 3;
constexpr uint32_t kQLatBox = 128 * 128;                  // 128 rows x 64 bf16
constexpr uint32_t kQBytes = 4 * kQLatBox + 128 * 64;     // + rope box 128 rows x 32 bf16
constexpr uint32_t kCLatBox = 64 * 128;                   // 64 rows x 64 bf16
constexpr uint32_t kStageBytes = 4 * kCLatBox + 64 * 64;  // + rope box 64 rows x 32 bf16
constexpr uint32_t kXBytes = 128 * 64 * 4;                // fp32 partial scores
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffStage = kQBytes;
constexpr uint32_t kOffX = kOffStage + kStages * kStageBytes;
constexpr uint32_t kOffBar = kOffX + kXBytes;
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;  // barriers + alignment slack
// TMEM columns
constexpr uint32_t kTmemO = 0, kTmemS = 256, kTmemP = 384, kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

static_assert(kSmemBytes <= 232448, "shared memory budget");

struct Params {
  int batch;
  int n_heads;
  int max_pages;
  int num_pages;
  int num_parts;  // clusters launched
  const int32_t* page_table;
  const int32_t* seq_lens;
  const int32_t* plan;
  float scale_log2;  // softmax scale * log2(e)
  float* o_lat;      // [B][H][512]
  float* lse;        // [B][H] or null
  float* part_o;     // [slots][H][512]
  float* part_lse;   // [slots][H]
  unsigned int* status;
  uint64_t wait_ns;
};

// Plan layout (int32 words in the workspace), written by plan_kernel.
struct PlanView {
  const int32_t* base;
  int B, C;
  __host__ __device__ PlanView(const int32_t* p, int b, int c) : base(p), B(b), C(c) {}
  __host__ __device__ int total_pages() const { return base[0]; }
  __host__ __device__ int parts() const { return base[1]; }
  __host__ __device__ const int32_t* seq_pages() const { return base + 4; }
  __host__ __device__ const int32_t* seq_prefix() const { return base + 4 + B; }
  __host__ __device__ const int32_t* seq_first_part() const { return base + 4 + 2 * B + 1; }
  __host__ __device__ const int32_t* seq_nparts() const { return base + 4 + 3 * B + 1; }
  __host__ __device__ const int32_t* seq_slot() const { return base + 4 + 4 * B + 1; }
  __host__ __device__ const int32_t* part_start() const { return base + 4 + 5 * B + 1; }
  __host__ __device__ const int32_t* part_seq() const { return base + 4 + 5 * B + 2 + C; }
  __host__ __device__ static size_t words(int B, int C) { return 4 + 5 * size_t(B) + 2 + 2 * size_t(C); }
};

// ------------------------------------------------------------------------------------------
// Planner: one block.  pages per sequence, prefix sums, equal division of the page list into
// parts, which parts touch which sequence, and where each sequence's partials go.
// ------------------------------------------------------------------------------------------
constexpr int kPlanThreads = 1024;

__device__ inline int block_exclusive_scan(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[w] = x;
  __syncthreads();
  if (w == 0) {
    int s = warp_sums[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    warp_sums[lane] = s;  // inclusive
  }
  __syncthreads();
  const int before = (w > 0 ? warp_sums[w - 1] : 0) + x - v;
  if (total) *total = warp_sums[31];
  __syncthreads();
  return before;
}

__global__ void __launch_bounds__(kPlanThreads)
    plan_kernel(const int32_t* __restrict__ seq_lens, int B, int max_pages, int C_req,
                int min_pages_per_part, int32_t* __restrict__ plan, unsigned int* status) {
  __shared__ int warp_sums[32];
  __shared__ int s_total;
  int32_t* pg = plan + 4;
  int32_t* prefix = plan + 4 + B;
  int32_t* first = plan + 4 + 2 * B + 1;
  int32_t* npart = plan + 4 + 3 * B + 1;
  int32_t* slot = plan + 4 + 4 * B + 1;
  int32_t* pstart = plan + 4 + 5 * B + 1;
  int32_t* pseq = plan + 4 + 5 * B + 2 + C_req;
  const int T = blockDim.x;
  const int chunk = (B + T - 1) / T;
  const int b0 = threadIdx.x * chunk, b1 = min(B, b0 + chunk);
  const int cap = max_pages * kPage;
  // 1. pages per sequence
  int local = 0;
  for (int b = b0; b < b1; ++b) {
    int len = seq_lens[b];
    if (len < 0 || len > cap) {
      atomicOr(status, MLA_STATUS_BAD_LENGTH);
      len = len < 0 ? 0 : cap;
    }
    const int n = (len + kPage - 1) / kPage;
    pg[b] = n;
    local += n;
  }
  // 2. prefix sums
  int run = block_exclusive_scan(local, warp_sums, &s_total);
  for (int b = b0; b < b1; ++b) {
    prefix[b] = run;
    run += pg[b];
  }
  const int P = s_total;
  if (threadIdx.x == 0) prefix[B] = P;
  int C = 0;
  if (P > 0) C = max(1, min(C_req, (P + min_pages_per_part - 1) / min_pages_per_part));
  if (threadIdx.x == 0) {
    plan[0] = P;
    plan[1] = C;
  }
  // 3. equal division of the page list
  for (int c = threadIdx.x; c <= C_req; c += T)
    pstart[c] = (c <= C && C > 0) ? static_cast<int>((static_cast<int64_t>(c) * P) / C) : P;
  // 4. parts covering each sequence
  int nloc = 0;
  for (int b = b0; b < b1; ++b) {
    const int n = pg[b];
    if (n == 0) {
      first[b] = 0;
      npart[b] = 0;
      continue;
    }
    const int64_t g_first = prefix[b], g_last = prefix[b] + n - 1;
    const int pf = static_cast<int>(((g_first + 1) * C - 1) / P);
    const int pl = static_cast<int>(((g_last + 1) * C - 1) / P);
    first[b] = pf;
    npart[b] = pl - pf + 1;
    nloc += pl - pf + 1;
  }
  __syncthreads();
  int srun = block_exclusive_scan(nloc, warp_sums, nullptr);
  for (int b = b0; b < b1; ++b) {
    slot[b] = srun;
    srun += npart[b];
  }
  // 5. first sequence of each part: last b with prefix[b] <= start
  for (int c = threadIdx.x; c < C_req; c += T) {
    if (c >= C) {
      pseq[c] = B;
      continue;
    }
    const int g0 = static_cast<int>((static_cast<int64_t>(c) * P) / C);
    int lo = 0, hi = B - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (prefix[mid] <= g0) lo = mid; else hi = mid - 1;
    }
    pseq[c] = lo;
  }
}

// ------------------------------------------------------------------------------------------
// The split kernel
// ------------------------------------------------------------------------------------------
struct Bars {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t q_full, q_empty;
  uint64_t s_full[2], s_free[2];
  uint64_t p_full[2], pv_done[2];
  uint64_t x_full, x_free;
  uint64_t o_free;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

// Iterates the segments (one per sequence touched) of a part.
struct SegIter {
  const int32_t* pages;
  const int32_t* prefix;
  int B, g, g_end, b;
  __device__ bool next(int& seq, int& p0, int& p1) {
    while (g < g_end && b < B) {
      const int n = pages[b], pre = prefix[b];
      if (n == 0 || g >= pre + n) {
        ++b;
        continue;
      }
      seq = b;
      p0 = g - pre;
      p1 = min(g_end - pre, n);
      g = pre + p1;
      ++b;
      return true;
    }
    return false;
  }
};

__device__ __forceinline__ uint32_t xbuf_off(int row, int chunk) {
  return static_cast<uint32_t>(row) * 256u + static_cast<uint32_t>((chunk ^ (row & 15)) * 16);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    split_kernel(const __grid_constant__ CUtensorMap tm_q_lat,
                 const __grid_constant__ CUtensorMap tm_q_rope,
                 const __grid_constant__ CUtensorMap tm_c_lat,
                 const __grid_constant__ CUtensorMap tm_c_rope, const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + kOffBar);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int part = blockIdx.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->s_free[i], 128);
      mbar_init(&bars->p_full[i], 128);
      mbar_init(&bars->pv_done[i], 1);
    }
    mbar_init(&bars->x_full, 1);
    mbar_init(&bars->x_free, 128);
    mbar_init(&bars->o_free, 128);
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    fence_mbar_init_cluster();
    mbar_arrive_expect_tx(&bars->x_full, kXBytes);  // arm for the first tile
  }
  if (warp == 5) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // peer barriers initialised before any remote traffic
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  WaitCtx wc{&bars->abort_flag, p.status, p.wait_ns};

  const PlanView plan(p.plan, p.batch, p.num_parts);
  const int n_parts = plan.parts();
  const bool active = part < n_parts;
  const int g_begin = active ? plan.part_start()[part] : 0;
  const int g_end = active ? plan.part_start()[part + 1] : 0;
  const int b_begin = active ? plan.part_seq()[part] : p.batch;

  uint8_t* sQ = smem + kOffQ;
  uint8_t* sStage = smem + kOffStage;
  uint8_t* sX = smem + kOffX;

  if (warp == 4) {
    // =================== TMA producer ===================
    SegIter it{plan.seq_pages(), plan.seq_prefix(), p.batch, g_begin, g_end, b_begin};
    int seq, p0, p1, t = 0, sg = 0, issued_stage = 0;
    bool ok = true;
    const uint64_t pol_stream = l2_policy_evict_first();
    if (lane == 0) {
      tma_prefetch_desc(&tm_q_lat);
      tma_prefetch_desc(&tm_q_rope);
      tma_prefetch_desc(&tm_c_lat);
      tma_prefetch_desc(&tm_c_rope);
    }
    while (ok && it.next(seq, p0, p1)) {
      if (lane == 0) {
        if (sg > 0) ok = mbar_wait(&bars->q_empty, (sg - 1) & 1, wc);
        if (ok) {
          mbar_arrive_expect_tx(&bars->q_full, kQBytes);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            tma_load_3d(sQ + i * kQLatBox, &tm_q_lat, &bars->q_full, 256 * rank + 64 * i, 0, seq);
          tma_load_3d(sQ + 4 * kQLatBox, &tm_q_rope, &bars->q_full, 512 + 32 * rank, 0, seq);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      const int32_t* pt = p.page_table + static_cast<size_t>(seq) * p.max_pages;
      for (int pb = p0; ok && pb < p1; pb += 32) {
        const int cnt = min(32, p1 - pb);
        int my_page = lane < cnt ? pt[pb + lane] : 0;
        if (lane < cnt && (my_page < 0 || my_page >= p.num_pages)) {
          atomicOr(p.status, MLA_STATUS_BAD_PAGE);
          my_page = 0;
        }
        for (int j = 0; j < cnt; ++j, ++t) {
          const int page = __shfl_sync(0xffffffffu, my_page, j);
          if (lane == 0) {
            const int s = t % kStages;
            if (t >= kStages) ok = mbar_wait(&bars->empty[s], ((t / kStages) - 1) & 1, wc);
            if (ok) {
              uint8_t* dst = sStage + s * kStageBytes;
              mbar_arrive_expect_tx(&bars->full[s], kStageBytes);
              const int y = page * kPage;
#pragma unroll
              for (int i = 0; i < 4; ++i)
                tma_load_2d_hint(dst + i * kCLatBox, &tm_c_lat, &bars->full[s],
                                 256 * rank + 64 * i, y, pol_stream);
              tma_load_2d_hint(dst + 4 * kCLatBox, &tm_c_rope, &bars->full[s], 512 + 32 * rank,
                               y, pol_stream);
              issued_stage = t + 1;
            }
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
        }
      }
      ++sg;
    }
    if (lane == 0 && bars->abort_flag) {
      volatile int never = 0;
      WaitCtx drain{&never, p.status, p.wait_ns};
      for (int i = max(0, issued_stage - kStages); i < issued_stage; ++i)
        mbar_wait(&bars->full[i % kStages], (i / kStages) & 1, drain);
      if (sg > 0) mbar_wait(&bars->q_full, (sg - 1) & 1, drain);
    }
  } else if (warp == 5) {
    // =================== MMA issuer ===================
    if (lane == 0) {
      const uint32_t idesc_qk = idesc_bf16(128, 64, 0, 0);
      const uint32_t idesc_pv = idesc_bf16(128, 256, 0, 1);
      const uint32_t q_base = smem_u32(sQ);
      SegIter it{plan.seq_pages(), plan.seq_prefix(), p.batch, g_begin, g_end, b_begin};
      int seq, p0, p1, t = 0, sg = 0;
      bool ok = true;
      auto issue_pv = [&](int tt, bool first_of_seg) -> bool {
        if (first_of_seg && sg > 0 && !mbar_wait(&bars->o_free, (sg - 1) & 1, wc)) return false;
        if (!mbar_wait(&bars->p_full[tt & 1], (tt >> 1) & 1, wc)) return false;
        tc_fence_after();
        const uint32_t st = smem_u32(sStage + (tt % kStages) * kStageBytes);
        const uint32_t a_tmem = tmem + kTmemP + (tt & 1) * 32;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t bdesc = smem_desc(st + kk * 2048, 8192, 1024, kSwizzle128B);
          mma_ts(tmem + kTmemO, a_tmem + kk * 8, bdesc, idesc_pv,
                 (first_of_seg && kk == 0) ? 0u : 1u);
        }
        mma_commit(&bars->pv_done[tt & 1]);
        mma_commit(&bars->empty[tt % kStages]);
        return true;
      };
      while (ok && it.next(seq, p0, p1)) {
        const int n_tiles = p1 - p0;
        ok = mbar_wait(&bars->q_full, sg & 1, wc);
        for (int i = 0; ok && i < n_tiles; ++i, ++t) {
          const int s = t % kStages;
          const int sb = t & 1;
          if (!mbar_wait(&bars->full[s], (t / kStages) & 1, wc)) { ok = false; break; }
          if (t >= 2 && !mbar_wait(&bars->s_free[sb], ((t >> 1) - 1) & 1, wc)) { ok = false; break; }
          tc_fence_after();
          const uint32_t st = smem_u32(sStage + s * kStageBytes);
          const uint32_t d = tmem + kTmemS + sb * 64;
          int n_mma = 0;
#pragma unroll
          for (int box = 0; box < 4; ++box)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk, ++n_mma)
              mma_ss(d, smem_desc(q_base + box * kQLatBox + kk * 32, 16, 1024, kSwizzle128B),
                     smem_desc(st + box * kCLatBox + kk * 32, 16, 1024, kSwizzle128B), idesc_qk,
                     n_mma > 0 ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            mma_ss(d, smem_desc(q_base + 4 * kQLatBox + kk * 32, 16, 512, kSwizzle64B),
                   smem_desc(st + 4 * kCLatBox + kk * 32, 16, 512, kSwizzle64B), idesc_qk, 1u);
          mma_commit(&bars->s_full[sb]);
          if (i == n_tiles - 1) mma_commit(&bars->q_empty);
          if (i > 0 && !issue_pv(t - 1, i == 1)) { ok = false; break; }
        }
        if (ok && !issue_pv(t - 1, n_tiles == 1)) ok = false;
        ++sg;
      }
      // no MMA may be in flight when TMEM is released
      if (bars->abort_flag) {
        mma_commit(&bars->drain);
        volatile int never = 0;
        WaitCtx drain{&never, p.status, p.wait_ns};
        mbar_wait(&bars->drain, 0, drain);
      }
    }
  } else {
    // =================== softmax / correction / epilogue (warps 0-3) ===================
    const int row = threadIdx.x;  // head row = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t x_base = smem_u32(sX);
    const uint32_t peer_x_base = mapa_shared(smem_u32(sX), peer);
    const uint32_t peer_xfull = mapa_shared(smem_u32(&bars->x_full), peer);
    const uint32_t peer_xfree = mapa_shared(smem_u32(&bars->x_free), peer);
    SegIter it{plan.seq_pages(), plan.seq_prefix(), p.batch, g_begin, g_end, b_begin};
    int seq, p0, p1, t = 0, sg = 0;
    bool ok = true;
    const float NEG_INF = -__int_as_float(0x7f800000);
    while (ok && it.next(seq, p0, p1)) {
      const int n_tiles = p1 - p0;
      const int len = min(p.seq_lens[seq], p.max_pages * kPage);
      float m_ref = NEG_INF, l_sum = 0.f;
      for (int i = 0; ok && i < n_tiles; ++i, ++t) {
        const int sb = t & 1;
        if (!warp_wait(&bars->s_full[sb], (t >> 1) & 1, wc)) { ok = false; break; }
        tc_fence_after();
        float s[64];
        {
          uint32_t r[32];
          tmem_ld32(tmem + kTmemS + sb * 64 + lane_off, r);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) s[k] = __uint_as_float(r[k]);
          tmem_ld32(tmem + kTmemS + sb * 64 + 32 + lane_off, r);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) s[32 + k] = __uint_as_float(r[k]);
        }
        tc_fence_before();
        mbar_arrive(&bars->s_free[sb]);
        // ---- exchange partial scores with the peer CTA ----
        if (t >= 1 && !warp_wait<true>(&bars->x_free, (t - 1) & 1, wc)) { ok = false; break; }
#pragma unroll
        for (int c = 0; c < 16; ++c)
          st_async_v4(peer_x_base + xbuf_off(row, c), s[4 * c], s[4 * c + 1], s[4 * c + 2],
                      s[4 * c + 3], peer_xfull);
        if (!warp_wait<true>(&bars->x_full, t & 1, wc)) { ok = false; break; }
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          float4 v;
          asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                       : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                       : "r"(x_base + xbuf_off(row, c)));
          s[4 * c] += v.x;
          s[4 * c + 1] += v.y;
          s[4 * c + 2] += v.z;
          s[4 * c + 3] += v.w;
        }
        mbar_arrive_remote(peer_xfree);
        if (row == 0) mbar_arrive_expect_tx(&bars->x_full, kXBytes);
        // ---- online softmax (identical in both CTAs) ----
        const int valid = min(kPage, len - (p0 + i) * kPage);
        float mx = NEG_INF;
#pragma unroll
        for (int k = 0; k < 64; ++k) {
          s[k] = (k < valid) ? s[k] * p.scale_log2 : NEG_INF;
          mx = fmaxf(mx, s[k]);
        }
        float alpha = 1.f;
        bool rescale = false;
        if (i == 0) {
          m_ref = mx;
        } else if (mx > m_ref + kRescaleThreshold) {
          alpha = ex2_approx(m_ref - mx);
          m_ref = mx;
          rescale = true;
        }
        float rs = 0.f;
        uint32_t pk[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          const float e0 = ex2_approx(s[2 * k] - m_ref);
          const float e1 = ex2_approx(s[2 * k + 1] - m_ref);
          rs += e0 + e1;
          pk[k] = pack_bf16x2(e0, e1);
        }
        l_sum = l_sum * alpha + rs;
        if (__any_sync(0xffffffffu, rescale)) {
          // O must hold PV of the previous tile before it is rescaled
          const int tp = t - 1;
          if (!warp_wait(&bars->pv_done[tp & 1], (tp >> 1) & 1, wc)) { ok = false; break; }
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < 256; c += 32) {
            uint32_t r[32];
            tmem_ld32(tmem + kTmemO + c + lane_off, r);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; ++k) r[k] = __float_as_uint(__uint_as_float(r[k]) * alpha);
            tmem_st32(tmem + kTmemO + c + lane_off, r);
          }
          tmem_wait_st();
        }
        tmem_st32(tmem + kTmemP + sb * 32 + lane_off, pk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->p_full[sb]);
      }
      if (!ok) break;
      // ---- segment epilogue: O / l -> global ----
      const int tl = t - 1;
      if (!warp_wait(&bars->pv_done[tl & 1], (tl >> 1) & 1, wc)) { ok = false; break; }
      tc_fence_after();
      const int nparts = plan.seq_nparts()[seq];
      const float lse_nat = (m_ref + __log2f(l_sum)) * 0.69314718055994531f;
      const float inv_l = 1.f / l_sum;
      float* dst;
      float* dst_lse;
      if (nparts == 1) {
        dst = p.o_lat + (static_cast<size_t>(seq) * p.n_heads + row) * 512 + 256 * rank;
        dst_lse = p.lse ? p.lse + static_cast<size_t>(seq) * p.n_heads + row : nullptr;
      } else {
        const int slot = plan.seq_slot()[seq] + (part - plan.seq_first_part()[seq]);
        dst = p.part_o + (static_cast<size_t>(slot) * p.n_heads + row) * 512 + 256 * rank;
        dst_lse = p.part_lse + static_cast<size_t>(slot) * p.n_heads + row;
      }
      const bool row_ok = row < p.n_heads;
#pragma unroll 1
      for (int c = 0; c < 256; c += 32) {
        uint32_t r[32];
        tmem_ld32(tmem + kTmemO + c + lane_off, r);
        tmem_wait_ld();
        if (row_ok) {
          float4* d4 = reinterpret_cast<float4*>(dst + c);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            d4[k] = make_float4(__uint_as_float(r[4 * k]) * inv_l, __uint_as_float(r[4 * k + 1]) * inv_l,
                                __uint_as_float(r[4 * k + 2]) * inv_l,
                                __uint_as_float(r[4 * k + 3]) * inv_l);
        }
      }
      if (row_ok && rank == 0 && dst_lse) *dst_lse = lse_nat;
      tc_fence_before();
      mbar_arrive(&bars->o_free);
      ++sg;
    }
    // the peer's last remote operations on this CTA's shared memory must have landed
    if (t > 0) {
      volatile int never = 0;
      WaitCtx drain{&never, p.status, p.wait_ns};
      mbar_wait<true>(&bars->x_free, (t - 1) & 1, ok ? wc : drain);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  cluster_sync();
}

// ------------------------------------------------------------------------------------------
// Combine: log-sum-exp merge of the parts of sequences split over several ranges.
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(128)
    combine_kernel(const int32_t* __restrict__ plan_words, int B, int C, int H,
                   const float* __restrict__ part_o, const float* __restrict__ part_lse,
                   float* __restrict__ o_lat, float* __restrict__ lse) {
  const PlanView plan(plan_words, B, C);
  const int h = blockIdx.x, b = blockIdx.y;
  const int n = plan.seq_nparts()[b];
  if (n == 1) return;
  float4* out = reinterpret_cast<float4*>(o_lat + (static_cast<size_t>(b) * H + h) * 512);
  if (n == 0) {
    out[threadIdx.x] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (threadIdx.x == 0 && lse) lse[static_cast<size_t>(b) * H + h] = -__int_as_float(0x7f800000);
    return;
  }
  const int slot0 = plan.seq_slot()[b];
  float m = -__int_as_float(0x7f800000);
  for (int s = 0; s < n; ++s) m = fmaxf(m, part_lse[static_cast<size_t>(slot0 + s) * H + h]);
  float tot = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s = 0; s < n; ++s) {
    const float w = __expf(part_lse[static_cast<size_t>(slot0 + s) * H + h] - m);
    tot += w;
    const float4 v = reinterpret_cast<const float4*>(
        part_o + (static_cast<size_t>(slot0 + s) * H + h) * 512)[threadIdx.x];
    acc.x += w * v.x;
    acc.y += w * v.y;
    acc.z += w * v.z;
    acc.w += w * v.w;
  }
  const float inv = 1.f / tot;
  out[threadIdx.x] = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  if (threadIdx.x == 0 && lse) lse[static_cast<size_t>(b) * H + h] = m + __logf(tot);
}

}  // namespace attn
}  // namespace mla
