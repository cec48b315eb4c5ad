// Split-KV flash-decode over the paged latent cache, on tcgen05 tensor cores.
//
// What it computes ([LP] "Classic attention and the cost of the KV cache" and "MLA: compress
// the pair, not the heads"): for each sequence b and head h, with the absorbed query
// q = [q_lat | q_rope] (576) and cache rows c_j = [c_KV,j | k_R,j] (576),
//     s_j = scale * <q, c_j>,  p = softmax_j(s),  o_lat = sum_j p_j c_KV,j   (512 wide),
// every cached row j < len_b being visible to the newest token.
//
// Design (B200).  All H = 128 heads of a sequence share every cache row, so the per-page work
// is two dense contractions, S = Q C^T ([128 x 576] x [576 x 64]) and O += P C_lat
// ([128 x 64] x [64 x 512]).  O (128 x 512 fp32) alone would fill a whole SM's tensor memory,
// so each work unit runs on a CLUSTER OF TWO CTAs that split the 576 columns of every row:
// CTA r owns latent columns [256r, 256r+256) and RoPE columns [512+32r, 512+32r+32).
//   * TMEM (512 columns): O half 256 | query latent half 128 (A operand of QK) | two S
//     buffers of 64.  The 32 RoPE columns of the query half sit in shared memory (A operand,
//     64B swizzle), and so does P (bf16, 128B swizzle, A operand of PV), so an S buffer is
//     free again as soon as it has been drained and QK runs two pages ahead of the softmax.
//   * Pages arrive by TMA (128B/64B swizzle) into a 4-stage ring; each byte leaves HBM once.
//     Four pages ahead of the ring each CTA issues a bulk L2 prefetch of half of the page's
//     rows, so the ring's loads find their lines in L2.
//   * S_r = Q_r C_r^T is a partial score; the pair exchanges partials.  Distributed shared
//     memory moves ~16 B/clk per SM, so a partial travels as 16-bit fixed point relative to
//     its row's largest magnitude (error <= 2^-16 of it, ~1e-4 in the softmax logit), staged
//     in shared memory and sent with ONE bulk copy (cp.async.bulk, completion counted in bytes
//     on the peer's mbarrier).
//   * Two warpgroups share the per-page softmax work: the "send" warpgroup drains S_t,
//     quantises and stages it; the "softmax" warpgroup drains S_t again, adds the peer's
//     decoded partial, runs the online softmax and writes P_t.  With S double-buffered, QK of
//     page t+1 and the exchange of page t+1 run while page t is being softmaxed.
//   * Each CTA normalises its own half of O with its own running sum (its copy of the scores
//     differs from the peer's only by the 16-bit rounding of the received half), so the halves
//     need no further agreement.
//
// The concatenated page list of all sequences is cut into `num_parts` contiguous ranges of
// (nearly) equal length, one per cluster; a range may end inside a sequence and may span
// several.  A sequence covered by one range gets its final o_lat/lse written directly; one
// split over several ranges gets normalised partials that the combine kernel merges with
// log-sum-exp weights.
//
// Extended-precision query.  Rounding the absorbed query to bf16 perturbs every logit by about
// 2^-9 of its size; with large logits (inputs scaled x4 give a logit spread of ~16) that is
// enough to move the output by ~1e-2.  When the caller passes the rounding remainder q_lo as
// well (q = q_cat + q_lo to ~16 bits), each cluster takes 64 heads instead of 128 and stacks,
// for each of them, a row of q_cat and a row of q_lo in the 128 rows of the MMA: in every
// quarter of the rows (one warp's TMEM lanes), rows 0-15 hold heads 16w..16w+15 of the group
// from q_cat and rows 16-31 the same heads from q_lo.  The score of a head is then the sum of
// its two rows (one shuffle), the softmax runs identically on both rows, O gets the same P in
// both, and only the q_cat row is written out.  Launch: `groups` = ceil(H/64) clusters per
// part, so the tensor work per token doubles; the page bytes are read by the part's clusters
// at about the same time and mostly come from L2 the second time.
//
// Roles (384 threads): warps 0-3 softmax + epilogue (thread i owns head row i = TMEM lane i),
// warps 4-7 send, warp 8 TMA producer, warp 9 MMA issuer, warp 10 bulk-copy sender (warp 11
// has no role).  Each softmax warp hands its rows of the receive buffer back to the peer
// itself once it has decoded them.  The online softmax keeps a per-row reference maximum and rescales O
// only when the running maximum grows by more than 2^8.
#pragma once
#include "ptx_sm100.cuh"

namespace mla {
namespace attn {

constexpr int kThreads = 384;
constexpr int kPage = 64;
constexpr int kRow = 576;
constexpr int kStages = 4;
constexpr uint32_t kCLatBox = 64 * 128;                   // 64 rows x 64 bf16
constexpr uint32_t kStageBytes = 4 * kCLatBox + 64 * 64;  // + rope box 64 rows x 32 bf16
constexpr uint32_t kXPayload = 128 * 128;                 // 128 rows x 64 x 16-bit
constexpr uint32_t kXBytes = kXPayload + 128 * 4;         // + one fp32 step per row
constexpr uint32_t kQRopeBytes = 128 * 64;                // 128 rows x 32 bf16
constexpr uint32_t kPBytes = 128 * 128;                   // P: 128 rows x 64 bf16
constexpr uint32_t kOffStage = 0;
constexpr uint32_t kOffP = kOffStage + kStages * kStageBytes;  // one P buffer
constexpr uint32_t kOffQRope = kOffP + kPBytes;
constexpr uint32_t kOffSend = kOffQRope + kQRopeBytes;  // two send buffers
constexpr uint32_t kOffRecv = kOffSend + 2 * kXBytes;   // one receive buffer
constexpr uint32_t kOffBar = kOffRecv + kXBytes;
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;  // barriers + alignment slack
// TMEM columns
constexpr uint32_t kTmemO = 0, kTmemQ = 256, kTmemS = 384, kTmemCols = 512;
constexpr int kAhead = 4;  // pages prefetched into L2 ahead of the TMA ring
constexpr uint32_t kPageBytes = kPage * kRow * 2;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(kTmemS + 2 * 64 == kTmemCols, "tensor memory budget");
static_assert(kXBytes % 16 == 0 && kOffP % 1024 == 0 && kOffQRope % 1024 == 0, "alignment");

struct Params {
  int batch;
  int n_heads;
  int max_pages;
  int num_pages;
  int num_parts;  // ranges of the page list (the plan's parts)
  int groups;     // clusters per part: 1, or ceil(H / 64) with the query remainder (q_lo)
  const __nv_bfloat16* q_cat;  // [B][H][576]
  const __nv_bfloat16* q_lo;   // [B][H][576] rounding remainder of the query, or null
  const uint8_t* pool;         // cache pages, [num_pages][64][576] bf16
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

// Pages of sequence b, its length clamped to the cache (a bad length is reported once, by the
// thread that first reads it).
__device__ inline int plan_pages(const int32_t* seq_lens, int b, int cap, unsigned int* status) {
  int len = seq_lens[b];
  if (len < 0 || len > cap) {
    if (status) atomicOr(status, MLA_STATUS_BAD_LENGTH);
    len = len < 0 ? 0 : cap;
  }
  return (len + kPage - 1) / kPage;
}

// The part that holds global page g of the concatenated list (g = -1 gives -1).
__device__ inline int part_of_page(int64_t g, int C, int P) {
  return g < 0 ? -1 : static_cast<int>(((g + 1) * C - 1) / P);
}

// Every value a thread needs comes from its own sequences and two block-wide scans: the parts
// whose first page lies inside sequence b are written by b's thread, so no thread searches the
// prefix sums that other threads wrote.
__global__ void __launch_bounds__(kPlanThreads)
    plan_kernel(const int32_t* __restrict__ seq_lens, int B, int max_pages, int C_req,
                int min_pages_per_part, int32_t* __restrict__ plan, unsigned int* status) {
  griddep_launch_dependents();
  griddep_wait();
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
  // 1. pages of this thread's sequences, and their exclusive prefix over the whole batch
  int local = 0;
  for (int b = b0; b < b1; ++b) local += plan_pages(seq_lens, b, cap, status);
  const int run0 = block_exclusive_scan(local, warp_sums, &s_total);
  const int P = s_total;
  int C = 0;
  if (P > 0) C = max(1, min(C_req, (P + min_pages_per_part - 1) / min_pages_per_part));
  if (threadIdx.x == 0) {
    plan[0] = P;
    plan[1] = C;
    prefix[B] = P;
  }
  // 2. equal division of the page list; parts beyond C are empty and start no sequence
  for (int c = threadIdx.x; c <= C_req; c += T) {
    pstart[c] = (c <= C && C > 0) ? static_cast<int>((static_cast<int64_t>(c) * P) / C) : P;
    if (c < C_req && c >= C) pseq[c] = B;
  }
  // 3. per sequence: its pages, prefix, the parts that cover it, and the parts starting in it
  int run = run0, nloc = 0;
  for (int b = b0; b < b1; ++b) {
    const int n = plan_pages(seq_lens, b, cap, nullptr);
    pg[b] = n;
    prefix[b] = run;
    if (n == 0) {
      first[b] = 0;
      npart[b] = 0;
      continue;
    }
    const int pf = part_of_page(run, C, P);
    const int pl = part_of_page(static_cast<int64_t>(run) + n - 1, C, P);
    first[b] = pf;
    npart[b] = pl - pf + 1;
    nloc += pl - pf + 1;
    for (int c = part_of_page(static_cast<int64_t>(run) - 1, C, P) + 1; c <= pl; ++c) pseq[c] = b;
    run += n;
  }
  // 4. where each sequence's partials go
  int srun = block_exclusive_scan(nloc, warp_sums, nullptr);
  run = run0;
  for (int b = b0; b < b1; ++b) {
    const int n = plan_pages(seq_lens, b, cap, nullptr);
    slot[b] = srun;
    if (n > 0)
      srun += part_of_page(static_cast<int64_t>(run) + n - 1, C, P) - part_of_page(run, C, P) + 1;
    run += n;
  }
}

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

// Exchange buffer row layout: 8 chunks of 16 B, XOR-swizzled so that 8 consecutive rows hit
// 8 different bank groups.
__device__ __forceinline__ uint32_t xrow_off(int row, int chunk) {
  return static_cast<uint32_t>(row) * 128u + static_cast<uint32_t>((chunk ^ (row & 7)) * 16);
}

// Reductions over a row's 64 values as 8 independent chains (a single 64-long chain of
// dependent instructions would dominate a page's softmax time).
__device__ __forceinline__ float max64(const float* s) {
  float m[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) m[j] = s[j];
#pragma unroll
  for (int k = 8; k < 64; ++k) m[k & 7] = fmaxf(m[k & 7], s[k]);
  return fmaxf(fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3])),
               fmaxf(fmaxf(m[4], m[5]), fmaxf(m[6], m[7])));
}
__device__ __forceinline__ float maxabs64(const float* s) {
  float m[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) m[j] = fabsf(s[j]);
#pragma unroll
  for (int k = 8; k < 64; ++k) m[k & 7] = fmaxf(m[k & 7], fabsf(s[k]));
  return fmaxf(fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3])),
               fmaxf(fmaxf(m[4], m[5]), fmaxf(m[6], m[7])));
}

// 16-bit fixed point (offset binary: u = q + 32768 for q in [-32767, 32767]) without the
// quarter-rate int<->float conversion instructions.  Encoding: fma(x, 1/step, 1.5*2^23 + 32768)
// rounds to nearest even and leaves u in the low 16 mantissa bits.  Decoding: the bits
// 0x4B000000 | u are the float 2^23 + u exactly.
constexpr float kEncBias = 12615680.0f;  // 1.5 * 2^23 + 32768
constexpr float kDecBias = 8421376.0f;   // 2^23 + 32768
constexpr uint32_t kDecBits = 0x4B000000u;

__device__ __forceinline__ uint32_t enc_u16x2(float a, float b, float inv_step) {
  const uint32_t ua = __float_as_uint(fmaf(a, inv_step, kEncBias));
  const uint32_t ub = __float_as_uint(fmaf(b, inv_step, kEncBias));
  return __byte_perm(ua, ub, 0x5410);  // low halves: a -> bits 0-15, b -> bits 16-31
}
__device__ __forceinline__ float dec_lo(uint32_t v) {
  return __uint_as_float(__byte_perm(v, kDecBits, 0x7610)) - kDecBias;
}
__device__ __forceinline__ float dec_hi(uint32_t v) {
  return __uint_as_float(__byte_perm(v, kDecBits, 0x7632)) - kDecBias;
}


// ------------------------------------------------------------------------------------------
// The split kernel
// ------------------------------------------------------------------------------------------
// Every mbarrier below completes one phase per use and is waited phase by phase, never more
// than one phase behind its current state (buffers that could run two pages ahead of their
// waiter have one barrier per buffer), so parity waits cannot alias.
struct Bars {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t q_full;        // TMA: the segment's query RoPE half landed in shared memory
  uint64_t q_empty;       // MMA: the segment's last QK finished (commit)
  uint64_t q_ready;       // softmax WG: the segment's query latent half is in TMEM (128)
  uint64_t s_full[2];     // MMA: S buffer i written (commit)
  uint64_t s_free[2];     // both warpgroups drained S buffer i (256)
  uint64_t staged[2];     // send WG: partial staged in send[i] (128)
  uint64_t p_full;        // softmax WG: P written (128)
  uint64_t pv_done;       // MMA: PV finished, P buffer free (commit, once per page)
  uint64_t x_full;        // the peer's partial landed in recv (bulk-copy bytes)
  uint64_t peer_done[2];  // the peer's 4 softmax warps decoded our partial of a page of
                          // parity i (4 remote arrivals)
  uint64_t o_free;        // softmax WG: the epilogue drained O (128)
  uint64_t seg_done;      // MMA: every PV of the segment finished (commit, once per segment)
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    split_kernel(const __grid_constant__ CUtensorMap tm_c_lat,
                 const __grid_constant__ CUtensorMap tm_c_rope,
                 const __grid_constant__ CUtensorMap tm_q_rope,
                 const __grid_constant__ CUtensorMap tm_ql_rope, const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + kOffBar);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  // clusters of one part are adjacent, so they stream the same pages at about the same time
  const int part = static_cast<int>(blockIdx.x >> 1) / p.groups;
  const int group = static_cast<int>(blockIdx.x >> 1) - part * p.groups;
  const bool hi_lo = p.q_lo != nullptr;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    mbar_init(&bars->q_ready, 128);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->s_free[i], 256);
      mbar_init(&bars->staged[i], 128);
      mbar_init(&bars->peer_done[i], 4);
    }
    mbar_init(&bars->p_full, 128);
    mbar_init(&bars->pv_done, 1);
    mbar_init(&bars->x_full, 1);
    mbar_init(&bars->o_free, 128);
    mbar_init(&bars->seg_done, 1);
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    fence_mbar_init_cluster();
    mbar_arrive_expect_tx(&bars->x_full, kXBytes);  // armed for page 0
  }
  if (warp == 9) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // peer barriers initialised before any remote traffic
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  WaitCtx wc{&bars->abort_flag, p.status, p.wait_ns};
  // everything below reads what the preceding kernels wrote (plan, q_cat, the appended rows)
  griddep_launch_dependents();
  griddep_wait();

  const PlanView plan(p.plan, p.batch, p.num_parts);
  const int n_parts = plan.parts();
  const bool active = part < n_parts;
  const int g_begin = active ? plan.part_start()[part] : 0;
  const int g_end = active ? plan.part_start()[part + 1] : 0;
  const int b_begin = active ? plan.part_seq()[part] : p.batch;
  uint8_t* sStage = smem + kOffStage;
  uint8_t* sQRope = smem + kOffQRope;
  const uint32_t send_base = smem_u32(smem + kOffSend);
  const uint32_t recv_base = smem_u32(smem + kOffRecv);

  if (warp == 8) {
    // =================== TMA producer: page ring + query RoPE half ===================
    SegIter it{plan.seq_pages(), plan.seq_prefix(), p.batch, g_begin, g_end, b_begin};
    int seq, p0, p1, t = 0, sg = 0, issued = 0;
    bool ok = true;
    const uint64_t pol_stream = l2_policy_evict_first();
    if (lane == 0) {
      tma_prefetch_desc(&tm_c_lat);
      tma_prefetch_desc(&tm_c_rope);
      tma_prefetch_desc(&tm_q_rope);
      if (hi_lo) tma_prefetch_desc(&tm_ql_rope);
    }
    while (ok && it.next(seq, p0, p1)) {
      if (lane == 0) {
        if (sg > 0) ok = mbar_wait(&bars->q_empty, (sg - 1) & 1, wc);
        if (ok) {
          mbar_arrive_expect_tx(&bars->q_full, kQRopeBytes);
          if (!hi_lo) {
            tma_load_3d(sQRope, &tm_q_rope, &bars->q_full, 512 + 32 * rank, 0, seq);
          } else {
            // 16-row boxes: rows 32w..32w+15 from q_cat, rows 32w+16..32w+31 from q_lo, both
            // for heads 64 group + 16w .. +15 (rows past H are zero-filled by the copy)
#pragma unroll
            for (int w4 = 0; w4 < 4; ++w4) {
              const int h0 = 64 * group + 16 * w4;
              tma_load_3d(sQRope + (32 * w4) * 64, &tm_q_rope, &bars->q_full, 512 + 32 * rank,
                          h0, seq);
              tma_load_3d(sQRope + (32 * w4 + 16) * 64, &tm_ql_rope, &bars->q_full,
                          512 + 32 * rank, h0, seq);
            }
          }
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
        // warm L2 ahead of the ring: each CTA of the pair fetches half of a page's rows
        if (lane < min(cnt, kAhead))
          prefetch_l2(p.pool + static_cast<size_t>(my_page) * kPageBytes + rank * (kPageBytes / 2),
                      kPageBytes / 2);
        for (int j = 0; j < cnt; ++j, ++t) {
          const int page = __shfl_sync(0xffffffffu, my_page, j);
          const int later = __shfl_sync(0xffffffffu, my_page, min(j + kAhead, 31));
          if (lane == 0 && j + kAhead < cnt)
            prefetch_l2(p.pool + static_cast<size_t>(later) * kPageBytes + rank * (kPageBytes / 2),
                        kPageBytes / 2);
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
              issued = t + 1;
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
      for (int i = max(0, issued - kStages); i < issued; ++i)
        mbar_wait(&bars->full[i % kStages], (i / kStages) & 1, drain);
      if (sg > 0) mbar_wait(&bars->q_full, (sg - 1) & 1, drain);
    }
  } else if (warp == 9) {
    // =================== MMA issuer ===================
    if (lane == 0) {
      const uint32_t idesc_qk = idesc_bf16(128, 64, 0, 0);
      const uint32_t idesc_pv = idesc_bf16(128, 256, 0, 1);
      const uint32_t qrope = smem_u32(sQRope);
      SegIter it{plan.seq_pages(), plan.seq_prefix(), p.batch, g_begin, g_end, b_begin};
      int seq, p0, p1, t = 0, sg = 0;
      bool ok = true;
      // S_tt = Q_r C_r^T into S buffer tt & 1: latent half A from TMEM, RoPE half A from smem
      auto issue_qk = [&](int tt, bool last_of_seg) -> bool {
        const int s = tt % kStages;
        if (!mbar_wait(&bars->full[s], (tt / kStages) & 1, wc)) return false;
        tc_fence_after();
        const uint32_t st = smem_u32(sStage + s * kStageBytes);
        const uint32_t d = tmem + kTmemS + (tt & 1) * 64;
#pragma unroll
        for (int j = 0; j < 16; ++j)
          mma_ts(d, tmem + kTmemQ + 8 * j,
                 smem_desc(st + (j >> 2) * kCLatBox + (j & 3) * 32, 16, 1024, kSwizzle128B),
                 idesc_qk, j > 0 ? 1u : 0u);
#pragma unroll
        for (int j = 0; j < 2; ++j)
          mma_ss(d, smem_desc(qrope + j * 32, 16, 512, kSwizzle64B),
                 smem_desc(st + 4 * kCLatBox + j * 32, 16, 512, kSwizzle64B), idesc_qk, 1u);
        mma_commit(&bars->s_full[tt & 1]);
        if (last_of_seg) mma_commit(&bars->q_empty);
        return true;
      };
      // O += P_tt C_lat: A = P (bf16, shared memory), B = the page's latent half
      const uint32_t p_base = smem_u32(smem + kOffP);
      auto issue_pv = [&](int tt, bool first_of_seg) -> bool {
        if (first_of_seg && sg > 0 && !mbar_wait(&bars->o_free, (sg - 1) & 1, wc)) return false;
        if (!mbar_wait(&bars->p_full, tt & 1, wc)) return false;
        tc_fence_after();
        const uint32_t st = smem_u32(sStage + (tt % kStages) * kStageBytes);
        const uint32_t pa = p_base;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ss(tmem + kTmemO, smem_desc(pa + kk * 32, 16, 1024, kSwizzle128B),
                 smem_desc(st + kk * 2048, 8192, 1024, kSwizzle128B), idesc_pv,
                 (first_of_seg && kk == 0) ? 0u : 1u);
        mma_commit(&bars->pv_done);
        mma_commit(&bars->empty[tt % kStages]);
        return true;
      };
      // S buffer of page tt (tt >= 2) is free once both warpgroups drained page tt - 2
      auto s_ready = [&](int tt) -> bool {
        return tt < 2 || mbar_wait(&bars->s_free[tt & 1], ((tt >> 1) - 1) & 1, wc);
      };
      while (ok && it.next(seq, p0, p1)) {
        const int n = p1 - p0, t0 = t;
        ok = mbar_wait(&bars->q_ready, sg & 1, wc) && mbar_wait(&bars->q_full, sg & 1, wc);
        if (ok) ok = s_ready(t0) && issue_qk(t0, n == 1);
        if (ok && n > 1) ok = s_ready(t0 + 1) && issue_qk(t0 + 1, n == 2);
        // softmax order per page: drain S_i (s_free) ... write P_i (p_full)
        for (int i = 0; ok && i < n; ++i) {
          const int tt = t0 + i;
          if (i + 2 < n && !(ok = s_ready(tt + 2) && issue_qk(tt + 2, i + 3 == n))) break;
          if (!(ok = issue_pv(tt, i == 0))) break;
        }
        if (ok) mma_commit(&bars->seg_done);
        t += n;
        ++sg;
      }
      if (bars->abort_flag) {  // no MMA may be in flight when TMEM is released
        mma_commit(&bars->drain);
        volatile int never = 0;
        WaitCtx drain{&never, p.status, p.wait_ns};
        mbar_wait(&bars->drain, 0, drain);
      }
    }
  } else if (warp == 10) {
    // =================== exchange: bulk copies out ===================
    if (lane == 0) {
      const uint32_t peer_recv = mapa_shared(recv_base, peer);
      const uint32_t peer_xfull = mapa_shared(smem_u32(&bars->x_full), peer);
      SegIter it{plan.seq_pages(), plan.seq_prefix(), p.batch, g_begin, g_end, b_begin};
      int seq, p0, p1, t = 0;
      bool ok = true;
      while (ok && it.next(seq, p0, p1)) {
        const int n = p1 - p0;
        for (int tt = t; ok && tt < t + n; ++tt) {
          const int buf = tt & 1;
          // the page's partial is staged in send[buf] and the peer's (single) receive buffer
          // has been decoded for page tt - 1: ship it
          if (!(ok = mbar_wait(&bars->staged[buf], (tt >> 1) & 1, wc))) break;
          if (tt >= 1 && !(ok = mbar_wait<true>(&bars->peer_done[(tt - 1) & 1],
                                               ((tt - 1) >> 1) & 1, wc)))
            break;
          bulk_copy_s2cluster(peer_recv, send_base + buf * kXBytes, kXBytes, peer_xfull);
        }
        t += n;
      }
    }
  } else if (warp == 11) {
    // no role
  } else if (warp >= 4) {
    // =================== send warpgroup (warps 4-7) ===================
    const int row = threadIdx.x - 128;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    SegIter it{plan.seq_pages(), plan.seq_prefix(), p.batch, g_begin, g_end, b_begin};
    int seq, p0, p1, t = 0;
    bool ok = true;
    while (ok && it.next(seq, p0, p1)) {
      const int n = p1 - p0;
      const int len = min(p.seq_lens[seq], p.max_pages * kPage);
      for (int i = 0; i < n; ++i) {
        const int tt = t + i, buf = tt & 1;
        if (!(ok = warp_wait(&bars->s_full[buf], (tt >> 1) & 1, wc))) break;
        tc_fence_after();
        float s[64];
        {
          uint32_t r[32];
          tmem_ld32(tmem + kTmemS + buf * 64 + lane_off, r);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) s[k] = __uint_as_float(r[k]);
          tmem_ld32(tmem + kTmemS + buf * 64 + 32 + lane_off, r);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) s[32 + k] = __uint_as_float(r[k]);
        }
        tc_fence_before();
        mbar_arrive(&bars->s_free[buf]);
        const int valid = min(kPage, len - (p0 + i) * kPage);
        if (valid < kPage) {
#pragma unroll
          for (int k = 0; k < 64; ++k) s[k] = k < valid ? s[k] : 0.f;  // never sent
        }
        const float mabs = maxabs64(s);
        const float inv = mabs > 0.f ? 32767.f / mabs : 0.f;
        if (tt >= 2 && !(ok = warp_wait<true>(&bars->peer_done[buf], ((tt >> 1) - 1) & 1, wc)))
          break;
        const uint32_t base = send_base + buf * kXBytes;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint32_t a = enc_u16x2(s[8 * c], s[8 * c + 1], inv);
          const uint32_t b = enc_u16x2(s[8 * c + 2], s[8 * c + 3], inv);
          const uint32_t cc = enc_u16x2(s[8 * c + 4], s[8 * c + 5], inv);
          const uint32_t d = enc_u16x2(s[8 * c + 6], s[8 * c + 7], inv);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(base + xrow_off(row, c)),
                       "r"(a), "r"(b), "r"(cc), "r"(d)
                       : "memory");
        }
        asm volatile("st.shared.f32 [%0], %1;" ::"r"(base + kXPayload + row * 4),
                     "f"(mabs * (1.f / 32767.f))
                     : "memory");
        fence_proxy_async_smem();  // generic-proxy writes -> visible to the bulk copy
        mbar_arrive(&bars->staged[buf]);
      }
      t += n;
    }
  } else {
    // =================== softmax warpgroup (warps 0-3) + epilogue ===================
    const int row = threadIdx.x;  // head row = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const float NEG_INF = -__int_as_float(0x7f800000);
    // the head this row computes, and whether it carries the query's remainder (q_lo)
    const int head = hi_lo ? 64 * group + 16 * warp + (lane & 15) : row;
    const bool lo_row = hi_lo && (lane & 16);
    const bool row_ok = head < p.n_heads;
    const bool row_out = row_ok && !lo_row;  // rows whose result is written
    const uint32_t peer_done_r[2] = {mapa_shared(smem_u32(&bars->peer_done[0]), peer),
                                     mapa_shared(smem_u32(&bars->peer_done[1]), peer)};
    SegIter it{plan.seq_pages(), plan.seq_prefix(), p.batch, g_begin, g_end, b_begin};
    int seq, p0, p1, t = 0, sg = 0;
    bool ok = true;
    while (ok && it.next(seq, p0, p1)) {
      const int n = p1 - p0, t0 = t;
      const int len = min(p.seq_lens[seq], p.max_pages * kPage);
      // ---- this CTA's latent half of the query row -> TMEM (A operand of QK) ----
      {
        const uint4* src = reinterpret_cast<const uint4*>(
            (lo_row ? p.q_lo : p.q_cat) +
            (static_cast<size_t>(seq) * p.n_heads + (row_ok ? head : 0)) * kRow);
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint4 v = row_ok ? __ldg(src + (256 * rank + 64 * c) / 8 + k)
                                   : make_uint4(0u, 0u, 0u, 0u);
            r[4 * k] = v.x;
            r[4 * k + 1] = v.y;
            r[4 * k + 2] = v.z;
            r[4 * k + 3] = v.w;
          }
          tmem_st32(tmem + kTmemQ + 32 * c + lane_off, r);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->q_ready);
      }
      float m_ref = NEG_INF, l_sum = 0.f;
      for (int i = 0; i < n; ++i) {
        const int tt = t0 + i, buf = tt & 1;
        const bool first = i == 0;
        // ---- own exact partial ----
        if (!(ok = warp_wait(&bars->s_full[buf], (tt >> 1) & 1, wc))) break;
        tc_fence_after();
        float s[64];
        {
          uint32_t r[32];
          tmem_ld32(tmem + kTmemS + buf * 64 + lane_off, r);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) s[k] = __uint_as_float(r[k]);
          tmem_ld32(tmem + kTmemS + buf * 64 + 32 + lane_off, r);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) s[32 + k] = __uint_as_float(r[k]);
        }
        tc_fence_before();
        mbar_arrive(&bars->s_free[buf]);
        // ---- plus the peer's decoded partial ----
        if (!(ok = warp_wait<true>(&bars->x_full, tt & 1, wc))) break;
        {
          const uint32_t base = recv_base;
          float dq;
          asm volatile("ld.shared.f32 %0, [%1];" : "=f"(dq) : "r"(base + kXPayload + row * 4));
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint32_t v[4];
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
                         : "r"(base + xrow_off(row, c)));
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              s[8 * c + 2 * k] = fmaf(dec_lo(v[k]), dq, s[8 * c + 2 * k]);
              s[8 * c + 2 * k + 1] = fmaf(dec_hi(v[k]), dq, s[8 * c + 2 * k + 1]);
            }
          }
          // this warp's rows are decoded: warp 0 re-arms recv for the next page (its phase
          // cannot complete before all four warps have handed their rows back), and every
          // warp tells the peer its rows may be refilled
          __syncwarp();
          if (lane == 0) {
            if (warp == 0) mbar_arrive_expect_tx(&bars->x_full, kXBytes);
            mbar_arrive_remote_relaxed(peer_done_r[buf]);
          }
        }
        // ---- extended-precision query: a head's score is the sum of its q_cat and q_lo rows
        // (lanes l and l ^ 16 of this warp); both rows continue with the same scores ----
        if (hi_lo) {
#pragma unroll
          for (int k = 0; k < 64; ++k) s[k] += __shfl_xor_sync(0xffffffffu, s[k], 16);
        }
        // ---- online softmax ----
        const int valid = min(kPage, len - (p0 + i) * kPage);
        if (valid < kPage) {
#pragma unroll
          for (int k = 0; k < 64; ++k) s[k] = k < valid ? s[k] : NEG_INF;
        }
        float mx = max64(s);
        mx *= p.scale_log2;  // log2 units (scale > 0 keeps the arg max)
        float alpha = 1.f;
        bool rescale = false;
        if (first) {
          m_ref = mx;
        } else if (mx > m_ref + kRescaleThreshold) {
          alpha = ex2_approx(m_ref - mx);
          m_ref = mx;
          rescale = true;
        }
        float rsum[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        uint32_t pk[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          const float e0 = ex2_approx(fmaf(s[2 * k], p.scale_log2, -m_ref));
          const float e1 = ex2_approx(fmaf(s[2 * k + 1], p.scale_log2, -m_ref));
          rsum[k & 7] += e0 + e1;
          pk[k] = pack_bf16x2(e0, e1);
        }
        const float rs = ((rsum[0] + rsum[1]) + (rsum[2] + rsum[3])) +
                         ((rsum[4] + rsum[5]) + (rsum[6] + rsum[7]));
        l_sum = l_sum * alpha + rs;
        if (!first && __any_sync(0xffffffffu, rescale)) {
          // O must hold PV of the previous page before it is rescaled
          if (!(ok = warp_wait(&bars->pv_done, (tt - 1) & 1, wc))) break;
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
        }
        // ---- P -> shared memory (canonical K-major, 128B swizzle) once PV of page tt - 1
        // has read it ----
        if (tt >= 1 && !(ok = warp_wait(&bars->pv_done, (tt - 1) & 1, wc))) break;
        {
          const uint32_t pa = smem_u32(smem + kOffP);
#pragma unroll
          for (int c = 0; c < 8; ++c)
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(pa + xrow_off(row, c)),
                         "r"(pk[4 * c]), "r"(pk[4 * c + 1]), "r"(pk[4 * c + 2]),
                         "r"(pk[4 * c + 3])
                         : "memory");
        }
        fence_proxy_async_smem();  // generic-proxy writes -> visible to the tensor core
        mbar_arrive(&bars->p_full);
      }
      if (!ok) break;
      // ---- segment epilogue: O / l -> global ----
      if (!(ok = warp_wait(&bars->seg_done, sg & 1, wc))) break;
      tc_fence_after();
      const int nparts = plan.seq_nparts()[seq];
      const float lse_nat = (m_ref + __log2f(l_sum)) * 0.69314718055994531f;
      const float inv_l = 1.f / l_sum;
      float* dst;
      float* dst_lse;
      if (nparts == 1) {
        dst = p.o_lat + (static_cast<size_t>(seq) * p.n_heads + head) * 512 + 256 * rank;
        dst_lse = p.lse ? p.lse + static_cast<size_t>(seq) * p.n_heads + head : nullptr;
      } else {
        const int slot = plan.seq_slot()[seq] + (part - plan.seq_first_part()[seq]);
        dst = p.part_o + (static_cast<size_t>(slot) * p.n_heads + head) * 512 + 256 * rank;
        dst_lse = p.part_lse + static_cast<size_t>(slot) * p.n_heads + head;
      }
#pragma unroll 1
      for (int c = 0; c < 256; c += 32) {
        uint32_t r[32];
        tmem_ld32(tmem + kTmemO + c + lane_off, r);
        tmem_wait_ld();
        if (row_out) {
          float4* d4 = reinterpret_cast<float4*>(dst + c);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            d4[k] = make_float4(__uint_as_float(r[4 * k]) * inv_l,
                                __uint_as_float(r[4 * k + 1]) * inv_l,
                                __uint_as_float(r[4 * k + 2]) * inv_l,
                                __uint_as_float(r[4 * k + 3]) * inv_l);
        }
      }
      if (row_out && rank == 0 && dst_lse) *dst_lse = lse_nat;
      tc_fence_before();
      mbar_arrive(&bars->o_free);
      t += n;
      ++sg;
    }
    // The peer's remote arrivals for our last two partials must land before this CTA exits.
    {
      volatile int never = 0;
      WaitCtx drain{&never, p.status, p.wait_ns};
      for (int u = max(0, t - 2); u < t; ++u)
        mbar_wait<true>(&bars->peer_done[u & 1], (u >> 1) & 1, ok ? wc : drain);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  cluster_sync();
}

// ------------------------------------------------------------------------------------------
// Combine: log-sum-exp merge of the parts of sequences split over several ranges.
// ------------------------------------------------------------------------------------------
constexpr int kCombineWarps = 8;

// One warp per (sequence, head); lane l owns float4 columns l, l + 32, l + 64 and l + 96.  The
// parts are merged in slot order; every part's loads of a chunk are issued before any is used.
__global__ void __launch_bounds__(32 * kCombineWarps)
    combine_kernel(const int32_t* __restrict__ plan_words, int B, int C, int H,
                   const float* __restrict__ part_o, const float* __restrict__ part_lse,
                   float* __restrict__ o_lat, float* __restrict__ lse) {
  griddep_launch_dependents();
  griddep_wait();
  const PlanView plan(plan_words, B, C);
  const int wid = blockIdx.x * kCombineWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (wid >= B * H) return;
  const int b = wid / H, h = wid - b * H;
  const int n = plan.seq_nparts()[b];
  if (n == 1) return;
  float4* out = reinterpret_cast<float4*>(o_lat + (static_cast<size_t>(b) * H + h) * 512);
  const float NEG_INF = -__int_as_float(0x7f800000);
  if (n == 0) {
#pragma unroll
    for (int k = 0; k < 4; ++k) out[lane + 32 * k] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (lane == 0 && lse) lse[static_cast<size_t>(b) * H + h] = NEG_INF;
    return;
  }
  const int slot0 = plan.seq_slot()[b];
  float m = NEG_INF;
  for (int s = lane; s < n; s += 32)
    m = fmaxf(m, part_lse[static_cast<size_t>(slot0 + s) * H + h]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float tot = 0.f;
  float4 acc[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = 0; s0 < n; s0 += 32) {
    const int cnt = min(32, n - s0);
    const float wl =
        lane < cnt ? __expf(part_lse[static_cast<size_t>(slot0 + s0 + lane) * H + h] - m) : 0.f;
#pragma unroll 4
    for (int j = 0; j < cnt; ++j) {
      const float w = __shfl_sync(0xffffffffu, wl, j);
      const float4* src = reinterpret_cast<const float4*>(
          part_o + (static_cast<size_t>(slot0 + s0 + j) * H + h) * 512);
      tot += w;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float4 v = src[lane + 32 * k];
        acc[k].x += w * v.x;
        acc[k].y += w * v.y;
        acc[k].z += w * v.z;
        acc[k].w += w * v.w;
      }
    }
  }
  const float inv = 1.f / tot;
#pragma unroll
  for (int k = 0; k < 4; ++k)
    out[lane + 32 * k] = make_float4(acc[k].x * inv, acc[k].y * inv, acc[k].z * inv, acc[k].w * inv);
  if (lane == 0 && lse) lse[static_cast<size_t>(b) * H + h] = m + __logf(tot);
}

}  // namespace attn
}  // namespace mla
