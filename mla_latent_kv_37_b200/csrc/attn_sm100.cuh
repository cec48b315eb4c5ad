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
//   * TMEM (512 columns): O half 256 | query latent half 128 (A operand of QK) | S of two
//     pages, 2 x 64 (page parity), so the QK of page t+1 never waits for the softmax of page t.
//   * Pages arrive by TMA into a 4-slot ring laid out box-major.  Four pages ahead of the ring
//     each CTA issues a bulk L2 prefetch of its half of the page's rows, so the ring's loads
//     find their lines in L2.
//   * S_r = Q_r C_r^T is a partial score; every row's softmax needs both CTAs' partials.  Both
//     CTAs run the same softmax over all 128 rows (symmetric), so each holds the full P of the
//     page for its own PV and no P or rescale factor crosses the pair.  Per page:
//       - four send warps (one per TMEM quarter, one thread per row) read this CTA's partial,
//         quantise it to 16-bit fixed point relative to the row's largest magnitude (error
//         <= 2^-16 of it, ~1e-4 in a logit) and store it straight from registers into the
//         peer's receive buffer (st.async, completion counted in bytes on the peer's
//         mbarrier; two receive buffers, by page parity);
//       - eight softmax warps, two per TMEM quarter, each own 16 whole rows (two threads per
//         row, 32 columns each: the 16x32bx2 TMEM load), so a row's maximum and sum take one
//         shuffle.  They add the peer's decoded partial to their own, run the online softmax
//         on packed f32x2 arithmetic, write P (bf16) into the page's P buffer, rescale their
//         rows of O when needed, and hand the receive buffer back to the peer;
//       - PV runs as soon as P is complete; its completion frees the P buffer and the slot.
//   * The MMA warp issues from an event loop with precomputed descriptors: each page's QK as
//     soon as the page has landed and its S buffer is free, each PV as soon as its P is
//     written, whichever comes first; it backs off with nanosleep while idle.
//   * The next segment's query half goes into TMEM as soon as the last QK of the previous one
//     has run, before that segment's epilogue, so a sequence boundary costs no pipeline drain.
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
// well (q = q_cat + q_lo to ~16 bits), each cluster takes 64 heads instead of 128 and puts, for
// each of them, a row of q_cat and a row of q_lo in the same 16-lane half of a warp's TMEM
// lanes (see RowMap).  The score of a head is then the sum of its two rows (one shuffle), the
// softmax runs identically on both rows, O gets the same P in both, and only the q_cat row is
// written out.  Launch: `groups` = ceil(H/64) clusters per part, so the tensor work per token
// doubles; the page bytes are read by the part's clusters at about the same time and mostly
// come from L2 the second time.
//
// Roles (448 threads, 128 registers each): warps 0-7 softmax, query load (warps 0-3), O
// rescale and epilogue; warps 8-11 send; warp 12 TMA producer; warp 13 MMA issuer and TMEM
// owner.  The online softmax keeps a per-row reference maximum and rescales O only when the
// running maximum grows by more than 2^8.
#pragma once
#include "ptx_sm100.cuh"

namespace mla {
namespace attn {

constexpr int kThreads = 448;  // 14 warps: 8 softmax, 4 send, TMA producer, MMA issuer
constexpr int kPage = 64;
constexpr int kRow = 576;
constexpr int kSlots = 4;  // page slots of the ring
constexpr uint32_t kBoxBytes = 64 * 128;      // one page's 64 rows x 64 latent columns (bf16)
constexpr uint32_t kRopeBoxBytes = 64 * 64;   // one page's 64 rows x 32 RoPE columns (bf16)
constexpr uint32_t kSlotBytes = 4 * kBoxBytes + kRopeBoxBytes;  // this CTA's half of a page
// The ring is box-major: latent box i of slot s at i * kSlots * kBoxBytes + s * kBoxBytes; the
// RoPE boxes of the slots follow.
constexpr uint32_t kOffRing = 0;
constexpr uint32_t kBoxStride = kSlots * kBoxBytes;
constexpr uint32_t kOffRope = kOffRing + 4 * kBoxStride;
constexpr uint32_t kPBytes = 128 * 128;  // P of one page: 128 rows x 64 bf16
constexpr uint32_t kOffP = kOffRope + kSlots * kRopeBoxBytes;  // two P buffers (page parity)
constexpr uint32_t kQRopeBytes = 128 * 64;                    // 128 rows x 32 bf16
constexpr uint32_t kOffQRope = kOffP + 2 * kPBytes;
constexpr uint32_t kXPayload = 128 * 128;         // 128 rows x 64 partial scores x 16 bits
constexpr uint32_t kXBytes = kXPayload + 128 * 4;  // + one fp32 step per row
constexpr uint32_t kOffX = kOffQRope + kQRopeBytes;  // two receive buffers (page parity)
constexpr uint32_t kOffBar = kOffX + 2 * kXBytes;
constexpr uint32_t kSmemBytes = kOffBar + 512 + 1024;  // barriers + alignment slack
// TMEM columns: O half | query latent half | S of two pages (page parity)
constexpr uint32_t kTmemO = 0, kTmemQ = 256, kTmemS = 384, kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(kTmemS + 2 * 64 == kTmemCols, "tensor memory budget");
static_assert(kXBytes % 16 == 0 && kOffP % 1024 == 0 && kOffQRope % 1024 == 0 &&
                  kOffRope % 1024 == 0 && kOffX % 16 == 0 && kOffBar % 8 == 0,
              "alignment");

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
  int stall_test;  // 1: warp 0 first waits on a barrier nothing arrives on (timeout-path test)
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
// Planner: one block.  pages per sequence, prefix sums, division of the page list into parts of
// equal cost, which parts touch which sequence, and where each sequence's partials go.
//
// Cost model: a part pays for its pages and, for every sequence that starts inside it, one more
// segment (a query load, a drained pipeline and an O write-back), which costs about as much as
// kSegPages pages.  So the division is equal in "virtual pages": every non-empty sequence is
// kSegPages virtual pages of start-up followed by its real pages, and part c covers the virtual
// range [c V / C, (c + 1) V / C).  A part whose range begins inside a sequence's start-up begins
// at that sequence's first page.
// ------------------------------------------------------------------------------------------
constexpr int kPlanThreads = 1024;
constexpr int kSegPages = 3;

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

// The part that holds virtual position v of the list (v = -1 gives -1): part c holds
// [floor(c V / C), floor((c + 1) V / C)).
__device__ inline int part_of_page(int64_t v, int C, int64_t V) {
  return v < 0 ? -1 : static_cast<int>(((v + 1) * C - 1) / V);
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
  // 1. pages of this thread's sequences, and their exclusive prefix over the whole batch; the
  //    same for the count of non-empty sequences (each adds kSegPages virtual pages)
  int local = 0, nonempty = 0;
  for (int b = b0; b < b1; ++b) {
    const int n = plan_pages(seq_lens, b, cap, status);
    local += n;
    nonempty += n > 0;
  }
  const int run0 = block_exclusive_scan(local, warp_sums, &s_total);
  const int P = s_total;
  __shared__ int s_seqs;
  const int rank0 = block_exclusive_scan(nonempty, warp_sums, &s_seqs);
  const int64_t V = static_cast<int64_t>(P) + static_cast<int64_t>(kSegPages) * s_seqs;
  int C = 0;
  if (P > 0) C = max(1, min(C_req, (P + min_pages_per_part - 1) / min_pages_per_part));
  if (threadIdx.x == 0) {
    plan[0] = P;
    plan[1] = C;
    prefix[B] = P;
  }
  // 2. parts beyond C are empty and start no sequence; every other part start is written by
  //    the thread of the sequence it starts in (step 3)
  for (int c = threadIdx.x; c <= C_req; c += T) {
    if (c >= C) pstart[c] = P;
    if (c < C_req && c >= C) pseq[c] = B;
  }
  // 3. per sequence: its pages, prefix, the parts that cover it, and the parts starting in it
  int run = run0, rank = rank0, nloc = 0;
  for (int b = b0; b < b1; ++b) {
    const int n = plan_pages(seq_lens, b, cap, nullptr);
    pg[b] = n;
    prefix[b] = run;
    if (n == 0) {
      first[b] = 0;
      npart[b] = 0;
      continue;
    }
    // virtual positions: start-up [vs, vs + kSegPages), pages from vp (page k at vp + k)
    const int64_t vs = static_cast<int64_t>(run) + static_cast<int64_t>(kSegPages) * rank;
    const int64_t vp = vs + kSegPages;
    const int pf = part_of_page(vp, C, V);
    const int pl = part_of_page(vp + n - 1, C, V);
    first[b] = pf;
    npart[b] = pl - pf + 1;
    nloc += pl - pf + 1;
    for (int c = part_of_page(vs - 1, C, V) + 1; c <= pl; ++c) {
      const int64_t u = (static_cast<int64_t>(c) * V) / C;  // the part's first virtual position
      pstart[c] = run + static_cast<int>(u > vp ? u - vp : 0);
      pseq[c] = b;
    }
    run += n;
    ++rank;
  }
  // 4. where each sequence's partials go
  int srun = block_exclusive_scan(nloc, warp_sums, nullptr);
  run = run0;
  rank = rank0;
  for (int b = b0; b < b1; ++b) {
    const int n = plan_pages(seq_lens, b, cap, nullptr);
    slot[b] = srun;
    if (n > 0) {
      const int64_t vp =
          static_cast<int64_t>(run) + static_cast<int64_t>(kSegPages) * rank + kSegPages;
      srun += part_of_page(vp + n - 1, C, V) - part_of_page(vp, C, V) + 1;
      ++rank;
    }
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
// TMEM lanes (MMA rows) and heads.  Without the query remainder, lane L computes head L.  With
// it, in quarter q of the lanes (one warp's 32) lanes 16h + 8k + j (h, k in {0, 1}, j < 8)
// compute head 64 group + 16q + 8h + j, from q_cat for k = 0 and from q_lo for k = 1, so that
// the two rows of a head sit in the same 16-lane half of the quarter (one softmax warp).
struct RowMap {
  bool hi_lo;
  int group;
  __device__ int head(int L) const {
    return hi_lo ? 64 * group + 16 * (L >> 5) + 8 * ((L >> 4) & 1) + (L & 7) : L;
  }
  __device__ bool lo(int L) const { return hi_lo && ((L >> 3) & 1); }
};

// Every mbarrier below completes one phase per use and is waited phase by phase, never more
// than one phase behind its current state (buffers that could run two pages ahead of their
// waiter have one barrier per buffer), so parity waits cannot alias.  Barriers marked "bytes"
// complete when the stated number of bytes has landed (TMA, or st.async from the peer CTA);
// the ones the peer writes are armed here, one use ahead.
struct Bars {
  uint64_t full[kSlots];   // TMA: the page slot is filled (bytes)
  uint64_t empty[kSlots];  // MMA: the PV that read the slot finished (commit)
  uint64_t q_full;         // TMA: the segment's query RoPE half landed (bytes)
  uint64_t q_empty;        // MMA: the segment's last QK finished (commit)
  uint64_t q_ready;        // softmax warps 0-3: the query latent half is in TMEM (4)
  uint64_t s_full[2];      // MMA: S of a page is written (commit)
  uint64_t s_free[2];      // the 8 softmax and 4 send warps drained S of the page (12)
  uint64_t x_full[2];      // the peer's partial scores of a page landed (bytes)
  uint64_t x_free[2];      // the peer's softmax warps decoded our partials of a page (8 remote)
  uint64_t p_full[2];      // softmax warps: P of the page written, O rescaled (8)
  uint64_t pv_done[2];     // MMA: PV of the page finished, its P buffer is free (commit)
  uint64_t seg_done;       // MMA: every PV of the segment finished (commit)
  uint64_t o_free;         // softmax warps: the epilogue drained O (8)
  uint64_t drain;          // MMA: final drain after an abort
  uint64_t stall;          // nothing ever arrives here (timeout-path test)
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(Bars) <= 512, "barrier block");

constexpr uint64_t kDrainNs = 200000000ull;  // waits for copies and MMAs already in flight
constexpr uint32_t kFull = 0xffffffffu;

__device__ __forceinline__ float max32(const float* s) {
  float m[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) m[j] = s[j];
#pragma unroll
  for (int k = 8; k < 32; ++k) m[k & 7] = fmaxf(m[k & 7], s[k]);
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

__device__ __forceinline__ void spin_ns(uint64_t ns) {
  const uint64_t t0 = globaltimer_ns();
  while (globaltimer_ns() - t0 < ns) {
  }
}

// Advance the start-address field (bits 0-13, in 16-byte units) of a shared-memory matrix
// descriptor by `bytes` (addresses stay below 256 KiB, so the field cannot overflow).
__device__ __forceinline__ uint64_t desc_add(uint64_t d, uint32_t bytes) {
  return d + static_cast<uint64_t>(bytes >> 4);
}

__global__ void __cluster_dims__(2, 1, 1) __maxnreg__(128)
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
  const RowMap rows{p.q_lo != nullptr, group};

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    mbar_init(&bars->q_ready, 4);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->s_free[i], 12);
      mbar_init(&bars->x_full[i], 1);
      mbar_init(&bars->x_free[i], 8);
      mbar_init(&bars->p_full[i], 8);
      mbar_init(&bars->pv_done[i], 1);
    }
    mbar_init(&bars->seg_done, 1);
    mbar_init(&bars->o_free, 8);
    mbar_init(&bars->drain, 1);
    mbar_init(&bars->stall, 1);
    bars->abort_flag = 0;
    fence_mbar_init_cluster();
    // receive buffers armed for their first use
    mbar_arrive_expect_tx(&bars->x_full[0], kXBytes);
    mbar_arrive_expect_tx(&bars->x_full[1], kXBytes);
  }
  if (warp == 13) {
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
  uint8_t* sQRope = smem + kOffQRope;
  volatile int never = 0;
  const WaitCtx drain_ctx{&never, p.status, kDrainNs};

  if (warp == 12) {
    // =================== TMA producer: page ring + query RoPE half ===================
    SegIter it{plan.seq_pages(), plan.seq_prefix(), p.batch, g_begin, g_end, b_begin};
    int seq, p0, p1, t = 0, sg = 0, issued = 0;
    bool ok = true;
    const uint64_t pol_stream = l2_policy_evict_first();
    if (lane == 0) {
      tma_prefetch_desc(&tm_c_lat);
      tma_prefetch_desc(&tm_c_rope);
      tma_prefetch_desc(&tm_q_rope);
      if (rows.hi_lo) tma_prefetch_desc(&tm_ql_rope);
    }
    while (ok && it.next(seq, p0, p1)) {
      if (lane == 0) {
        if (sg > 0) ok = mbar_wait(&bars->q_empty, (sg - 1) & 1, wc);
        if (ok) {
          mbar_arrive_expect_tx(&bars->q_full, kQRopeBytes);
          if (!rows.hi_lo) {
            tma_load_3d(sQRope, &tm_q_rope, &bars->q_full, 512 + 32 * rank, 0, seq);
          } else {
            // 8-row boxes in the lane order of RowMap (rows past H are zero-filled)
#pragma unroll
            for (int qq = 0; qq < 4; ++qq)
#pragma unroll
              for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                for (int k = 0; k < 2; ++k)
                  tma_load_3d(sQRope + (32 * qq + 16 * hh + 8 * k) * 64,
                              k ? &tm_ql_rope : &tm_q_rope, &bars->q_full, 512 + 32 * rank,
                              64 * group + 16 * qq + 8 * hh, seq);
          }
        }
      }
      ok = __shfl_sync(kFull, ok, 0);
      const int32_t* pt = p.page_table + static_cast<size_t>(seq) * p.max_pages;
      for (int pb = p0; ok && pb < p1; pb += 32) {
        const int cnt = min(32, p1 - pb);
        int my_page = lane < cnt ? pt[pb + lane] : 0;
        if (lane < cnt && (my_page < 0 || my_page >= p.num_pages)) {
          atomicOr(p.status, MLA_STATUS_BAD_PAGE);
          my_page = 0;
        }
        for (int j = 0; j < cnt; ++j, ++t) {
          const int page = __shfl_sync(kFull, my_page, j);
          if (lane == 0) {
            const int s = t % kSlots;
            if (t >= kSlots) ok = mbar_wait(&bars->empty[s], ((t / kSlots) - 1) & 1, wc);
            if (ok) {
              mbar_arrive_expect_tx(&bars->full[s], kSlotBytes);
              const int y = page * kPage;
#pragma unroll
              for (int i = 0; i < 4; ++i)
                tma_load_2d_hint(smem + kOffRing + i * kBoxStride + s * kBoxBytes, &tm_c_lat,
                                 &bars->full[s], 256 * rank + 64 * i, y, pol_stream);
              tma_load_2d_hint(smem + kOffRope + s * kRopeBoxBytes, &tm_c_rope, &bars->full[s],
                               512 + 32 * rank, y, pol_stream);
              issued = t + 1;
            }
          }
          ok = __shfl_sync(kFull, ok, 0);
          if (!ok) break;
        }
      }
      ++sg;
    }
    // No copy may still be landing when the CTA exits.  Normally every load has been consumed
    // by now and these return at once; after an abort (raised by any role, at any time) they
    // wait for the copies still in flight.
    if (lane == 0) {
      for (int i = max(0, issued - kSlots); i < issued; ++i)
        mbar_wait(&bars->full[i % kSlots], (i / kSlots) & 1, drain_ctx);
      if (sg > 0) mbar_wait(&bars->q_full, (sg - 1) & 1, drain_ctx);
    }
  } else if (warp == 13) {
    // =================== MMA issuer: QK and PV per page, each as soon as it is ready ==========
    if (lane == 0) {
      const uint32_t idesc_qk = idesc_bf16(128, 64, 0, 0);
      const uint32_t idesc_pv = idesc_bf16(128, 256, 0, 1);
      // descriptors at the buffers' starts; every operand below is one of these advanced
      const uint64_t d_ring = smem_desc(smem_u32(smem + kOffRing), 16, 1024, kSwizzle128B);
      const uint64_t d_rope = smem_desc(smem_u32(smem + kOffRope), 16, 512, kSwizzle64B);
      const uint64_t d_qrope = smem_desc(smem_u32(sQRope), 16, 512, kSwizzle64B);
      const uint64_t d_p = smem_desc(smem_u32(smem + kOffP), 16, 1024, kSwizzle128B);
      const uint64_t d_pv_b = smem_desc(smem_u32(smem + kOffRing), kBoxStride, 1024, kSwizzle128B);
      // S_t = Q_r C_r^T into S buffer t & 1: latent half A from TMEM, RoPE half A from smem
      auto issue_qk = [&](int t) {
        const uint32_t s = static_cast<uint32_t>(t % kSlots);
        const uint32_t d = tmem + kTmemS + 64 * (t & 1);
        const uint64_t b0 = desc_add(d_ring, s * kBoxBytes);
#pragma unroll
        for (int j = 0; j < 16; ++j)
          mma_ts(d, tmem + kTmemQ + 8 * j, desc_add(b0, (j >> 2) * kBoxStride + (j & 3) * 32),
                 idesc_qk, j > 0 ? 1u : 0u);
        const uint64_t r0 = desc_add(d_rope, s * kRopeBoxBytes);
        mma_ss(d, d_qrope, r0, idesc_qk, 1u);
        mma_ss(d, desc_add(d_qrope, 32), desc_add(r0, 32), idesc_qk, 1u);
        mma_commit(&bars->s_full[t & 1]);
      };
      // O += P_t C_lat,t: A = P (bf16, shared memory), B = the page's latent half (MN-major)
      auto issue_pv = [&](int t, bool first) {
        const uint32_t s = static_cast<uint32_t>(t % kSlots);
        const uint64_t a0 = desc_add(d_p, (t & 1) * kPBytes);
        const uint64_t b0 = desc_add(d_pv_b, s * kBoxBytes);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ss(tmem + kTmemO, desc_add(a0, kk * 32), desc_add(b0, kk * 2048), idesc_pv,
                 (first && kk == 0) ? 0u : 1u);
        mma_commit(&bars->pv_done[t & 1]);
        mma_commit(&bars->empty[s]);
      };
      SegIter itq{plan.seq_pages(), plan.seq_prefix(), p.batch, g_begin, g_end, b_begin};
      SegIter itv = itq;
      int qs, q0, q1, vs, v0, v1;
      bool q_more = itq.next(qs, q0, q1), v_more = itv.next(vs, v0, v1);
      int q_i = 0, q_t = 0, q_sg = 0;  // QK: page in segment, global page, segment
      int v_i = 0, v_t = 0, v_sg = 0;  // PV: page in segment, global page, segment
      uint64_t idle_since = 0;
      uint32_t spins = 0;
      bool ok = true;
      while (ok && (q_more || v_more)) {
        bool progress = false;
        // PV first: it frees the ring slot and the P buffer the rest of the pipe waits for
        if (v_more && mbar_test(&bars->p_full[v_t & 1], (v_t >> 1) & 1) &&
            (v_i > 0 || v_sg == 0 || mbar_test(&bars->o_free, (v_sg - 1) & 1))) {
          tc_fence_after();
          issue_pv(v_t, v_i == 0);
          ++v_t;
          if (++v_i == v1 - v0) {
            mma_commit(&bars->seg_done);
            ++v_sg;
            v_i = 0;
            v_more = itv.next(vs, v0, v1);
          }
          progress = true;
        }
        if (q_more &&
            (q_i > 0 ||
             (mbar_test(&bars->q_ready, q_sg & 1) && mbar_test(&bars->q_full, q_sg & 1))) &&
            (q_t < 2 || mbar_test(&bars->s_free[q_t & 1], ((q_t >> 1) - 1) & 1)) &&
            mbar_test(&bars->full[q_t % kSlots], (q_t / kSlots) & 1)) {
          tc_fence_after();
          issue_qk(q_t);
          ++q_t;
          if (++q_i == q1 - q0) {
            mma_commit(&bars->q_empty);
            ++q_sg;
            q_i = 0;
            q_more = itq.next(qs, q0, q1);
          }
          progress = true;
        }
        if (progress) {
          idle_since = 0;
          spins = 0;
        } else {
          // back off briefly: this warp shares its SM sub-partition with softmax and send warps
          __nanosleep(32);
          if ((++spins & 63) != 0) continue;
          if (bars->abort_flag) {
            ok = false;
          } else {
            const uint64_t now = globaltimer_ns();
            if (idle_since == 0) {
              idle_since = now;
            } else if (now - idle_since > p.wait_ns) {
              bars->abort_flag = 1;
              atomicOr(p.status, MLA_STATUS_TIMEOUT);
              ok = false;
            }
          }
        }
      }
      // No MMA may be in flight when TMEM is released: normally they have all completed, after
      // an abort (by any role) the commit waits for the last ones.
      mma_commit(&bars->drain);
      mbar_wait(&bars->drain, 0, drain_ctx);
    }
  } else if (warp >= 8) {
    // =================== send warps: this CTA's partial scores, quantised, into the peer ======
    // Thread = TMEM lane 32q + lane = row; all 64 columns of the page; row 32q + lane of the
    // peer's receive buffer.
    const int q = warp & 3;
    const int row = 32 * q + lane;
    const uint32_t lanes = static_cast<uint32_t>(32 * q) << 16;
    const uint32_t x_peer = mapa_shared(smem_u32(smem + kOffX), peer);
    // the peer's x_full[0]; x_full[1] is the next 8 bytes
    const uint32_t xfull_peer = mapa_shared(smem_u32(&bars->x_full[0]), peer);
    SegIter it{plan.seq_pages(), plan.seq_prefix(), p.batch, g_begin, g_end, b_begin};
    int seq, p0, p1, t = 0;
    bool ok = true;
    while (ok && it.next(seq, p0, p1)) {
      const int len = min(p.seq_lens[seq], p.max_pages * kPage);
      for (int i = 0; i < p1 - p0; ++i, ++t) {
        const int pb = t & 1;
        if (!(ok = warp_wait(&bars->s_full[pb], (t >> 1) & 1, wc))) break;
        tc_fence_after();
        float s[64];
        {
          uint32_t r[32];
          tmem_ld32(tmem + kTmemS + 64 * pb + lanes, r);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) s[k] = __uint_as_float(r[k]);
          tmem_ld32(tmem + kTmemS + 64 * pb + 32 + lanes, r);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) s[32 + k] = __uint_as_float(r[k]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->s_free[pb]);
        // columns past the sequence's end are never used: they travel as zeros
        const int valid = min(kPage, len - (p0 + i) * kPage);
        if (valid < kPage) {
#pragma unroll
          for (int k = 0; k < 64; ++k) s[k] = k < valid ? s[k] : 0.f;
        }
        const float mabs = maxabs64(s);
        const float inv = mabs > 0.f ? 32767.f / mabs : 0.f;
        if (t >= 2 && !(ok = warp_wait<true>(&bars->x_free[pb], ((t >> 1) - 1) & 1, wc))) break;
        const uint32_t xb = x_peer + pb * kXBytes;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          st_async_u4(xb + xrow_off(row, c), enc_u16x2(s[8 * c], s[8 * c + 1], inv),
                      enc_u16x2(s[8 * c + 2], s[8 * c + 3], inv),
                      enc_u16x2(s[8 * c + 4], s[8 * c + 5], inv),
                      enc_u16x2(s[8 * c + 6], s[8 * c + 7], inv), xfull_peer + 8 * pb);
        st_async_u1(xb + kXPayload + row * 4, __float_as_uint(mabs * (1.f / 32767.f)),
                    xfull_peer + 8 * pb);
      }
    }
    if (ok) {  // the peer's hand-backs for our last two pages land before this CTA exits
      for (int u = max(0, t - 2); u < t; ++u)
        mbar_wait<true>(&bars->x_free[u & 1], (u >> 1) & 1, drain_ctx);
    }
  } else {
    // =================== softmax warps, query load, epilogue ===================
    // 16x32bx2 view: warp w owns the 16 rows 32q + 16k .. 32q + 16k + 15 (q = w & 3, k = w >> 2),
    // two threads per row: thread (j, h) = (lane & 15, lane >> 4) takes columns 32h .. 32h + 31
    // of each page and O columns 128h .. 128h + 127.  A row lives in one warp, so its maximum
    // and sum take one shuffle.  Warps 0-3 load the query (32x32b view, thread = lane 32q + lane).
    const int q = warp & 3, kh = warp >> 2, j = lane & 15, hcol = lane >> 4;
    const int row = 32 * q + 16 * kh + j;
    const uint32_t lanes_own = static_cast<uint32_t>(32 * q + 16 * kh) << 16;
    const uint32_t lanes_all = static_cast<uint32_t>(32 * q) << 16;
    const float NEG_INF = -__int_as_float(0x7f800000);
    const uint32_t x_loc = smem_u32(smem + kOffX);
    const uint32_t p_loc = smem_u32(smem + kOffP);
    // the peer's x_free[0]; x_free[1] is the next 8 bytes
    const uint32_t xfree_rem = mapa_shared(smem_u32(&bars->x_free[0]), peer);
    const int hd = rows.head(row);
    const bool out_row = hd < p.n_heads && !rows.lo(row);
    // this CTA's latent half of the query rows of sequence sq -> TMEM (A operand of QK), in two
    // batches of 16 loads issued before their first use
    auto load_q = [&](int sq) {
      const int qrow = 32 * q + lane;
      const int qhd = rows.head(qrow);
      const bool in = qhd < p.n_heads;
      const uint4* src = reinterpret_cast<const uint4*>(
          (rows.lo(qrow) ? p.q_lo : p.q_cat) +
          (static_cast<size_t>(sq) * p.n_heads + (in ? qhd : 0)) * kRow) + 32 * rank;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint4 v[16];
#pragma unroll
        for (int k = 0; k < 16; ++k)
          v[k] = in ? __ldg(src + 16 * half + k) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t r[32];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            r[4 * k] = v[8 * c + k].x;
            r[4 * k + 1] = v[8 * c + k].y;
            r[4 * k + 2] = v[8 * c + k].z;
            r[4 * k + 3] = v[8 * c + k].w;
          }
          tmem_st32(tmem + kTmemQ + 32 * (2 * half + c) + lanes_all, r);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->q_ready);
    };
    SegIter it{plan.seq_pages(), plan.seq_prefix(), p.batch, g_begin, g_end, b_begin};
    int seq, p0, p1, t = 0, sg = 0;
    bool ok = true;
    bool have = it.next(seq, p0, p1);
    // timeout-path test: a wait that can only run out, raising the status and the abort
    if (p.stall_test && warp == 0) ok = warp_wait(&bars->stall, 0, wc);
    if (have && kh == 0) load_q(seq);
    while (ok && have) {
      const int n = p1 - p0;
      const int len = min(p.seq_lens[seq], p.max_pages * kPage);
      float m_ref = NEG_INF, l_sum = 0.f;
      for (int i = 0; ok && i < n; ++i, ++t) {
        const int pb = t & 1;
        const bool first = i == 0;
        // ---- own exact partial: this thread's 32 columns of its row ----
        if (!(ok = warp_wait(&bars->s_full[pb], (t >> 1) & 1, wc))) break;
        tc_fence_after();
        float s[32];
        {
          uint32_t r[32];
          tmem_ld16x2_32(tmem + kTmemS + 64 * pb + lanes_own, r);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) s[k] = __uint_as_float(r[k]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->s_free[pb]);
        // ---- plus the peer's partial (16-bit, relative to its row's largest magnitude) ----
        // The bits 0x4B000000 | u are the float 2^23 + u exactly; subtracting 2^23 + 32768 is
        // exact too, and one FMA per value scales and adds the result (pairs at a time).
        if (!(ok = warp_wait(&bars->x_full[pb], (t >> 1) & 1, wc))) break;
        {
          const uint32_t xb = x_loc + pb * kXBytes;
          float dq;
          asm volatile("ld.shared.f32 %0, [%1];" : "=f"(dq) : "r"(xb + kXPayload + row * 4));
          const uint64_t dq2 = f2_pack(dq, dq);
          const uint64_t nbias2 = f2_pack(-kDecBias, -kDecBias);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t v[4];
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
                         : "r"(xb + xrow_off(row, 4 * hcol + c)));
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint64_t d2 = f2_add(
                  f2_pack(__uint_as_float(__byte_perm(v[k], kDecBits, 0x7610)),
                          __uint_as_float(__byte_perm(v[k], kDecBits, 0x7632))),
                  nbias2);
              const uint64_t r2 = f2_fma(d2, dq2, f2_pack(s[8 * c + 2 * k], s[8 * c + 2 * k + 1]));
              f2_unpack(r2, s[8 * c + 2 * k], s[8 * c + 2 * k + 1]);
            }
          }
        }
        // ---- a head's score with the query remainder: the sum of its two rows ----
        if (rows.hi_lo) {
#pragma unroll
          for (int k = 0; k < 32; ++k) s[k] += __shfl_xor_sync(kFull, s[k], 8);
        }
        // ---- online softmax over the row (two threads) ----
        const int valid = min(kPage, len - (p0 + i) * kPage) - 32 * hcol;
        if (valid < 32) {
#pragma unroll
          for (int k = 0; k < 32; ++k) s[k] = k < valid ? s[k] : NEG_INF;
        }
        float mx;
        {
          float m[5];
#pragma unroll
          for (int k = 0; k < 5; ++k) m[k] = max3f(s[6 * k], s[6 * k + 1], s[6 * k + 2]);
#pragma unroll
          for (int k = 0; k < 5; ++k) m[k] = max3f(m[k], s[6 * k + 3], s[6 * k + 4]);
#pragma unroll
          for (int k = 0; k < 5; ++k) m[k] = fmaxf(m[k], s[6 * k + 5]);
          mx = max3f(max3f(m[0], m[1], m[2]), max3f(m[3], m[4], s[30]), s[31]);
        }
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
        mx *= p.scale_log2;  // log2 units (scale > 0 keeps the arg max)
        float alpha = 1.f;
        bool resc = false;
        if (first) {
          m_ref = mx;
        } else if (mx > m_ref + kRescaleThreshold) {
          alpha = ex2_approx(m_ref - mx);
          m_ref = mx;
          resc = true;
        }
        uint32_t pk[16];
        float tot;
        {
          const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2);
          const uint64_t nb2 = f2_pack(-m_ref, -m_ref);
          uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            float x0, x1;
            f2_unpack(f2_fma(f2_pack(s[2 * k], s[2 * k + 1]), sc2, nb2), x0, x1);
            const float e0 = ex2_approx(x0);
            const float e1 = ex2_approx(x1);
            acc[k & 3] = f2_add(acc[k & 3], f2_pack(e0, e1));
            pk[k] = pack_bf16x2(e0, e1);
          }
          float a0, a1;
          f2_unpack(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), a0, a1);
          tot = a0 + a1;
        }
        tot += __shfl_xor_sync(kFull, tot, 16);
        l_sum = l_sum * alpha + tot;
        // ---- O rescale (rare): O must hold PV of the previous page first ----
        if (!first && __any_sync(kFull, resc)) {
          if (!(ok = warp_wait(&bars->pv_done[pb ^ 1], ((t - 1) >> 1) & 1, wc))) break;
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < 256; c += 64) {
            uint32_t r[32];
            tmem_ld16x2_32(tmem + kTmemO + c + lanes_own, r);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; ++k) r[k] = __float_as_uint(__uint_as_float(r[k]) * alpha);
            tmem_st16x2_32(tmem + kTmemO + c + lanes_own, r);
          }
          tmem_wait_st();
          tc_fence_before();
        }
        // ---- P -> shared memory (K-major, 128B swizzle) once PV(t - 2) has read buffer pb ----
        if (t >= 2 && !(ok = warp_wait(&bars->pv_done[pb], ((t >> 1) - 1) & 1, wc))) break;
#pragma unroll
        for (int c = 0; c < 4; ++c)
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                           p_loc + pb * kPBytes + xrow_off(row, 4 * hcol + c)),
                       "r"(pk[4 * c]), "r"(pk[4 * c + 1]), "r"(pk[4 * c + 2]), "r"(pk[4 * c + 3])
                       : "memory");
        fence_proxy_async_smem();  // generic-proxy writes -> visible to the tensor core
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bars->p_full[pb]);
          // the receive buffer was decoded long ago: warp 0 re-arms it for page t + 2 and every
          // warp hands it back (off the page's critical path)
          if (warp == 0) mbar_arrive_expect_tx(&bars->x_full[pb], kXBytes);
          mbar_arrive_remote_relaxed(xfree_rem + 8 * pb);
        }
      }
      if (!ok) break;
      // ---- the next segment's query half, as soon as the last QK of this one has run ----
      int nseq = 0, np0 = 0, np1 = 0;
      const bool next = it.next(nseq, np0, np1);
      if (next && kh == 0) {
        if (!(ok = warp_wait(&bars->q_empty, sg & 1, wc))) break;
        load_q(nseq);
      }
      // ---- segment epilogue: O / l -> global ----
      if (!(ok = warp_wait(&bars->seg_done, sg & 1, wc))) break;
      tc_fence_after();
      {
        const int nparts = plan.seq_nparts()[seq];
        float* dst;
        float* dst_lse;
        if (nparts == 1) {
          dst = p.o_lat + (static_cast<size_t>(seq) * p.n_heads + hd) * 512 + 256 * rank;
          dst_lse = p.lse ? p.lse + static_cast<size_t>(seq) * p.n_heads + hd : nullptr;
        } else {
          const int slot = plan.seq_slot()[seq] + (part - plan.seq_first_part()[seq]);
          dst = p.part_o + (static_cast<size_t>(slot) * p.n_heads + hd) * 512 + 256 * rank;
          dst_lse = p.part_lse + static_cast<size_t>(slot) * p.n_heads + hd;
        }
        const float inv_l = 1.f / l_sum;
#pragma unroll 1
        for (int c = 0; c < 256; c += 64) {
          uint32_t r[32];
          // thread (j, h) gets O columns c + 32h .. c + 32h + 31 of its row
          tmem_ld16x2_32(tmem + kTmemO + c + lanes_own, r);
          tmem_wait_ld();
          if (out_row) {
            float4* d4 = reinterpret_cast<float4*>(dst + c + 32 * hcol);
#pragma unroll
            for (int k = 0; k < 8; ++k)
              d4[k] = make_float4(__uint_as_float(r[4 * k]) * inv_l,
                                  __uint_as_float(r[4 * k + 1]) * inv_l,
                                  __uint_as_float(r[4 * k + 2]) * inv_l,
                                  __uint_as_float(r[4 * k + 3]) * inv_l);
          }
        }
        if (hcol == 0 && rank == 0 && out_row && dst_lse)
          *dst_lse = (m_ref + __log2f(l_sum)) * 0.69314718055994531f;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->o_free);
      ++sg;
      seq = nseq;
      p0 = np0;
      p1 = np1;
      have = next;
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();
  uint32_t peer_abort;
  asm volatile("ld.shared::cluster.u32 %0, [%1];"
               : "=r"(peer_abort)
               : "r"(mapa_shared(smem_u32(&bars->abort_flag), peer)));
  const bool aborted = bars->abort_flag != 0 || peer_abort != 0;
  // After an abort, remote stores and arrivals of the peer that nothing waited for may still be
  // in flight towards this CTA's shared memory: give them time to land before it is released.
  if (aborted) spin_ns(200000);
  if (warp == 13) {
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

// ------------------------------------------------------------------------------------------
// Merge of partial results that were computed apart (e.g. one per GPU, each over a range of a
// sequence's pages): part_o [n][rows][512] normalised, part_lse [n][rows]; for every row
//     lse = log sum_r exp(lse_r),   o = sum_r exp(lse_r - lse) o_r,
// the same log-sum-exp weights as the combine kernel.  A part with lse = -inf (no tokens)
// weighs nothing; a row whose parts are all empty gets o = 0, lse = -inf.
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(32 * kCombineWarps)
    merge_kernel(int n, int rows, const float* __restrict__ part_o,
                 const float* __restrict__ part_lse, float* __restrict__ o_lat,
                 float* __restrict__ lse) {
  griddep_launch_dependents();
  griddep_wait();
  const int row = blockIdx.x * kCombineWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const float NEG_INF = -__int_as_float(0x7f800000);
  float m = NEG_INF;
  for (int r = lane; r < n; r += 32) m = fmaxf(m, part_lse[static_cast<size_t>(r) * rows + row]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float4* out = reinterpret_cast<float4*>(o_lat + static_cast<size_t>(row) * 512);
  if (m == NEG_INF) {
#pragma unroll
    for (int k = 0; k < 4; ++k) out[lane + 32 * k] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (lane == 0 && lse) lse[row] = NEG_INF;
    return;
  }
  float tot = 0.f;
  float4 acc[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int r = 0; r < n; ++r) {
    const float l = part_lse[static_cast<size_t>(r) * rows + row];
    if (l == NEG_INF) continue;  // warp-uniform
    const float w = __expf(l - m);
    tot += w;
    const float4* src = reinterpret_cast<const float4*>(
        part_o + (static_cast<size_t>(r) * rows + row) * 512);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float4 v = src[lane + 32 * k];
      acc[k].x += w * v.x;
      acc[k].y += w * v.y;
      acc[k].z += w * v.z;
      acc[k].w += w * v.w;
    }
  }
  const float inv = 1.f / tot;
#pragma unroll
  for (int k = 0; k < 4; ++k)
    out[lane + 32 * k] = make_float4(acc[k].x * inv, acc[k].y * inv, acc[k].z * inv, acc[k].w * inv);
  if (lane == 0 && lse) lse[row] = m + __logf(tot);
}

}  // namespace attn
}  // namespace mla
