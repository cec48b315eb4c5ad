// Persistent "stream-K" weight-streaming GEMM on tcgen05 with the product's epilogue fused in.
//
//   Y_g[m][n] = sum_k A_g[m][k] * X_g[n][k]       (A = weights, X = a few activation rows)
//
// Decode projections multiply large weight matrices by a handful of token vectors, so their
// cost is the time to stream the weights from HBM once.  The work -- every (128-row tile,
// K block) pair of every group, a K block being one 128-byte piece of a row (64 bf16 or 128
// E4M3 values) -- is one list of I iterations cut into P equal
// contiguous ranges, one per CTA (P <= number of SMs), so every SM streams the same number of
// weight bytes in one wave and its TMA -> shared memory -> tcgen05.mma pipeline never drains
// between tiles.  A CTA's range splits into segments at tile boundaries; each segment is
// accumulated in one of two TMEM buffers (so the epilogue of one segment overlaps the MMAs of
// the next).
//
// A tile covered by one CTA is finished straight from TMEM.  A tile shared by several CTAs is
// finished by its first contributor, the CTA that accumulates the tile's first K blocks: that
// segment is the last of the CTA's range, while the other contributors cover the tile at the
// start (or all) of theirs, so by the time it gets there their partial sums are long written.
// Each other contributor writes its partial sum (column planes already added) to slot (its CTA
// index - the tile's first CTA index) of the tile's partial area, and each of its epilogue
// warps counts itself on the tile's counter; the finisher waits (bounded) for the full count,
// adds slots 1, 2, ... in slot order to its own sum from TMEM (so the result does not depend on
// arrival order) and runs the epilogue.  Only the finisher ever waits, and only for CTAs that
// wait for nobody.  Counters are tagged with a per-launch epoch in their upper 32 bits, so
// stale counts from earlier launches read as zero and the workspace never needs clearing; the
// finisher also clears its tile's counter, so a launch replayed with the same epoch (from a
// CUDA graph) starts from zero too.
//
// Roles (192 threads): warp 0 TMA producer, warp 1 MMA issuer + TMEM owner, warps 2-5
// epilogue (warp w reads TMEM lanes 32*(w%4) .. +31, i.e. tile rows).
//
// Launched with programmatic stream serialisation: the kernel may start while the previous
// kernel on its stream drains.  The producer requests its first ring of weight tiles at once
// (weights never depend on an earlier kernel), then waits for that kernel (griddepcontrol.wait)
// before it loads any activation; the epilogue warps wait before they touch global memory.
//
// Operand layouts in shared memory (128-byte swizzle, filled by TMA):
//   A K-major : box (64 k, 128 m)   -> [128 rows][128 B], SBO = 1024 B
//   A MN-major: 2 boxes (64 m, 64 k) -> [64 k rows][128 B] per 64-m half, LBO = 8 KiB
//   A tiled   : box (128 B, 128 m, kbs) from weights stored as 16 KB tiles -> the K-major layout
//   X         : box (64 k, 1, n_pad) -> [n_pad rows][128 B], SBO = 1024 B
//
// E4M3 instantiation (kFp8): weights and activations are E4M3 bytes, so a K block is 128 values
// in the same 128-byte rows, and tcgen05.mma.kind::f8f6f4 covers 32 of them per instruction
// with the bf16 path's descriptors and 32-byte K step.  The activations arrive as n_planes
// column planes (E4M3 pieces of one activation row) that the epilogue sums, then scales by the
// weight row's and the activation row's scales.
#pragma once
#include "ptx_sm100.cuh"
#include "rope.cuh"

namespace mla {
namespace sk {

constexpr int kThreads = 192;
constexpr uint64_t kDrainNs = 200000000ull;  // waits for copies and MMAs already in flight
constexpr uint32_t kATileBytes = 128 * 64 * 2;
constexpr int kRopePairs = 32;  // d_rope / 2

struct Params {
  int m_total;        // rows per group
  int m_tiles;        // 128-row tiles per group
  int groups;         // independent products (heads) sharing the launch
  int a1_tile_start;  // tiles (within a group) >= this read map A1, rows relative to it
  int a2_tile_start;  // tiles >= this read map A2, rows relative to it (>= a1_tile_start)
  int k_blocks;       // 64-wide K blocks per tile
  int kbs;            // K blocks per pipeline stage (one TMA box of A per stage)
  int units;          // stages' worth of work per tile: ceil(k_blocks / kbs)
  int n_pad;          // MMA N (multiple of 16, <= 256)
  int n_lo;           // > 0: columns [n_lo, 2 n_lo) hold the low halves of columns [0, n_lo)
  int n_out;          // valid output columns (the batch)
  int a_mn_major;     // 0: A K-major, 1: A MN-major
  int a_tiled;        // 1: the weights behind each map stored as contiguous tiles of 128 rows x
                      //    128 bytes, [row tiles][K / 128 bytes][128][128 B] (groups == 1 when
                      //    several maps are used)
  int stages;         // shared-memory ring depth
  int max_slots;      // partial slots per tile
  long long iters;    // m_tiles * groups * units
  uint32_t epoch;     // launch tag for the tile counters (never 0)
  float* partial;     // [tiles][max_slots][n_cols / 4][128][4], n_cols = n_lo or n_pad
  unsigned long long* counters;  // [tiles]
  const int32_t* positions;      // RoPE positions [n_out] (products with RoPE rows)
  float rope_theta;
  unsigned int* status;
  uint64_t wait_ns;
  int n_planes;          // X column planes summed into each output: 1, 2 (hi/lo) or 3
  const float* a_scale[3];  // E4M3: one scale per row of the weights behind map A0, A1, A2
  int a_rows[3];            //        and those weights' row counts
  const float* x_scale;     // E4M3: one scale per output column (an activation row)
};

// A stage holds kbs K blocks: A [kbs][128 rows][128 B] (K-major) or [2][64 kbs][128 B]
// (MN-major), then X [kbs][n_pad][128 B].
__host__ __device__ inline uint32_t stage_bytes(int n_pad, int kbs) {
  return static_cast<uint32_t>(kbs) * (kATileBytes + static_cast<uint32_t>(n_pad) * 128u);
}

// E4M3 operands (tcgen05 kind::f8f6f4): a 128-byte row of a K block holds 128 elements, so the
// shared-memory tiles, their descriptors and the 32-byte K step of one MMA are those of the
// bf16 path byte for byte.  Instruction descriptor: D f32, both operand formats 0 (E4M3).
__host__ __device__ constexpr uint32_t idesc_e4m3(int M, int N) {
  return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}
__device__ __forceinline__ void mma_ss_e4m3(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// First iteration of CTA c's range, and the CTA whose range holds iteration i.
__host__ __device__ inline long long range_start(long long c, long long iters, long long ctas) {
  return c * iters / ctas;
}
__host__ __device__ inline int cta_of(long long i, long long iters, long long ctas) {
  return static_cast<int>(((i + 1) * ctas - 1) / iters);
}

// Count this contributor in on the tile counter; returns the count including itself.
__device__ __forceinline__ uint32_t count_in(unsigned long long* ctr, uint32_t epoch,
                                             unsigned int* status) {
  unsigned long long cur = *reinterpret_cast<volatile unsigned long long*>(ctr);
  for (int it = 0; it < (1 << 20); ++it) {
    const unsigned long long nv = (static_cast<uint32_t>(cur >> 32) == epoch)
                                      ? cur + 1ull
                                      : ((static_cast<unsigned long long>(epoch) << 32) | 1ull);
    const unsigned long long prev = atomicCAS(ctr, cur, nv);
    if (prev == cur) return static_cast<uint32_t>(nv);
    cur = prev;
  }
  atomicOr(status, MLA_STATUS_TIMEOUT);
  return 0;
}

// ---------------------------------------------------------------------------------------------
// Epilogues.  apply() is called by all 32 lanes of a warp together (lane = tile row), for 16
// output columns c0 .. c0+15 of row r of group g; v[j] is the finished value of column c0 + j.
// RoPE rows exchange their pair partner with the neighbouring lane (pairs are (even, odd)
// rows, and a warp's 32 rows never straddle a RoPE boundary).
// ---------------------------------------------------------------------------------------------
// Fill the [n][32] (cos, sin) table for the n RoPE positions (epilogue warps, once per CTA).
__device__ __forceinline__ void rope_table(float2* tab, const int32_t* positions, int n,
                                           float theta, int tid, int nthreads) {
  for (int e = tid; e < n * kRopePairs; e += nthreads)
    tab[e] = rope_cs(theta, e % kRopePairs, positions[e / kRopePairs]);
}

__device__ __forceinline__ void rope_rotate(const float2* tab, int b, int pair, bool odd,
                                            float v, float partner, float& out) {
  const float2 cs = tab[b * kRopePairs + pair];
  // (x0, x1) -> (x0 c - x1 s, x0 s + x1 c); this lane holds x1 when odd.
  out = odd ? (partner * cs.y + v * cs.x) : (v * cs.x - partner * cs.y);
}

// Every epilogue gets a shared-memory area of smem_bytes(n_out) bytes that its prepare()
// fills once per CTA (epilogue warps only, before the first tile is finished), so that the
// per-element work reads no global memory besides the partial sums.
// Cache append: rows 0..511 = c_KV, 512..575 = k_R (rotated); scattered into the page slot.
struct EpiAppend {
  static constexpr bool kRope = true;
  const int32_t* positions;
  const int32_t* page_table;
  int max_pages;
  __nv_bfloat16* pool;
  int num_pages;
  unsigned int* status;
  float theta;
  // [n][32] float2 RoPE table, then [n] int64 offsets of the destination rows (-1: invalid)
  __host__ __device__ static size_t smem_bytes(int n) {
    return static_cast<size_t>(n) * (kRopePairs * 8 + 8);
  }
  __device__ void prepare(uint8_t* sm, int n, int tid, int nthreads) const {
    constexpr int kRow = 576, kPage = 64;
    rope_table(reinterpret_cast<float2*>(sm), positions, n, theta, tid, nthreads);
    long long* off = reinterpret_cast<long long*>(sm + static_cast<size_t>(n) * kRopePairs * 8);
    for (int b = tid; b < n; b += nthreads) {
      long long o = -1;
      const int pos = positions[b];
      if (pos < 0 || pos >= max_pages * kPage) {
        atomicOr(status, MLA_STATUS_BAD_POSITION);
      } else {
        const int page = page_table[static_cast<size_t>(b) * max_pages + pos / kPage];
        if (page < 0 || page >= num_pages)
          atomicOr(status, MLA_STATUS_BAD_PAGE);
        else
          o = (static_cast<long long>(page) * kPage + pos % kPage) * kRow;
      }
      off[b] = o;
    }
  }
  __device__ void apply(const uint8_t* sm, int, int r, bool valid, int c0, int n_out,
                        float (&v)[16]) const {
    constexpr int kDc = 512;
    const float2* tab = reinterpret_cast<const float2*>(sm);
    const long long* off =
        reinterpret_cast<const long long*>(sm + static_cast<size_t>(n_out) * kRopePairs * 8);
    const bool rope = r >= kDc;  // warp-uniform
    float p[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) p[j] = __shfl_xor_sync(0xffffffffu, v[j], 1);
    if (!valid) return;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int b = c0 + j;
      if (b >= n_out) break;
      const long long o = off[b];
      if (o < 0) continue;
      float x = v[j];
      if (rope) rope_rotate(tab, b, (r - kDc) >> 1, r & 1, v[j], p[j], x);
      pool[o + r] = __float2bfloat16_rn(x);
    }
  }
};

// q = W_Q h: per head rows 0..127 -> q_nope as bf16 hi/lo planes [2][n_lo_pad][H][128],
// rows 128..191 -> RoPE(q_rope) into q_cat[b][h][512..575] (+ its bf16 remainder in q_lo).
struct EpiWq {
  static constexpr bool kRope = true;
  int H;
  int b_pad;  // rows per hi/lo plane
  __nv_bfloat16* q_cat;
  __nv_bfloat16* q_lo;
  __nv_bfloat16* qn;
  const int32_t* positions;
  float theta;
  __host__ __device__ static size_t smem_bytes(int n) {
    return static_cast<size_t>(n) * kRopePairs * 8;
  }
  __device__ void prepare(uint8_t* sm, int n, int tid, int nthreads) const {
    rope_table(reinterpret_cast<float2*>(sm), positions, n, theta, tid, nthreads);
  }
  __device__ void apply(const uint8_t* sm, int, int r, bool valid, int c0, int n_out,
                        float (&v)[16]) const {
    constexpr int kDn = 128, kDq = 192, kRow = 576, kDc = 512;
    const float2* tab = reinterpret_cast<const float2*>(sm);
    const int h = r / kDq, d = r - h * kDq;
    const bool rope = d >= kDn;  // warp-uniform
    float p[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) p[j] = __shfl_xor_sync(0xffffffffu, v[j], 1);
    if (!valid) return;
    const size_t plane = static_cast<size_t>(b_pad) * H * kDn;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int b = c0 + j;
      if (b >= n_out) break;
      if (!rope) {
        const size_t o = (static_cast<size_t>(b) * H + h) * kDn + d;
        const __nv_bfloat16 hi = __float2bfloat16_rn(v[j]);
        qn[o] = hi;
        qn[plane + o] = __float2bfloat16_rn(v[j] - __bfloat162float(hi));
      } else {
        float x;
        rope_rotate(tab, b, (d - kDn) >> 1, d & 1, v[j], p[j], x);
        const size_t o = (static_cast<size_t>(b) * H + h) * kRow + kDc + (d - kDn);
        const __nv_bfloat16 e = __float2bfloat16_rn(x);
        q_cat[o] = e;
        if (q_lo) q_lo[o] = __float2bfloat16_rn(x - __bfloat162float(e));
      }
    }
  }
};

// Folded query: with W_UK absorbed into W_Q offline, the folded matrix has 576 rows per head
// (512 latent rows W_UK_h^T W_Q,nope,h, then W_Q's 64 RoPE rows) and its product with h maps
// row for row onto q_cat[b][h][0..575]; the last 64 rows of a head are rotated at the token's
// position.  Head boundaries and the 512 split fall on 32-row (warp) boundaries.
struct EpiWqFold {
  static constexpr bool kRope = true;
  int H;
  __nv_bfloat16* q_cat;
  __nv_bfloat16* q_lo;
  const int32_t* positions;
  float theta;
  __host__ __device__ static size_t smem_bytes(int n) {
    return static_cast<size_t>(n) * kRopePairs * 8;
  }
  __device__ void prepare(uint8_t* sm, int n, int tid, int nthreads) const {
    rope_table(reinterpret_cast<float2*>(sm), positions, n, theta, tid, nthreads);
  }
  __device__ void apply(const uint8_t* sm, int, int r, bool valid, int c0, int n_out,
                        float (&v)[16]) const {
    constexpr int kRow = 576, kDc = 512;
    const float2* tab = reinterpret_cast<const float2*>(sm);
    const int h = r / kRow, d = r - h * kRow;
    const bool rope = d >= kDc;  // warp-uniform
    float p[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) p[j] = __shfl_xor_sync(0xffffffffu, v[j], 1);
    if (!valid) return;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int b = c0 + j;
      if (b >= n_out) break;
      float x = v[j];
      if (rope) rope_rotate(tab, b, (d - kDc) >> 1, d & 1, v[j], p[j], x);
      const size_t o = (static_cast<size_t>(b) * H + h) * kRow + d;
      const __nv_bfloat16 e = __float2bfloat16_rn(x);
      q_cat[o] = e;
      if (q_lo) q_lo[o] = __float2bfloat16_rn(x - __bfloat162float(e));
    }
  }
};

// q_lat_h = W_UK_h^T q_nope_h (hi + lo already summed) -> q_cat[b][h][0..511] (+ q_lo).
// Cache append and a query product in one launch (both multiply the same hidden states): rows
// [0, 640) are the append tiles (W_DKV then W_KR; rows 576..639 padding), rows from 640 on are
// the query's.  Both use the RoPE table that EpiAppend::prepare builds at the start of the area.
template <class Q>
struct EpiAppendQ {
  static constexpr bool kRope = true;
  static constexpr int kSplitRow = 640;
  EpiAppend a;
  Q q;
  __host__ __device__ static size_t smem_bytes(int n) { return EpiAppend::smem_bytes(n); }
  __device__ void prepare(uint8_t* sm, int n, int tid, int nthreads) const {
    a.prepare(sm, n, tid, nthreads);
  }
  __device__ void apply(const uint8_t* sm, int g, int r, bool valid, int c0, int n_out,
                        float (&v)[16]) const {
    if (r < kSplitRow)  // warp-uniform: a warp's rows lie in one tile
      a.apply(sm, g, r, valid && r < 576, c0, n_out, v);
    else
      q.apply(sm, g, r - kSplitRow, valid, c0, n_out, v);
  }
};
using EpiAppendWq = EpiAppendQ<EpiWq>;
using EpiAppendWqFold = EpiAppendQ<EpiWqFold>;

struct EpiWuk {
  static constexpr bool kRope = false;
  int H;
  __nv_bfloat16* q_cat;
  __nv_bfloat16* q_lo;
  __host__ __device__ static size_t smem_bytes(int) { return 0; }
  __device__ void prepare(uint8_t*, int, int, int) const {}
  __device__ void apply(const uint8_t*, int g, int r, bool valid, int c0, int n_out,
                        float (&v)[16]) const {
    constexpr int kRow = 576;
    if (!valid) return;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int b = c0 + j;
      if (b >= n_out) break;
      const size_t o = (static_cast<size_t>(b) * H + g) * kRow + r;
      const __nv_bfloat16 e = __float2bfloat16_rn(v[j]);
      q_cat[o] = e;
      if (q_lo) q_lo[o] = __float2bfloat16_rn(v[j] - __bfloat162float(e));
    }
  }
};

// o_h = W_UV_h o_lat_h -> o_heads[b][h][0..127] and/or bf16 hi/lo planes [2][b_pad][H*128].
struct EpiWuv {
  static constexpr bool kRope = false;
  int H;
  int b_pad;
  __nv_bfloat16* o_heads;
  __nv_bfloat16* oh;
  float* oh32 = nullptr;  // or o_heads in fp32 [b][h][128] (split into E4M3 planes next),
  unsigned int* rowmax = nullptr;  // with max_{h,i} |o_heads[b][h][i]| per b (fp32 bits,
                                   // zeroed before the launch) raised by atomicMax
  __host__ __device__ static size_t smem_bytes(int) { return 0; }
  __device__ void prepare(uint8_t*, int, int, int) const {}
  __device__ void apply(const uint8_t*, int g, int r, bool valid, int c0, int n_out,
                        float (&v)[16]) const {
    constexpr int kDv = 128;
    if (rowmax) {
      // |v| over the warp's 32 rows for each of the 16 columns; lane j raises column c0 + j
      float mine = 0.f;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        float m = valid ? fabsf(v[j]) : 0.f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if ((threadIdx.x & 31) == j) mine = m;
      }
      const int lane = threadIdx.x & 31;
      if (lane < 16 && c0 + lane < n_out) atomicMax(rowmax + c0 + lane, __float_as_uint(mine));
    }
    if (!valid) return;
    const size_t plane = static_cast<size_t>(b_pad) * H * kDv;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int b = c0 + j;
      if (b >= n_out) break;
      const size_t o = (static_cast<size_t>(b) * H + g) * kDv + r;
      const __nv_bfloat16 hi = __float2bfloat16_rn(v[j]);
      if (o_heads) o_heads[o] = hi;
      if (oh) {
        oh[o] = hi;
        oh[plane + o] = __float2bfloat16_rn(v[j] - __bfloat162float(hi));
      }
      if (oh32) oh32[o] = v[j];
    }
  }
};

// out = W_O [o_1 .. o_H] -> out[b][0..D-1].
struct EpiWo {
  static constexpr bool kRope = false;
  int D;
  __nv_bfloat16* out;
  __host__ __device__ static size_t smem_bytes(int) { return 0; }
  __device__ void prepare(uint8_t*, int, int, int) const {}
  __device__ void apply(const uint8_t*, int, int r, bool valid, int c0, int n_out,
                        float (&v)[16]) const {
    if (!valid) return;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int b = c0 + j;
      if (b >= n_out) break;
      out[static_cast<size_t>(b) * D + r] = __float2bfloat16_rn(v[j]);
    }
  }
};

// Adds 16 columns of one row from slots 1 .. n-1, in slot order, to v.  src points at the row's
// first float4 of the 16 columns in slot 0; the loads of four slots are in flight at once.
__device__ __forceinline__ void add_slots(const float4* src, size_t slot_stride, int n,
                                          float (&v)[16]) {
  for (int s0 = 1; s0 < n; s0 += 4) {
    float4 y[4][4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (s0 + u < n)
#pragma unroll
        for (int q = 0; q < 4; ++q) y[u][q] = __ldcg(src + (s0 + u) * slot_stride + q * 128);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (s0 + u >= n) break;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        v[4 * q] += y[u][q].x;
        v[4 * q + 1] += y[u][q].y;
        v[4 * q + 2] += y[u][q].z;
        v[4 * q + 3] += y[u][q].w;
      }
    }
  }
}

// The finishing CTA of a shared tile waits until the other contributors' warps (4 each) have
// counted in under this launch's epoch.  Bounded like every wait: false on abort or timeout.
__device__ __forceinline__ bool wait_count(const unsigned long long* ctr, uint32_t epoch,
                                           uint32_t target, const WaitCtx& w) {
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 1;; ++i) {
    const unsigned long long v = *reinterpret_cast<const volatile unsigned long long*>(ctr);
    if (static_cast<uint32_t>(v >> 32) == epoch && static_cast<uint32_t>(v) >= target)
      return true;
    if ((i & 15) == 0) {
      if (*w.abort_flag) return false;
      if (globaltimer_ns() - t0 > w.limit_ns) {
        *w.abort_flag = 1;
        atomicOr(w.status, MLA_STATUS_TIMEOUT);
        return false;
      }
    }
  }
}

// 16 accumulator columns c0 .. c0+15 of this warp's TMEM lanes, summed over the n_planes column
// planes (plane pl at columns pl * n_lo + c): all planes' loads are issued before one wait.
__device__ __forceinline__ void tmem_sum_planes(uint32_t tacc, int c0, int n_planes, int n_lo,
                                                float (&v)[16]) {
  uint32_t a[3][16];
  tmem_ld16(tacc + c0, a[0]);
  if (n_planes > 1) tmem_ld16(tacc + n_lo + c0, a[1]);
  if (n_planes > 2) tmem_ld16(tacc + 2 * n_lo + c0, a[2]);
  tmem_wait_ld();
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    float x = __uint_as_float(a[0][j]);
    if (n_planes > 1) x += __uint_as_float(a[1][j]);
    if (n_planes > 2) x += __uint_as_float(a[2][j]);
    v[j] = x;
  }
}

// E4M3 products: the fp32 sum of a row times its weight row's scale and the column's scale.
// Row r (within a group) lies in tile r / 128, which selects the weights (map A0, A1 or A2)
// exactly as the producer does; rows past those weights' end get scale 0.
__device__ __forceinline__ void scale_e4m3(const Params& p, int r, bool valid, int c0,
                                           float (&v)[16]) {
  const int mt = r >> 7;
  const int m = mt >= p.a2_tile_start ? 2 : mt >= p.a1_tile_start ? 1 : 0;
  const int rr = r - (m == 2 ? p.a2_tile_start * 128 : m == 1 ? p.a1_tile_start * 128 : 0);
  const float sr = valid && rr < p.a_rows[m] ? p.a_scale[m][rr] : 0.f;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int b = c0 + j;
    v[j] *= b < p.n_out ? sr * p.x_scale[b] : 0.f;
  }
}

// ---------------------------------------------------------------------------------------------
template <class Epi, bool kFp8 = false>
__global__ void __launch_bounds__(kThreads, 1)
    streamk_gemm_kernel(const __grid_constant__ CUtensorMap tmA0,
                        const __grid_constant__ CUtensorMap tmA1,
                        const __grid_constant__ CUtensorMap tmA2,
                        const __grid_constant__ CUtensorMap tmX, const Params p, const Epi epi) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbytes = stage_bytes(p.n_pad, p.kbs);
  const uint32_t a_bytes = static_cast<uint32_t>(p.kbs) * kATileBytes;
  uint8_t* epi_smem = smem + p.stages * sbytes;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(
      epi_smem + ((Epi::smem_bytes(p.n_out) + 15) & ~static_cast<size_t>(15)));
  uint64_t* empty_bar = full_bar + p.stages;
  uint64_t* acc_full = empty_bar + p.stages;   // [2]
  uint64_t* acc_empty = acc_full + 2;          // [2], 4 arrivals (one per epilogue warp)
  uint64_t* fin_ready = acc_empty + 2;         // 1 arrival: a shared tile's count is complete
  uint64_t* mma_done = fin_ready + 1;          // final drain of the MMA pipe
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* fin_flag = abort_flag + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const long long c = blockIdx.x;
  const long long P = gridDim.x;
  const long long i_begin = range_start(c, p.iters, P);
  const long long i_end = range_start(c + 1, p.iters, P);
  const long long kb = p.units;  // work units per tile
  uint32_t tmem_cols = 32;
  while (tmem_cols < 2u * static_cast<uint32_t>(p.n_pad)) tmem_cols <<= 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    mbar_init(fin_ready, 1);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    *fin_flag = 0;
    fence_mbar_init_cluster();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  WaitCtx wc{abort_flag, p.status, p.wait_ns};
  griddep_launch_dependents();

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      tma_prefetch_desc(&tmA0);
      tma_prefetch_desc(&tmA1);
      tma_prefetch_desc(&tmA2);
      tma_prefetch_desc(&tmX);
      const uint64_t pol_w = l2_policy_evict_first();
      const uint64_t pol_x = l2_policy_evict_last();
      auto load_a = [&](long long i, int s) {
        const long long t = i / kb;
        const int kb0 = static_cast<int>(i - t * kb) * p.kbs;
        const int g = static_cast<int>(t / p.m_tiles);
        const int mt = static_cast<int>(t - static_cast<long long>(g) * p.m_tiles);
        const CUtensorMap* tmA = &tmA0;
        int m_row0 = mt * 128;
        if (mt >= p.a2_tile_start) {
          tmA = &tmA2;
          m_row0 = (mt - p.a2_tile_start) * 128;
        } else if (mt >= p.a1_tile_start) {
          tmA = &tmA1;
          m_row0 = (mt - p.a1_tile_start) * 128;
        }
        uint8_t* a_dst = smem + s * sbytes;
        if (p.a_tiled) {
          // view (128 B, 128 rows, K blocks, row tiles): box (128 B, 128, kbs, 1) is one
          // contiguous run of kbs tiles in HBM
          tma_load_4d_hint(a_dst, tmA, &full_bar[s], 0, 0, kb0, g * p.m_tiles + m_row0 / 128,
                           pol_w);
        } else if (p.a_mn_major) {
          // [g][k][m] with m contiguous: box (64 m, 64 kbs k) per 64-row half of the tile
          tma_load_3d_hint(a_dst, tmA, &full_bar[s], m_row0, kb0 * 64, g, pol_w);
          tma_load_3d_hint(a_dst + a_bytes / 2, tmA, &full_bar[s], m_row0 + 64, kb0 * 64, g,
                           pol_w);
        } else {
          // view (64 k, rows, groups, k blocks): box (64, 128, 1, kbs)
          tma_load_4d_hint(a_dst, tmA, &full_bar[s], 0, m_row0, g, kb0, pol_w);
        }
      };
      auto load_x = [&](long long i, int s) {
        const long long t = i / kb;
        const int kb0 = static_cast<int>(i - t * kb) * p.kbs;
        const int g = static_cast<int>(t / p.m_tiles);
        // view (64 k, groups, n, k blocks): box (64, 1, n_pad, kbs)
        tma_load_4d_hint(smem + s * sbytes + a_bytes, &tmX, &full_bar[s], 0, g, 0, kb0, pol_x);
      };
      // The weights never depend on the preceding kernel: the first ring's worth of weight
      // tiles is requested before waiting for that kernel to finish, the activations after.
      const long long pre = min(i_end - i_begin, static_cast<long long>(p.stages));
      for (long long j = 0; j < pre; ++j) {
        mbar_arrive_expect_tx(&full_bar[j], sbytes);
        load_a(i_begin + j, static_cast<int>(j));
      }
      griddep_wait();
      for (long long j = 0; j < pre; ++j) load_x(i_begin + j, static_cast<int>(j));
      long long issued = pre;
      for (long long i = i_begin + pre; i < i_end; ++i, ++issued) {
        const int s = static_cast<int>(issued % p.stages);
        const uint32_t ph = static_cast<uint32_t>((issued / p.stages) & 1);
        if (!mbar_wait(&empty_bar[s], ph ^ 1, wc)) break;
        mbar_arrive_expect_tx(&full_bar[s], sbytes);
        load_a(i, s);
        load_x(i, s);
      }
      // No copy may still be landing when the CTA exits: normally the MMA warp has consumed
      // every stage and these return at once; after an abort (raised by any role, at any
      // time) they wait, on their own limit, for the copies still in flight.
      {
        volatile int never = 0;
        WaitCtx drain{&never, p.status, kDrainNs};
        for (long long j = (issued > p.stages ? issued - p.stages : 0); j < issued; ++j)
          mbar_wait(&full_bar[j % p.stages], static_cast<uint32_t>((j / p.stages) & 1), drain);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc =
          kFp8 ? idesc_e4m3(128, p.n_pad) : idesc_bf16(128, p.n_pad, p.a_mn_major, 0);
      long long it = 0;  // iteration counter (ring position)
      int seg = 0;
      bool ok = true;
      for (long long i = i_begin; i < i_end && ok; ++seg) {
        const long long t = i / kb;
        const long long seg_end = min(i_end, (t + 1) * kb);
        const int buf = seg & 1;
        if (!mbar_wait(&acc_empty[buf], static_cast<uint32_t>(((seg >> 1) & 1) ^ 1), wc)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * p.n_pad);
        for (; i < seg_end; ++i, ++it) {
          const int s = static_cast<int>(it % p.stages);
          if (!mbar_wait(&full_bar[s], static_cast<uint32_t>((it / p.stages) & 1), wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + s * sbytes);
          const uint32_t x_base = a_base + a_bytes;
          const bool first = (i == t * kb) || (i == i_begin);
          for (int kk = 0; kk < 4 * p.kbs; ++kk) {
            const uint32_t kq = static_cast<uint32_t>(kk >> 2), kr = static_cast<uint32_t>(kk & 3);
            const uint64_t xdesc =
                smem_desc(x_base + kq * static_cast<uint32_t>(p.n_pad) * 128u + kr * 32, 16, 1024,
                          kSwizzle128B);
            const uint64_t adesc =
                p.a_mn_major
                    ? smem_desc(a_base + kk * 2048, a_bytes / 2, 1024, kSwizzle128B)
                    : smem_desc(a_base + kq * kATileBytes + kr * 32, 16, 1024, kSwizzle128B);
            if (kFp8)
              mma_ss_e4m3(d_tmem, adesc, xdesc, idesc, (first && kk == 0) ? 0u : 1u);
            else
              mma_ss(d_tmem, adesc, xdesc, idesc, (first && kk == 0) ? 0u : 1u);
          }
          mma_commit(&empty_bar[s]);
        }
        if (ok) mma_commit(&acc_full[buf]);
      }
      mma_commit(mma_done);  // fires once every issued MMA has completed
    }
  } else {
    // ---------------- epilogue ----------------
    const int quarter = warp & 3;
    const int m_local = quarter * 32 + lane;
    // per-CTA epilogue tables while the first tiles stream in (epilogue warps only), once the
    // preceding kernel's writes are visible
    griddep_wait();
    epi.prepare(epi_smem, p.n_out, threadIdx.x - 64, 128);
    asm volatile("bar.sync 1, 128;" ::: "memory");
    const int n_cols = p.n_lo > 0 ? p.n_lo : p.n_pad;  // columns that are outputs
    int seg = 0, multi = 0;
    for (long long i = i_begin; i < i_end; ++seg) {
      const long long t = i / kb;
      const long long seg_end = min(i_end, (t + 1) * kb);
      i = seg_end;
      const int g = static_cast<int>(t / p.m_tiles);
      const int mt = static_cast<int>(t - static_cast<long long>(g) * p.m_tiles);
      const int r = mt * 128 + m_local;
      const bool valid = r < p.m_total;
      const int c_first = cta_of(t * kb, p.iters, P);
      const int c_last = cta_of((t + 1) * kb - 1, p.iters, P);
      const int buf = seg & 1;
      if (!warp_wait(&acc_full[buf], static_cast<uint32_t>((seg >> 1) & 1), wc)) break;
      tc_fence_after();
      const uint32_t tacc = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                            static_cast<uint32_t>(buf * p.n_pad);
      if (c_first == c_last) {
        // whole tile in this CTA: finish from TMEM
        for (int c0 = 0; c0 < n_cols; c0 += 16) {
          float v[16];
          tmem_sum_planes(tacc, c0, p.n_planes, p.n_lo, v);
          if (kFp8) scale_e4m3(p, r, valid, c0, v);
          epi.apply(epi_smem, g, r, valid, c0, p.n_out, v);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[buf]);
        continue;
      }
      const int n_contrib = c_last - c_first + 1;
      // slot layout [n_cols / 4][128 rows][4 columns]: a warp moves 512 contiguous bytes
      float4* part_tile = reinterpret_cast<float4*>(p.partial) +
                          static_cast<size_t>(t) * p.max_slots * (n_cols / 4) * 128 + m_local;
      const size_t slot_stride = static_cast<size_t>(n_cols / 4) * 128;  // in float4
      if (c != c_first) {
        // shared tile, not ours to finish: publish the partial sum, count this warp in
        float4* dst = part_tile + static_cast<size_t>(c - c_first) * slot_stride;
        for (int c0 = 0; c0 < n_cols; c0 += 16) {
          float v[16];
          tmem_sum_planes(tacc, c0, p.n_planes, p.n_lo, v);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
            __stcg(dst + (c0 / 4 + q4) * 128,
                   make_float4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]));
        }
        tc_fence_before();
        __threadfence();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&acc_empty[buf]);
          count_in(&p.counters[t], p.epoch, p.status);
        }
        continue;
      }
      // shared tile to finish: wait for the other contributors' 4 (n_contrib - 1) warps
      const uint32_t ph = static_cast<uint32_t>(multi & 1);
      ++multi;
      if (warp == 2 && lane == 0) {
        const bool ok = wait_count(&p.counters[t], p.epoch,
                                   4u * static_cast<uint32_t>(n_contrib - 1), wc);
        if (ok) atomicExch(&p.counters[t], 0ull);  // last user of this counter in the launch
        __threadfence();
        *fin_flag = ok ? 1 : 0;
        mbar_arrive(fin_ready);
      }
      if (!warp_wait(fin_ready, ph, wc)) break;
      if (*fin_flag) {
        for (int c0 = 0; c0 < n_cols; c0 += 16) {
          float v[16];
          tmem_sum_planes(tacc, c0, p.n_planes, p.n_lo, v);
          add_slots(part_tile + (c0 / 4) * 128, slot_stride, n_contrib, v);
          if (kFp8) scale_e4m3(p, r, valid, c0, v);
          epi.apply(epi_smem, g, r, valid, c0, p.n_out, v);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
    }
  }

  // Never release TMEM while issued MMAs may still write it.
  if (warp == 1 && lane == 0) {
    volatile int never = 0;
    WaitCtx drain{&never, p.status, kDrainNs};
    mbar_wait(mma_done, 0, drain);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, tmem_cols);
  }
}

}  // namespace sk
}  // namespace mla
