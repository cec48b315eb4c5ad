// C ABI of the MLA decode library (see include/mla.h for the contract of every entry point).
// Host side: argument validation (before any CUDA call), per-device context, TMA descriptor
// encoding, workspace layout, launch configuration.  All device work is in the included
// kernel headers.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <atomic>
#include <mutex>
#include <utility>

#include "attn_f32.cuh"
#include "attn_sm100.cuh"
#include "epilogue.cuh"
#include "fold.cuh"
#include "fp8.cuh"
#include "gemm_streamk.cuh"

namespace mla {

__device__ unsigned int g_status_word;

namespace {

constexpr int kDc = 512, kDr = 64, kDn = 128, kDv = 128, kRowN = 576, kPageN = 64;
constexpr uint64_t kDefaultWaitNs = 2000000000ull;  // 2 s per bounded wait

// Time limit of one bounded wait inside a kernel: 2 s, or MLA_WAIT_NS (nanoseconds, >= 1) from
// the environment, read at every call.  A small value makes the waits give up early, which is
// how the timeout path (status bit, abort and drain, usable context afterwards) is exercised.
uint64_t wait_limit_ns() {
  const char* e = std::getenv("MLA_WAIT_NS");
  if (!e || !*e) return kDefaultWaitNs;
  char* end = nullptr;
  const unsigned long long v = std::strtoull(e, &end, 10);
  return (end && *end == '\0' && v >= 1) ? static_cast<uint64_t>(v) : kDefaultWaitNs;
}

// MLA_TEST_STALL=1 in the environment (read at each call): one warp of every split-KV CTA
// first waits on a barrier nothing arrives on, so that the wait runs out and the timeout path
// is taken.  A test hook; results of such a call are meaningless and the status says so.
int stall_test_requested() {
  const char* e = std::getenv("MLA_TEST_STALL");
  return (e && e[0] == '1' && e[1] == '\0') ? 1 : 0;
}
constexpr int kMinPagesPerPart = 4;
constexpr int kMaxParts = 1 << 16;  // upper bound on num_splits (host check before any arithmetic)
constexpr int kSkMinUnits = 2;    // fewest stages' worth of weights a stream-K CTA streams
constexpr int kSkMaxContrib = 4;  // aim for at most this many CTAs sharing one tile
constexpr int kSkMaxStages = 12;
constexpr int kFp8MaxBatch = 128;  // E4M3 products: planes x round16(B) <= 256 MMA columns
constexpr size_t kSmemPerBlockMax = 232448;  // 227 KiB opt-in limit per CTA

// ------------------------------------------------------------------------------------------
// validation
// ------------------------------------------------------------------------------------------
bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_dims(const mla_dims* d) {
  if (!d) return MLA_ERR_NULL_ARG;
  if (d->d_c != kDc || d->d_rope != kDr || d->d_nope != kDn || d->d_v != kDv ||
      d->page_size != kPageN)
    return MLA_ERR_DIMS;
  if (d->n_heads < 16 || d->n_heads > 128 || d->n_heads % 16) return MLA_ERR_DIMS;
  if (d->d_model <= 0 || d->d_model % 64) return MLA_ERR_DIMS;
  if (d->batch < 1) return MLA_ERR_DIMS;
  if (d->dtype != MLA_BF16 && d->dtype != MLA_FP32) return MLA_ERR_DIMS;
  if (d->dtype == MLA_BF16 && d->batch > 128) return MLA_ERR_DIMS;  // 2B <= 256 MMA columns
  if (!(d->rope_theta > 0.f) || !std::isfinite(d->rope_theta)) return MLA_ERR_DIMS;
  return MLA_OK;
}

size_t elem_size(const mla_dims* d) { return d->dtype == MLA_BF16 ? 2 : 4; }

// ------------------------------------------------------------------------------------------
// per-device context
// ------------------------------------------------------------------------------------------
struct DevCtx {
  bool init = false;
  int cc_major = 0;
  int sms = 0;
  int max_clusters = 0;
  unsigned int* status = nullptr;
};
DevCtx g_dev[64];
std::mutex g_mu;
std::atomic<unsigned long long> g_launches{0};
// profiling hook: events recorded around the split-KV kernel of successive decode calls
cudaEvent_t* g_prof_begin = nullptr;
cudaEvent_t* g_prof_end = nullptr;
int g_prof_count = 0;
int g_prof_next = 0;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// Description of the last CUDA call of this thread that failed inside the library.
thread_local char g_err_detail[256] = "";

int cuda_fail(cudaError_t e, const char* where) {
  std::snprintf(g_err_detail, sizeof(g_err_detail), "%s: %s (%s)", where, cudaGetErrorName(e),
                cudaGetErrorString(e));
  return MLA_ERR_CUDA;
}

int device_ctx(DevCtx** out) {
  int dev = 0;
  cudaError_t e;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return MLA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  DevCtx& c = g_dev[dev];
  if (!c.init) {
    if ((e = cudaDeviceGetAttribute(&c.cc_major, cudaDevAttrComputeCapabilityMajor, dev)) !=
        cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute");
    if (c.cc_major != 10) return MLA_ERR_DEVICE;
    if ((e = cudaDeviceGetAttribute(&c.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute");
    void* sym = nullptr;
    if ((e = cudaGetSymbolAddress(&sym, g_status_word)) != cudaSuccess)
      return cuda_fail(e, "cudaGetSymbolAddress(status word)");
    c.status = static_cast<unsigned int*>(sym);
    if (!g_encode) {
      cudaDriverEntryPointQueryResult q;
      void* fn = nullptr;
      if ((e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q)) !=
          cudaSuccess)
        return cuda_fail(e, "cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)");
      if (q != cudaDriverEntryPointSuccess || !fn) return MLA_ERR_CUDA;
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    // kernel attributes (once per device)
    const int attn_smem = static_cast<int>(attn::kSmemBytes);
    if ((e = cudaFuncSetAttribute(attn::split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  attn_smem)) != cudaSuccess)
      return cuda_fail(e, "cudaFuncSetAttribute(split_kernel)");
    const int sk_smem = static_cast<int>(kSmemPerBlockMax);
    const void* sk_kernels[9] = {
        reinterpret_cast<const void*>(sk::streamk_gemm_kernel<sk::EpiAppend>),
        reinterpret_cast<const void*>(sk::streamk_gemm_kernel<sk::EpiWq>),
        reinterpret_cast<const void*>(sk::streamk_gemm_kernel<sk::EpiWuk>),
        reinterpret_cast<const void*>(sk::streamk_gemm_kernel<sk::EpiWuv>),
        reinterpret_cast<const void*>(sk::streamk_gemm_kernel<sk::EpiWo>),
        reinterpret_cast<const void*>(sk::streamk_gemm_kernel<sk::EpiAppendWq>),
        reinterpret_cast<const void*>(sk::streamk_gemm_kernel<sk::EpiAppendWqFold>),
        reinterpret_cast<const void*>(sk::streamk_gemm_kernel<sk::EpiWo, true>),
        reinterpret_cast<const void*>(sk::streamk_gemm_kernel<sk::EpiAppendWq, true>)};
    for (const void* k : sk_kernels)
      if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, sk_smem)) !=
          cudaSuccess)
        return cuda_fail(e, "cudaFuncSetAttribute(streamk_gemm_kernel)");
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(attn::kThreads, 1, 1);
    cfg.dynamicSmemBytes = attn::kSmemBytes;
    int nclusters = 0;
    if (cudaOccupancyMaxActiveClusters(&nclusters, attn::split_kernel, &cfg) != cudaSuccess ||
        nclusters <= 0) {
      (void)cudaGetLastError();  // a failed query only means: fall back to one per SM pair
      nclusters = c.sms / 2;
    }
    c.max_clusters = nclusters;
    c.init = true;
  }
  *out = &c;
  return MLA_OK;
}

int default_parts(int sms, int max_clusters) { return max_clusters > 0 ? max_clusters : sms / 2; }

// ------------------------------------------------------------------------------------------
// GEMM configuration
// ------------------------------------------------------------------------------------------
int round16(int x) { return (x + 15) / 16 * 16; }

// One weight product of a layer: rows per group, 128-row tiles per group, K, groups, and the
// activation columns (n_pad on the MMA's N side; n_lo > 0 when the columns are n_pad / n_lo
// planes of n_lo columns each, summed by the epilogue: the bf16 high and low halves of an fp32
// input, or three E4M3 pieces); elem = bytes per element (2 bf16, 1 E4M3).  A K block is one
// 128-byte row piece.
struct GemmShape {
  int m_total, m_tiles, k, groups, n_pad, n_lo;
  int elem = 2;
  int k_blocks() const { return (k * elem + 127) / 128; }
  int planes() const { return n_lo > 0 ? n_pad / n_lo : 1; }
};

// the five products of a layer on the bf16 path
GemmShape shape_append(const mla_dims* d) {
  return {kRowN, 5, d->d_model, 1, round16(d->batch), 0};
}
// cache append and W_Q in one product: 5 append tiles (W_DKV, W_KR) then W_Q's
GemmShape shape_append_wq(const mla_dims* d) {
  const int m = d->n_heads * (kDn + kDr);
  return {sk::EpiAppendWq::kSplitRow + m, 5 + m / 128, d->d_model, 1, round16(d->batch), 0};
}
GemmShape shape_wq(const mla_dims* d) {
  const int m = d->n_heads * (kDn + kDr);
  return {m, m / 128, d->d_model, 1, round16(d->batch), 0};
}
GemmShape shape_wuk(const mla_dims* d) {
  return {kDc, kDc / 128, kDn, d->n_heads, 2 * round16(d->batch), round16(d->batch)};
}
GemmShape shape_wuv(const mla_dims* d) {
  return {kDv, 1, kDc, d->n_heads, 2 * round16(d->batch), round16(d->batch)};
}
GemmShape shape_wo(const mla_dims* d) {
  return {d->d_model, (d->d_model + 127) / 128, d->n_heads * kDv, 1, 2 * round16(d->batch),
          round16(d->batch)};
}
// the folded execution mode: cache append + the folded query (576 rows per head) in one
// product, and the folded output product over all heads' latent columns (K = H * 512)
GemmShape shape_append_wq_fold(const mla_dims* d) {
  const int m = d->n_heads * kRowN;
  return {sk::EpiAppendWqFold::kSplitRow + m, 5 + m / 128, d->d_model, 1, round16(d->batch), 0};
}
GemmShape shape_wo_fold(const mla_dims* d) {
  return {d->d_model, (d->d_model + 127) / 128, d->n_heads * kDc, 1, 2 * round16(d->batch),
          round16(d->batch)};
}
// cache append and W_Q in E4M3 against h as two E4M3 planes
GemmShape shape_append_wq_e4m3(const mla_dims* d) {
  const int m = d->n_heads * (kDn + kDr);
  return {sk::EpiAppendWq::kSplitRow + m, 5 + m / 128, d->d_model, 1, 2 * round16(d->batch),
          round16(d->batch), 1};
}
// W_O in E4M3 against o_heads as E4M3 planes (tcgen05 kind::f8f6f4): three planes (~12
// significant bits) while they fit the MMA cheaply, two (~8 bits) above 32 rows
int oh_planes(const mla_dims* d) { return round16(d->batch) <= 32 ? 3 : 2; }
GemmShape shape_wo_e4m3(const mla_dims* d) {
  return {d->d_model, (d->d_model + 127) / 128, d->n_heads * kDv, 1,
          oh_planes(d) * round16(d->batch), round16(d->batch), 1};
}

// Stream-K launch plan: K blocks per stage, CTAs, partial slots per tile, ring depth, smem.
struct SkPlan {
  int kbs = 1, units = 1, ctas = 1, max_slots = 1, stages = 2, tiles = 0;
  long long iters = 0;
  size_t smem = 0, partial_bytes = 0;
};

SkPlan sk_plan(const GemmShape& s, size_t epi_bytes, int sms) {
  SkPlan q;
  q.tiles = s.m_tiles * s.groups;
  const size_t fixed = 1024 + (epi_bytes + 15) / 16 * 16 + 256;  // alignment, tables, barriers
  const size_t budget = kSmemPerBlockMax - fixed;
  // Large TMA boxes (several K blocks of 128 weight rows) stream HBM more efficiently: the
  // largest box (up to 4 K blocks) that still leaves a double-buffered ring.
  q.kbs = 1;
  for (int kbs = 2; kbs <= 4 && kbs <= s.k_blocks(); kbs *= 2)
    if (budget / sk::stage_bytes(s.n_pad, kbs) >= 2) q.kbs = kbs;
  q.units = (s.k_blocks() + q.kbs - 1) / q.kbs;
  q.iters = static_cast<long long>(q.tiles) * q.units;
  long long P = std::min<long long>(sms, (q.iters + kSkMinUnits - 1) / kSkMinUnits);
  P = std::min<long long>(P, static_cast<long long>(q.tiles) * kSkMaxContrib);
  P = std::max<long long>(1, std::min(P, q.iters));
  q.ctas = static_cast<int>(P);
  for (long long t = 0; t < q.tiles; ++t) {
    const int cf = sk::cta_of(t * q.units, q.iters, P);
    const int cl = sk::cta_of((t + 1) * q.units - 1, q.iters, P);
    q.max_slots = std::max(q.max_slots, cl - cf + 1);
  }
  const size_t sb = sk::stage_bytes(s.n_pad, q.kbs);
  q.stages = static_cast<int>(std::min<size_t>(kSkMaxStages, budget / sb));
  q.smem = fixed + static_cast<size_t>(q.stages) * sb;
  // a partial slot holds the output columns only (the column planes are summed before it)
  const int n_cols = s.n_lo > 0 ? s.n_lo : s.n_pad;
  q.partial_bytes = q.max_slots > 1 ? static_cast<size_t>(q.tiles) * q.max_slots * n_cols * 128 *
                                          sizeof(float)
                                    : 0;
  return q;
}

std::atomic<uint32_t> g_sk_epoch{0x5EED0000u};
uint32_t next_epoch() {
  uint32_t e = g_sk_epoch.fetch_add(1, std::memory_order_relaxed) + 1;
  if (e == 0) e = g_sk_epoch.fetch_add(1, std::memory_order_relaxed) + 1;
  return e;
}

// ------------------------------------------------------------------------------------------
// workspace layout
// ------------------------------------------------------------------------------------------
// [partial, counters, qn, o_split, oh_split, xmax) serve the projection products and are the
// same for every split count; [plan, part_o, part_lse) serve the decode call and grow with its
// parts.  A projection call therefore needs only `plan` bytes, the decode call all `total`.
struct Workspace {
  size_t partial, counters, qn, o_split, oh_split, xmax, plan, part_o, part_lse, total;
};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

Workspace layout(const mla_dims* d, int num_parts, int sms) {
  const size_t B = d->batch, H = d->n_heads, Bp = round16(d->batch);
  size_t part = 0, ctr = 0;
  if (d->dtype == MLA_BF16) {
    // the same (shape, epilogue table size) pairs the launches use
    const GemmShape shapes[8] = {shape_append(d), shape_wq(d), shape_wuk(d),
                                 shape_wuv(d), shape_wo(d), shape_append_wq(d),
                                 shape_append_wq_fold(d), shape_wo_fold(d)};
    const size_t epi[8] = {sk::EpiAppend::smem_bytes(d->batch), sk::EpiWq::smem_bytes(d->batch),
                           0, 0, 0, sk::EpiAppendWq::smem_bytes(d->batch),
                           sk::EpiAppendWqFold::smem_bytes(d->batch), 0};
    for (int i = 0; i < 8; ++i) {
      const SkPlan q = sk_plan(shapes[i], epi[i], sms);
      part = std::max(part, q.partial_bytes);
      ctr = std::max(ctr, static_cast<size_t>(q.tiles) * 8);
    }
    if (d->batch <= kFp8MaxBatch) {
      const SkPlan qs[2] = {sk_plan(shape_wo_e4m3(d), 0, sms),
                            sk_plan(shape_append_wq_e4m3(d), sk::EpiAppendWq::smem_bytes(d->batch),
                                    sms)};
      for (const SkPlan& q : qs) {
        part = std::max(part, q.partial_bytes);
        ctr = std::max(ctr, static_cast<size_t>(q.tiles) * 8);
      }
    }
  } else {
    part = std::max({static_cast<size_t>(kRowN) * B, H * (kDn + kDr) * B, H * kDc * B,
                     H * kDv * B, static_cast<size_t>(d->d_model) * B}) *
           sizeof(float);
  }
  Workspace w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  w.partial = take(part);
  w.counters = take(ctr);
  w.qn = take(std::max(2 * Bp * H * kDn * 2, B * H * kDn * 4));      // bf16 hi/lo, or fp32
  // bf16 hi/lo of o_lat; once the W_UV product has read them, the E4M3 W_O call puts o_heads'
  // three E4M3 planes [3][Bp][H*128] and their Bp scales here
  w.o_split = take(2 * Bp * H * kDc * 2);
  w.oh_split = take(std::max(2 * Bp * H * kDv * 2, B * H * kDv * 4)); // bf16 hi/lo, or fp32
  w.xmax = take(Bp * 4);  // E4M3 W_O call: max |o_heads[b]| per batch row (fp32 bits)
  w.plan = take(attn::PlanView::words(static_cast<int>(B), num_parts) * 4);
  w.part_o = take((B + num_parts) * H * kDc * 4);
  w.part_lse = take((B + num_parts) * H * 4);
  w.total = off;
  return w;
}

// Parts of the page list: num_splits, or about one cluster per co-resident cluster slot, shared
// by the `groups` clusters that each part runs on (2 for 128 heads with the query remainder).
int resolve_parts(int num_splits, const DevCtx* c, int groups = 1) {
  if (num_splits > 0) return num_splits;
  return std::max(1, default_parts(c ? c->sms : 148, c ? c->max_clusters : 74) / groups);
}

// ------------------------------------------------------------------------------------------
// TMA descriptors
// ------------------------------------------------------------------------------------------
int encode(CUtensorMap* m, CUtensorMapDataType dt, const void* base, int rank,
           const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
           CUtensorMapSwizzle sw) {
  cuuint64_t gdim[5];
  cuuint64_t gstr[4];
  cuuint32_t bdim[5], estr[5];
  for (int i = 0; i < rank; ++i) {
    gdim[i] = dims[i];
    bdim[i] = box[i];
    estr[i] = 1;
  }
  for (int i = 0; i < rank - 1; ++i) gstr[i] = strides_bytes[i];
  const CUresult r = g_encode(m, dt, rank, const_cast<void*>(base), gdim, gstr, bdim, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_ARG;
}

// 3-D bf16 map (k contiguous, then rows_a, then rows_b), box (64, box_a, box_b), 128B swizzle.
int map3(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1,
         uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2,
         CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B) {
  const uint64_t dims[3] = {d0, d1, d2};
  const uint64_t str[2] = {s1, s2};
  const uint32_t box[3] = {b0, b1, b2};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, 3, dims, str, box, sw);
}

// 2-D bf16 map (k contiguous, rows), box (b0, b1).
int map2(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t s1, uint32_t b0,
         uint32_t b1, CUtensorMapSwizzle sw) {
  const uint64_t dims[2] = {d0, d1};
  const uint64_t str[1] = {s1};
  const uint32_t box[2] = {b0, b1};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, 2, dims, str, box, sw);
}

// Weights [groups][rows][K] (K contiguous) as a 4-D view (64 k, rows, groups, K / 64) so that
// one box (64, 128, 1, kbs) brings kbs consecutive 128-byte pieces of 128 weight rows.
int map_weights(CUtensorMap* m, const void* base, uint64_t rows, uint64_t groups, uint64_t K,
                int kbs) {
  const uint64_t dims[4] = {64, rows, groups, K / 64};
  const uint64_t str[3] = {K * 2, rows * K * 2, 128};
  const uint32_t box[4] = {64, 128, 1, static_cast<uint32_t>(kbs)};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, 4, dims, str, box,
                CU_TENSOR_MAP_SWIZZLE_128B);
}

// E4M3 weights in 128 x 128 tiles (the layout mla_quantize_weights_fp8 writes) as the view
// (128 k, 128 rows, K / 128, row tiles), box (128, 128, kbs, 1): kbs tiles in one contiguous run,
// landing as the same 128-byte swizzled row pieces as map_weights.
int map_weights_e4m3(CUtensorMap* m, const void* base, uint64_t rows, uint64_t K, int kbs) {
  const uint64_t dims[4] = {128, 128, K / 128, (rows + 127) / 128};
  const uint64_t str[3] = {128, 128 * 128, K * 128};
  const uint32_t box[4] = {128, 128, static_cast<uint32_t>(kbs), 1};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, 4, dims, str, box,
                CU_TENSOR_MAP_SWIZZLE_128B);
}

// E4M3 activation planes [n_rows][K] bytes as the view (128 k, 1, n_rows, K / 128), box
// (128, 1, n_pad, kbs).
int map_acts_e4m3(CUtensorMap* m, const void* base, uint64_t n_rows, uint64_t K, int n_pad,
                  int kbs) {
  const uint64_t dims[4] = {128, 1, n_rows, K / 128};
  const uint64_t str[3] = {K, K, 128};
  const uint32_t box[4] = {128, 1, static_cast<uint32_t>(n_pad), static_cast<uint32_t>(kbs)};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, 4, dims, str, box,
                CU_TENSOR_MAP_SWIZZLE_128B);
}

// Activations X: element (k, g, n) at n * n_stride + g * g_stride + 2 k (bytes), as the view
// (64 k, groups, n, K / 64) with box (64, 1, n_pad, kbs); rows n >= n_rows read as zero.
int map_acts(CUtensorMap* m, const void* base, uint64_t groups, uint64_t n_rows, uint64_t K,
             uint64_t g_stride, uint64_t n_stride, int n_pad, int kbs) {
  const uint64_t dims[4] = {64, groups, n_rows, K / 64};
  const uint64_t str[3] = {g_stride, n_stride, 128};
  const uint32_t box[4] = {64, 1, static_cast<uint32_t>(n_pad), static_cast<uint32_t>(kbs)};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, 4, dims, str, box,
                CU_TENSOR_MAP_SWIZZLE_128B);
}

// ------------------------------------------------------------------------------------------
// launches
// ------------------------------------------------------------------------------------------
int last_launch(int kernels = 1) {
  g_launches.fetch_add(static_cast<unsigned long long>(kernels), std::memory_order_relaxed);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MLA_OK : cuda_fail(e, "kernel launch");
}

// The kernels of the bf16 decode path are launched with programmatic stream serialisation:
// each may be scheduled while its predecessor on the stream drains, and waits for it
// (griddep_wait) before it touches that kernel's results.  MLA_NO_PDL=1 in the environment
// launches them as ordinary stream-ordered kernels.  A failure is reported by last_launch().
bool pdl_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("MLA_NO_PDL");
    return !(e && e[0] == '1');
  }();
  return on;
}

template <typename... KArgs, typename... Args>
void launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr{};
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  (void)cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// A profiling event on `st`.  Under stream capture it becomes an external event node, which
// records a timestamp every time the graph runs (a plain record inside a capture does not).
cudaError_t record_profile_event(cudaEvent_t ev, cudaStream_t st) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) return cudaErrorUnknown;
  return cudaEventRecordWithFlags(
      ev, st, cs == cudaStreamCaptureStatusActive ? cudaEventRecordExternal : cudaEventRecordDefault);
}

// Scales of an E4M3 product: per weight row of the weights behind maps A0, A1, A2 (with their row
// counts), per activation row.
struct E4m3Scales {
  const float* a[3] = {nullptr, nullptr, nullptr};
  int rows[3] = {0, 0, 0};
  const float* x = nullptr;
};

// One weight product on the tensor cores, its epilogue fused (stream-K, see gemm_streamk.cuh).
template <class Epi, bool kFp8 = false>
int run_streamk(const DevCtx* c, const GemmShape& s, const SkPlan& q, int n_out,
                const int32_t* positions, float theta, const CUtensorMap& a0,
                const CUtensorMap& a1, int a1_tile_start, int a_mn_major,
                const CUtensorMap& xmap, char* ws, const Workspace& w, const Epi& epi,
                cudaStream_t st, const CUtensorMap* a2 = nullptr, int a2_tile_start = 1 << 30,
                const E4m3Scales& scales = E4m3Scales{}, int a_tiled = 0) {
  sk::Params p{};
  p.m_total = s.m_total;
  p.m_tiles = s.m_tiles;
  p.groups = s.groups;
  p.a1_tile_start = a1_tile_start;
  p.a2_tile_start = a2_tile_start;
  p.k_blocks = s.k_blocks();
  p.kbs = q.kbs;
  p.units = q.units;
  p.n_pad = s.n_pad;
  p.n_lo = s.n_lo;
  p.n_planes = s.planes();
  p.n_out = n_out;
  p.a_mn_major = a_mn_major;
  p.a_tiled = a_tiled;
  p.stages = q.stages;
  p.max_slots = q.max_slots;
  p.iters = q.iters;
  p.epoch = next_epoch();
  p.partial = reinterpret_cast<float*>(ws + w.partial);
  p.counters = reinterpret_cast<unsigned long long*>(ws + w.counters);
  p.positions = positions;
  p.rope_theta = theta;
  p.status = c->status;
  p.wait_ns = wait_limit_ns();
  for (int m = 0; m < 3; ++m) {
    p.a_scale[m] = scales.a[m];
    p.a_rows[m] = scales.rows[m];
  }
  p.x_scale = scales.x;
  launch_pdl(sk::streamk_gemm_kernel<Epi, kFp8>, dim3(q.ctas), dim3(sk::kThreads), q.smem, st, a0,
             a1, a2 ? *a2 : a1, xmap, p, epi);
  return last_launch();
}

// q_lat_h = W_UK_h^T [q_nope_hi | q_nope_lo] into q_cat[..., :512] (+ q_lo), bf16 path; the
// q_nope hi/lo planes are in the workspace (written by the W_Q product).  A is MN-major: the
// rows of W_UK are the K side.
int run_wuk(const DevCtx* c, const mla_dims* dims, const void* w_uk, char* ws,
            const Workspace& w, __nv_bfloat16* qc, __nv_bfloat16* ql, cudaStream_t st) {
  const int B = dims->batch, H = dims->n_heads;
  const GemmShape s2 = shape_wuk(dims);
  const int Bp = s2.n_lo;
  const SkPlan q2 = sk_plan(s2, 0, c->sms);
  CUtensorMap a2, b2;
  int rc;
  if ((rc = map3(&a2, w_uk, kDc, kDn, H, kDc * 2ull, kDc * 2ull * kDn, 64, 64 * q2.kbs, 1)))
    return rc;
  if ((rc = map_acts(&b2, ws + w.qn, H, 2 * Bp, kDn, kDn * 2ull, kDn * 2ull * H, s2.n_pad,
                     q2.kbs)))
    return rc;
  sk::EpiWuk e2{H, qc, ql};
  return run_streamk(c, s2, q2, B, nullptr, 0.f, a2, a2, 1 << 30, 1, b2, ws, w, e2, st);
}


// Host checks shared by both decode entry points (everything but the workspace).
int check_decode_args(const mla_dims* dims, const void* q_cat, const void* q_lo,
                      const void* cache_pool, int32_t num_pages, const int32_t* page_table,
                      int32_t max_pages, const int32_t* seq_lens, float softmax_scale,
                      int32_t num_splits, const float* o_lat, const float* lse) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (!q_cat || !cache_pool || !page_table || !seq_lens || !o_lat) return MLA_ERR_NULL_ARG;
  if (num_pages < 1 || max_pages < 1 || num_splits < 0 || num_splits > kMaxParts)
    return MLA_ERR_ARG;
  if (q_lo && dims->dtype != MLA_BF16) return MLA_ERR_ARG;
  if (!(softmax_scale >= 0.f) || !std::isfinite(softmax_scale)) return MLA_ERR_ARG;
  if (!aligned(q_cat, 16) || !aligned(cache_pool, 16) || !aligned(o_lat, 16) ||
      (q_lo && !aligned(q_lo, 16)) || !aligned(page_table, 4) || !aligned(seq_lens, 4) ||
      (lse && !aligned(lse, 4)))
    return MLA_ERR_ALIGN;
  // page ids and lengths are int32 token counts on the device
  if (static_cast<int64_t>(num_pages) * kPageN > INT32_MAX ||
      static_cast<int64_t>(max_pages) * kPageN > INT32_MAX)
    return MLA_ERR_ARG;
  return MLA_OK;
}

// Clusters per part: 1, or one per 64 heads when the query remainder q_lo is given.
int decode_groups(const mla_dims* dims, const void* q_lo) {
  return (q_lo && dims->dtype == MLA_BF16) ? (dims->n_heads + 63) / 64 : 1;
}

// plan -> split-KV attention -> combine, on `st`, with the scratch the caller placed.
int enqueue_decode(const DevCtx* c, const mla_dims* dims, const void* q_cat, const void* q_lo,
                   const void* cache_pool, int32_t num_pages, const int32_t* page_table,
                   int32_t max_pages, const int32_t* seq_lens, float softmax_scale, int parts,
                   int32_t* plan, float* part_o, float* part_lse, float* o_lat, float* lse,
                   cudaStream_t st) {
  int rc;
  const int B = dims->batch, H = dims->n_heads;
  const int groups = decode_groups(dims, q_lo);
  const float scale =
      softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(kDn + kDr));
  launch_pdl(attn::plan_kernel, dim3(1), dim3(attn::kPlanThreads), 0, st, seq_lens, B, max_pages,
             parts, kMinPagesPerPart, plan, c->status);
  if ((rc = last_launch())) return rc;
  if (dims->dtype == MLA_BF16) {
    CUtensorMap tc_lat, tc_rope, tq_rope, tql_rope;
    const uint64_t rows = static_cast<uint64_t>(num_pages) * kPageN;
    // query RoPE halves: one 128-head box, or 8-head boxes from q_cat and q_lo
    const uint32_t qbox = q_lo ? 8 : 128;
    if ((rc = map3(&tq_rope, q_cat, kRowN, H, B, kRowN * 2ull, kRowN * 2ull * H, 32, qbox, 1,
                   CU_TENSOR_MAP_SWIZZLE_64B)))
      return rc;
    if (q_lo) {
      if ((rc = map3(&tql_rope, q_lo, kRowN, H, B, kRowN * 2ull, kRowN * 2ull * H, 32, qbox, 1,
                     CU_TENSOR_MAP_SWIZZLE_64B)))
        return rc;
    } else {
      tql_rope = tq_rope;
    }
    if ((rc = map2(&tc_lat, cache_pool, kRowN, rows, kRowN * 2ull, 64, 64,
                   CU_TENSOR_MAP_SWIZZLE_128B)))
      return rc;
    if ((rc = map2(&tc_rope, cache_pool, kRowN, rows, kRowN * 2ull, 32, 64,
                   CU_TENSOR_MAP_SWIZZLE_64B)))
      return rc;
    attn::Params p{};
    p.batch = B;
    p.n_heads = H;
    p.max_pages = max_pages;
    p.num_pages = num_pages;
    p.num_parts = parts;
    p.groups = groups;
    p.q_cat = static_cast<const __nv_bfloat16*>(q_cat);
    p.q_lo = static_cast<const __nv_bfloat16*>(q_lo);
    p.pool = static_cast<const uint8_t*>(cache_pool);
    p.page_table = page_table;
    p.seq_lens = seq_lens;
    p.plan = plan;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.o_lat = o_lat;
    p.lse = lse;
    p.part_o = part_o;
    p.part_lse = part_lse;
    p.status = c->status;
    p.wait_ns = wait_limit_ns();
    p.stall_test = stall_test_requested();
    const bool prof = g_prof_next < g_prof_count;
    if (prof && record_profile_event(g_prof_begin[g_prof_next], st) != cudaSuccess)
      return MLA_ERR_CUDA;
    launch_pdl(attn::split_kernel, dim3(2 * parts * groups), dim3(attn::kThreads),
               attn::kSmemBytes, st, tc_lat, tc_rope, tq_rope, tql_rope, p);
    if (prof) {
      if ((rc = last_launch())) return rc;
      if (record_profile_event(g_prof_end[g_prof_next++], st) != cudaSuccess) return MLA_ERR_CUDA;
      g_launches.fetch_sub(1, std::memory_order_relaxed);  // counted again below
    }
  } else {
    attn::f32_split_kernel<<<dim3(parts, H), 128, 0, st>>>(
        static_cast<const float*>(q_cat), static_cast<const float*>(cache_pool), page_table,
        max_pages, num_pages, seq_lens, plan, B, parts, H, scale, o_lat, lse, part_o, part_lse,
        c->status);
  }
  if ((rc = last_launch())) return rc;
  launch_pdl(attn::combine_kernel,
             dim3(static_cast<unsigned>((static_cast<size_t>(B) * H + attn::kCombineWarps - 1) /
                                        attn::kCombineWarps)),
             dim3(32 * attn::kCombineWarps), 0, st, plan, B, parts, H, part_o, part_lse, o_lat,
             lse);
  return last_launch();
}
}  // namespace
}  // namespace mla

using namespace mla;

// =============================================================================================
// C ABI
// =============================================================================================
extern "C" {

size_t mla_workspace_size(const mla_dims* dims, int32_t num_splits) {
  if (check_dims(dims) != MLA_OK || num_splits < 0 || num_splits > kMaxParts) return 0;
  DevCtx* c = nullptr;
  const bool have = device_ctx(&c) == MLA_OK;
  const int sms = have ? c->sms : 148;
  const int parts = num_splits > 0 ? num_splits : (have ? resolve_parts(0, c) : 74);
  return layout(dims, parts, sms).total;
}

int64_t mla_cache_row_bytes(const mla_dims* dims) {
  if (check_dims(dims) != MLA_OK) return 0;
  return static_cast<int64_t>(dims->d_c + dims->d_rope) * static_cast<int64_t>(elem_size(dims));
}

int mla_cache_append(const mla_dims* dims, const void* h, const void* w_dkv, const void* w_kr,
                     const int32_t* positions, const int32_t* page_table, int32_t max_pages,
                     void* cache_pool, int32_t num_pages, void* workspace,
                     size_t workspace_bytes, mla_stream_t stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (!h || !positions || !page_table || !cache_pool) return MLA_ERR_NULL_ARG;
  const bool scatter_only = (w_dkv == nullptr && w_kr == nullptr);
  if (!scatter_only && (!w_dkv || !w_kr)) return MLA_ERR_NULL_ARG;
  if (max_pages < 1 || num_pages < 1) return MLA_ERR_ARG;
  if (!aligned(h, 16) || !aligned(cache_pool, 16) || (w_dkv && !aligned(w_dkv, 16)) ||
      (w_kr && !aligned(w_kr, 16)) || !aligned(positions, 4) || !aligned(page_table, 4))
    return MLA_ERR_ALIGN;
  if (!scatter_only && (!workspace)) return MLA_ERR_WORKSPACE;
  if (workspace && !aligned(workspace, 256)) return MLA_ERR_ALIGN;
  DevCtx* c = nullptr;
  if ((rc = device_ctx(&c))) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int B = dims->batch, D = dims->d_model;
  const dim3 eg((kRowN / 2 + 95) / 96, B);
  if (scatter_only) {
    if (dims->dtype == MLA_BF16)
      append_epilogue_kernel<__nv_bfloat16><<<eg, 96, 0, st>>>(
          nullptr, 0, 0, static_cast<const __nv_bfloat16*>(h), positions, page_table, max_pages,
          static_cast<__nv_bfloat16*>(cache_pool), num_pages, dims->rope_theta, c->status);
    else
      append_epilogue_kernel<float><<<eg, 96, 0, st>>>(
          nullptr, 0, 0, static_cast<const float*>(h), positions, page_table, max_pages,
          static_cast<float*>(cache_pool), num_pages, dims->rope_theta, c->status);
    return last_launch();
  }
  const Workspace w = layout(dims, resolve_parts(0, c), c->sms);
  if (workspace_bytes < w.plan) return MLA_ERR_WORKSPACE;  // projection scratch only
  char* ws = static_cast<char*>(workspace);
  float* part = reinterpret_cast<float*>(ws + w.partial);
  if (dims->dtype == MLA_BF16) {
    const GemmShape s = shape_append(dims);
    const SkPlan q = sk_plan(s, sk::EpiAppend::smem_bytes(B), c->sms);
    CUtensorMap a0, a1, bm;
    if ((rc = map_weights(&a0, w_dkv, kDc, 1, D, q.kbs))) return rc;
    if ((rc = map_weights(&a1, w_kr, kDr, 1, D, q.kbs))) return rc;
    if ((rc = map_acts(&bm, h, 1, B, D, D * 2ull, D * 2ull, s.n_pad, q.kbs))) return rc;
    sk::EpiAppend e{positions, page_table, max_pages, static_cast<__nv_bfloat16*>(cache_pool),
                    num_pages, c->status, dims->rope_theta};
    return run_streamk(c, s, q, B, positions, dims->rope_theta, a0, a1, kDc / 128, 0, bm, ws, w,
                       e, st);
  } else {
    // fp32: rows 0..511 from W_DKV, 512..575 from W_KR, written as one [576][B] partial
    f32_gemm_k_kernel<<<dim3(kDc / 8, 1), 256, 0, st>>>(static_cast<const float*>(w_dkv), 0, D,
                                                       static_cast<const float*>(h), D, 0, kDc, D,
                                                       B, part);
    if ((rc = last_launch())) return rc;
    f32_gemm_k_kernel<<<dim3(kDr / 8, 1), 256, 0, st>>>(static_cast<const float*>(w_kr), 0, D,
                                                       static_cast<const float*>(h), D, 0, kDr, D,
                                                       B, part + static_cast<size_t>(kDc) * B);
    if ((rc = last_launch())) return rc;
    append_epilogue_kernel<float><<<eg, 96, 0, st>>>(
        part, 1, B, nullptr, positions, page_table, max_pages, static_cast<float*>(cache_pool),
        num_pages, dims->rope_theta, c->status);
  }
  return last_launch();
}

int mla_absorb_q(const mla_dims* dims, const void* h, const void* w_q, const void* w_uk,
                 const int32_t* positions, void* q_cat, void* q_lo, void* workspace,
                 size_t workspace_bytes, mla_stream_t stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (!h || !w_q || !w_uk || !positions || !q_cat) return MLA_ERR_NULL_ARG;
  if (!workspace) return MLA_ERR_WORKSPACE;
  if (q_lo && dims->dtype != MLA_BF16) return MLA_ERR_ARG;
  if (!aligned(h, 16) || !aligned(w_q, 16) || !aligned(w_uk, 16) || !aligned(q_cat, 16) ||
      (q_lo && !aligned(q_lo, 16)) || !aligned(positions, 4))
    return MLA_ERR_ALIGN;
  if (!aligned(workspace, 256)) return MLA_ERR_ALIGN;
  DevCtx* c = nullptr;
  if ((rc = device_ctx(&c))) return rc;
  const Workspace w = layout(dims, resolve_parts(0, c), c->sms);
  if (workspace_bytes < w.plan) return MLA_ERR_WORKSPACE;  // projection scratch only
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int B = dims->batch, D = dims->d_model, H = dims->n_heads;
  char* ws = static_cast<char*>(workspace);
  float* part = reinterpret_cast<float*>(ws + w.partial);
  void* qn = ws + w.qn;
  const float theta = dims->rope_theta;
  if (dims->dtype == MLA_BF16) {
    __nv_bfloat16* qc = static_cast<__nv_bfloat16*>(q_cat);
    __nv_bfloat16* ql = static_cast<__nv_bfloat16*>(q_lo);
    // q = W_Q h -> q_nope hi/lo planes [2][Bp][H][128] and RoPE(q_rope) into q_cat
    const GemmShape s1 = shape_wq(dims);
    const int Bp = s1.n_pad;
    const SkPlan q1 = sk_plan(s1, sk::EpiWq::smem_bytes(B), c->sms);
    CUtensorMap a, bm;
    if ((rc = map_weights(&a, w_q, s1.m_total, 1, D, q1.kbs))) return rc;
    if ((rc = map_acts(&bm, h, 1, B, D, D * 2ull, D * 2ull, s1.n_pad, q1.kbs))) return rc;
    __nv_bfloat16* qnb = static_cast<__nv_bfloat16*>(qn);
    sk::EpiWq e1{H, Bp, qc, ql, qnb, positions, theta};
    if ((rc = run_streamk(c, s1, q1, B, positions, theta, a, a, 1 << 30, 0, bm, ws, w, e1, st)))
      return rc;
    return run_wuk(c, dims, w_uk, ws, w, qc, ql, st);
  } else {
    float* qc = static_cast<float*>(q_cat);
    const int M = H * (kDn + kDr);
    f32_gemm_k_kernel<<<dim3((M + 7) / 8, 1), 256, 0, st>>>(static_cast<const float*>(w_q), 0, D,
                                                           static_cast<const float*>(h), D, 0, M,
                                                           D, B, part);
    if ((rc = last_launch())) return rc;
    wq_epilogue_kernel<float><<<dim3(H, B), 96, 0, st>>>(part, 1, B, B, H, positions, theta, qc,
                                                         nullptr, qn);
    if ((rc = last_launch())) return rc;
    // q_lat_h[m] = sum_k W_UK[h*128 + k][m] q_nope[b][h][k]
    f32_gemm_mn_kernel<<<dim3(kDc / 128, H), 128, 0, st>>>(
        static_cast<const float*>(w_uk), static_cast<size_t>(kDn) * kDc, kDc,
        static_cast<const float*>(qn), static_cast<size_t>(H) * kDn, kDn, kDc, kDn, B, part);
    if ((rc = last_launch())) return rc;
    wuk_epilogue_kernel<float, false><<<dim3(H, B), 128, 0, st>>>(part, B, B, H, qc, nullptr);
  }
  return last_launch();
}

int mla_append_absorb(const mla_dims* dims, const void* h, const void* w_dkv, const void* w_kr,
                      const void* w_q, const void* w_uk, const int32_t* positions,
                      const int32_t* page_table, int32_t max_pages, void* cache_pool,
                      int32_t num_pages, void* q_cat, void* q_lo, void* workspace,
                      size_t workspace_bytes, mla_stream_t stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (!h || !w_dkv || !w_kr || !w_q || !w_uk || !positions || !page_table || !cache_pool ||
      !q_cat)
    return MLA_ERR_NULL_ARG;
  if (!workspace) return MLA_ERR_WORKSPACE;
  if (max_pages < 1 || num_pages < 1) return MLA_ERR_ARG;
  if (q_lo && dims->dtype != MLA_BF16) return MLA_ERR_ARG;
  if (!aligned(h, 16) || !aligned(w_dkv, 16) || !aligned(w_kr, 16) || !aligned(w_q, 16) ||
      !aligned(w_uk, 16) || !aligned(cache_pool, 16) || !aligned(q_cat, 16) ||
      (q_lo && !aligned(q_lo, 16)) || !aligned(positions, 4) || !aligned(page_table, 4))
    return MLA_ERR_ALIGN;
  if (!aligned(workspace, 256)) return MLA_ERR_ALIGN;
  if (dims->dtype != MLA_BF16) {
    // fp32 path: the two calls in order
    if ((rc = mla_cache_append(dims, h, w_dkv, w_kr, positions, page_table, max_pages,
                               cache_pool, num_pages, workspace, workspace_bytes, stream)))
      return rc;
    return mla_absorb_q(dims, h, w_q, w_uk, positions, q_cat, q_lo, workspace, workspace_bytes,
                        stream);
  }
  DevCtx* c = nullptr;
  if ((rc = device_ctx(&c))) return rc;
  const Workspace w = layout(dims, resolve_parts(0, c), c->sms);
  if (workspace_bytes < w.plan) return MLA_ERR_WORKSPACE;  // projection scratch only
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int B = dims->batch, D = dims->d_model, H = dims->n_heads;
  char* ws = static_cast<char*>(workspace);
  __nv_bfloat16* qc = static_cast<__nv_bfloat16*>(q_cat);
  __nv_bfloat16* ql = static_cast<__nv_bfloat16*>(q_lo);
  // [W_DKV; W_KR; W_Q] h in one stream-K product: cache rows + q_nope planes + RoPE(q_rope)
  const GemmShape s = shape_append_wq(dims);
  const SkPlan q = sk_plan(s, sk::EpiAppendWq::smem_bytes(B), c->sms);
  CUtensorMap a0, a1, a2, bm;
  if ((rc = map_weights(&a0, w_dkv, kDc, 1, D, q.kbs))) return rc;
  if ((rc = map_weights(&a1, w_kr, kDr, 1, D, q.kbs))) return rc;
  if ((rc = map_weights(&a2, w_q, static_cast<uint64_t>(H) * (kDn + kDr), 1, D, q.kbs)))
    return rc;
  if ((rc = map_acts(&bm, h, 1, B, D, D * 2ull, D * 2ull, s.n_pad, q.kbs))) return rc;
  sk::EpiAppendWq e{
      sk::EpiAppend{positions, page_table, max_pages, static_cast<__nv_bfloat16*>(cache_pool),
                    num_pages, c->status, dims->rope_theta},
      sk::EpiWq{H, s.n_pad, qc, ql, reinterpret_cast<__nv_bfloat16*>(ws + w.qn), positions,
                dims->rope_theta}};
  if ((rc = run_streamk(c, s, q, B, positions, dims->rope_theta, a0, a1, kDc / 128, 0, bm, ws, w,
                        e, st, &a2, sk::EpiAppendWq::kSplitRow / 128)))
    return rc;
  return run_wuk(c, dims, w_uk, ws, w, qc, ql, st);
}

int mla_decode_attn(const mla_dims* dims, const void* q_cat, const void* q_lo,
                    const void* cache_pool, int32_t num_pages, const int32_t* page_table,
                    int32_t max_pages, const int32_t* seq_lens, float softmax_scale,
                    int32_t num_splits, void* workspace, size_t workspace_bytes, float* o_lat,
                    float* lse, mla_stream_t stream) {
  int rc = check_decode_args(dims, q_cat, q_lo, cache_pool, num_pages, page_table, max_pages,
                             seq_lens, softmax_scale, num_splits, o_lat, lse);
  if (rc) return rc;
  if (!workspace) return MLA_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return MLA_ERR_ALIGN;
  DevCtx* c = nullptr;
  if ((rc = device_ctx(&c))) return rc;
  const int parts = resolve_parts(num_splits, c, decode_groups(dims, q_lo));
  const Workspace w = layout(dims, parts, c->sms);
  if (workspace_bytes < w.total) return MLA_ERR_WORKSPACE;
  char* ws = static_cast<char*>(workspace);
  return enqueue_decode(c, dims, q_cat, q_lo, cache_pool, num_pages, page_table, max_pages,
                        seq_lens, softmax_scale, parts, reinterpret_cast<int32_t*>(ws + w.plan),
                        reinterpret_cast<float*>(ws + w.part_o),
                        reinterpret_cast<float*>(ws + w.part_lse), o_lat, lse,
                        reinterpret_cast<cudaStream_t>(stream));
}

int mla_out_proj(const mla_dims* dims, const float* o_lat, const void* w_uv, const void* w_o,
                 void* o_heads, void* out, void* workspace, size_t workspace_bytes,
                 mla_stream_t stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (!o_lat || !w_uv) return MLA_ERR_NULL_ARG;
  if ((w_o == nullptr) != (out == nullptr)) return MLA_ERR_NULL_ARG;
  if (!o_heads && !out) return MLA_ERR_NULL_ARG;
  if (!workspace) return MLA_ERR_WORKSPACE;
  if (!aligned(o_lat, 16) || !aligned(w_uv, 16) || (w_o && !aligned(w_o, 16)) ||
      (o_heads && !aligned(o_heads, 16)) || (out && !aligned(out, 16)))
    return MLA_ERR_ALIGN;
  if (!aligned(workspace, 256)) return MLA_ERR_ALIGN;
  DevCtx* c = nullptr;
  if ((rc = device_ctx(&c))) return rc;
  const Workspace w = layout(dims, resolve_parts(0, c), c->sms);
  if (workspace_bytes < w.plan) return MLA_ERR_WORKSPACE;  // projection scratch only
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int B = dims->batch, D = dims->d_model, H = dims->n_heads;
  char* ws = static_cast<char*>(workspace);
  float* part = reinterpret_cast<float*>(ws + w.partial);
  void* oh_split = out ? static_cast<void*>(ws + w.oh_split) : nullptr;
  if (dims->dtype == MLA_BF16) {
    __nv_bfloat16* os = reinterpret_cast<__nv_bfloat16*>(ws + w.o_split);
    const GemmShape s1 = shape_wuv(dims);
    const int Bp = s1.n_lo;
    const size_t n = static_cast<size_t>(B) * H * kDc;
    launch_pdl(split_hi_lo_kernel,
               dim3(static_cast<unsigned>(std::min<size_t>((n / 8 + 255) / 256, 4096))), dim3(256),
               0, st, o_lat, n, static_cast<size_t>(Bp) * H * kDc, os,
               static_cast<unsigned int*>(nullptr), 0);
    if ((rc = last_launch())) return rc;
    // o_h = W_UV_h [o_lat_hi | o_lat_lo]
    const SkPlan q1 = sk_plan(s1, 0, c->sms);
    CUtensorMap a, bm;
    if ((rc = map_weights(&a, w_uv, kDv, H, kDc, q1.kbs))) return rc;
    if ((rc = map_acts(&bm, os, H, 2 * Bp, kDc, kDc * 2ull, kDc * 2ull * H, s1.n_pad, q1.kbs)))
      return rc;
    sk::EpiWuv e1{H, Bp, static_cast<__nv_bfloat16*>(o_heads),
                  static_cast<__nv_bfloat16*>(oh_split)};
    if ((rc = run_streamk(c, s1, q1, B, nullptr, 0.f, a, a, 1 << 30, 0, bm, ws, w, e1, st)))
      return rc;
    if (out) {
      const GemmShape s2 = shape_wo(dims);
      const uint64_t K = static_cast<uint64_t>(H) * kDv;
      const SkPlan q2 = sk_plan(s2, 0, c->sms);
      CUtensorMap a2, b2;
      if ((rc = map_weights(&a2, w_o, D, 1, K, q2.kbs))) return rc;
      if ((rc = map_acts(&b2, oh_split, 1, 2 * Bp, K, K * 2, K * 2, s2.n_pad, q2.kbs))) return rc;
      sk::EpiWo e2{D, static_cast<__nv_bfloat16*>(out)};
      if ((rc = run_streamk(c, s2, q2, B, nullptr, 0.f, a2, a2, 1 << 30, 0, b2, ws, w, e2, st)))
        return rc;
    }
  } else {
    f32_gemm_k_kernel<<<dim3(kDv / 8, H), 256, 0, st>>>(
        static_cast<const float*>(w_uv), static_cast<size_t>(kDv) * kDc, kDc, o_lat,
        static_cast<size_t>(H) * kDc, kDc, kDv, kDc, B, part);
    if ((rc = last_launch())) return rc;
    wuv_epilogue_kernel<float, false><<<dim3(H, B), kDv, 0, st>>>(
        part, 1, B, B, H, static_cast<float*>(o_heads), oh_split);
    if ((rc = last_launch())) return rc;
    if (out) {
      const int K = H * kDv;
      f32_gemm_k_kernel<<<dim3((D + 7) / 8, 1), 256, 0, st>>>(
          static_cast<const float*>(w_o), 0, K, static_cast<const float*>(oh_split), K, 0, D, K,
          B, part);
      if ((rc = last_launch())) return rc;
      wo_epilogue_kernel<float, false><<<dim3((D + 255) / 256, B), 256, 0, st>>>(
          part, 1, B, B, D, static_cast<float*>(out));
      if ((rc = last_launch())) return rc;
    }
  }
  return MLA_OK;
}

// ------------------------------------------------------------------------------------------
// folded execution mode
// ------------------------------------------------------------------------------------------
int mla_fold_weights(const mla_dims* dims, const void* w_q, const void* w_uk, const void* w_uv,
                     const void* w_o, void* w_qf, void* w_of, mla_stream_t stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (dims->dtype != MLA_BF16) return MLA_ERR_ARG;
  if (!w_qf && !w_of) return MLA_ERR_NULL_ARG;
  if (w_qf && (!w_q || !w_uk)) return MLA_ERR_NULL_ARG;
  if (w_of && (!w_uv || !w_o)) return MLA_ERR_NULL_ARG;
  if ((w_q && !aligned(w_q, 16)) || (w_uk && !aligned(w_uk, 16)) || (w_uv && !aligned(w_uv, 16)) ||
      (w_o && !aligned(w_o, 16)) || (w_qf && !aligned(w_qf, 16)) || (w_of && !aligned(w_of, 16)))
    return MLA_ERR_ALIGN;
  DevCtx* c = nullptr;
  if ((rc = device_ctx(&c))) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int D = dims->d_model, H = dims->n_heads;
  using fold::kTile;
  const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(w_q);
  const __nv_bfloat16* uk = static_cast<const __nv_bfloat16*>(w_uk);
  const __nv_bfloat16* uv = static_cast<const __nv_bfloat16*>(w_uv);
  const __nv_bfloat16* o = static_cast<const __nv_bfloat16*>(w_o);
  if (w_qf) {
    __nv_bfloat16* qf = static_cast<__nv_bfloat16*>(w_qf);
    // rows m < 512 of head h: sum_k W_UK[h*128 + k][m] W_Q[h*192 + k][:]
    fold::batched_gemm_kernel<<<dim3((D + kTile - 1) / kTile, kDc / kTile, H), fold::kThreads, 0,
                                st>>>(uk, static_cast<long long>(kDn) * kDc, 1, kDc, q,
                                      static_cast<long long>(kDn + kDr) * D, D, 1, qf,
                                      static_cast<long long>(kRowN) * D, D, 1, kDc, D, kDn);
    if ((rc = last_launch())) return rc;
    // rows 512..575 of head h: W_Q's RoPE rows as they are
    fold::copy_rows_kernel<<<1024, 256, 0, st>>>(q + static_cast<size_t>(kDn) * D,
                                                 static_cast<long long>(kDn + kDr) * D,
                                                 qf + static_cast<size_t>(kDc) * D,
                                                 static_cast<long long>(kRowN) * D, H, kDr, D);
    if ((rc = last_launch())) return rc;
  }
  if (w_of) {
    // column h*512 + m of row n: sum_k W_O[n][h*128 + k] W_UV[h*128 + k][m]
    fold::batched_gemm_kernel<<<dim3(kDc / kTile, (D + kTile - 1) / kTile, H), fold::kThreads, 0,
                                st>>>(o, kDv, static_cast<long long>(H) * kDv, 1, uv,
                                      static_cast<long long>(kDv) * kDc, kDc, 1,
                                      static_cast<__nv_bfloat16*>(w_of), kDc,
                                      static_cast<long long>(H) * kDc, 1, D, kDc, kDv);
    if ((rc = last_launch())) return rc;
  }
  return MLA_OK;
}

int mla_append_absorb_folded(const mla_dims* dims, const void* h, const void* w_dkv,
                             const void* w_kr, const void* w_qf, const int32_t* positions,
                             const int32_t* page_table, int32_t max_pages, void* cache_pool,
                             int32_t num_pages, void* q_cat, void* q_lo, void* workspace,
                             size_t workspace_bytes, mla_stream_t stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (dims->dtype != MLA_BF16) return MLA_ERR_ARG;
  if (!h || !w_dkv || !w_kr || !w_qf || !positions || !page_table || !cache_pool || !q_cat)
    return MLA_ERR_NULL_ARG;
  if (!workspace) return MLA_ERR_WORKSPACE;
  if (max_pages < 1 || num_pages < 1) return MLA_ERR_ARG;
  if (!aligned(h, 16) || !aligned(w_dkv, 16) || !aligned(w_kr, 16) || !aligned(w_qf, 16) ||
      !aligned(cache_pool, 16) || !aligned(q_cat, 16) || (q_lo && !aligned(q_lo, 16)) ||
      !aligned(positions, 4) || !aligned(page_table, 4))
    return MLA_ERR_ALIGN;
  if (!aligned(workspace, 256)) return MLA_ERR_ALIGN;
  DevCtx* c = nullptr;
  if ((rc = device_ctx(&c))) return rc;
  const Workspace w = layout(dims, resolve_parts(0, c), c->sms);
  if (workspace_bytes < w.plan) return MLA_ERR_WORKSPACE;  // projection scratch only
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int B = dims->batch, D = dims->d_model, H = dims->n_heads;
  char* ws = static_cast<char*>(workspace);
  // [W_DKV; W_KR; W_QF] h in one stream-K product: cache rows + q_cat rows
  const GemmShape s = shape_append_wq_fold(dims);
  const SkPlan q = sk_plan(s, sk::EpiAppendWqFold::smem_bytes(B), c->sms);
  CUtensorMap a0, a1, a2, bm;
  if ((rc = map_weights(&a0, w_dkv, kDc, 1, D, q.kbs))) return rc;
  if ((rc = map_weights(&a1, w_kr, kDr, 1, D, q.kbs))) return rc;
  if ((rc = map_weights(&a2, w_qf, static_cast<uint64_t>(H) * kRowN, 1, D, q.kbs))) return rc;
  if ((rc = map_acts(&bm, h, 1, B, D, D * 2ull, D * 2ull, s.n_pad, q.kbs))) return rc;
  sk::EpiAppendWqFold e{
      sk::EpiAppend{positions, page_table, max_pages, static_cast<__nv_bfloat16*>(cache_pool),
                    num_pages, c->status, dims->rope_theta},
      sk::EpiWqFold{H, static_cast<__nv_bfloat16*>(q_cat), static_cast<__nv_bfloat16*>(q_lo),
                    positions, dims->rope_theta}};
  return run_streamk(c, s, q, B, positions, dims->rope_theta, a0, a1, kDc / 128, 0, bm, ws, w, e,
                     st, &a2, sk::EpiAppendWqFold::kSplitRow / 128);
}

int mla_out_proj_folded(const mla_dims* dims, const float* o_lat, const void* w_of, void* out,
                        void* workspace, size_t workspace_bytes, mla_stream_t stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (dims->dtype != MLA_BF16) return MLA_ERR_ARG;
  if (!o_lat || !w_of || !out) return MLA_ERR_NULL_ARG;
  if (!workspace) return MLA_ERR_WORKSPACE;
  if (!aligned(o_lat, 16) || !aligned(w_of, 16) || !aligned(out, 16)) return MLA_ERR_ALIGN;
  if (!aligned(workspace, 256)) return MLA_ERR_ALIGN;
  DevCtx* c = nullptr;
  if ((rc = device_ctx(&c))) return rc;
  const Workspace w = layout(dims, resolve_parts(0, c), c->sms);
  if (workspace_bytes < w.plan) return MLA_ERR_WORKSPACE;  // projection scratch only
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int B = dims->batch, D = dims->d_model, H = dims->n_heads;
  char* ws = static_cast<char*>(workspace);
  __nv_bfloat16* os = reinterpret_cast<__nv_bfloat16*>(ws + w.o_split);
  const GemmShape s = shape_wo_fold(dims);
  const int Bp = s.n_lo;
  const size_t n = static_cast<size_t>(B) * H * kDc;
  // o_lat -> bf16 hi/lo planes [2][Bp][H * 512], the K layout of the folded product
  launch_pdl(split_hi_lo_kernel,
             dim3(static_cast<unsigned>(std::min<size_t>((n / 8 + 255) / 256, 4096))), dim3(256),
             0, st, o_lat, n, static_cast<size_t>(Bp) * H * kDc, os,
             static_cast<unsigned int*>(nullptr), 0);
  if ((rc = last_launch())) return rc;
  const uint64_t K = static_cast<uint64_t>(H) * kDc;
  const SkPlan q = sk_plan(s, 0, c->sms);
  CUtensorMap a, bm;
  if ((rc = map_weights(&a, w_of, D, 1, K, q.kbs))) return rc;
  if ((rc = map_acts(&bm, os, 1, 2 * Bp, K, K * 2, K * 2, s.n_pad, q.kbs))) return rc;
  sk::EpiWo e{D, static_cast<__nv_bfloat16*>(out)};
  return run_streamk(c, s, q, B, nullptr, 0.f, a, a, 1 << 30, 0, bm, ws, w, e, st);
}

// ------------------------------------------------------------------------------------------
// E4M3 weights
// ------------------------------------------------------------------------------------------
int mla_quantize_weights_fp8(const void* w, int64_t rows, int64_t cols, void* codes,
                             float* scale, mla_stream_t stream) {
  if (!w || !codes || !scale) return MLA_ERR_NULL_ARG;
  if (rows < 1 || rows > INT32_MAX || cols < 128 || cols % 128) return MLA_ERR_ARG;
  if (!aligned(w, 16) || !aligned(codes, 16) || !aligned(scale, 4)) return MLA_ERR_ALIGN;
  DevCtx* c = nullptr;
  int rc = device_ctx(&c);
  if (rc) return rc;
  fp8::quantize_rows_kernel<<<static_cast<unsigned>(rows), 256, 0,
                              reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(w), cols, static_cast<uint8_t*>(codes), scale);
  return last_launch();
}

int mla_append_absorb_fp8(const mla_dims* dims, const void* h, const void* w_dkv_codes,
                          const float* w_dkv_scale, const void* w_kr_codes,
                          const float* w_kr_scale, const void* w_q_codes, const float* w_q_scale,
                          const void* w_uk, const int32_t* positions, const int32_t* page_table,
                          int32_t max_pages, void* cache_pool, int32_t num_pages, void* q_cat,
                          void* q_lo, void* workspace, size_t workspace_bytes,
                          mla_stream_t stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (dims->dtype != MLA_BF16) return MLA_ERR_ARG;
  if (dims->batch > kFp8MaxBatch || dims->d_model % 128) return MLA_ERR_DIMS;
  if (!h || !w_dkv_codes || !w_dkv_scale || !w_kr_codes || !w_kr_scale || !w_q_codes ||
      !w_q_scale || !w_uk || !positions || !page_table || !cache_pool || !q_cat)
    return MLA_ERR_NULL_ARG;
  if (!workspace) return MLA_ERR_WORKSPACE;
  if (max_pages < 1 || num_pages < 1) return MLA_ERR_ARG;
  if (!aligned(h, 16) || !aligned(w_dkv_codes, 16) || !aligned(w_kr_codes, 16) ||
      !aligned(w_q_codes, 16) || !aligned(w_uk, 16) || !aligned(cache_pool, 16) ||
      !aligned(q_cat, 16) || (q_lo && !aligned(q_lo, 16)) || !aligned(positions, 4) ||
      !aligned(page_table, 4) || !aligned(w_dkv_scale, 4) || !aligned(w_kr_scale, 4) ||
      !aligned(w_q_scale, 4))
    return MLA_ERR_ALIGN;
  if (!aligned(workspace, 256)) return MLA_ERR_ALIGN;
  DevCtx* c = nullptr;
  if ((rc = device_ctx(&c))) return rc;
  const Workspace w = layout(dims, resolve_parts(0, c), c->sms);
  if (workspace_bytes < w.plan) return MLA_ERR_WORKSPACE;  // projection scratch only
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int B = dims->batch, D = dims->d_model, H = dims->n_heads;
  char* ws = static_cast<char*>(workspace);
  __nv_bfloat16* qc = static_cast<__nv_bfloat16*>(q_cat);
  __nv_bfloat16* ql = static_cast<__nv_bfloat16*>(q_lo);
  const GemmShape s = shape_append_wq_e4m3(dims);
  const int Bp = s.n_lo;
  // h -> a power-of-two scale and two E4M3 planes per row, in the out-projection's o_split area
  // (unused until mla_out_proj runs)
  if (align_up(2ull * Bp * D, 256) + 4ull * Bp > w.oh_split - w.o_split) return MLA_ERR_DIMS;
  uint8_t* planes = reinterpret_cast<uint8_t*>(ws + w.o_split);
  float* x_scale = reinterpret_cast<float*>(ws + w.o_split + align_up(2ull * Bp * D, 256));
  const int slices = (D / 8) % 8 == 0 ? 8 : 1;
  launch_pdl(fp8::split_planes_bf16_kernel, dim3(static_cast<unsigned>(Bp), slices), dim3(256),
             0, st, static_cast<const __nv_bfloat16*>(h), B, static_cast<long long>(D), Bp,
             planes, x_scale);
  if ((rc = last_launch())) return rc;
  // [W_DKV; W_KR; W_Q] (E4M3) x [h planes] in one stream-K product, epilogue as in
  // mla_append_absorb: cache rows + q_nope planes + RoPE(q_rope)
  const SkPlan q = sk_plan(s, sk::EpiAppendWq::smem_bytes(B), c->sms);
  const int m_q = H * (kDn + kDr);
  CUtensorMap a0, a1, a2, bm;
  if ((rc = map_weights_e4m3(&a0, w_dkv_codes, kDc, D, q.kbs))) return rc;
  if ((rc = map_weights_e4m3(&a1, w_kr_codes, kDr, D, q.kbs))) return rc;
  if ((rc = map_weights_e4m3(&a2, w_q_codes, m_q, D, q.kbs))) return rc;
  if ((rc = map_acts_e4m3(&bm, planes, 2 * Bp, D, s.n_pad, q.kbs))) return rc;
  sk::EpiAppendWq e{
      sk::EpiAppend{positions, page_table, max_pages, static_cast<__nv_bfloat16*>(cache_pool),
                    num_pages, c->status, dims->rope_theta},
      sk::EpiWq{H, Bp, qc, ql, reinterpret_cast<__nv_bfloat16*>(ws + w.qn), positions,
                dims->rope_theta}};
  E4m3Scales sc;
  sc.a[0] = w_dkv_scale;
  sc.rows[0] = kDc;
  sc.a[1] = w_kr_scale;
  sc.rows[1] = kDr;
  sc.a[2] = w_q_scale;
  sc.rows[2] = m_q;
  sc.x = x_scale;
  if ((rc = run_streamk<sk::EpiAppendWq, true>(c, s, q, B, positions, dims->rope_theta, a0, a1,
                                               kDc / 128, 0, bm, ws, w, e, st, &a2,
                                               sk::EpiAppendWq::kSplitRow / 128, sc, 1)))
    return rc;
  return run_wuk(c, dims, w_uk, ws, w, qc, ql, st);
}

int mla_out_proj_fp8(const mla_dims* dims, const float* o_lat, const void* w_uv,
                     const void* w_o_codes, const float* w_o_scale, void* o_heads, void* out,
                     void* workspace, size_t workspace_bytes, mla_stream_t stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (dims->dtype != MLA_BF16) return MLA_ERR_ARG;
  if (dims->batch > kFp8MaxBatch) return MLA_ERR_DIMS;
  if (!o_lat || !w_uv || !w_o_codes || !w_o_scale || !out) return MLA_ERR_NULL_ARG;
  if (!workspace) return MLA_ERR_WORKSPACE;
  if (!aligned(o_lat, 16) || !aligned(w_uv, 16) || !aligned(w_o_codes, 16) ||
      !aligned(w_o_scale, 4) || (o_heads && !aligned(o_heads, 16)) || !aligned(out, 16))
    return MLA_ERR_ALIGN;
  if (!aligned(workspace, 256)) return MLA_ERR_ALIGN;
  DevCtx* c = nullptr;
  if ((rc = device_ctx(&c))) return rc;
  const Workspace w = layout(dims, resolve_parts(0, c), c->sms);
  if (workspace_bytes < w.plan) return MLA_ERR_WORKSPACE;  // projection scratch only
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int B = dims->batch, D = dims->d_model, H = dims->n_heads;
  char* ws = static_cast<char*>(workspace);
  __nv_bfloat16* os = reinterpret_cast<__nv_bfloat16*>(ws + w.o_split);
  float* oh32 = reinterpret_cast<float*>(ws + w.oh_split);
  unsigned int* xmax = reinterpret_cast<unsigned int*>(ws + w.xmax);
  // o_h = W_UV_h [o_lat_hi | o_lat_lo] (bf16 weights, as in mla_out_proj); o_heads kept in fp32
  const GemmShape s1 = shape_wuv(dims);
  const int Bp = s1.n_lo;
  const size_t n = static_cast<size_t>(B) * H * kDc;
  launch_pdl(split_hi_lo_kernel,
             dim3(static_cast<unsigned>(std::min<size_t>((n / 8 + 255) / 256, 4096))), dim3(256),
             0, st, o_lat, n, static_cast<size_t>(Bp) * H * kDc, os, xmax, Bp);
  if ((rc = last_launch())) return rc;
  const SkPlan q1 = sk_plan(s1, 0, c->sms);
  CUtensorMap a, bm;
  if ((rc = map_weights(&a, w_uv, kDv, H, kDc, q1.kbs))) return rc;
  if ((rc = map_acts(&bm, os, H, 2 * Bp, kDc, kDc * 2ull, kDc * 2ull * H, s1.n_pad, q1.kbs)))
    return rc;
  sk::EpiWuv e1{H, Bp, static_cast<__nv_bfloat16*>(o_heads), nullptr, oh32, xmax};
  if ((rc = run_streamk(c, s1, q1, B, nullptr, 0.f, a, a, 1 << 30, 0, bm, ws, w, e1, st)))
    return rc;
  // o_heads row b -> E4M3 planes and a scale (the W_UV input is consumed by now)
  const GemmShape s2 = shape_wo_e4m3(dims);
  const int n_planes = oh_planes(dims);
  const uint64_t K = static_cast<uint64_t>(H) * kDv;
  uint8_t* planes = reinterpret_cast<uint8_t*>(ws + w.o_split);
  float* x_scale =
      reinterpret_cast<float*>(ws + w.o_split + align_up(n_planes * Bp * K, 256));
  const size_t groups8 = static_cast<size_t>(Bp) * K / 8;
  launch_pdl(fp8::split_planes_kernel,
             dim3(static_cast<unsigned>(std::min<size_t>((groups8 + 255) / 256, 4 * c->sms))),
             dim3(256), 0, st, static_cast<const float*>(oh32),
             static_cast<const unsigned int*>(xmax), B, static_cast<long long>(K), Bp, n_planes,
             planes, x_scale);
  if ((rc = last_launch())) return rc;
  // out = s_W,r * s_x,b * sum over planes of (W_O codes) x (plane codes), kind::f8f6f4
  const SkPlan q2 = sk_plan(s2, 0, c->sms);
  CUtensorMap a2, b2;
  if ((rc = map_weights_e4m3(&a2, w_o_codes, D, K, q2.kbs))) return rc;
  if ((rc = map_acts_e4m3(&b2, planes, n_planes * Bp, K, s2.n_pad, q2.kbs))) return rc;
  sk::EpiWo e2{D, static_cast<__nv_bfloat16*>(out)};
  E4m3Scales sc;
  sc.a[0] = w_o_scale;
  sc.rows[0] = D;
  sc.x = x_scale;
  return run_streamk<sk::EpiWo, true>(c, s2, q2, B, nullptr, 0.f, a2, a2, 1 << 30, 0, b2, ws, w,
                                      e2, st, nullptr, 1 << 30, sc, 1);
}

int mla_merge_partials(const mla_dims* dims, int32_t n_parts, const float* part_o,
                       const float* part_lse, float* o_lat, float* lse, mla_stream_t stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (!part_o || !part_lse || !o_lat) return MLA_ERR_NULL_ARG;
  if (n_parts < 1 || n_parts > kMaxParts) return MLA_ERR_ARG;
  if (!aligned(part_o, 16) || !aligned(o_lat, 16) || !aligned(part_lse, 4) ||
      (lse && !aligned(lse, 4)))
    return MLA_ERR_ALIGN;
  DevCtx* c = nullptr;
  if ((rc = device_ctx(&c))) return rc;
  const int rows = dims->batch * dims->n_heads;
  launch_pdl(attn::merge_kernel,
             dim3(static_cast<unsigned>((rows + attn::kCombineWarps - 1) / attn::kCombineWarps)),
             dim3(32 * attn::kCombineWarps), 0, reinterpret_cast<cudaStream_t>(stream), n_parts,
             rows, part_o, part_lse, o_lat, lse);
  return last_launch();
}

int mla_get_status(mla_stream_t stream) {
  DevCtx* c = nullptr;
  int rc = device_ctx(&c);
  if (rc) return rc;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MLA_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpy(&v, c->status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess)
    return MLA_ERR_CUDA;
  if (cudaMemset(c->status, 0, sizeof(unsigned int)) != cudaSuccess) return MLA_ERR_CUDA;
  return static_cast<int>(v & 0x7fffffffu);
}

const char* mla_error_string(int code) {
  switch (code) {
    case MLA_OK: return "ok";
    case MLA_ERR_NULL_ARG: return "a required pointer is NULL";
    case MLA_ERR_DIMS: return "unsupported shape or dtype";
    case MLA_ERR_ALIGN: return "misaligned pointer";
    case MLA_ERR_WORKSPACE: return "workspace missing or too small";
    case MLA_ERR_ARG: return "invalid argument";
    case MLA_ERR_CUDA: return "CUDA runtime error";
    case MLA_ERR_DEVICE: return "device is not sm_100 (B200)";
    default: break;
  }
  if (code > 0) {
    if (code & MLA_STATUS_TIMEOUT) return "device: bounded wait timed out";
    if (code & MLA_STATUS_BAD_PAGE) return "device: page id out of range";
    if (code & MLA_STATUS_BAD_LENGTH) return "device: sequence length out of range";
    if (code & MLA_STATUS_BAD_POSITION) return "device: append position out of range";
  }
  return "unknown code";
}

const char* mla_error_detail(void) { return g_err_detail; }

const char* mla_version(void) { return "mla_latent_kv_37_b200 0.1 (sm_100a)"; }

uint64_t mla_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int mla_set_profile_events(void* const* begin, void* const* end, int32_t count) {
  if (count < 0 || (count > 0 && (!begin || !end))) return MLA_ERR_ARG;
  std::lock_guard<std::mutex> lock(g_mu);
  g_prof_begin = reinterpret_cast<cudaEvent_t*>(const_cast<void**>(begin));
  g_prof_end = reinterpret_cast<cudaEvent_t*>(const_cast<void**>(end));
  g_prof_count = count;
  g_prof_next = 0;
  return MLA_OK;
}

int32_t mla_profile_events_used(void) { return g_prof_next; }

}  // extern "C"

// =============================================================================================
// Decode attention with scratch memory owned by the library (no allocation by anyone).
//
// Some callers cannot allocate device memory for a workspace: a process whose memory manager
// has already reserved all of the GPU's memory for itself, or a code path where a cudaMalloc
// (which can synchronise the device or fail under memory pressure) is not acceptable.  For them
// the split-KV scratch of mla_decode_attn (the page plan and the per-part partial results)
// lives in one fixed-size array in the library's own device data.  Every GPU that loads the
// library holds MLA_STATIC_SCRATCH_BYTES for it until the process exits.
// =============================================================================================
static __device__ __align__(256) unsigned char g_decode_scratch[MLA_STATIC_SCRATCH_BYTES];

namespace {
void* g_scratch_addr[64];  // device address of g_decode_scratch, per device
std::mutex g_scratch_mu;

// Host code sees `g_decode_scratch` only as a stand-in symbol: its device address is looked
// up once per device, with that device current, and cached.
int decode_scratch_addr(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MLA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return MLA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return MLA_OK;
}

struct DecodeScratch {
  size_t plan, part_o, part_lse, total;
};

DecodeScratch decode_scratch_layout(int B, int H, int parts) {
  DecodeScratch d{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  d.plan = take(attn::PlanView::words(B, parts) * 4);
  d.part_o = take((static_cast<size_t>(B) + static_cast<size_t>(parts)) * H * kDc * 4);
  d.part_lse = take((static_cast<size_t>(B) + static_cast<size_t>(parts)) * H * 4);
  d.total = off;
  return d;
}
}  // namespace

extern "C" int mla_decode_attn_static_scratch(const mla_dims* dims, const void* q_cat,
                                              const void* q_lo, const void* cache_pool,
                                              int32_t num_pages, const int32_t* page_table,
                                              int32_t max_pages, const int32_t* seq_lens,
                                              float softmax_scale, int32_t num_splits,
                                              float* o_lat, float* lse, mla_stream_t stream) {
  int rc = check_decode_args(dims, q_cat, q_lo, cache_pool, num_pages, page_table, max_pages,
                             seq_lens, softmax_scale, num_splits, o_lat, lse);
  if (rc) return rc;
  if (q_lo) return MLA_ERR_ARG;  // this entry point takes the bf16 query alone
  DevCtx* c = nullptr;
  if ((rc = device_ctx(&c))) return rc;
  const int B = dims->batch, H = dims->n_heads;
  const int parts = resolve_parts(num_splits, c);
  const DecodeScratch w = decode_scratch_layout(B, H, parts);
  if (w.total > MLA_STATIC_SCRATCH_BYTES) return MLA_ERR_WORKSPACE;  // beyond the fixed size
  void* scratch = nullptr;
  if ((rc = decode_scratch_addr(&scratch))) return rc;
  // Nothing in the scratch has to start at zero: the plan kernel writes every plan word and
  // the split kernel writes every partial slot before the combine kernel reads it.
  char* ws = static_cast<char*>(scratch);
  return enqueue_decode(c, dims, q_cat, nullptr, cache_pool, num_pages, page_table, max_pages,
                        seq_lens, softmax_scale, parts, reinterpret_cast<int32_t*>(ws + w.plan),
                        reinterpret_cast<float*>(ws + w.part_o),
                        reinterpret_cast<float*>(ws + w.part_lse), o_lat, lse,
                        reinterpret_cast<cudaStream_t>(stream));
}
