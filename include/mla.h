/*
 * mla.h -- C ABI for weight-absorbed Multi-Head Latent Attention (MLA) decode on NVIDIA B200
 * (sm_100a).  One new query token per sequence attends, across n_heads heads, to a paged
 * per-layer cache that stores 576 numbers per token: the 512-wide latent c_KV plus the
 * 64-wide decoupled RoPE key k_R.
 *
 * Sources (web pages on MLA, cited by title and section):
 *   [LP] linuxpro.com.br, "Como a DeepSeek reescreveu o Transformer (MLA)":
 *        "Classic attention and the cost of the KV cache" (softmax(QK^T/sqrt(d_k) + M)V, the
 *        new token computes one query row and reads the whole cache), "MLA: compress the pair,
 *        not the heads" (c^KV 512 + k^R 64 cached; W^UK and W^UV absorbed by associativity).
 *   [TN] technova-ai.online, "DeepSeek AI efficiency architecture benchmarks", section
 *        "Architectural Innovations: Multi-Head Latent Attention (MLA)": c_KV = W_DKV h_t,
 *        K_t = W_UK c_KV, V_t = W_UV c_KV.
 *   [IA] ia.com.br, "Como a MLA da DeepSeek cortou 93% da memoria ...", section
 *        "Um resumo no lugar de 128 copias": RoPE kept out of the compression as 64 numbers.
 *
 * Conventions shared by every call
 *   - All pointers except `dims` are DEVICE pointers owned by the caller; the library never
 *     allocates or frees memory and keeps no state between calls other than one device status
 *     word per GPU (see mla_get_status).
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream).
 *     The bf16 kernels are launched with programmatic stream serialisation: one may be
 *     scheduled while the work before it on the stream drains, but it reads and writes nothing
 *     until that work has completed, so stream order holds exactly as for ordinary launches.
 *     Setting MLA_NO_PDL=1 in the environment before the first call turns this off.
 *   - Every wait inside a kernel is bounded (2 s; MLA_WAIT_NS in the environment, in
 *     nanoseconds, read at each call, overrides it).  A wait that runs out raises
 *     MLA_STATUS_TIMEOUT; the kernel then waits (on its own, longer limit) for the copies and
 *     tensor-core operations it has in flight, releases its resources and returns, and the
 *     CUDA context stays usable.  MLA_TEST_STALL=1 (read at each call) makes one warp of the
 *     decode kernel wait on a barrier nothing arrives on, to exercise that path in tests.
 *   - Weights are row-major [out_features, in_features] (column-vector form, [TN]):
 *       w_dkv [d_c, D], w_kr [d_rope, D], w_q [H*(d_nope+d_rope), D] (per head d_nope rows then
 *       d_rope rows), w_uk [H*d_nope, d_c], w_uv [H*d_v, d_c], w_o [D, H*d_v].
 *   - Element type: dims.dtype = MLA_BF16 -> h, weights, cache, q_cat, o_heads, out are bf16;
 *     MLA_FP32 -> all of them fp32.  o_lat and lse are fp32 in both cases.
 *   - Cache pool: [num_pages, page_size, d_c + d_rope] rows of one layer; row = [c_KV | k_R].
 *     page_table [batch, max_pages] int32 (row-major) maps a sequence's page index to a pool
 *     page; only entries [0, ceil(len/page_size)) of a row are read.  Cache slots past a
 *     sequence's length must hold finite values; they never influence a result.
 *   - RoPE: interleaved pairs (x[2i], x[2i+1]) rotated by pos * rope_theta^(-2i/d_rope); the
 *     same rotation is applied to k_R (shared by all heads) and to every head's query part.
 *   - Return value: MLA_OK (0) or a negative MLA_ERR_* detected on the host before any launch
 *     (nothing was enqueued).  Errors found on the device while a kernel runs (bad page id,
 *     over-long sequence, timed-out wait) are OR-ed into the status word; kernels never trap.
 *   - A workspace (device, >= 256-byte aligned, size from mla_workspace_size) is scratch
 *     shared by the four compute calls; calls that share one workspace must be ordered (same
 *     stream or synchronised).
 */
#ifndef MLA_B200_H_
#define MLA_B200_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* mla_stream_t; /* same type as cudaStream_t */

enum { MLA_BF16 = 0, MLA_FP32 = 1 };

/* Shapes.  Supported: d_c = 512, d_rope = 64, d_nope = 128, d_v = 128, page_size = 64,
 * n_heads in {16, 32, ..., 128}, d_model a positive multiple of 64, batch >= 1.
 * rope_theta > 0 (10000 for DeepSeek-V2/V3). */
typedef struct mla_dims {
  int32_t batch;     /* B: sequences, one new token each */
  int32_t n_heads;   /* H */
  int32_t d_c;       /* latent width of c_KV */
  int32_t d_rope;    /* width of the decoupled RoPE key k_R and of each head's q_rope */
  int32_t d_nope;    /* per-head non-rotary query/key width */
  int32_t d_v;       /* per-head value width */
  int32_t d_model;   /* D: hidden size of h_t */
  int32_t page_size; /* tokens per cache page */
  int32_t dtype;     /* MLA_BF16 or MLA_FP32 */
  float rope_theta;  /* RoPE base */
} mla_dims;

/* Host-detected errors (returned). */
#define MLA_OK 0
#define MLA_ERR_NULL_ARG (-1)    /* a required pointer is NULL */
#define MLA_ERR_DIMS (-2)        /* unsupported shape or dtype */
#define MLA_ERR_ALIGN (-3)       /* a pointer is not 16-byte aligned (workspace: 256) */
#define MLA_ERR_WORKSPACE (-4)   /* workspace missing or smaller than mla_workspace_size */
#define MLA_ERR_ARG (-5)         /* other bad argument (negative count, bad option) */
#define MLA_ERR_CUDA (-6)        /* a CUDA runtime call failed (launch, attribute, device) */
#define MLA_ERR_DEVICE (-7)      /* current device is not sm_100 */

/* Device-detected conditions (bits of the status word, see mla_get_status). */
#define MLA_STATUS_BAD_PAGE 0x1u     /* a page id outside [0, num_pages) was skipped */
#define MLA_STATUS_BAD_LENGTH 0x2u   /* a sequence length outside [0, max_pages*page_size] */
#define MLA_STATUS_TIMEOUT 0x4u      /* a bounded wait inside a kernel gave up */
#define MLA_STATUS_BAD_POSITION 0x8u /* an append position outside the sequence's pages */

/* Scratch bytes needed by every compute call for these dims when the decode call is split
 * into at most `num_splits` parts (0 = the library's automatic choice).  Never fails.  The
 * projection calls use only the part that does not depend on the split count, so a workspace
 * sized for any num_splits serves them; mla_decode_attn needs the size for its own count. */
size_t mla_workspace_size(const mla_dims* dims, int32_t num_splits);

/* Bytes one cached token occupies in one layer's pool: (d_c + d_rope) * element size.
 * For DeepSeek-V3 shapes in bf16 this is 1152; times 61 layers, 70,272 bytes per token
 * ([LP] "MLA: compress the pair, not the heads"). Returns 0 for unsupported dims. */
int64_t mla_cache_row_bytes(const mla_dims* dims);

/*
 * mla_cache_append -- the new token's cache row ([TN]; [LP] "MLA: compress the pair ..."):
 *   c_KV = W_DKV h_t,   k_R = RoPE(W_KR h_t, positions[b]),
 * rounded to the cache dtype (round-to-nearest-even) and written to slot
 * positions[b] % page_size of pool page page_table[b][positions[b] / page_size].
 *   h        [B, D]
 *   w_dkv, w_kr: the two projections; if BOTH are NULL, h is taken as ready rows
 *            [B, d_c + d_rope] (already rotated) and only the paged scatter runs.
 *   positions [B] int32, 0-based index of the new token (= rows already cached).
 * Only the addressed slot of each sequence is written; all other pool bytes are untouched.
 */
int mla_cache_append(const mla_dims* dims, const void* h, const void* w_dkv, const void* w_kr,
                     const int32_t* positions, const int32_t* page_table, int32_t max_pages,
                     void* cache_pool, int32_t num_pages, void* workspace,
                     size_t workspace_bytes, mla_stream_t stream);

/*
 * mla_absorb_q -- absorbed query ([LP] "MLA: compress the pair ...", associativity
 * Q (c W_UK)^T = (Q W_UK^T) c^T):
 *   q = W_Q h_t;  per head q_nope = q[h*192 : h*192+128],  q_rope = RoPE(q[h*192+128 : +64]);
 *   q_lat_h = W_UK_h^T q_nope_h (512);   q_cat[b][h] = [q_lat_h | q_rope_h]   (576).
 *   q_cat    [B, H, d_c + d_rope] (dims.dtype)
 *   q_lo     nullable; bf16 only: [B, H, d_c + d_rope] receives the rounding remainder
 *            q - bf16(q) of every element, so that q_cat + q_lo carries ~16 significant bits.
 *            It is meant for large score logits (|logit| >> 10), where the bf16 rounding of
 *            q_cat alone costs accuracy; pass it on to mla_decode_attn.
 * q_nope is kept at ~16 bits (bf16 hi + lo) through the W_UK product; accumulation is fp32.
 */
int mla_absorb_q(const mla_dims* dims, const void* h, const void* w_q, const void* w_uk,
                 const int32_t* positions, void* q_cat, void* q_lo, void* workspace,
                 size_t workspace_bytes, mla_stream_t stream);

/*
 * mla_append_absorb -- mla_cache_append followed by mla_absorb_q in one call, same arguments
 * and same results (up to the order of fp32 additions).  Both start by multiplying the new
 * hidden states h by a weight matrix; here W_DKV, W_KR and W_Q stream through one product, so
 * the small cache-append projection shares the launch of the large query projection.  All
 * pointers are required except q_lo.  The fp32 path runs the two calls in order.
 */
int mla_append_absorb(const mla_dims* dims, const void* h, const void* w_dkv, const void* w_kr,
                      const void* w_q, const void* w_uk, const int32_t* positions,
                      const int32_t* page_table, int32_t max_pages, void* cache_pool,
                      int32_t num_pages, void* q_cat, void* q_lo, void* workspace,
                      size_t workspace_bytes, mla_stream_t stream);

/*
 * mla_decode_attn -- attention of each sequence's new query over its whole cache
 * ([LP] "Classic attention ...": softmax(Q K^T / sqrt(d_k) + M) V, causal mask M admits every
 * cached row since the query is the newest token), in latent space:
 *   s_j = scale * (q_lat . c_j + q_rope . k_R,j),  j < seq_lens[b];   p = softmax(s);
 *   o_lat[b][h] = sum_j p_j c_j (d_c wide),   lse[b][h] = log sum_j exp(s_j).
 *   q_cat    [B, H, d_c + d_rope] (dims.dtype).
 *   q_lo     nullable; bf16 only: [B, H, d_c + d_rope], the query's rounding remainder as
 *            written by mla_absorb_q.  When given, the scores use q_cat + q_lo (~16 significant
 *            bits instead of 8), for inputs whose logits are large enough (spread >> 10) that
 *            the bf16 rounding of the query alone moves the output by more than ~1e-3.  It
 *            costs about twice the tensor work (each cluster then handles 64 heads) and reads
 *            the same cache bytes.  The workspace size does not change.
 *   seq_lens [B] int32 (rows to attend, including the token just appended); 0 is allowed
 *            and yields o_lat = 0, lse = -inf.
 *   softmax_scale: 0 selects 1/sqrt(d_nope + d_rope).
 *   num_splits: number of parts the concatenated page list of all sequences is divided into
 *            (split-KV); 0 = automatic (about one part per pair of SMs, or per four SMs with
 *            q_lo).  At most 65536, and not more than the value used for mla_workspace_size.
 *   num_pages * page_size and max_pages * page_size must fit in int32 (MLA_ERR_ARG).
 *   o_lat    [B, H, d_c] fp32;  lse [B, H] fp32, nullable.
 */
int mla_decode_attn(const mla_dims* dims, const void* q_cat, const void* q_lo,
                    const void* cache_pool, int32_t num_pages, const int32_t* page_table,
                    int32_t max_pages, const int32_t* seq_lens, float softmax_scale,
                    int32_t num_splits, void* workspace, size_t workspace_bytes, float* o_lat,
                    float* lse, mla_stream_t stream);

/*
 * mla_out_proj -- value up-projection and output projection ([TN] V = W_UV c_KV, moved after
 * the weighted sum by associativity; [LP] W_O):
 *   o_heads[b][h] = W_UV_h o_lat[b][h]  (d_v wide),   out[b] = W_O concat_h o_heads[b][h].
 *   o_lat    [B, H, d_c] fp32 (from mla_decode_attn).
 *   o_heads  [B, H, d_v] (dims.dtype), nullable if only `out` is wanted.
 *   w_o, out nullable together (then only o_heads is produced).
 */
int mla_out_proj(const mla_dims* dims, const float* o_lat, const void* w_uv, const void* w_o,
                 void* o_heads, void* out, void* workspace, size_t workspace_bytes,
                 mla_stream_t stream);

/*
 * mla_merge_partials -- merge attention results computed apart over disjoint parts of the
 * cached rows, e.g. one per GPU when a long sequence's pages are spread over several GPUs
 * (split-KV across devices; each GPU runs mla_decode_attn over its own pages and the results
 * are gathered).  For every (b, h):
 *   lse = log sum_r exp(lse_r),   o_lat = sum_r exp(lse_r - lse) o_lat_r
 * ([LP] "Classic attention ...": softmax over the union of the parts equals this weighting of
 * the parts' softmaxes; the same merge the decode call applies to its own split-KV parts).
 *   part_o   [n_parts, B, H, d_c] fp32, each normalised (mla_decode_attn's o_lat).
 *   part_lse [n_parts, B, H] fp32 (mla_decode_attn's lse); -inf marks a part without rows.
 *   o_lat    [B, H, d_c] fp32;  lse [B, H] fp32, nullable.  Rows whose parts are all empty
 *            get o_lat = 0, lse = -inf.
 */
int mla_merge_partials(const mla_dims* dims, int32_t n_parts, const float* part_o,
                       const float* part_lse, float* o_lat, float* lse, mla_stream_t stream);

/*
 * Folded execution mode (bf16 only).  The absorbed form multiplies by W_UK_h and W_UV_h at
 * every step; the associativity that allows it ([LP] "MLA: compress the pair, not the heads":
 * Q K^T = (Q W_UK^T) c^T) also allows multiplying the weights together once, ahead of time
 * ([IA] "O preço da economia: mais contas": the mode that reuses pre-multiplied matrices).  For
 * decode the folded matrices are larger (576 x D per head instead of 192 x D plus 128 x 512,
 * and D x 512 per head instead of D x 128 plus 128 x 512), so every step streams more weight
 * bytes; the mode exists to measure that trade.
 *
 * mla_fold_weights -- the one-time folding, fp32 accumulation, bf16 (round to nearest even):
 *   w_qf [H, d_c + d_R, D]: rows m < d_c of head h = sum_k W_UK[h*d_nope + k][m] W_Q[h*192 + k]
 *                           (W_UK_h^T W_Q,nope,h); rows d_c + i = W_Q[h*192 + d_nope + i].
 *   w_of [D, H*d_c]:        column h*d_c + m = sum_k W_O[:, h*d_v + k] W_UV[h*d_v + k][m].
 *   Either output may be NULL (then its two inputs may be NULL too).  Caller-owned buffers.
 */
int mla_fold_weights(const mla_dims* dims, const void* w_q, const void* w_uk, const void* w_uv,
                     const void* w_o, void* w_qf, void* w_of, mla_stream_t stream);

/*
 * mla_append_absorb_folded -- mla_append_absorb with the folded query weights: one product
 * [W_DKV; W_KR; W_QF] h writes the cache row (as mla_cache_append) and
 *   q_cat[b][h][m] = (W_QF h)[h*576 + m],  m < d_c;   q_cat[b][h][d_c..] = RoPE(rows d_c..).
 *   q_lo optional, as in mla_absorb_q.  Same arguments otherwise; bf16 only (MLA_ERR_ARG).
 */
int mla_append_absorb_folded(const mla_dims* dims, const void* h, const void* w_dkv,
                             const void* w_kr, const void* w_qf, const int32_t* positions,
                             const int32_t* page_table, int32_t max_pages, void* cache_pool,
                             int32_t num_pages, void* q_cat, void* q_lo, void* workspace,
                             size_t workspace_bytes, mla_stream_t stream);

/*
 * mla_out_proj_folded -- out[b] = W_OF o_lat[b] (o_lat flattened to H*d_c), the output of
 * mla_out_proj without the per-head o_heads.  o_lat fp32 [B, H, d_c]; out [B, D] bf16.
 */
int mla_out_proj_folded(const mla_dims* dims, const float* o_lat, const void* w_of, void* out,
                        void* workspace, size_t workspace_bytes, mla_stream_t stream);

/*
 * E4M3 (FP8) weights ([IA] "De onde vem o 93%": the pages' throughput figure was measured with
 * the weights converted to FP8).  A weight matrix is stored as one byte per element, E4M3
 * (sign, 4 exponent bits with bias 7, 3 mantissa bits, subnormals, largest finite 448), and
 * one fp32 scale per row: weight = decode(code) * scale[row].
 *
 * mla_quantize_weights_fp8 -- w [rows, cols] bf16 -> codes, scale [rows]:
 *   scale[r] = max_j |w[r][j]| / 448 (fp32, round to nearest; 1 for a zero row),
 *   code(r, j) = w[r][j] / scale[r] (fp32) rounded to the nearest E4M3 value, ties to even,
 *   saturating at +-448.  cols a positive multiple of 128.  No dims: any bf16 matrix.
 *   Layout of codes (round_up(rows, 128) * cols bytes): tiles of 128 rows x 128 columns, each
 *   contiguous and row-major inside, ordered by row tile, then column tile, so that code(r, j)
 *   is at byte ((r / 128) * (cols / 128) + j / 128) * 16384 + (r % 128) * 128 + j % 128.  A
 *   product then streams whole 16 KB tiles from HBM.  The padding rows of the last row tile
 *   are not written and never reach a result.
 *
 * mla_append_absorb_fp8 -- mla_append_absorb with W_DKV, W_KR and W_Q stored as E4M3 (each
 *   as mla_quantize_weights_fp8 writes it, with its row scales); W_UK stays bf16.  bf16 path
 *   only, d_model a multiple of 128 (else MLA_ERR_DIMS).  Each hidden-state
 *   row h_b enters the E4M3 x E4M3 product as a power-of-two scale s_b (the smallest power of
 *   two >= max|h_b| / 448) and two E4M3 planes whose sum is h_b / s_b exactly (a bf16 value has
 *   8 significant bits; only parts below E4M3's smallest subnormal, under about 2^-8 of the
 *   row's largest element, are dropped).  Each product row is w_scale[row] * s_b * (sum over
 *   planes) in fp32; the epilogue (cache rows, RoPE, q_nope planes, W_UK absorption, q_lo) is
 *   that of mla_append_absorb.  Workspace as mla_append_absorb.
 *
 * mla_out_proj_fp8 -- mla_out_proj with W_O stored as E4M3 codes + row scales (w_o_codes:
 *   W_O [D, H*d_v] as mla_quantize_weights_fp8 writes it, w_o_scale [D]); W_UV stays bf16.
 *   out is required, o_heads optional.  bf16 path only.  The codes stream from HBM at one
 *   byte per weight into E4M3 x E4M3 tensor-core products (fp32 sums).  Each o_heads row b
 *   enters as a scale s_b = max|o_b| / 448 and E4M3 planes whose sum approximates o_b / s_b:
 *   three planes (about 12 significant bits) for batches up to 32, two (about 8) above, so that
 *   planes x round16(batch) fit the 256 columns of one MMA up to batch 128;
 *   out[b][r] = w_o_scale[r] * s_b * (sum over planes), rounded to bf16.
 *   The workspace of mla_workspace_size serves it (projection part only, as mla_out_proj).
 */
int mla_quantize_weights_fp8(const void* w, int64_t rows, int64_t cols, void* codes,
                             float* scale, mla_stream_t stream);

int mla_append_absorb_fp8(const mla_dims* dims, const void* h, const void* w_dkv_codes,
                          const float* w_dkv_scale, const void* w_kr_codes,
                          const float* w_kr_scale, const void* w_q_codes, const float* w_q_scale,
                          const void* w_uk, const int32_t* positions, const int32_t* page_table,
                          int32_t max_pages, void* cache_pool, int32_t num_pages, void* q_cat,
                          void* q_lo, void* workspace, size_t workspace_bytes,
                          mla_stream_t stream);

int mla_out_proj_fp8(const mla_dims* dims, const float* o_lat, const void* w_uv,
                     const void* w_o_codes, const float* w_o_scale, void* o_heads, void* out,
                     void* workspace, size_t workspace_bytes, mla_stream_t stream);

/*
 * Native decode step over a stack of layers, end to end from host memory.
 *
 * mla_layer -- one layer's device-resident weights and paged cache (layouts as in the calls
 * above; w_o must be given: the step's result is `out`).  With w_q_scale non-NULL the layer's
 * w_dkv, w_kr, w_q and w_o are E4M3 codes as mla_quantize_weights_fp8 writes them, with the
 * four row-scale arrays (all required then), and the layer runs mla_append_absorb_fp8 and
 * mla_out_proj_fp8; with w_q_scale NULL the four scale pointers are ignored.
 *
 * mla_step_workspace_size -- bytes of device workspace mla_decode_step_host needs: device
 *   copies of every layer's h and out, positions, lengths, q_cat, o_lat, lse, o_heads, and the
 *   workspace of the per-layer calls.  0 for unsupported dims or n_layers < 1.
 *
 * mla_decode_step_host -- for every layer l in order ([TN] MLA equations; [LP] "MLA: compress
 * the pair, not the heads"):  mla_append_absorb -> mla_decode_attn -> mla_out_proj, with
 *   h_host        [n_layers, B, D] (dims.dtype) host memory: layer l's hidden states,
 *   positions_host, seq_lens_host [B] int32 host memory (the same for every layer),
 *   out_host      [n_layers, B, D] (dims.dtype) host memory: layer l's output W_O concat_h o_h.
 * The inputs are copied up on a copy stream ahead of the layers, each layer's output is copied
 * back on another as soon as it is written (page-locked host memory lets the copies overlap the
 * kernels; pageable memory works but copies synchronously), and `stream` waits for the last
 * copy: the host buffers may be read (out) or reused (inputs) once `stream` has reached that
 * point.  Host-detected errors return before anything is enqueued; a failure of a layer's call
 * returns its code, with the earlier layers' work already enqueued.  Calls from several host
 * threads on one device are serialised.
 */
typedef struct mla_layer {
  const void* w_dkv;
  const void* w_kr;
  const void* w_q;
  const void* w_uk;
  const void* w_uv;
  const void* w_o;
  void* cache_pool;
  int32_t num_pages;
  const int32_t* page_table;
  int32_t max_pages;
  const float* w_dkv_scale;
  const float* w_kr_scale;
  const float* w_q_scale;
  const float* w_o_scale;
} mla_layer;

size_t mla_step_workspace_size(const mla_dims* dims, int32_t n_layers, int32_t num_splits);

int mla_decode_step_host(const mla_dims* dims, int32_t n_layers, const mla_layer* layers,
                         const void* h_host, const int32_t* positions_host,
                         const int32_t* seq_lens_host, void* out_host, int32_t num_splits,
                         void* workspace, size_t workspace_bytes, mla_stream_t stream);

/*
 * mla_decode_attn_static_scratch -- mla_decode_attn for callers that cannot allocate device
 * memory.  (The MLA pages have no counterpart to this: it is a deployment convenience.)
 * A process whose memory manager already owns all of the GPU's memory, or a code path where a
 * cudaMalloc -- which may synchronise the device or fail under memory pressure -- is not
 * acceptable, cannot provide the workspace mla_decode_attn needs.  This entry point takes the
 * same arguments minus the workspace (q_lo must be NULL here too) and keeps the split-KV
 * scratch (page plan and per-part partial results) in a fixed array of
 * MLA_STATIC_SCRATCH_BYTES in the library's own device data, which every GPU that loads the
 * library holds until the process exits.  It allocates
 * nothing.  Results equal mla_decode_attn's for the same arguments.
 *   - The scratch needed is about (batch + parts) * n_heads * 2 KiB (parts = num_splits, or
 *     the automatic choice); calls needing more than MLA_STATIC_SCRATCH_BYTES return
 *     MLA_ERR_WORKSPACE without launching anything (pass a smaller num_splits).
 *   - The first call on each device looks the array's device address up (one-time set-up,
 *     cached per device); make that first call before any stream capture.
 *   - All calls on a device share the one array and leave their contents in it; nothing in it
 *     needs to start at zero.  Calls that overlap on the GPU (different streams, or threads
 *     without synchronisation) race on the scratch: order them on one stream.
 */
#define MLA_STATIC_SCRATCH_BYTES (64u * 1024u * 1024u)
int mla_decode_attn_static_scratch(const mla_dims* dims, const void* q_cat, const void* q_lo,
                                   const void* cache_pool, int32_t num_pages,
                                   const int32_t* page_table, int32_t max_pages,
                                   const int32_t* seq_lens, float softmax_scale,
                                   int32_t num_splits, float* o_lat, float* lse,
                                   mla_stream_t stream);

/* Synchronises `stream`, returns the device status word of the current device (a bitwise OR
 * of MLA_STATUS_* raised since the last call, 0 if none) and clears it.  Returns a negative
 * MLA_ERR_CUDA if the synchronisation itself failed. */
int mla_get_status(mla_stream_t stream);

/* Static description of a return code or status bit set. */
const char* mla_error_string(int code);

/* The CUDA error behind the last MLA_ERR_CUDA returned to the calling thread: the failing
 * call, the error's name and its description ("" if there was none).  The string belongs to
 * the library and stays valid until the thread's next call into it. */
const char* mla_error_detail(void);

/* Library build string (for logs). */
const char* mla_version(void);

/* Number of kernels this library has launched in this process (all devices, all calls). */
uint64_t mla_launch_count(void);

/* Profiling hook.  After this call, the i-th bf16 mla_decode_attn call (i < count) records
 * begin[i] just before and end[i] just after its split-KV kernel on the call's stream, so the
 * caller can time that kernel alone with cudaEventElapsedTime.  begin/end are host arrays of
 * cudaEvent_t created by the caller (timing enabled), kept alive until the calls are done.
 * count = 0 switches recording off.  Returns MLA_OK or MLA_ERR_ARG. */
int mla_set_profile_events(void* const* begin, void* const* end, int32_t count);

/* How many event pairs have been recorded since the last mla_set_profile_events. */
int32_t mla_profile_events_used(void);

#ifdef __cplusplus
}
#endif
#endif /* MLA_B200_H_ */
