// Native decode-step executor: one MLA decode step over a stack of layers, end to end from host
// memory, built only on the library's public calls (mla.h).  Per layer l:
//   mla_append_absorb -> mla_decode_attn -> mla_out_proj
// ([TN] MLA equations; [LP] "MLA: compress the pair, not the heads").  The hidden states of
// every layer go up on one copy stream ahead of that layer, every layer's output comes back on
// another as soon as the layer has written it, and the step ends when the last output is on
// the host; only the first layer's input and the last layer's output are exposed.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>
#include <vector>

#include "mla.h"

namespace {

size_t elem_bytes(const mla_dims* d) { return d->dtype == MLA_BF16 ? 2 : 4; }
size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// device buffers of a step inside the caller's workspace
struct StepLayout {
  size_t h, pos, lens, q_cat, o_lat, lse, o_heads, out, call, total;
};

StepLayout step_layout(const mla_dims* d, int32_t n_layers, int32_t num_splits) {
  const size_t B = d->batch, H = d->n_heads, D = d->d_model, e = elem_bytes(d);
  StepLayout s{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  s.h = take(static_cast<size_t>(n_layers) * B * D * e);
  s.pos = take(B * 4);
  s.lens = take(B * 4);
  s.q_cat = take(B * H * (d->d_c + d->d_rope) * e);
  s.o_lat = take(B * H * d->d_c * 4);
  s.lse = take(B * H * 4);
  s.o_heads = take(B * H * d->d_v * e);
  s.out = take(static_cast<size_t>(n_layers) * B * D * e);
  const size_t call = mla_workspace_size(d, num_splits);
  s.call = take(call);
  s.total = call ? off : 0;
  return s;
}

// Copy streams and per-layer events, one set per device, reused by every step (enqueue is
// serialised by the mutex; stream order makes reuse of an event safe across steps).
struct StepStreams {
  bool init = false;
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, done = nullptr;
  std::vector<cudaEvent_t> ev_in, ev_out;
};
StepStreams g_step[64];
std::mutex g_step_mu;

int step_streams(int dev, int n_layers, StepStreams** out) {
  if (dev < 0 || dev >= 64) return MLA_ERR_DEVICE;
  StepStreams& s = g_step[dev];
  if (!s.init) {
    if (cudaStreamCreateWithFlags(&s.in, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&s.out, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&s.start, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&s.done, cudaEventDisableTiming) != cudaSuccess)
      return MLA_ERR_CUDA;
    s.init = true;
  }
  while (static_cast<int>(s.ev_in.size()) < n_layers) {
    cudaEvent_t a = nullptr, b = nullptr;
    if (cudaEventCreateWithFlags(&a, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&b, cudaEventDisableTiming) != cudaSuccess)
      return MLA_ERR_CUDA;
    s.ev_in.push_back(a);
    s.ev_out.push_back(b);
  }
  *out = &s;
  return MLA_OK;
}

int cuda_rc(cudaError_t e) { return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA; }

}  // namespace

extern "C" {

size_t mla_step_workspace_size(const mla_dims* dims, int32_t n_layers, int32_t num_splits) {
  if (!dims || n_layers < 1) return 0;
  return step_layout(dims, n_layers, num_splits).total;
}

int mla_decode_step_host(const mla_dims* dims, int32_t n_layers, const mla_layer* layers,
                         const void* h_host, const int32_t* positions_host,
                         const int32_t* seq_lens_host, void* out_host, int32_t num_splits,
                         void* workspace, size_t workspace_bytes, mla_stream_t stream) {
  if (!dims) return MLA_ERR_NULL_ARG;
  if (n_layers < 1 || num_splits < 0) return MLA_ERR_ARG;
  if (!layers || !h_host || !positions_host || !seq_lens_host || !out_host)
    return MLA_ERR_NULL_ARG;
  for (int l = 0; l < n_layers; ++l) {
    const mla_layer& ly = layers[l];
    if (!ly.w_o) return MLA_ERR_NULL_ARG;  // the step's result is `out`
    if (ly.w_q_scale && (!ly.w_dkv_scale || !ly.w_kr_scale || !ly.w_o_scale))
      return MLA_ERR_NULL_ARG;  // an E4M3 layer needs every row scale
  }
  if (!workspace) return MLA_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) % 256) return MLA_ERR_ALIGN;
  const StepLayout s = step_layout(dims, n_layers, num_splits);
  if (s.total == 0) return MLA_ERR_DIMS;
  if (workspace_bytes < s.total) return MLA_ERR_WORKSPACE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_step_mu);
  StepStreams* ss = nullptr;
  int rc = step_streams(dev, n_layers, &ss);
  if (rc) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  const size_t B = dims->batch, D = dims->d_model, e = elem_bytes(dims);
  const size_t layer_bytes = B * D * e;
  char* h_dev = ws + s.h;
  char* out_dev = ws + s.out;
  int32_t* pos_dev = reinterpret_cast<int32_t*>(ws + s.pos);
  int32_t* lens_dev = reinterpret_cast<int32_t*>(ws + s.lens);
  void* q_cat = ws + s.q_cat;
  float* o_lat = reinterpret_cast<float*>(ws + s.o_lat);
  float* lse = reinterpret_cast<float*>(ws + s.lse);
  void* o_heads = ws + s.o_heads;
  void* call_ws = ws + s.call;
  const size_t call_bytes = workspace_bytes - s.call;
  // the device buffers are free once everything already queued on `st` has run
  if ((rc = cuda_rc(cudaEventRecord(ss->start, st)))) return rc;
  if ((rc = cuda_rc(cudaStreamWaitEvent(ss->in, ss->start, 0)))) return rc;
  if ((rc = cuda_rc(cudaStreamWaitEvent(ss->out, ss->start, 0)))) return rc;
  if ((rc = cuda_rc(cudaMemcpyAsync(pos_dev, positions_host, B * 4, cudaMemcpyHostToDevice,
                                    ss->in))))
    return rc;
  if ((rc = cuda_rc(cudaMemcpyAsync(lens_dev, seq_lens_host, B * 4, cudaMemcpyHostToDevice,
                                    ss->in))))
    return rc;
  for (int l = 0; l < n_layers; ++l) {
    if ((rc = cuda_rc(cudaMemcpyAsync(h_dev + l * layer_bytes,
                                      static_cast<const char*>(h_host) + l * layer_bytes,
                                      layer_bytes, cudaMemcpyHostToDevice, ss->in))))
      return rc;
    if ((rc = cuda_rc(cudaEventRecord(ss->ev_in[l], ss->in)))) return rc;
  }
  for (int l = 0; l < n_layers; ++l) {
    const mla_layer& ly = layers[l];
    if ((rc = cuda_rc(cudaStreamWaitEvent(st, ss->ev_in[l], 0)))) return rc;
    void* hl = h_dev + l * layer_bytes;
    void* outl = out_dev + l * layer_bytes;
    const bool e4m3 = ly.w_q_scale != nullptr;
    rc = e4m3 ? mla_append_absorb_fp8(dims, hl, ly.w_dkv, ly.w_dkv_scale, ly.w_kr, ly.w_kr_scale,
                                      ly.w_q, ly.w_q_scale, ly.w_uk, pos_dev, ly.page_table,
                                      ly.max_pages, ly.cache_pool, ly.num_pages, q_cat, nullptr,
                                      call_ws, call_bytes, stream)
              : mla_append_absorb(dims, hl, ly.w_dkv, ly.w_kr, ly.w_q, ly.w_uk, pos_dev,
                                  ly.page_table, ly.max_pages, ly.cache_pool, ly.num_pages,
                                  q_cat, nullptr, call_ws, call_bytes, stream);
    if (rc) return rc;
    if ((rc = mla_decode_attn(dims, q_cat, nullptr, ly.cache_pool, ly.num_pages, ly.page_table,
                              ly.max_pages, lens_dev, 0.f, num_splits, call_ws, call_bytes,
                              o_lat, lse, stream)))
      return rc;
    rc = e4m3 ? mla_out_proj_fp8(dims, o_lat, ly.w_uv, ly.w_o, ly.w_o_scale, o_heads, outl,
                                 call_ws, call_bytes, stream)
              : mla_out_proj(dims, o_lat, ly.w_uv, ly.w_o, o_heads, outl, call_ws, call_bytes,
                             stream);
    if (rc) return rc;
    if ((rc = cuda_rc(cudaEventRecord(ss->ev_out[l], st)))) return rc;
    if ((rc = cuda_rc(cudaStreamWaitEvent(ss->out, ss->ev_out[l], 0)))) return rc;
    if ((rc = cuda_rc(cudaMemcpyAsync(static_cast<char*>(out_host) + l * layer_bytes, outl,
                                      layer_bytes, cudaMemcpyDeviceToHost, ss->out))))
      return rc;
  }
  if ((rc = cuda_rc(cudaEventRecord(ss->done, ss->out)))) return rc;
  return cuda_rc(cudaStreamWaitEvent(st, ss->done, 0));
}

}  // extern "C"
