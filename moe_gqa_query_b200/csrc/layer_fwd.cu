// layer_fwd.cu -- the whole prefill forward of a GQE layer behind one C-ABI
// call (gqe_layer_forward, device buffers) and its host-buffer form
// (gqe_layer_forward_host), which pipelines the host<->device copies of
// sequence chunks with the compute.  Both chain the per-step entry points of
// gqe_api.cu on the caller's streams; nothing here launches a kernel of its
// own, allocates device memory or synchronises.
#include <cuda_runtime.h>

#include "../../include/gqe.h"

namespace gqe {

namespace {

inline size_t up256(size_t n) { return (n + 255) & ~size_t(255); }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline cudaStream_t S(gqe_stream s) { return reinterpret_cast<cudaStream_t>(s); }

#define GQE_TRY(x)                 \
  do {                             \
    gqe_status _s = (x);           \
    if (_s != GQE_OK) return _s;   \
  } while (0)

// Byte offsets of one forward's intermediates inside its scratch.  Every
// region starts on a 256-byte boundary.
struct LayerLayout {
  size_t idx, tw, q, qs, K, V, o, os, ws_q, ws_o;
  size_t ws_q_bytes, ws_o_bytes, bytes;
};

gqe_status layer_layout(const gqe_dims* d, size_t base, LayerLayout* L) {
  size_t wq = 0, wo = 0;
  GQE_TRY(gqe_workspace_size(d, GQE_OP_ROUTED_QPROJ, 0, &wq));
  GQE_TRY(gqe_workspace_size(d, GQE_OP_COMBINE_OUT_PROJ, 0, &wo));
  const size_t N = (size_t)d->B * d->T, G = d->G, k = d->k, dh = d->d_head, sh = d->n_shared;
  size_t off = base;
  auto take = [&off](size_t n) {
    const size_t o = off;
    off += up256(n);
    return o;
  };
  L->idx = take(N * G * k * 4);      // top-k expert indices, int32 [N, G, k]
  L->tw = take(N * G * k * 4);       // renormalised weights, fp32 [N, G, k]
  L->q = take(N * G * k * dh * 2);   // routed queries [B, G, T, k, d]
  L->qs = take(N * sh * dh * 2);     // shared-head queries [B, T, d]
  L->K = take(N * G * dh * 2);       // [B, G, T, d]
  L->V = take(N * G * dh * 2);
  L->o = take(N * G * k * dh * 2);   // routed attention outputs [B, G, T, k, d]
  L->os = take(N * sh * dh * 2);     // shared-head output [B, T, d]
  L->ws_q = take(wq);
  L->ws_q_bytes = wq;
  L->ws_o = take(wo);
  L->ws_o_bytes = wo;
  L->bytes = off;
  return GQE_OK;
}

// Bytes of one of the host form's double-buffered x or y chunks.
inline size_t chunk_bytes(const gqe_dims* d) { return up256((size_t)d->B * d->T * d->d_model * 2); }

gqe_status check_weights(const gqe_dims* d, const gqe_layer_weights* w) {
  if (!w || !w->Wr || !w->Wq || !w->Wk || !w->Wv || !w->Wo) return GQE_ERR_INVALID_ARG;
  if (d->n_shared && !w->Wsh) return GQE_ERR_INVALID_ARG;
  if (!aligned16(w->Wq) || !aligned16(w->Wk) || !aligned16(w->Wv) || !aligned16(w->Wo)) return GQE_ERR_INVALID_ARG;
  if (d->n_shared && !aligned16(w->Wsh)) return GQE_ERR_INVALID_ARG;
  return GQE_OK;
}

// The five steps of the forward on one stream, intermediates at L's offsets.
gqe_status forward_steps(const gqe_dims* d, const gqe_layer_weights* w, const gqe_bf16* x, gqe_bf16* y,
                         uint8_t* ws, const LayerLayout& L, gqe_stream s) {
  int32_t* idx = reinterpret_cast<int32_t*>(ws + L.idx);
  float* tw = reinterpret_cast<float*>(ws + L.tw);
  gqe_bf16* q = reinterpret_cast<gqe_bf16*>(ws + L.q);
  gqe_bf16* qs = d->n_shared ? reinterpret_cast<gqe_bf16*>(ws + L.qs) : nullptr;
  gqe_bf16* K = reinterpret_cast<gqe_bf16*>(ws + L.K);
  gqe_bf16* V = reinterpret_cast<gqe_bf16*>(ws + L.V);
  gqe_bf16* o = reinterpret_cast<gqe_bf16*>(ws + L.o);
  gqe_bf16* os = d->n_shared ? reinterpret_cast<gqe_bf16*>(ws + L.os) : nullptr;
  GQE_TRY(gqe_router_topk(d, x, w->Wr, w->bias, idx, tw, nullptr, s));
  GQE_TRY(gqe_routed_qproj(d, x, w->Wq, w->Wsh, idx, q, qs, nullptr, ws + L.ws_q, L.ws_q_bytes, s));
  GQE_TRY(gqe_kv_proj(d, x, w->Wk, w->Wv, K, V, s));
  GQE_TRY(gqe_attn_prefill(d, q, qs, K, V, o, os, nullptr, s));
  return gqe_combine_out_proj(d, o, os, tw, w->Wo, y, ws + L.ws_o, L.ws_o_bytes, s);
}

}  // namespace

// Scratch of gqe_layer_forward (host = false) or of gqe_layer_forward_host
// for chunks of dims->B sequences (host = true: two x and two y chunk
// buffers in front of one forward's intermediates).
gqe_status layer_workspace_bytes(const gqe_dims* dims, bool host, size_t* bytes) {
  LayerLayout L;
  GQE_TRY(layer_layout(dims, host ? 4 * chunk_bytes(dims) : 0, &L));
  *bytes = L.bytes;
  return GQE_OK;
}

}  // namespace gqe

using namespace gqe;

extern "C" {

gqe_status gqe_layer_forward(const gqe_dims* dims, const gqe_layer_weights* w, const gqe_bf16* x, gqe_bf16* y,
                             void* ws, size_t ws_bytes, gqe_stream stream) {
  LayerLayout L;
  GQE_TRY(layer_layout(dims, 0, &L));     // also validates dims
  GQE_TRY(check_weights(dims, w));
  if (!x || !y || !aligned16(x) || !aligned16(y)) return GQE_ERR_INVALID_ARG;
  if (!ws || !aligned16(ws) || ws_bytes < L.bytes) return GQE_ERR_WORKSPACE;
  return forward_steps(dims, w, x, y, static_cast<uint8_t*>(ws), L, stream);
}

gqe_status gqe_layer_forward_host(const gqe_dims* dims, const gqe_layer_weights* w, const gqe_bf16* x_host,
                                  gqe_bf16* y_host, int chunk_seqs, void* ws, size_t ws_bytes,
                                  gqe_stream stream_in, gqe_stream stream_compute, gqe_stream stream_out) {
  size_t full = 0;
  GQE_TRY(gqe_workspace_size(dims, GQE_OP_LAYER_FORWARD, 0, &full));   // validates dims
  GQE_TRY(check_weights(dims, w));
  if (!x_host || !y_host || chunk_seqs < 1) return GQE_ERR_INVALID_ARG;
  gqe_dims cd = *dims;
  cd.B = chunk_seqs;
  size_t need = 0;
  GQE_TRY(layer_workspace_bytes(&cd, true, &need));
  if (!ws || !aligned16(ws) || ws_bytes < need) return GQE_ERR_WORKSPACE;

  uint8_t* base = static_cast<uint8_t*>(ws);
  const size_t cb = chunk_bytes(&cd);
  gqe_bf16* xd[2] = {reinterpret_cast<gqe_bf16*>(base), reinterpret_cast<gqe_bf16*>(base + cb)};
  gqe_bf16* yd[2] = {reinterpret_cast<gqe_bf16*>(base + 2 * cb), reinterpret_cast<gqe_bf16*>(base + 3 * cb)};
  const size_t seq_elems = (size_t)dims->T * dims->d_model;

  // e_in: chunk copied in; e_cmp[j] / e_out[j]: the last forward / copy-back
  // that used buffer slot j.  An event wait binds to the record made before
  // it, so re-recording an event for a later chunk leaves earlier waits as
  // they were.
  cudaEvent_t ev[5] = {nullptr, nullptr, nullptr, nullptr, nullptr};
  for (int i = 0; i < 5; ++i) {
    if (cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming) != cudaSuccess) {
      for (int j = 0; j < i; ++j) cudaEventDestroy(ev[j]);
      return GQE_ERR_CUDA;
    }
  }
  cudaEvent_t e_in = ev[0], e_cmp[2] = {ev[1], ev[2]}, e_out[2] = {ev[3], ev[4]};
  cudaStream_t s_in = S(stream_in), s_cmp = S(stream_compute), s_out = S(stream_out);

  gqe_status st = GQE_OK;
  const int n_chunks = (dims->B + chunk_seqs - 1) / chunk_seqs;
  int last = 0;
  for (int i = 0; i < n_chunks && st == GQE_OK; ++i) {
    const int j = i & 1;
    last = j;
    const int b0 = i * chunk_seqs;
    cd.B = dims->B - b0 < chunk_seqs ? dims->B - b0 : chunk_seqs;
    const size_t bytes = (size_t)cd.B * seq_elems * 2;
    LayerLayout L;
    st = layer_layout(&cd, 4 * cb, &L);
    if (st != GQE_OK) break;
    // copy in: x slot j is free once the forward of chunk i-2 is done
    if (i >= 2 && cudaStreamWaitEvent(s_in, e_cmp[j], 0) != cudaSuccess) { st = GQE_ERR_CUDA; break; }
    if (cudaMemcpyAsync(xd[j], x_host + (size_t)b0 * seq_elems, bytes, cudaMemcpyHostToDevice, s_in) != cudaSuccess ||
        cudaEventRecord(e_in, s_in) != cudaSuccess) { st = GQE_ERR_CUDA; break; }
    // forward: after its input landed and once y slot j was read back (chunk i-2)
    if (cudaStreamWaitEvent(s_cmp, e_in, 0) != cudaSuccess) { st = GQE_ERR_CUDA; break; }
    if (i >= 2 && cudaStreamWaitEvent(s_cmp, e_out[j], 0) != cudaSuccess) { st = GQE_ERR_CUDA; break; }
    st = forward_steps(&cd, w, xd[j], yd[j], base, L, stream_compute);
    if (st != GQE_OK) break;
    if (cudaEventRecord(e_cmp[j], s_cmp) != cudaSuccess) { st = GQE_ERR_CUDA; break; }
    // copy back
    if (cudaStreamWaitEvent(s_out, e_cmp[j], 0) != cudaSuccess ||
        cudaMemcpyAsync(y_host + (size_t)b0 * seq_elems, yd[j], bytes, cudaMemcpyDeviceToHost, s_out) != cudaSuccess ||
        cudaEventRecord(e_out[j], s_out) != cudaSuccess) { st = GQE_ERR_CUDA; break; }
  }
  if (st == GQE_OK) {
    // the next call's copies into the x slots wait for this call's last
    // forward; its forwards (which write the y slots) for the last copy-back
    if (cudaStreamWaitEvent(s_in, e_cmp[last], 0) != cudaSuccess ||
        cudaStreamWaitEvent(s_cmp, e_out[last], 0) != cudaSuccess)
      st = GQE_ERR_CUDA;
  }
  // released once the work recorded on them has completed
  for (int i = 0; i < 5; ++i) cudaEventDestroy(ev[i]);
  return st;
}

}  // extern "C"
