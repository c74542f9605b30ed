// fake_cuda_runtime.cpp -- test infrastructure, host only.  Stands in for the
// CUDA runtime calls and the per-step entry points that the whole-layer
// forward (csrc/layer_fwd.cu) makes, so that file can be compiled unchanged
// into a host library and its stream/event ordering checked on a machine
// without a GPU.  Nothing is executed: every call appends one line to a log
// (kind, stream, events, and the device or host byte ranges it reads and
// writes), which tests/test_host_pipeline_order.py turns into the
// happens-before graph that CUDA's stream and event rules define.  A step or
// a copy can be made to fail on the host (fake_fail) to check the error paths.
#include <cuda_runtime.h>

#include <cstdio>
#include <string>
#include <vector>

#include "../include/gqe.h"

namespace gqe {
gqe_status layer_workspace_bytes(const gqe_dims* dims, bool host, size_t* bytes);
}

namespace {

std::vector<std::string> g_log;
long g_next_event = 1;
// host-side failure injection: the n-th step call returns g_fail_status, the
// n-th copy returns an error (-1: never)
int g_fail_step = -1, g_fail_status = 0, g_steps = 0;
int g_fail_copy = -1, g_copies = 0;

bool step_fails(gqe_status* st) {
  if (g_steps++ != g_fail_step) return false;
  *st = static_cast<gqe_status>(g_fail_status);
  return true;
}

std::string hex(const void* p) {
  char b[32];
  snprintf(b, sizeof b, "%lx", (unsigned long)(uintptr_t)p);
  return b;
}

std::string range(const void* p, size_t n) { return hex(p) + ":" + std::to_string(n); }

void log_line(const std::string& s) { g_log.push_back(s); }

// one kernel step: "kernel <stream> <name> r=<ranges> w=<ranges>"
void log_kernel(gqe_stream s, const char* name, const std::vector<std::string>& reads,
                const std::vector<std::string>& writes) {
  std::string line = std::string("kernel ") + hex(s) + " " + name + " r=";
  for (size_t i = 0; i < reads.size(); ++i) line += (i ? "," : "") + reads[i];
  line += " w=";
  for (size_t i = 0; i < writes.size(); ++i) line += (i ? "," : "") + writes[i];
  log_line(line);
}

size_t n_tok(const gqe_dims* d) { return (size_t)d->B * d->T; }

}  // namespace

extern "C" {

// ---- log access for the test
int fake_log_size() { return (int)g_log.size(); }
const char* fake_log_line(int i) { return g_log[i].c_str(); }
void fake_log_clear() {
  g_log.clear();
  g_steps = g_copies = 0;
}
void fake_fail(int step, int status, int copy) {
  g_fail_step = step;
  g_fail_status = status;
  g_fail_copy = copy;
}

// ---- CUDA runtime stand-ins
cudaError_t cudaEventCreateWithFlags(cudaEvent_t* e, unsigned int) {
  *e = reinterpret_cast<cudaEvent_t>(g_next_event++);
  log_line("create " + hex(*e));
  return cudaSuccess;
}
cudaError_t cudaEventDestroy(cudaEvent_t e) {
  log_line("destroy " + hex(e));
  return cudaSuccess;
}
cudaError_t cudaEventRecord(cudaEvent_t e, cudaStream_t s) {
  log_line("record " + hex(e) + " " + hex(s));
  return cudaSuccess;
}
cudaError_t cudaStreamWaitEvent(cudaStream_t s, cudaEvent_t e, unsigned int) {
  log_line("wait " + hex(s) + " " + hex(e));
  return cudaSuccess;
}
cudaError_t cudaMemcpyAsync(void* dst, const void* src, size_t n, enum cudaMemcpyKind kind, cudaStream_t s) {
  if (g_copies++ == g_fail_copy) return cudaErrorInvalidValue;
  log_line(std::string("copy ") + hex(s) + " " + (kind == cudaMemcpyHostToDevice ? "h2d" : "d2h") + " r=" +
           range(src, n) + " w=" + range(dst, n));
  return cudaSuccess;
}

// ---- the per-step entry points: the ranges each one reads and writes
gqe_status gqe_workspace_size(const gqe_dims* d, int op, int, size_t* bytes) {
  if (!d || !bytes || d->B < 1 || d->T < 1 || d->k < 1 || d->k > d->E || d->G < 1) return GQE_ERR_INVALID_ARG;
  const size_t N = n_tok(d);
  if (op == GQE_OP_ROUTED_QPROJ) {
    *bytes = N * d->G * d->k * 8 + 4096;   // permutation tables
    return GQE_OK;
  }
  if (op == GQE_OP_COMBINE_OUT_PROJ) {
    *bytes = N * d->d_head * 2;            // the weighted-sum slot
    return GQE_OK;
  }
  if (op == GQE_OP_LAYER_FORWARD || op == GQE_OP_LAYER_FORWARD_HOST)
    return gqe::layer_workspace_bytes(d, op == GQE_OP_LAYER_FORWARD_HOST, bytes);
  return GQE_ERR_INVALID_ARG;
}

gqe_status gqe_router_topk(const gqe_dims* d, const gqe_bf16* x, const gqe_bf16* Wr, const float*, int32_t* idx,
                           float* w, float*, gqe_stream s) {
  gqe_status st;
  if (step_fails(&st)) return st;
  const size_t N = n_tok(d), sel = N * d->G * d->k * 4;
  log_kernel(s, "router", {range(x, N * d->d_model * 2), range(Wr, 2)}, {range(idx, sel), range(w, sel)});
  return GQE_OK;
}

gqe_status gqe_routed_qproj(const gqe_dims* d, const gqe_bf16* x, const gqe_bf16* Wq, const gqe_bf16*,
                            const int32_t* idx, gqe_bf16* q, gqe_bf16* qs, int32_t*, void* ws, size_t ws_bytes,
                            gqe_stream s) {
  gqe_status st;
  if (step_fails(&st)) return st;
  const size_t N = n_tok(d);
  std::vector<std::string> w = {range(q, N * d->G * d->k * d->d_head * 2), range(ws, ws_bytes)};
  if (d->n_shared) w.push_back(range(qs, N * d->d_head * 2));
  log_kernel(s, "qproj", {range(x, N * d->d_model * 2), range(idx, N * d->G * d->k * 4), range(Wq, 2)}, w);
  return GQE_OK;
}

gqe_status gqe_kv_proj(const gqe_dims* d, const gqe_bf16* x, const gqe_bf16* Wk, const gqe_bf16*, gqe_bf16* K,
                       gqe_bf16* V, gqe_stream s) {
  gqe_status st;
  if (step_fails(&st)) return st;
  const size_t N = n_tok(d), kv = N * d->G * d->d_head * 2;
  log_kernel(s, "kv", {range(x, N * d->d_model * 2), range(Wk, 2)}, {range(K, kv), range(V, kv)});
  return GQE_OK;
}

gqe_status gqe_attn_prefill(const gqe_dims* d, const gqe_bf16* q, const gqe_bf16* qs, const gqe_bf16* K,
                            const gqe_bf16* V, gqe_bf16* o, gqe_bf16* os, float*, gqe_stream s) {
  gqe_status st;
  if (step_fails(&st)) return st;
  const size_t N = n_tok(d), kv = N * d->G * d->d_head * 2, qo = N * d->G * d->k * d->d_head * 2;
  std::vector<std::string> r = {range(q, qo), range(K, kv), range(V, kv)};
  std::vector<std::string> w = {range(o, qo)};
  if (d->n_shared) {
    r.push_back(range(qs, N * d->d_head * 2));
    w.push_back(range(os, N * d->d_head * 2));
  }
  log_kernel(s, "attn", r, w);
  return GQE_OK;
}

gqe_status gqe_combine_out_proj(const gqe_dims* d, const gqe_bf16* o, const gqe_bf16* os, const float* tw,
                                const gqe_bf16* Wo, gqe_bf16* y, void* ws, size_t ws_bytes, gqe_stream s) {
  gqe_status st;
  if (step_fails(&st)) return st;
  const size_t N = n_tok(d);
  std::vector<std::string> r = {range(o, N * d->G * d->k * d->d_head * 2), range(tw, N * d->G * d->k * 4),
                                range(Wo, 2)};
  if (d->n_shared) r.push_back(range(os, N * d->d_head * 2));
  log_kernel(s, "combine_out", r, {range(ws, ws_bytes), range(y, N * d->d_model * 2)});
  return GQE_OK;
}

}  // extern "C"
