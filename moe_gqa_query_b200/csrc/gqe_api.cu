// gqe_api.cu -- the C ABI declared in include/gqe.h: argument validation,
// TMA descriptor construction and kernel launches.  Nothing here allocates or
// synchronises (except gqe_device_error, which is a synchronous query).
#include <math.h>
#include <string.h>

#include <mutex>

#include "../../include/gqe.h"
#include "attn.cuh"
#include "bwd.cuh"
#include "gemm.cuh"
#include "route.cuh"

using namespace gqe;

namespace {

// Device error word set by kernels whose internal waits run out of time.
__device__ unsigned int g_device_error = 0;

// Device address of g_device_error for the current device (looked up once per
// device; host code cannot take the address of a __device__ variable).
unsigned* error_word() {
  static unsigned* cache[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (!cache[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) == cudaSuccess) cache[dev] = static_cast<unsigned*>(p);
  }
  return cache[dev];
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Tensor map (bf16 unless `f32`), 128-byte swizzle, zero fill out of bounds.
// dims/box innermost first; strides in bytes for dims 1..rank-1.
bool encode_map(CUtensorMap* m, const void* ptr, int rank, const uint64_t* dims, const uint64_t* strides,
                const uint32_t* box, bool f32 = false) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gd[5], gs[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i < rank - 1; ++i) gs[i] = strides[i];
  memset(m, 0, sizeof(*m));
  CUresult r = fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(ptr), gd, gs, bx, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Encoded maps are cached (a layer call re-encodes the same few maps every
// step); a small direct-mapped table keyed by everything the encoding reads.
struct MapKey {
  const void* ptr;
  int rank;
  bool f32;
  uint64_t dims[3];
  uint32_t box[3];
  bool operator==(const MapKey& o) const {
    return ptr == o.ptr && rank == o.rank && f32 == o.f32 && !memcmp(dims, o.dims, sizeof(dims)) &&
           !memcmp(box, o.box, sizeof(box));
  }
};

bool make_map(CUtensorMap* m, const void* ptr, int rank, const uint64_t* dims, const uint64_t* strides,
              const uint32_t* box, bool f32 = false) {
  constexpr int kSlots = 256;
  static MapKey keys[kSlots];
  static CUtensorMap maps[kSlots];
  static bool used[kSlots];
  static std::mutex mu;
  MapKey k{};
  k.ptr = ptr;
  k.rank = rank;
  k.f32 = f32;
  for (int i = 0; i < rank && i < 3; ++i) {
    k.dims[i] = dims[i];
    k.box[i] = box[i];
  }
  uint64_t h = (reinterpret_cast<uintptr_t>(ptr) + (f32 ? 1 : 0)) * 0x9E3779B97F4A7C15ull;
  for (int i = 0; i < 3; ++i) h = (h ^ (k.dims[i] + 0x632BE5ABull * k.box[i])) * 0x100000001B3ull;
  const int slot = (int)(h >> 56);
  {
    std::lock_guard<std::mutex> lock(mu);
    if (used[slot] && keys[slot] == k) {
      *m = maps[slot];
      return true;
    }
  }
  if (!encode_map(m, ptr, rank, dims, strides, box, f32)) return false;
  std::lock_guard<std::mutex> lock(mu);
  keys[slot] = k;
  maps[slot] = *m;
  used[slot] = true;
  return true;
}

// fp32 [rows, cols], box 32 cols (128 bytes) x box_rows rows
bool map2d_f32(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t rows, uint32_t box_rows) {
  const uint64_t dims[2] = {cols, rows};
  const uint64_t strides[1] = {cols * 4};
  const uint32_t box[2] = {32, box_rows};
  return make_map(m, ptr, 2, dims, strides, box, true);
}

bool map2d(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t rows, uint32_t box_rows) {
  const uint64_t dims[2] = {cols, rows};
  const uint64_t strides[1] = {cols * 2};
  const uint32_t box[2] = {64, box_rows};
  return make_map(m, ptr, 2, dims, strides, box);
}

// [outer, rows, cols] contiguous, box 64 cols x box_rows rows x 1
bool map3d(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t rows, uint64_t outer, uint32_t box_rows) {
  const uint64_t dims[3] = {cols, rows, outer};
  const uint64_t strides[2] = {cols * 2, cols * rows * 2};
  const uint32_t box[3] = {64, box_rows, 1};
  return make_map(m, ptr, 3, dims, strides, box);
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

gqe_status check_dims(const gqe_dims* d) {
  if (!d) return GQE_ERR_INVALID_ARG;
  if (d->B < 1 || d->T < 1 || d->d_model < 1 || d->G < 1 || d->E < 1 || d->k < 1 || d->k > d->E)
    return GQE_ERR_INVALID_ARG;
  if (d->n_shared < 0 || d->n_shared > 1 || d->renorm_scope < 0 || d->renorm_scope > 2)
    return GQE_ERR_INVALID_ARG;
  if (d->output_mode < 0 || d->output_mode > 2) return GQE_ERR_INVALID_ARG;
  if (d->shared_kv_group < 0 || d->shared_kv_group >= d->G) return GQE_ERR_INVALID_ARG;
  if (!(d->scale >= 0.f) || isinf(d->scale)) return GQE_ERR_INVALID_ARG;
  if (d->d_head != 64 && d->d_head != 128) return GQE_ERR_UNSUPPORTED;
  if (d->E > 8 || d->G * d->E > 64) return GQE_ERR_UNSUPPORTED;
  if (d->d_model % 64 != 0) return GQE_ERR_UNSUPPORTED;
  const long long N = (long long)d->B * d->T;
  if (N * d->G * d->k * d->d_head >= (1ll << 31) || N * d->d_model >= (1ll << 31)) return GQE_ERR_UNSUPPORTED;
  return GQE_OK;
}

inline float scale_log2(const gqe_dims* d) {
  const float s = d->scale > 0.f ? d->scale : 1.0f / sqrtf((float)d->d_head);
  return s * 1.4426950408889634f;
}

inline cudaStream_t S(gqe_stream s) { return reinterpret_cast<cudaStream_t>(s); }
inline gqe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? GQE_OK : GQE_ERR_CUDA; }

#define GQE_CHECK(x)               \
  do {                             \
    gqe_status _s = (x);           \
    if (_s != GQE_OK) return _s;   \
  } while (0)
#define GQE_REQUIRE(c, code) \
  do {                       \
    if (!(c)) return code;   \
  } while (0)

}  // namespace

namespace gqe {

// Scratch of the whole-layer forward (layer_fwd.cu).
gqe_status layer_workspace_bytes(const gqe_dims* dims, bool host, size_t* bytes);

// Argument checks, tensor maps and parameters of a decode call, all but the
// partial-state scratch, which the caller attaches (gqe_attn_decode: the
// caller's workspace; gqe_attn_decode_noalloc in attn_decode.cu: the
// library's fixed array).
gqe_status decode_setup(const gqe_dims* dims, const gqe_bf16* q_routed, const gqe_bf16* q_sh, const gqe_bf16* Kc,
                        const gqe_bf16* Vc, int L_max, const int32_t* cache_len, gqe_bf16* o_routed,
                        gqe_bf16* o_sh, CUtensorMap* mK, CUtensorMap* mV, DecodeParams* p) {
  GQE_CHECK(check_dims(dims));
  GQE_REQUIRE(dims->T == 1 && L_max >= 1, GQE_ERR_INVALID_ARG);
  GQE_REQUIRE(q_routed && Kc && Vc && cache_len && o_routed, GQE_ERR_INVALID_ARG);
  GQE_REQUIRE(!dims->n_shared || (q_sh && o_sh), GQE_ERR_INVALID_ARG);
  GQE_REQUIRE(aligned16(q_routed) && aligned16(Kc) && aligned16(Vc), GQE_ERR_INVALID_ARG);
  GQE_REQUIRE(!dims->n_shared || aligned16(q_sh), GQE_ERR_INVALID_ARG);
  const int B = dims->B, G = dims->G, d = dims->d_head;
  GQE_REQUIRE(map3d(mK, Kc, d, L_max, (uint64_t)B * G, 64), GQE_ERR_CUDA);
  GQE_REQUIRE(map3d(mV, Vc, d, L_max, (uint64_t)B * G, 64), GQE_ERR_CUDA);
  *p = DecodeParams{};
  p->q_routed = q_routed;
  p->q_sh = q_sh;
  p->Kc = Kc;
  p->Vc = Vc;
  p->cache_len = cache_len;
  p->o_routed = o_routed;
  p->o_sh = o_sh;
  p->B = B;
  p->G = G;
  p->k = dims->k;
  p->d = d;
  p->n_shared = dims->n_shared;
  p->sg = dims->shared_kv_group;
  p->L_max = L_max;
  decode_split_plan(L_max, &p->chunk, &p->n_chunks);
  p->nq_max = dims->k + dims->n_shared;
  p->scale_log2 = scale_log2(dims);
  p->err = error_word();
  return GQE_OK;
}

}  // namespace gqe

extern "C" {

const char* gqe_status_string(gqe_status s) {
  switch (s) {
    case GQE_OK: return "ok";
    case GQE_ERR_INVALID_ARG: return "invalid argument";
    case GQE_ERR_UNSUPPORTED: return "unsupported shape";
    case GQE_ERR_WORKSPACE: return "workspace too small";
    case GQE_ERR_CUDA: return "CUDA error";
    case GQE_ERR_DEVICE_CHECK: return "device-side check failed";
  }
  return "unknown status";
}

gqe_status gqe_workspace_size(const gqe_dims* dims, int op, int L_max, size_t* bytes) {
  GQE_CHECK(check_dims(dims));
  GQE_REQUIRE(bytes, GQE_ERR_INVALID_ARG);
  const int N = dims->B * dims->T;
  if (op == GQE_OP_ROUTED_QPROJ) {
    *bytes = perm_layout(N, dims->G, dims->E, dims->k).bytes;
    return GQE_OK;
  }
  if (op == GQE_OP_COMBINE_OUT_PROJ) {
    const size_t slots = (size_t)dims->k * dims->G + (dims->output_mode == 0 ? 1 : 0) + dims->n_shared;
    *bytes = (size_t)N * slots * dims->d_head * 2;
    return GQE_OK;
  }
  if (op == GQE_OP_ATTN_BWD) {
    AttnBwdLayout L;
    attn_bwd_layout(dims->B, dims->T, dims->G, dims->k, dims->n_shared, dims->d_head, &L);
    *bytes = L.bytes;
    return GQE_OK;
  }
  if (op == GQE_OP_ATTN_DECODE) {
    GQE_REQUIRE(L_max >= 1, GQE_ERR_INVALID_ARG);
    *bytes = decode_workspace_bytes(dims->B, dims->G, dims->k, dims->d_head, dims->n_shared, L_max);
    return GQE_OK;
  }
  if (op == GQE_OP_LAYER_FORWARD || op == GQE_OP_LAYER_FORWARD_HOST)
    return layer_workspace_bytes(dims, op == GQE_OP_LAYER_FORWARD_HOST, bytes);
  return GQE_ERR_INVALID_ARG;
}

gqe_status gqe_router_topk(const gqe_dims* dims, const gqe_bf16* x, const gqe_bf16* Wr, const float* bias,
                           int32_t* topk_idx, float* topk_w, float* probs, gqe_stream stream) {
  GQE_CHECK(check_dims(dims));
  GQE_REQUIRE(x && Wr && topk_idx && topk_w, GQE_ERR_INVALID_ARG);
  GQE_REQUIRE(aligned16(x), GQE_ERR_INVALID_ARG);
  RouterParams p{};
  p.x = x;
  p.Wr = Wr;
  p.bias = bias;
  p.topk_idx = topk_idx;
  p.topk_w = topk_w;
  p.probs = probs;
  p.N = dims->B * dims->T;
  p.D = dims->d_model;
  p.G = dims->G;
  p.E = dims->E;
  p.k = dims->k;
  p.scope = dims->renorm_scope;
  p.err = error_word();
  // tcgen05 router with x and Wr streamed by TMA for prefill-sized batches
  // (Wr rows must be 16-byte strided: G*E a multiple of 8)
  const int GE = p.G * p.E;
  if (p.N >= 1024 && p.D % 64 == 0 && GE % 8 == 0 && GE <= 64 && aligned16(Wr)) {
    const int R = router_tc_tile_rows(p.N);
    CUtensorMap mX, mW;
    if (map2d(&mX, x, p.D, p.N, R) && map2d(&mW, Wr, GE, p.D, 64)) {
      const cudaError_t e = launch_router_tc(mX, mW, p, R, S(stream));
      if (e != cudaErrorNotSupported) return cuda_status(e);
    }
  }
  return cuda_status(launch_router(p, S(stream)));
}

gqe_status gqe_router_stats(const gqe_dims* dims, const float* probs, const int32_t* topk_idx, int32_t* counts,
                            float* prob_sum, gqe_stream stream) {
  GQE_CHECK(check_dims(dims));
  GQE_REQUIRE(probs && topk_idx && counts && prob_sum, GQE_ERR_INVALID_ARG);
  return cuda_status(launch_router_stats(probs, topk_idx, dims->B * dims->T, dims->G, dims->E, dims->k, counts,
                                         prob_sum, S(stream)));
}

gqe_status gqe_routed_qproj(const gqe_dims* dims, const gqe_bf16* x, const gqe_bf16* Wq, const gqe_bf16* Wsh,
                            const int32_t* topk_idx, gqe_bf16* q_routed, gqe_bf16* q_sh, int32_t* expert_counts,
                            void* ws, size_t ws_bytes, gqe_stream stream) {
  GQE_CHECK(check_dims(dims));
  GQE_REQUIRE(x && Wq && topk_idx && q_routed, GQE_ERR_INVALID_ARG);
  GQE_REQUIRE(!dims->n_shared || (Wsh && q_sh), GQE_ERR_INVALID_ARG);
  GQE_REQUIRE(aligned16(x) && aligned16(Wq) && aligned16(q_routed), GQE_ERR_INVALID_ARG);
  GQE_REQUIRE(!dims->n_shared || (aligned16(Wsh) && aligned16(q_sh)), GQE_ERR_INVALID_ARG);
  const int N = dims->B * dims->T, G = dims->G, E = dims->E, k = dims->k, d = dims->d_head, D = dims->d_model;
  const PermLayout L = perm_layout(N, G, E, k);
  GQE_REQUIRE(ws && aligned16(ws), GQE_ERR_WORKSPACE);
  GQE_REQUIRE(ws_bytes >= L.bytes, GQE_ERR_WORKSPACE);

  cudaError_t e = launch_permutation(topk_idx, N, dims->T, G, E, k, ws, L, S(stream));
  if (e != cudaSuccess) return GQE_ERR_CUDA;

  CUtensorMap mWq, mWsh;
  GQE_REQUIRE(map2d(&mWq, Wq, D, (uint64_t)G * E * d, d), GQE_ERR_CUDA);
  if (dims->n_shared) GQE_REQUIRE(map2d(&mWsh, Wsh, D, d, d), GQE_ERR_CUDA);
  else mWsh = mWq;

  uint8_t* w = static_cast<uint8_t*>(ws);
  RoutedParams rp{};
  rp.src_row = reinterpret_cast<const int*>(w + L.off_src_row);
  rp.dst_row = reinterpret_cast<const int*>(w + L.off_dst_row);
  rp.seg_cnt = reinterpret_cast<const int*>(w + L.off_seg_cnt);
  rp.expert_counts = expert_counts;
  rp.seg_cap = L.cap;
  rp.n_seg = G * E;
  rp.max_routed_tiles = (int)(((long long)N * G * k) / 128) + G * E;
  rp.n_tokens = N;
  rp.K = D;
  rp.d = d;
  EpiParams epr{};
  epr.out0 = q_routed;
  epr.mode = kEpiRows;
  epr.ldo = d;
  epr.n_limit = d;
  epr.err = error_word();
  EpiParams eps = epr;
  eps.out0 = q_sh;
  rp.shared_tiles = dims->n_shared ? (N + 127) / 128 : 0;
  return cuda_status(launch_gemm_routed(mWq, mWsh, x, rp, epr, eps, S(stream)));
}

// CTA-pair GEMM (256 x 256 tiles) when the weights tile by 256 and there are
// enough rows to fill the pairs; single-CTA 128-row tiles otherwise.  (256 x
// 128 pair tiles fill the last wave better on 64 x 16 x 1024 shapes but ran
// 1.4x slower on B200: the k-block pipeline, not the tile count, bounds them.)
// Returns the pair tile width, 0 for the single-CTA kernel.
#ifndef GQE_GEMM_PAIR
#define GQE_GEMM_PAIR 1
#endif
static int pair_tile_n(int M, int n_per_weight) {
  return (GQE_GEMM_PAIR && M >= 2048 && n_per_weight % 256 == 0) ? 256 : 0;
}

static gqe_status kv_common(const gqe_dims* dims, const gqe_bf16* x, const gqe_bf16* Wk, const gqe_bf16* Wv,
                            EpiParams& ep, int M, gqe_stream stream) {
  const int G = dims->G, d = dims->d_head, D = dims->d_model;
  const int pbn = pair_tile_n(M, G * d);
  const int bn = pbn ? pbn : dense_tile_n(G * d, M);
  CUtensorMap mA, mK, mV;
  GQE_REQUIRE(map2d(&mA, x, D, M, 128), GQE_ERR_CUDA);
  GQE_REQUIRE(map2d(&mK, Wk, D, (uint64_t)G * d, pbn ? pbn / 2 : bn), GQE_ERR_CUDA);
  GQE_REQUIRE(map2d(&mV, Wv, D, (uint64_t)G * d, pbn ? pbn / 2 : bn), GQE_ERR_CUDA);
  ep.n_limit = G * d;
  ep.G = G;
  ep.d = d;
  ep.err = error_word();
  // head-layout output through TMA stores when 32-row groups stay inside one sequence
  CUtensorMap mOK{}, mOV{};
  ep.store_mode = kStorePerThread;
  if (ep.mode == kEpiHeads && ep.T % 32 == 0) {
    GQE_REQUIRE(map3d(&mOK, ep.out0, d, ep.T, (uint64_t)(M / ep.T) * G, 32), GQE_ERR_CUDA);
    GQE_REQUIRE(map3d(&mOV, ep.out1, d, ep.T, (uint64_t)(M / ep.T) * G, 32), GQE_ERR_CUDA);
    ep.store_mode = kStoreTmaHeads;
  }
  const int nt = (G * d + bn - 1) / bn;
  if (pbn)
    return cuda_status(launch_gemm_dense_pair(mA, mA, mA, ASource{kASingle, 0, 0, 0, 0, 0}, mK, mV, mOK, mOV, ep, M, D, nt,
                                              2 * nt, pbn, S(stream)));
  return cuda_status(launch_gemm_dense(mA, mK, mV, mOK, mOV, ep, M, D, nt, 2 * nt, bn, S(stream)));
}

gqe_status gqe_kv_proj(const gqe_dims* dims, const gqe_bf16* x, const gqe_bf16* Wk, const gqe_bf16* Wv,
                       gqe_bf16* K, gqe_bf16* V, gqe_stream stream) {
  GQE_CHECK(check_dims(dims));
  GQE_REQUIRE(x && Wk && Wv && K && V, GQE_ERR_INVALID_ARG);
  GQE_REQUIRE(aligned16(x) && aligned16(Wk) && aligned16(Wv) && aligned16(K) && aligned16(V), GQE_ERR_INVALID_ARG);
  EpiParams ep{};
  ep.out0 = K;
  ep.out1 = V;
  ep.mode = kEpiHeads;
  ep.T = dims->T;
  return kv_common(dims, x, Wk, Wv, ep, dims->B * dims->T, stream);
}

gqe_status gqe_kv_append(const gqe_dims* dims, const gqe_bf16* x, const gqe_bf16* Wk, const gqe_bf16* Wv,
                         gqe_bf16* Kc, gqe_bf16* Vc, int L_max, const int32_t* cache_len, gqe_stream stream) {
  GQE_CHECK(check_dims(dims));
  GQE_REQUIRE(dims->T == 1 && L_max >= 1, GQE_ERR_INVALID_ARG);
  GQE_REQUIRE(x && Wk && Wv && Kc && Vc && cache_len, GQE_ERR_INVALID_ARG);
  GQE_REQUIRE(aligned16(x) && aligned16(Wk) && aligned16(Wv) && aligned16(Kc) && aligned16(Vc), GQE_ERR_INVALID_ARG);
  EpiParams ep{};
  ep.out0 = Kc;
  ep.out1 = Vc;
  ep.mode = kEpiCacheRow;
  ep.cache_len = cache_len;
  ep.L_max = L_max;
  ep.T = 1;
  return kv_common(dims, x, Wk, Wv, ep, dims->B, stream);
}

gqe_status gqe_attn_prefill(const gqe_dims* dims, const gqe_bf16* q_routed, const gqe_bf16* q_sh,
                            const gqe_bf16* K, const gqe_bf16* V, gqe_bf16* o_routed, gqe_bf16* o_sh, float* lse,
                            gqe_stream stream) {
  GQE_CHECK(check_dims(dims));
  GQE_REQUIRE(q_routed && K && V && o_routed, GQE_ERR_INVALID_ARG);
  GQE_REQUIRE(!dims->n_shared || (q_sh && o_sh), GQE_ERR_INVALID_ARG);
  GQE_REQUIRE(aligned16(q_routed) && aligned16(K) && aligned16(V) && aligned16(o_routed), GQE_ERR_INVALID_ARG);
  GQE_REQUIRE(!dims->n_shared || (aligned16(q_sh) && aligned16(o_sh)), GQE_ERR_INVALID_ARG);
  const int B = dims->B, T = dims->T, G = dims->G, k = dims->k, d = dims->d_head;
  CUtensorMap mQ, mQs, mK, mV;
  GQE_REQUIRE(map3d(&mQ, q_routed, d, (uint64_t)T * k, (uint64_t)B * G, 128), GQE_ERR_CUDA);
  if (dims->n_shared) GQE_REQUIRE(map3d(&mQs, q_sh, d, T, B, 128), GQE_ERR_CUDA);
  else mQs = mQ;
  GQE_REQUIRE(map3d(&mK, K, d, T, (uint64_t)B * G, 128), GQE_ERR_CUDA);
  GQE_REQUIRE(map3d(&mV, V, d, T, (uint64_t)B * G, 128), GQE_ERR_CUDA);
  AttnParams p{};
  p.o_routed = o_routed;
  p.o_sh = o_sh;
  p.lse = lse;
  p.B = B;
  p.T = T;
  p.G = G;
  p.k = k;
  p.n_shared = dims->n_shared;
  p.sg = dims->shared_kv_group;
  p.scale_log2 = scale_log2(dims);
  p.err = error_word();
  return cuda_status(launch_attn_prefill(mQ, mQs, mK, mV, p, d, S(stream)));
}

gqe_status gqe_attn_prefill_bwd(const gqe_dims* dims, const gqe_bf16* q_routed, const gqe_bf16* q_sh,
                                const gqe_bf16* K, const gqe_bf16* V, const gqe_bf16* o_routed,
                                const gqe_bf16* o_sh, const float* lse, const gqe_bf16* do_routed,
                                const gqe_bf16* do_sh, gqe_bf16* dq_routed, gqe_bf16* dq_sh, gqe_bf16* dK,
                                gqe_bf16* dV, void* ws, size_t ws_bytes, gqe_stream stream) {
  GQE_CHECK(check_dims(dims));
  GQE_REQUIRE(q_routed && K && V && o_routed && lse && do_routed && dq_routed && dK && dV, GQE_ERR_INVALID_ARG);
  GQE_REQUIRE(!dims->n_shared || (q_sh && o_sh && do_sh && dq_sh), GQE_ERR_INVALID_ARG);
  const void* ptrs[] = {q_routed, K, V, o_routed, do_routed, dq_routed, dK, dV, lse};
  for (const void* q : ptrs) GQE_REQUIRE(aligned16(q), GQE_ERR_INVALID_ARG);
  if (dims->n_shared) {
    const void* sp[] = {q_sh, o_sh, do_sh, dq_sh};
    for (const void* q : sp) GQE_REQUIRE(aligned16(q), GQE_ERR_INVALID_ARG);
  }
  const int B = dims->B, T = dims->T, G = dims->G, k = dims->k, d = dims->d_head;
  AttnBwdLayout L;
  attn_bwd_layout(B, T, G, k, dims->n_shared, d, &L);
  GQE_REQUIRE(ws && (reinterpret_cast<uintptr_t>(ws) & 255u) == 0 && ws_bytes >= L.bytes, GQE_ERR_WORKSPACE);
  uint8_t* w = static_cast<uint8_t*>(ws);
  CUtensorMap mQ, mQs, mdO, mdOs, mK, mV, mdQ;
  GQE_REQUIRE(map3d(&mQ, q_routed, d, (uint64_t)T * k, (uint64_t)B * G, 128), GQE_ERR_CUDA);
  GQE_REQUIRE(map3d(&mdO, do_routed, d, (uint64_t)T * k, (uint64_t)B * G, 128), GQE_ERR_CUDA);
  if (dims->n_shared) {
    GQE_REQUIRE(map3d(&mQs, q_sh, d, T, B, 128), GQE_ERR_CUDA);
    GQE_REQUIRE(map3d(&mdOs, do_sh, d, T, B, 128), GQE_ERR_CUDA);
  } else {
    mQs = mQ;
    mdOs = mdO;
  }
  GQE_REQUIRE(map3d(&mK, K, d, T, (uint64_t)B * G, 128), GQE_ERR_CUDA);
  GQE_REQUIRE(map3d(&mV, V, d, T, (uint64_t)B * G, 128), GQE_ERR_CUDA);
  float* dq_acc = reinterpret_cast<float*>(w + L.off_dq);
  GQE_REQUIRE(map2d_f32(&mdQ, dq_acc, d, (uint64_t)L.n_rows_pad, 32), GQE_ERR_CUDA);
  AttnBwdParams p{};
  p.lse = lse;
  p.o_routed = o_routed;
  p.o_sh = o_sh;
  p.do_routed = do_routed;
  p.do_sh = do_sh;
  p.lse2 = reinterpret_cast<float*>(w + L.off_lse2);
  p.delta = reinterpret_cast<float*>(w + L.off_delta);
  p.dq_acc = dq_acc;
  p.dq_routed = dq_routed;
  p.dq_sh = dq_sh;
  p.dK = dK;
  p.dV = dV;
  p.B = B;
  p.T = T;
  p.G = G;
  p.k = k;
  p.n_shared = dims->n_shared;
  p.sg = dims->shared_kv_group;
  p.d = d;
  p.rows_pad = L.rows_pad;
  p.rows_pad_sh = L.rows_pad_sh;
  p.n_rows_pad = L.n_rows_pad;
  p.scale_log2 = scale_log2(dims);
  p.scale = p.scale_log2 / 1.4426950408889634f;
  p.err = error_word();
  return cuda_status(launch_attn_bwd(mQ, mQs, mdO, mdOs, mK, mV, mdQ, p, S(stream)));
}

gqe_status gqe_attn_decode(const gqe_dims* dims, const gqe_bf16* q_routed, const gqe_bf16* q_sh, const gqe_bf16* Kc,
                           const gqe_bf16* Vc, int L_max, const int32_t* cache_len, gqe_bf16* o_routed,
                           gqe_bf16* o_sh, void* ws, size_t ws_bytes, gqe_stream stream) {
  CUtensorMap mK, mV;
  DecodeParams p;
  GQE_CHECK(decode_setup(dims, q_routed, q_sh, Kc, Vc, L_max, cache_len, o_routed, o_sh, &mK, &mV, &p));
  const size_t need = decode_workspace_bytes(p.B, p.G, p.k, p.d, p.n_shared, L_max);
  GQE_REQUIRE(ws && aligned16(ws) && ws_bytes >= need, GQE_ERR_WORKSPACE);
  p.part = static_cast<float*>(ws);
  return cuda_status(launch_attn_decode_maps(mK, mV, p, S(stream)));
}

gqe_status gqe_combine(const gqe_dims* dims, const gqe_bf16* o_routed, const gqe_bf16* o_sh, const float* topk_w,
                       gqe_bf16* h, gqe_stream stream) {
  GQE_CHECK(check_dims(dims));
  GQE_REQUIRE(o_routed && topk_w && h, GQE_ERR_INVALID_ARG);
  GQE_REQUIRE(!dims->n_shared || o_sh, GQE_ERR_INVALID_ARG);
  GQE_REQUIRE(aligned16(o_routed) && aligned16(h) && (!dims->n_shared || aligned16(o_sh)), GQE_ERR_INVALID_ARG);
  CombineParams p{};
  p.o_routed = o_routed;
  p.o_sh = o_sh;
  p.w = topk_w;
  p.h = h;
  p.B = dims->B;
  p.T = dims->T;
  p.G = dims->G;
  p.k = dims->k;
  p.d = dims->d_head;
  p.n_shared = dims->n_shared;
  p.output_mode = dims->output_mode;
  return cuda_status(launch_combine(p, S(stream)));
}

gqe_status gqe_combine_out_proj(const gqe_dims* dims, const gqe_bf16* o_routed, const gqe_bf16* o_sh,
                                const float* topk_w, const gqe_bf16* Wo, gqe_bf16* y, void* ws, size_t ws_bytes,
                                gqe_stream stream) {
  GQE_CHECK(check_dims(dims));
  GQE_REQUIRE(o_routed && topk_w && Wo && y, GQE_ERR_INVALID_ARG);
  GQE_REQUIRE(!dims->n_shared || o_sh, GQE_ERR_INVALID_ARG);
  GQE_REQUIRE(aligned16(o_routed) && aligned16(Wo) && aligned16(y) && (!dims->n_shared || aligned16(o_sh)),
              GQE_ERR_INVALID_ARG);
  const int B = dims->B, T = dims->T, G = dims->G, k = dims->k, d = dims->d_head, D = dims->d_model;
  const int N = B * T;
  const int has_route = dims->output_mode == 0 ? 1 : 0;
  const int slots = k * G + has_route + dims->n_shared;
  const int Kdim = slots * d;
  size_t need = 0;
  GQE_CHECK(gqe_workspace_size(dims, GQE_OP_COMBINE_OUT_PROJ, 0, &need));
  GQE_REQUIRE(ws && aligned16(ws), GQE_ERR_WORKSPACE);
  GQE_REQUIRE(ws_bytes >= need, GQE_ERR_WORKSPACE);
  gqe_bf16* h = static_cast<gqe_bf16*>(ws);
  // without h: the hard slots come from o_routed in 128-token boxes (T % 128),
  // only the weighted-sum slot is written (into ws)
  // (the weighted hard slots of output_mode 2 are built in h)
  const bool direct = (T % 128 == 0) && pair_tile_n(N, D) == 256 && dims->output_mode != 2;
  CombineParams cp{};
  cp.o_routed = o_routed;
  cp.o_sh = o_sh;
  cp.w = topk_w;
  cp.h = h;
  cp.B = B;
  cp.T = T;
  cp.G = G;
  cp.k = k;
  cp.d = d;
  cp.n_shared = dims->n_shared;
  cp.route_only = direct ? 1 : 0;
  cp.output_mode = dims->output_mode;
  if (!direct || has_route) {     // direct without a weighted-sum slot needs no combine pass
    cudaError_t e = launch_combine(cp, S(stream));
    if (e != cudaSuccess) return GQE_ERR_CUDA;
  }
  if (!direct) return gqe_linear(N, D, Kdim, h, Wo, y, stream);
  CUtensorMap mO, mR, mS, mW, mY;
  GQE_REQUIRE(map2d(&mO, o_routed, (uint64_t)k * d, (uint64_t)B * G * T, 128), GQE_ERR_CUDA);
  GQE_REQUIRE(map2d(&mR, h, d, N, 128), GQE_ERR_CUDA);
  if (dims->n_shared) GQE_REQUIRE(map2d(&mS, o_sh, d, N, 128), GQE_ERR_CUDA);
  else mS = mR;
  GQE_REQUIRE(map2d(&mW, Wo, Kdim, D, 128), GQE_ERR_CUDA);
  GQE_REQUIRE(map2d(&mY, y, D, N, 32), GQE_ERR_CUDA);
  EpiParams ep{};
  ep.out0 = y;
  ep.out1 = y;
  ep.mode = kEpiRowMajor;
  ep.ldo = D;
  ep.n_limit = D;
  ep.err = error_word();
  ep.store_mode = kStoreTma2d;
  const int nt = D / 256;
  return cuda_status(launch_gemm_dense_pair(mO, mR, mS, ASource{kASlots, k, G, T, d, has_route}, mW, mW, mY, mY, ep, N, Kdim,
                                            nt, nt, 256, S(stream)));
}

gqe_status gqe_linear(int M, int N, int K, const gqe_bf16* A, const gqe_bf16* W, gqe_bf16* C, gqe_stream stream) {
  GQE_REQUIRE(M >= 1 && N >= 1 && K >= 1, GQE_ERR_INVALID_ARG);
  GQE_REQUIRE(A && W && C, GQE_ERR_INVALID_ARG);
  GQE_REQUIRE(K % 64 == 0 && N % 64 == 0, GQE_ERR_UNSUPPORTED);
  GQE_REQUIRE((long long)M * N < (1ll << 31) && (long long)M * K < (1ll << 31), GQE_ERR_UNSUPPORTED);
  GQE_REQUIRE(aligned16(A) && aligned16(W) && aligned16(C), GQE_ERR_INVALID_ARG);
  const int pbn = pair_tile_n(M, N);
  const int bn = pbn ? pbn : dense_tile_n(N, M);
  CUtensorMap mA, mW;
  GQE_REQUIRE(map2d(&mA, A, K, M, 128), GQE_ERR_CUDA);
  GQE_REQUIRE(map2d(&mW, W, K, N, pbn ? pbn / 2 : bn), GQE_ERR_CUDA);
  EpiParams ep{};
  ep.out0 = C;
  ep.out1 = C;
  ep.mode = kEpiRowMajor;
  ep.ldo = N;
  ep.n_limit = N;
  ep.err = error_word();
  CUtensorMap mO;
  GQE_REQUIRE(map2d(&mO, C, N, M, 32), GQE_ERR_CUDA);
  ep.store_mode = kStoreTma2d;
  const int nt = (N + bn - 1) / bn;
  if (pbn)
    return cuda_status(launch_gemm_dense_pair(mA, mA, mA, ASource{kASingle, 0, 0, 0, 0, 0}, mW, mW, mO, mO, ep, M, K, nt,
                                              nt, pbn, S(stream)));
  return cuda_status(launch_gemm_dense(mA, mW, mW, mO, mO, ep, M, K, nt, nt, bn, S(stream)));
}

gqe_status gqe_gemm_acc(int M, int N, int K, const gqe_bf16* A, int a_kn, const gqe_bf16* B, int b_kn, float* C,
                        int accumulate, gqe_stream stream) {
  GQE_REQUIRE(M >= 1 && N >= 1 && K >= 1, GQE_ERR_INVALID_ARG);
  GQE_REQUIRE(A && B && C && (a_kn == 0 || a_kn == 1) && (b_kn == 0 || b_kn == 1), GQE_ERR_INVALID_ARG);
  GQE_REQUIRE(N % 64 == 0, GQE_ERR_UNSUPPORTED);
  GQE_REQUIRE((a_kn ? M : K) % 8 == 0 && (b_kn ? N : K) % 8 == 0, GQE_ERR_UNSUPPORTED);
  GQE_REQUIRE((long long)M * N < (1ll << 31) && (long long)M * K < (1ll << 31) && (long long)N * K < (1ll << 31),
              GQE_ERR_UNSUPPORTED);
  GQE_REQUIRE(aligned16(A) && aligned16(B) && aligned16(C), GQE_ERR_INVALID_ARG);
  const int Kp = (K + 63) / 64 * 64;
  const int pbn = pair_tile_n(M, N);
  const int bn = pbn ? pbn : dense_tile_n(N, M);
  CUtensorMap mA, mW, mO;
  if (a_kn) GQE_REQUIRE(map2d(&mA, A, M, K, 64), GQE_ERR_CUDA);
  else GQE_REQUIRE(map2d(&mA, A, K, M, 128), GQE_ERR_CUDA);
  if (b_kn) GQE_REQUIRE(map2d(&mW, B, N, K, 64), GQE_ERR_CUDA);
  else GQE_REQUIRE(map2d(&mW, B, K, N, pbn ? pbn / 2 : bn), GQE_ERR_CUDA);
  GQE_REQUIRE(map2d_f32(&mO, C, N, M, 32), GQE_ERR_CUDA);
  const int nt = (N + bn - 1) / bn;
  // split K so that the output tiles times the slices fill the SMs once
  const int tiles = pbn ? ((M + 255) / 256) * nt : ((M + 127) / 128) * nt;
  const int slots = pbn ? num_sms() / 2 : num_sms();
  int ksplit = tiles >= slots ? 1 : slots / tiles;
  if (ksplit > Kp / 64) ksplit = Kp / 64;
  if (ksplit > 16) ksplit = 16;
  EpiParams ep{};
  ep.mode = kEpiRowMajor;
  ep.ldo = N;
  ep.n_limit = N;
  ep.err = error_word();
  ep.store_mode = kStoreReduceF32;
  ep.ksplit = ksplit;
  if (!accumulate && cudaMemsetAsync(C, 0, (size_t)M * N * sizeof(float), S(stream)) != cudaSuccess)
    return GQE_ERR_CUDA;
  const int mn = (a_kn ? 1 : 0) | (b_kn ? 2 : 0);
  if (pbn)
    return cuda_status(launch_gemm_dense_pair(mA, mA, mA, ASource{kASingle, 0, 0, 0, 0, 0}, mW, mW, mO, mO, ep, M, Kp,
                                              nt, nt, pbn, S(stream), mn));
  return cuda_status(launch_gemm_dense(mA, mW, mW, mO, mO, ep, M, Kp, nt, nt, bn, S(stream), mn));
}

gqe_status gqe_combine_bwd(const gqe_dims* dims, const gqe_bf16* o_routed, const gqe_bf16* o_sh,
                           const float* topk_w, const gqe_bf16* dh, gqe_bf16* do_routed, gqe_bf16* do_sh,
                           float* dtopk_w, gqe_stream stream) {
  GQE_CHECK(check_dims(dims));
  (void)o_sh;
  GQE_REQUIRE(o_routed && topk_w && dh && do_routed && dtopk_w, GQE_ERR_INVALID_ARG);
  GQE_REQUIRE(!dims->n_shared || do_sh, GQE_ERR_INVALID_ARG);
  GQE_REQUIRE(aligned16(o_routed) && aligned16(dh) && aligned16(do_routed), GQE_ERR_INVALID_ARG);
  CombineBwdParams p{};
  p.o_routed = o_routed;
  p.w = topk_w;
  p.dh = dh;
  p.do_routed = do_routed;
  p.do_sh = do_sh;
  p.dw = dtopk_w;
  p.B = dims->B;
  p.T = dims->T;
  p.G = dims->G;
  p.k = dims->k;
  p.d = dims->d_head;
  p.n_shared = dims->n_shared;
  p.output_mode = dims->output_mode;
  p.slots = dims->k * dims->G + (dims->output_mode == 0 ? 1 : 0) + dims->n_shared;
  return cuda_status(launch_combine_bwd(p, S(stream)));
}

gqe_status gqe_router_bwd(const gqe_dims* dims, const float* probs, const int32_t* topk_idx, const float* topk_w,
                          const float* dtopk_w, float* dlogits, float* dbias, gqe_stream stream) {
  GQE_CHECK(check_dims(dims));
  GQE_REQUIRE(probs && topk_idx && topk_w && dtopk_w && dlogits, GQE_ERR_INVALID_ARG);
  RouterBwdParams p{};
  p.probs = probs;
  p.idx = topk_idx;
  p.w = topk_w;
  p.dw = dtopk_w;
  p.dlogits = dlogits;
  p.dbias = dbias;
  p.N = dims->B * dims->T;
  p.G = dims->G;
  p.E = dims->E;
  p.k = dims->k;
  p.scope = dims->renorm_scope;
  return cuda_status(launch_router_bwd(p, S(stream)));
}

gqe_status gqe_bwd_pack_cols(const gqe_dims* dims, int* cols) {
  GQE_CHECK(check_dims(dims));
  GQE_REQUIRE(cols, GQE_ERR_INVALID_ARG);
  *cols = bwd_pack_cols(dims->G, dims->E, dims->d_head, dims->n_shared);
  return GQE_OK;
}

gqe_status gqe_bwd_pack(const gqe_dims* dims, const int32_t* topk_idx, const gqe_bf16* dq_routed,
                        const gqe_bf16* dq_sh, const gqe_bf16* dK, const gqe_bf16* dV, const float* dlogits,
                        gqe_bf16* A, gqe_stream stream) {
  GQE_CHECK(check_dims(dims));
  GQE_REQUIRE(topk_idx && dq_routed && dK && dV && dlogits && A, GQE_ERR_INVALID_ARG);
  GQE_REQUIRE(!dims->n_shared || dq_sh, GQE_ERR_INVALID_ARG);
  GQE_REQUIRE(aligned16(dq_routed) && aligned16(dK) && aligned16(dV) && aligned16(A), GQE_ERR_INVALID_ARG);
  GQE_REQUIRE(!dims->n_shared || aligned16(dq_sh), GQE_ERR_INVALID_ARG);
  PackParams p{};
  p.idx = topk_idx;
  p.dq = dq_routed;
  p.dq_sh = dq_sh;
  p.dK = dK;
  p.dV = dV;
  p.dlogits = dlogits;
  p.A = A;
  p.B = dims->B;
  p.T = dims->T;
  p.G = dims->G;
  p.E = dims->E;
  p.k = dims->k;
  p.d = dims->d_head;
  p.n_shared = dims->n_shared;
  p.Kc = bwd_pack_cols(dims->G, dims->E, dims->d_head, dims->n_shared);
  return cuda_status(launch_bwd_pack(p, S(stream)));
}

gqe_status gqe_transpose(int rows, int cols, const gqe_bf16* src, gqe_bf16* dst, int ld_dst, gqe_stream stream) {
  GQE_REQUIRE(rows >= 1 && cols >= 1 && ld_dst >= rows, GQE_ERR_INVALID_ARG);
  GQE_REQUIRE(src && dst, GQE_ERR_INVALID_ARG);
  GQE_REQUIRE((long long)rows * cols < (1ll << 31) && (long long)cols * ld_dst < (1ll << 31), GQE_ERR_UNSUPPORTED);
  return cuda_status(launch_transpose(src, dst, rows, cols, ld_dst, S(stream)));
}

gqe_status gqe_transpose_f32(int rows, int cols, const float* src, float* dst, int ld_dst, gqe_stream stream) {
  GQE_REQUIRE(rows >= 1 && cols >= 1 && ld_dst >= rows, GQE_ERR_INVALID_ARG);
  GQE_REQUIRE(src && dst, GQE_ERR_INVALID_ARG);
  GQE_REQUIRE((long long)rows * cols < (1ll << 31) && (long long)cols * ld_dst < (1ll << 31), GQE_ERR_UNSUPPORTED);
  return cuda_status(launch_transpose_f32(src, dst, rows, cols, ld_dst, S(stream)));
}

gqe_status gqe_bwd_pack_weights(const gqe_dims* dims, const gqe_bf16* Wr, const gqe_bf16* Wq, const gqe_bf16* Wsh,
                                const gqe_bf16* Wk, const gqe_bf16* Wv, gqe_bf16* Wcat, gqe_stream stream) {
  GQE_CHECK(check_dims(dims));
  GQE_REQUIRE(Wr && Wq && Wk && Wv && Wcat, GQE_ERR_INVALID_ARG);
  GQE_REQUIRE(!dims->n_shared || Wsh, GQE_ERR_INVALID_ARG);
  const int D = dims->d_model, G = dims->G, E = dims->E, d = dims->d_head, GE = G * E;
  const int Kc = bwd_pack_cols(G, E, d, dims->n_shared);
  // W_cat [Kc, D] = [Wq (G*E*d rows); Wsh; Wk; Wv; Wr^T; zero rows]
  uint16_t* W = Wcat;
  cudaStream_t st = S(stream);
  size_t row = 0;
  auto put = [&](const gqe_bf16* src, size_t rows) {
    const cudaError_t e = cudaMemcpyAsync(W + row * D, src, rows * D * 2, cudaMemcpyDeviceToDevice, st);
    row += rows;
    return e;
  };
  GQE_REQUIRE(put(Wq, (size_t)GE * d) == cudaSuccess, GQE_ERR_CUDA);
  if (dims->n_shared) GQE_REQUIRE(put(Wsh, d) == cudaSuccess, GQE_ERR_CUDA);
  GQE_REQUIRE(put(Wk, (size_t)G * d) == cudaSuccess, GQE_ERR_CUDA);
  GQE_REQUIRE(put(Wv, (size_t)G * d) == cudaSuccess, GQE_ERR_CUDA);
  GQE_REQUIRE(launch_transpose(Wr, W + row * D, D, GE, D, st) == cudaSuccess, GQE_ERR_CUDA);
  row += GE;
  if ((int)row < Kc)
    GQE_REQUIRE(cudaMemsetAsync(W + row * D, 0, ((size_t)Kc - row) * D * 2, st) == cudaSuccess, GQE_ERR_CUDA);
  return GQE_OK;
}

gqe_status gqe_gemm(int M, int N, int K, const gqe_bf16* A, int a_kn, const gqe_bf16* B, int b_kn, gqe_bf16* C,
                    gqe_stream stream) {
  GQE_REQUIRE(M >= 1 && N >= 1 && K >= 1, GQE_ERR_INVALID_ARG);
  GQE_REQUIRE(A && B && C && (a_kn == 0 || a_kn == 1) && (b_kn == 0 || b_kn == 1), GQE_ERR_INVALID_ARG);
  GQE_REQUIRE(N % 64 == 0, GQE_ERR_UNSUPPORTED);
  // TMA row pitches are multiples of 16 bytes
  GQE_REQUIRE((a_kn ? M : K) % 8 == 0 && (b_kn ? N : K) % 8 == 0, GQE_ERR_UNSUPPORTED);
  GQE_REQUIRE((long long)M * N < (1ll << 31) && (long long)M * K < (1ll << 31) && (long long)N * K < (1ll << 31),
              GQE_ERR_UNSUPPORTED);
  GQE_REQUIRE(aligned16(A) && aligned16(B) && aligned16(C), GQE_ERR_INVALID_ARG);
  const int Kp = (K + 63) / 64 * 64;
  const int pbn = pair_tile_n(M, N);
  const int bn = pbn ? pbn : dense_tile_n(N, M);
  CUtensorMap mA, mW;
  if (a_kn) GQE_REQUIRE(map2d(&mA, A, M, K, 64), GQE_ERR_CUDA);
  else GQE_REQUIRE(map2d(&mA, A, K, M, 128), GQE_ERR_CUDA);
  if (b_kn) GQE_REQUIRE(map2d(&mW, B, N, K, 64), GQE_ERR_CUDA);
  else GQE_REQUIRE(map2d(&mW, B, K, N, pbn ? pbn / 2 : bn), GQE_ERR_CUDA);
  EpiParams ep{};
  ep.out0 = C;
  ep.out1 = C;
  ep.mode = kEpiRowMajor;
  ep.ldo = N;
  ep.n_limit = N;
  ep.err = error_word();
  CUtensorMap mO;
  GQE_REQUIRE(map2d(&mO, C, N, M, 32), GQE_ERR_CUDA);
  ep.store_mode = kStoreTma2d;
  const int nt = (N + bn - 1) / bn;
  const int mn = (a_kn ? 1 : 0) | (b_kn ? 2 : 0);
  if (pbn)
    return cuda_status(launch_gemm_dense_pair(mA, mA, mA, ASource{kASingle, 0, 0, 0, 0, 0}, mW, mW, mO, mO, ep, M, Kp,
                                              nt, nt, pbn, S(stream), mn));
  return cuda_status(launch_gemm_dense(mA, mW, mW, mO, mO, ep, M, Kp, nt, nt, bn, S(stream), mn));
}

gqe_status gqe_debug_wait_timeout(gqe_stream stream) {
  unsigned* err = error_word();
  GQE_REQUIRE(err, GQE_ERR_CUDA);
  return cuda_status(launch_debug_wait(err, S(stream)));
}

gqe_status gqe_device_error(int* code, gqe_stream stream) {
  GQE_REQUIRE(code, GQE_ERR_INVALID_ARG);
  unsigned v = 0;
  if (cudaMemcpyFromSymbolAsync(&v, g_device_error, sizeof(v), 0, cudaMemcpyDeviceToHost, S(stream)) != cudaSuccess)
    return GQE_ERR_CUDA;
  if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return GQE_ERR_CUDA;
  *code = (int)v;
  if (v) {
    const unsigned zero = 0;
    if (cudaMemcpyToSymbolAsync(g_device_error, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, S(stream)) !=
            cudaSuccess ||
        cudaStreamSynchronize(S(stream)) != cudaSuccess)
      return GQE_ERR_CUDA;
  }
  return GQE_OK;
}

}  // extern "C"
