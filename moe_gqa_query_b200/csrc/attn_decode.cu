// attn_decode.cu -- GQE decode attention against a dense [B, G, L_max, d] cache.
//
// One new token per sequence: the k routed query rows of group g (plus the
// shared head's row when g is the shared head's KV group, so the cache is
// streamed once) attend to cache rows [0, cache_len[b]).  A decode step reads
// the whole KV cache (freeguideonline GQA tutorial, "自回归推理中的内存带宽优势"),
// so the kernel is built to stream it at HBM bandwidth:
//
//   split:  grid (chunks of `chunk` keys, G, B); 128 threads; TMA brings 64-row
//           K and V sub-tiles (128-byte swizzle, conflict-free reads) through a
//           4-deep ring; two threads per key row (half the head dims each)
//           keep an online-softmax state per query row in fp32; the CTA merges
//           its 64 row-states with warp shuffles and writes (m, l, acc[d]).
//   merge:  one CTA per (b, g) combines the chunk states and writes bf16.
#include <mutex>

#include "../../include/gqe.h"
#include "attn.cuh"
#include "launch.cuh"

namespace gqe {

namespace {

constexpr int kRows = 64;           // keys per sub-tile
constexpr int kStages = 4;
constexpr int kThreads = 128;

template <int D>
struct DecCfg {
  static constexpr int NB = D / 64;
  static constexpr int SubBytes = NB * kRows * 128;      // one of K or V
  static constexpr int QP = (D == 64) ? 2 : 1;            // query rows per pass
  static constexpr int HD = D / 2;                        // dims per thread
  static constexpr size_t Smem = 1024 + kStages * 2 * SubBytes + 4 * QP * (D + 2) * 4 + 64;
};

// logical 16-byte chunk `c` (0..D/8-1) of row `r` in a 128-byte swizzled sub-tile
template <int D>
__device__ __forceinline__ const uint4* swz_chunk(const uint8_t* base, int r, int c) {
  const int box = c >> 3, cc = c & 7;
  return reinterpret_cast<const uint4*>(base + box * (kRows * 128) + r * 128 + ((cc ^ (r & 7)) << 4));
}

template <int D>
__global__ void __launch_bounds__(kThreads)
decode_split_kernel(const __grid_constant__ CUtensorMap mapK, const __grid_constant__ CUtensorMap mapV,
                    DecodeParams p) {
  using C = DecCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  float* red = reinterpret_cast<float*>(ring + kStages * 2 * C::SubBytes);  // [4 warps][QP][D+2]
  uint64_t* full = reinterpret_cast<uint64_t*>(red + 4 * C::QP * (D + 2));
  __shared__ int s_abort;

  const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rr = tid >> 1, half = tid & 1;
  pdl_launch_dependents();
  pdl_wait();
  int len = p.cache_len[b];
  if (len < 1 || len > p.L_max) {
    // outside the documented range: flag it once per sequence and clamp, so
    // no key past the cache is counted and the merge stays finite
    if (tid == 0 && c == 0 && g == 0 && p.err) atomicCAS(p.err, 0u, (unsigned)kErrDecodeCacheLen);
    len = min(max(len, 0), p.L_max);
  }
  const int start = c * p.chunk;
  const int end = min(start + p.chunk, len);
  const int nq = p.k + ((p.n_shared && g == p.sg) ? 1 : 0);
  float* part = p.part + (((size_t)(b * p.G + g) * p.n_chunks + c) * p.nq_max) * (D + 2);

  if (start >= end) {
    for (int qi = tid; qi < nq; qi += kThreads) {
      part[qi * (D + 2) + 0] = -INFINITY;
      part[qi * (D + 2) + 1] = 0.f;
    }
    return;
  }
  const int n_sub = (end - start + kRows - 1) / kRows;
  const int n_pass = (nq + C::QP - 1) / C::QP;
  const int total = n_pass * n_sub;
  const int kvseq = b * p.G + g;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&full[s], 1);
    s_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  volatile int* abort = &s_abort;

  auto issue = [&](int it) {
    const int s = it % kStages;
    const int row = start + (it % n_sub) * kRows;
    mbar_arrive_expect_tx(&full[s], 2 * C::SubBytes);
    uint8_t* kd = ring + s * 2 * C::SubBytes;
    uint8_t* vd = kd + C::SubBytes;
    for (int bx = 0; bx < C::NB; ++bx) {
      tma_load_3d(kd + bx * kRows * 128, &mapK, &full[s], bx * 64, row, kvseq);
      tma_load_3d(vd + bx * kRows * 128, &mapV, &full[s], bx * 64, row, kvseq);
    }
  };
  if (tid == 0)
    for (int it = 0; it < min(kStages, total); ++it) issue(it);

  const float sl2 = p.scale_log2;
  int it = 0;
  for (int pass = 0; pass < n_pass; ++pass) {
    const int q0 = pass * C::QP;
    // query rows of this pass, this thread's half of the dims, fp32
    float q[C::QP][C::HD];
#pragma unroll
    for (int qp = 0; qp < C::QP; ++qp) {
      const int qi = q0 + qp;
      const gqe_bf16_t* src = nullptr;
      if (qi < p.k) src = p.q_routed + (((size_t)b * p.G + g) * p.k + qi) * D;
      else if (qi < nq) src = p.q_sh + (size_t)b * D;
#pragma unroll
      for (int i = 0; i < C::HD / 8; ++i) {
        uint4 v = src ? reinterpret_cast<const uint4*>(src + half * C::HD)[i] : make_uint4(0, 0, 0, 0);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          q[qp][8 * i + 2 * h] = bf16_lo(w[h]);
          q[qp][8 * i + 2 * h + 1] = bf16_hi(w[h]);
        }
      }
    }
    float m[C::QP], l[C::QP], acc[C::QP][C::HD];
#pragma unroll
    for (int qp = 0; qp < C::QP; ++qp) {
      m[qp] = -INFINITY;
      l[qp] = 0.f;
#pragma unroll
      for (int i = 0; i < C::HD; ++i) acc[qp][i] = 0.f;
    }

    for (int sub = 0; sub < n_sub; ++sub, ++it) {
      const int s = it % kStages;
      mbar_wait(&full[s], (it / kStages) & 1, abort, p.err, kErrTimeoutDecode);
      const uint8_t* kd = ring + s * 2 * C::SubBytes;
      const uint8_t* vd = kd + C::SubBytes;
      const bool valid = start + sub * kRows + rr < end;
      float sc[C::QP];
#pragma unroll
      for (int qp = 0; qp < C::QP; ++qp) sc[qp] = 0.f;
#pragma unroll
      for (int i = 0; i < C::HD / 8; ++i) {
        const uint4 kv = *swz_chunk<D>(kd, rr, half * (C::HD / 8) + i);
        const uint32_t w[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const float k0 = bf16_lo(w[h]), k1 = bf16_hi(w[h]);
#pragma unroll
          for (int qp = 0; qp < C::QP; ++qp) {
            sc[qp] = fmaf(q[qp][8 * i + 2 * h], k0, sc[qp]);
            sc[qp] = fmaf(q[qp][8 * i + 2 * h + 1], k1, sc[qp]);
          }
        }
      }
#pragma unroll
      for (int qp = 0; qp < C::QP; ++qp) sc[qp] += __shfl_xor_sync(0xffffffffu, sc[qp], 1);
      if (valid) {
        float pr[C::QP], al[C::QP];
#pragma unroll
        for (int qp = 0; qp < C::QP; ++qp) {
          const float x = sc[qp] * sl2;
          const float mn = fmaxf(m[qp], x);
          al[qp] = ex2(m[qp] - mn);
          pr[qp] = ex2(x - mn);
          l[qp] = fmaf(l[qp], al[qp], pr[qp]);
          m[qp] = mn;
        }
#pragma unroll
        for (int i = 0; i < C::HD / 8; ++i) {
          const uint4 vv = *swz_chunk<D>(vd, rr, half * (C::HD / 8) + i);
          const uint32_t w[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const float v0 = bf16_lo(w[h]), v1 = bf16_hi(w[h]);
#pragma unroll
            for (int qp = 0; qp < C::QP; ++qp) {
              acc[qp][8 * i + 2 * h] = fmaf(acc[qp][8 * i + 2 * h], al[qp], pr[qp] * v0);
              acc[qp][8 * i + 2 * h + 1] = fmaf(acc[qp][8 * i + 2 * h + 1], al[qp], pr[qp] * v1);
            }
          }
        }
      }
      __syncthreads();   // stage s fully read
      if (tid == 0 && it + kStages < total && !*abort) issue(it + kStages);
    }

    // ---- merge the 64 row states of this CTA: lanes with equal `half` first
#pragma unroll
    for (int qp = 0; qp < C::QP; ++qp) {
      float M = m[qp];
#pragma unroll
      for (int o = 2; o < 32; o <<= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
      const float f = (M == -INFINITY) ? 0.f : ex2(m[qp] - M);
      float L = l[qp] * f;
#pragma unroll
      for (int o = 2; o < 32; o <<= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
#pragma unroll
      for (int i = 0; i < C::HD; ++i) {
        float a = acc[qp][i] * f;
#pragma unroll
        for (int o = 2; o < 32; o <<= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
        acc[qp][i] = a;
      }
      if (lane < 2) {
        float* dst = red + (warp * C::QP + qp) * (D + 2);
        if (lane == 0) {
          dst[0] = M;
          dst[1] = L;
        }
#pragma unroll
        for (int i = 0; i < C::HD; ++i) dst[2 + half * C::HD + i] = acc[qp][i];
      }
    }
    __syncthreads();
    for (int e = tid; e < C::QP * D; e += kThreads) {
      const int qp = e / D, dim = e % D;
      const int qi = q0 + qp;
      if (qi >= nq) continue;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < 4; ++w) M = fmaxf(M, red[(w * C::QP + qp) * (D + 2)]);
      float L = 0.f, A = 0.f;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float* src = red + (w * C::QP + qp) * (D + 2);
        const float f = (src[0] == -INFINITY) ? 0.f : ex2(src[0] - M);
        L += src[1] * f;
        A += src[2 + dim] * f;
      }
      float* dst = part + qi * (D + 2);
      dst[2 + dim] = A;
      if (dim == 0) {
        dst[0] = M;
        dst[1] = L;
      }
    }
    __syncthreads();
  }
  drain_after_abort(abort);
}

template <int D>
__global__ void __launch_bounds__(128) decode_merge_kernel(DecodeParams p) {
  pdl_launch_dependents();
  pdl_wait();
  const int bg = blockIdx.x;
  const int b = bg / p.G, g = bg % p.G;
  const int nq = p.k + ((p.n_shared && g == p.sg) ? 1 : 0);
  const float* base = p.part + (size_t)bg * p.n_chunks * p.nq_max * (D + 2);
  for (int e = threadIdx.x; e < nq * D; e += blockDim.x) {
    const int qi = e / D, dim = e % D;
    float M = -INFINITY;
    for (int c = 0; c < p.n_chunks; ++c) M = fmaxf(M, base[(c * p.nq_max + qi) * (D + 2)]);
    float L = 0.f, A = 0.f;
    for (int c = 0; c < p.n_chunks; ++c) {
      const float* s = base + (c * p.nq_max + qi) * (D + 2);
      if (s[0] == -INFINITY) continue;   // chunk past cache_len: its acc was never written
      const float f = ex2(s[0] - M);
      L += s[1] * f;
      A += s[2 + dim] * f;
    }
    const float o = L > 0.f ? A / L : 0.f;   // L == 0 only for a flagged empty cache
    const uint32_t pk = pack_bf16x2(o, 0.f);
    gqe_bf16_t* dst = (qi < p.k) ? p.o_routed + (((size_t)b * p.G + g) * p.k + qi) * D + dim
                                 : p.o_sh + (size_t)b * D + dim;
    *dst = (gqe_bf16_t)(pk & 0xFFFFu);
  }
}

}  // namespace

void decode_split_plan(int L_max, int* chunk, int* n_chunks) {
  int c = 2048;
  if (L_max < 16384) {
    c = (L_max + 7) / 8;
    c = ((c + kRows - 1) / kRows) * kRows;
    if (c < kRows) c = kRows;
  }
  *chunk = c;
  *n_chunks = (L_max + c - 1) / c;
}

size_t decode_workspace_bytes(int B, int G, int k, int d, int n_shared, int L_max) {
  int chunk, n_chunks;
  decode_split_plan(L_max, &chunk, &n_chunks);
  return (size_t)B * G * n_chunks * (k + n_shared) * (d + 2) * sizeof(float);
}

template <int D>
static cudaError_t launch_dec(const CUtensorMap& mK, const CUtensorMap& mV, const DecodeParams& p,
                              cudaStream_t stream) {
  const size_t smem = DecCfg<D>::Smem;
  auto kern = decode_split_kernel<D>;
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  e = launch_kernel(kern, dim3(p.n_chunks, p.G, p.B), dim3(kThreads), smem, stream, 1, mK, mV, p);
  if (e != cudaSuccess) return e;
  return launch_kernel(decode_merge_kernel<D>, dim3(p.B * p.G), dim3(128), 0, stream, 1, p);
}

cudaError_t launch_attn_decode_maps(const CUtensorMap& mK, const CUtensorMap& mV, const DecodeParams& p,
                                   cudaStream_t stream) {
  if (p.d == 64) return launch_dec<64>(mK, mV, p, stream);
  return launch_dec<128>(mK, mV, p, stream);
}

}  // namespace gqe

// ---------------------------------------------------------------------------
// Decode without a caller workspace, for callers that cannot allocate device
// memory when they decode (an engine that reserved all device memory for its
// own pool, a decode loop that cannot pay cudaMalloc's implicit
// synchronisation).  The split-L partial states go to one fixed array in this
// file instead of a caller buffer; the kernels are the ones above.

namespace gqe {

gqe_status decode_setup(const gqe_dims* dims, const gqe_bf16* q_routed, const gqe_bf16* q_sh, const gqe_bf16* Kc,
                        const gqe_bf16* Vc, int L_max, const int32_t* cache_len, gqe_bf16* o_routed,
                        gqe_bf16* o_sh, CUtensorMap* mK, CUtensorMap* mV, DecodeParams* p);

namespace {

constexpr size_t kNoAllocScratchBytes = GQE_DECODE_NOALLOC_MAX_BYTES;

// Held by every GPU that loads the library, from load until process exit.
static __device__ __align__(256) float g_decode_noalloc_scratch[kNoAllocScratchBytes / sizeof(float)];

// Device address of the array on the current device.  Host code only sees a
// host-side stand-in under the array's name, so the address is looked up with
// the device current.  It is looked up again on every call made outside
// stream capture (a reset primary context reloads the module at another
// address); a call under capture uses the address the last uncaptured call
// on that device found, and fails when there is none.
float* noalloc_scratch(cudaStream_t stream) {
  static std::mutex mu;
  static float* cache[64] = {nullptr};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (cap == cudaStreamCaptureStatusNone) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_decode_noalloc_scratch) != cudaSuccess) return nullptr;
    cache[dev] = static_cast<float*>(ptr);
  }
  return cache[dev];
}

}  // namespace
}  // namespace gqe

extern "C" gqe_status gqe_attn_decode_noalloc(const gqe_dims* dims, const gqe_bf16* q_routed, const gqe_bf16* q_sh,
                                              const gqe_bf16* Kc, const gqe_bf16* Vc, int L_max,
                                              const int32_t* cache_len, gqe_bf16* o_routed, gqe_bf16* o_sh,
                                              gqe_stream stream) {
  using namespace gqe;
  CUtensorMap mK, mV;
  DecodeParams p;
  const gqe_status st = decode_setup(dims, q_routed, q_sh, Kc, Vc, L_max, cache_len, o_routed, o_sh, &mK, &mV, &p);
  if (st != GQE_OK) return st;
  // The partial states for these dims must fit the fixed array.  Every slot
  // the merge reads is written earlier in the same call (a chunk past
  // cache_len writes its empty state), so nothing is cleared beforehand.
  if (decode_workspace_bytes(p.B, p.G, p.k, p.d, p.n_shared, L_max) > kNoAllocScratchBytes)
    return GQE_ERR_WORKSPACE;
  float* scratch = noalloc_scratch(reinterpret_cast<cudaStream_t>(stream));
  if (!scratch) return GQE_ERR_CUDA;
  p.part = scratch;
  return launch_attn_decode_maps(mK, mV, p, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? GQE_OK
                                                                                                    : GQE_ERR_CUDA;
}
