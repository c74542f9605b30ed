// layer_bwd.cu -- the GQE layer's backward outside attention.
//
// combine_bwd: the output construction ("GQE" study note §3-2 3) hard slots,
//   4) weighted-sum slot, 5) shared head) differentiated: dh -> do, do_sh and
//   the gradient of the router weights p~ (the weighted-sum slot is the path on
//   which the router learns, §4-1).
// router_bwd: d p~ -> d logits through the renormalisation (§3-2 4)) and the
//   in-group softmax (§3-2 2)); TopK passes no gradient.  Also d bias.
// bwd_pack: the projection gradients as one bf16 matrix A = [dq scattered to
//   its expert's columns (zeros for unselected experts) | dq_sh | dK | dV |
//   d logits], so that dx = A W_cat and dW_cat = A^T x are two plain GEMMs over
//   the stacked weights W_cat = [Wq; Wsh; Wk; Wv; Wr^T].
// transpose: a tiled bf16 transpose (operand layouts for those GEMMs).
#include "bwd.cuh"
#include "launch.cuh"

namespace gqe {

namespace {

// ---------------------------------------------------------------- combine backward
// One thread per 8 elements (16 bytes) of a selected head row: d/8 threads
// per (token, g, j), the p~ gradient summed over them by shuffles; the shared
// slot is copied by the threads of (token, g = 0, j = 0).
__device__ __forceinline__ void unpack8(uint4 v, float* f) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    f[2 * e] = bf16_lo(w[e]);
    f[2 * e + 1] = bf16_hi(w[e]);
  }
}

__global__ void __launch_bounds__(256) combine_bwd_kernel(CombineBwdParams p) {
  pdl_launch_dependents();
  pdl_wait();
  const int tpr = p.d / 8;                     // threads per head row
  const int Gk = p.G * p.k;
  const long long gt = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long row = gt / tpr;              // (token, g, j)
  const int part = (int)(gt % tpr);
  const bool live = row < (long long)p.B * p.T * Gk;
  const long long rr = live ? row : 0;
  const int n = (int)(rr / Gk), gj = (int)(rr % Gk);
  const int g = gj / p.k, j = gj % p.k;
  const int b = n / p.T, t = n % p.T;
  const int d = p.d, e0 = part * 8;
  const gqe_bf16_t* dh = p.dh + (size_t)n * p.slots * d;
  const size_t orow = ((((size_t)b * p.G + g) * p.T + t) * p.k + j) * d;
  float hard[8], o[8], dov[8];
  unpack8(*reinterpret_cast<const uint4*>(dh + gj * d + e0), hard);
  unpack8(*reinterpret_cast<const uint4*>(p.o_routed + orow + e0), o);
  const float w = p.w[(size_t)n * Gk + gj];
  float dot = 0.f;
  if (p.output_mode == 0) {
    float route[8];
    unpack8(*reinterpret_cast<const uint4*>(dh + Gk * d + e0), route);
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      dov[v] = hard[v] + w * route[v];
      dot += route[v] * o[v];
    }
  } else if (p.output_mode == 1) {
#pragma unroll
    for (int v = 0; v < 8; ++v) dov[v] = hard[v];
  } else {
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      dov[v] = w * hard[v];
      dot += hard[v] * o[v];
    }
  }
  if (live)
    *reinterpret_cast<uint4*>(p.do_routed + orow + e0) =
        make_uint4(pack_bf16x2(dov[0], dov[1]), pack_bf16x2(dov[2], dov[3]), pack_bf16x2(dov[4], dov[5]),
                   pack_bf16x2(dov[6], dov[7]));
  for (int off = tpr >> 1; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
  if (live && part == 0) p.dw[(size_t)n * Gk + gj] = dot;
  if (live && p.n_shared && gj == 0) {
    const int col = Gk * d + (p.output_mode == 0 ? d : 0);
    *reinterpret_cast<uint4*>(p.do_sh + (size_t)n * d + e0) = *reinterpret_cast<const uint4*>(dh + col + e0);
  }
}

// ---------------------------------------------------------------- router backward
// One thread per (token, group): d p~ -> dp (renormalisation) -> ds (in-group
// softmax).  Token-scope sums are recomputed by each of the token's G threads.
constexpr int kRouterBwdThreads = 256;

__global__ void __launch_bounds__(kRouterBwdThreads) router_bwd_kernel(RouterBwdParams p) {
  __shared__ float sbias[kMaxBwdRouterCols];
  pdl_launch_dependents();
  pdl_wait();
  const int GE = p.G * p.E;
  if (p.dbias) {
    for (int i = threadIdx.x; i < GE; i += blockDim.x) sbias[i] = 0.f;
    __syncthreads();
  }
  const long long tg = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (tg < (long long)p.N * p.G) {
    const int n = (int)(tg / p.G), g = (int)(tg % p.G);
    const float* pr = p.probs + (size_t)n * GE;
    const int* idx = p.idx + (size_t)n * p.G * p.k;
    const float* dw = p.dw + (size_t)n * p.G * p.k;
    const float* wt = p.w + (size_t)n * p.G * p.k;
    // the renormalisation's sums: over all selections of the token (scope 0)
    // or of this group (scope 1)
    const int i0 = p.scope == 0 ? 0 : g * p.k;
    const int i1 = p.scope == 0 ? p.G * p.k : (g + 1) * p.k;
    float z = 0.f, sdw = 0.f;
    if (p.scope != 2) {
      for (int i = i0; i < i1; ++i) {
        z += pr[(i / p.k) * p.E + idx[i]];
        sdw += dw[i] * wt[i];
      }
    }
    // dp on the selected experts, and sum_e p_e dp_e over the group
    float pdp = 0.f;
    float dsel[8];
    for (int j = 0; j < p.k; ++j) {
      const float dwj = dw[g * p.k + j];
      dsel[j] = (p.scope == 2) ? dwj : (dwj - sdw) / z;
      pdp += pr[g * p.E + idx[g * p.k + j]] * dsel[j];
    }
    float* out = p.dlogits + (size_t)n * GE + g * p.E;
    for (int e = 0; e < p.E; ++e) {
      float dp = 0.f;
      for (int j = 0; j < p.k; ++j)
        if (idx[g * p.k + j] == e) dp = dsel[j];
      const float ds = pr[g * p.E + e] * (dp - pdp);
      out[e] = ds;
      if (p.dbias) atomicAdd(&sbias[g * p.E + e], ds);
    }
  }
  if (p.dbias) {
    __syncthreads();
    for (int i = threadIdx.x; i < GE; i += blockDim.x) atomicAdd(&p.dbias[i], sbias[i]);
  }
}

// ---------------------------------------------------------------- pack
// One thread per 16 bytes (8 columns) of A [N, Kc]: consecutive threads write
// consecutive chunks of a row.
__global__ void __launch_bounds__(256) bwd_pack_kernel(PackParams p) {
  pdl_launch_dependents();
  pdl_wait();
  const int cpr = p.Kc / 8;                    // chunks per row
  const long long gt = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (gt >= (long long)p.B * p.T * cpr) return;
  const int n = (int)(gt / cpr), c = (int)(gt % cpr) * 8;
  const int b = n / p.T, t = n % p.T;
  const int d = p.d;
  uint4 v = make_uint4(0u, 0u, 0u, 0u);
  const int n_q = p.G * p.E * d;
  const int c_sh = n_q, c_k = c_sh + p.n_shared * d, c_v = c_k + p.G * d, c_l = c_v + p.G * d;
  if (c < n_q) {
    // dq scattered into the expert columns: block (g, e) of d columns
    const int blk = c / d, e_in = c % d;
    const int g = blk / p.E, e = blk % p.E;
    const int* idx = p.idx + (size_t)n * p.G * p.k + g * p.k;
    for (int j = 0; j < p.k; ++j)
      if (idx[j] == e)
        v = *reinterpret_cast<const uint4*>(p.dq + ((((size_t)b * p.G + g) * p.T + t) * p.k + j) * d + e_in);
  } else if (c < c_k) {
    v = *reinterpret_cast<const uint4*>(p.dq_sh + (size_t)n * d + (c - c_sh));
  } else if (c < c_l) {
    const uint16_t* src = c < c_v ? p.dK : p.dV;
    const int cc = c < c_v ? c - c_k : c - c_v;
    const int g = cc / d, e_in = cc % d;
    v = *reinterpret_cast<const uint4*>(src + (((size_t)b * p.G + g) * p.T + t) * d + e_in);
  } else {
    const int GE = p.G * p.E;
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int c0 = c - c_l + 2 * e;
      const float lo = c0 < GE ? p.dlogits[(size_t)n * GE + c0] : 0.f;
      const float hi = c0 + 1 < GE ? p.dlogits[(size_t)n * GE + c0 + 1] : 0.f;
      w[e] = pack_bf16x2(lo, hi);
    }
    v = make_uint4(w[0], w[1], w[2], w[3]);
  }
  *reinterpret_cast<uint4*>(p.A + (size_t)n * p.Kc + c) = v;
}

// ---------------------------------------------------------------- transpose
// dst[c * ld_dst + r] = src[r * cols + c]; columns r in [rows, ld_dst) of dst
// are zeroed.  64 x 64 tiles through shared memory.
constexpr int kTr = 64;

template <typename Elem>
__global__ void __launch_bounds__(256) transpose_kernel(const Elem* __restrict__ src, Elem* __restrict__ dst,
                                                        int rows, int cols, int ld_dst) {
  __shared__ Elem tile[kTr][kTr + 2];
  pdl_launch_dependents();
  pdl_wait();
  const int r0 = blockIdx.y * kTr, c0 = blockIdx.x * kTr;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;   // 32 x 8
  for (int i = ty; i < kTr; i += 8) {
    const int r = r0 + i;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int c = c0 + tx * 2 + h;
      tile[i][tx * 2 + h] = (r < rows && c < cols) ? src[(size_t)r * cols + c] : Elem(0);
    }
  }
  __syncthreads();
  for (int i = ty; i < kTr; i += 8) {
    const int c = c0 + i;
    if (c >= cols) continue;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = r0 + tx * 2 + h;
      if (r < ld_dst) dst[(size_t)c * ld_dst + r] = tile[tx * 2 + h][i];
    }
  }
}

}  // namespace

cudaError_t launch_combine_bwd(const CombineBwdParams& p, cudaStream_t stream) {
  const long long threads = (long long)p.B * p.T * p.G * p.k * (p.d / 8);
  return launch_kernel(combine_bwd_kernel, dim3((unsigned)((threads + 255) / 256)), dim3(256), 0, stream, 1, p);
}

cudaError_t launch_router_bwd(const RouterBwdParams& p, cudaStream_t stream) {
  if (p.dbias) {
    cudaError_t e = cudaMemsetAsync(p.dbias, 0, sizeof(float) * p.G * p.E, stream);
    if (e != cudaSuccess) return e;
  }
  const long long threads = (long long)p.N * p.G;
  return launch_kernel(router_bwd_kernel, dim3((unsigned)((threads + kRouterBwdThreads - 1) / kRouterBwdThreads)),
                       dim3(kRouterBwdThreads), 0, stream, 1, p);
}

cudaError_t launch_bwd_pack(const PackParams& p, cudaStream_t stream) {
  const long long threads = (long long)p.B * p.T * (p.Kc / 8);
  return launch_kernel(bwd_pack_kernel, dim3((unsigned)((threads + 255) / 256)), dim3(256), 0, stream, 1, p);
}

cudaError_t launch_transpose(const uint16_t* src, uint16_t* dst, int rows, int cols, int ld_dst,
                             cudaStream_t stream) {
  const dim3 grid((cols + kTr - 1) / kTr, (ld_dst + kTr - 1) / kTr);
  return launch_kernel(transpose_kernel<uint16_t>, grid, dim3(256), 0, stream, 1, src, dst, rows, cols, ld_dst);
}

cudaError_t launch_transpose_f32(const float* src, float* dst, int rows, int cols, int ld_dst, cudaStream_t stream) {
  const dim3 grid((cols + kTr - 1) / kTr, (ld_dst + kTr - 1) / kTr);
  return launch_kernel(transpose_kernel<float>, grid, dim3(256), 0, stream, 1, src, dst, rows, cols, ld_dst);
}

}  // namespace gqe
