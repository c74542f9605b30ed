// combine.cu -- GQE output construction ("GQE" study note §3-2 3)-5)).
//
//   h_t = Concat( o_{t,g,e} for the selected e of every group g (group-major,
//                 ascending expert index: one head slot each, never averaged),
//                 sum_g sum_{e in S} p~_{t,g,e} o_{t,g,e}   (weighted-sum slot),
//                 o_shared_t )                               (shared head slot)
//
// One warp per token; each lane owns d/32 contiguous columns of every slot.
// The weighted sum accumulates in fp32 and is rounded to bf16 once.
#include <type_traits>

#include "route.cuh"

namespace gqe {

namespace {

template <int VPL>   // bf16 values per lane: d / 32
__global__ void __launch_bounds__(256) combine_kernel(CombineParams p) {
  const int warp_global = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int N = p.B * p.T;
  if (warp_global >= N) return;
  const int n = warp_global;
  const int b = n / p.T, t = n % p.T;
  const int d = p.d;
  const int slots = p.k * p.G + 1 + p.n_shared;
  uint16_t* hrow = p.h + (size_t)n * slots * d + lane * VPL;
  float acc[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) acc[i] = 0.f;
  typedef typename std::conditional<VPL == 2, uint32_t, uint2>::type vec_t;
  const int GK = p.G * p.k;
  const uint16_t* obase = p.o_routed + (((size_t)b * p.G) * p.T + t) * p.k * d + lane * VPL;
  const size_t gstride = (size_t)p.T * p.k * d;   // next group, same token
  const float* wrow = p.w + (size_t)n * GK;
  for (int s0 = 0; s0 < GK; s0 += 8) {
    vec_t v[8];
    float wv[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int s = s0 + u;
      if (s < GK) {
        const int g = s / p.k, j = s % p.k;
        v[u] = __ldg(reinterpret_cast<const vec_t*>(obase + g * gstride + (size_t)j * d));
        wv[u] = __ldg(wrow + s);
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int s = s0 + u;
      if (s < GK) {
        *reinterpret_cast<vec_t*>(hrow + s * d) = v[u];
        const uint32_t* uu = reinterpret_cast<const uint32_t*>(&v[u]);
#pragma unroll
        for (int i = 0; i < VPL / 2; ++i) {
          acc[2 * i] = fmaf(wv[u], bf16_lo(uu[i]), acc[2 * i]);
          acc[2 * i + 1] = fmaf(wv[u], bf16_hi(uu[i]), acc[2 * i + 1]);
        }
      }
    }
  }
  vec_t r;
  uint32_t* ru = reinterpret_cast<uint32_t*>(&r);
#pragma unroll
  for (int i = 0; i < VPL / 2; ++i) ru[i] = pack_bf16x2(acc[2 * i], acc[2 * i + 1]);
  *reinterpret_cast<vec_t*>(hrow + (p.k * p.G) * d) = r;
  if (p.n_shared) {
    const vec_t v = *reinterpret_cast<const vec_t*>(p.o_sh + (size_t)n * d + lane * VPL);
    *reinterpret_cast<vec_t*>(hrow + (p.k * p.G + 1) * d) = v;
  }
}

}  // namespace

cudaError_t launch_combine(const CombineParams& p, cudaStream_t stream) {
  const int N = p.B * p.T;
  const int grid = (N * 32 + 255) / 256;
  if (p.d == 64) combine_kernel<2><<<grid, 256, 0, stream>>>(p);
  else combine_kernel<4><<<grid, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace gqe
