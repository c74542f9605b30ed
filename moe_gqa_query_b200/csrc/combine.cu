// combine.cu -- GQE output construction ("GQE" study note §3-2 3)-5)) and the
// two ablation variants of §5-1's accuracy table (output_mode 1: hard slots
// and shared head only; 2: hard slots each times its router weight, shared
// head, no weighted-sum slot).
//
//   h_t = Concat( o_{t,g,e} for the selected e of every group g (group-major,
//                 ascending expert index: one head slot each, never averaged),
//                 sum_g sum_{e in S} p~_{t,g,e} o_{t,g,e}   (weighted-sum slot),
//                 o_shared_t )                               (shared head slot)
//
// One thread per (token, 16-byte column chunk): it reads that chunk of every
// hard slot row of the token (independent loads), accumulates the weighted sum
// in fp32 registers over the slots in order, and rounds it to bf16 once.  The
// d/8 threads of a token read each slot row as one contiguous d*2-byte run.
#include "launch.cuh"
#include "route.cuh"

namespace gqe {

namespace {

template <int D>
__global__ void __launch_bounds__(256) combine_kernel(CombineParams p) {
  constexpr int CPT = D / 8;       // 16-byte chunks per slot row
  const int gid = blockIdx.x * blockDim.x + threadIdx.x;
  const int n = gid / CPT;
  const int c8 = (gid % CPT) * 8;
  const int N = p.B * p.T;
  pdl_launch_dependents();
  if (n >= N) return;
  pdl_wait();
  const int b = n / p.T, t = n - b * p.T;
  const int GK = p.G * p.k;
  const int has_route = p.output_mode == 0 ? 1 : 0;
  const int slots = GK + has_route + p.n_shared;
  // route_only: h is the [N, d] weighted-sum slot; the hard and shared slots
  // are read from o_routed and o_sh by the projection itself
  uint16_t* hrow = p.h + (size_t)n * (p.route_only ? D : slots * D) + c8;
  uint16_t* route_dst = p.route_only ? hrow : hrow + (size_t)GK * D;
  const size_t gstride = (size_t)p.T * p.k * D;     // next group, same token
  const uint16_t* obase = p.o_routed + (((size_t)b * p.G) * p.T + t) * p.k * D + c8;
  const float* wrow = p.w + (size_t)n * GK;
  const bool copy_hard = !p.route_only || p.output_mode == 2;
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  int g = 0, j = 0;
#pragma unroll 8
  for (int s = 0; s < GK; ++s) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(obase + g * gstride + (size_t)j * D));
    const float w = __ldg(wrow + s);
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
    if (p.output_mode == 2) {
      // weighted concat: the hard slot times its router weight
      const uint4 wv = make_uint4(pack_bf16x2(w * bf16_lo(u[0]), w * bf16_hi(u[0])),
                                  pack_bf16x2(w * bf16_lo(u[1]), w * bf16_hi(u[1])),
                                  pack_bf16x2(w * bf16_lo(u[2]), w * bf16_hi(u[2])),
                                  pack_bf16x2(w * bf16_lo(u[3]), w * bf16_hi(u[3])));
      *reinterpret_cast<uint4*>(hrow + (size_t)s * D) = wv;
    } else if (copy_hard) {
      *reinterpret_cast<uint4*>(hrow + (size_t)s * D) = v;     // hard slot: a copy
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[2 * i] = fmaf(w, bf16_lo(u[i]), acc[2 * i]);
      acc[2 * i + 1] = fmaf(w, bf16_hi(u[i]), acc[2 * i + 1]);
    }
    if (++j == p.k) {
      j = 0;
      ++g;
    }
  }
  if (has_route) {
    uint4 r;
    r.x = pack_bf16x2(acc[0], acc[1]);
    r.y = pack_bf16x2(acc[2], acc[3]);
    r.z = pack_bf16x2(acc[4], acc[5]);
    r.w = pack_bf16x2(acc[6], acc[7]);
    *reinterpret_cast<uint4*>(route_dst) = r;
  }
  if (p.n_shared && !p.route_only) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(p.o_sh + (size_t)n * D + c8));
    *reinterpret_cast<uint4*>(hrow + (size_t)(GK + has_route) * D) = v;
  }
}

}  // namespace

cudaError_t launch_combine(const CombineParams& p, cudaStream_t stream) {
  const long long threads = (long long)p.B * p.T * (p.d / 8);
  const int grid = (int)((threads + 255) / 256);
  if (p.d == 64) return launch_kernel(combine_kernel<64>, dim3(grid), dim3(256), 0, stream, 1, p);
  return launch_kernel(combine_kernel<128>, dim3(grid), dim3(256), 0, stream, 1, p);
}

}  // namespace gqe
