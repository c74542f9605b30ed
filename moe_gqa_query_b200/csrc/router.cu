// router.cu -- GQE router: logits, in-group softmax, TopK and renormalised weights.
//
// "GQE" study note §3-2 2): s_{t,g,e} = r_g(x_t)_e (a linear map of x_t),
// p = softmax over the E experts of the group, S_{t,g} = TopK(p, k); §3-2 4):
// p~ = p normalised over the selected experts (all k*G of the token by
// default, or within the group).
//
// The router reads x once and is HBM bound.  A CTA of 4 warps owns 32 tokens
// (many CTAs per SM keep enough bytes in flight): x streams through a 4-deep
// cp.async ring (128-byte rows, XOR-swizzled); the logits x Wr are accumulated
// in fp32 on the tensor cores (mma.sync m16n8k16: the products of bf16 inputs
// are exact, so this is the fp32 dot product), two warps per 16 tokens each
// taking half of every 64-column chunk, the halves added in shared memory; one
// thread per token then runs the softmax and TopK of every group in fp32
// registers.  Selection uses the fp32 logits (softmax is monotone within a
// group); ties go to the lower expert index; selected experts are emitted in
// ascending index order.
#include "route.cuh"

namespace gqe {

namespace {

constexpr int kTok = 32;       // tokens per CTA
constexpr int kKC = 64;        // reduction chunk (d_model columns)
constexpr int kXStages = 4;

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float* c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int GEP>
__global__ void __launch_bounds__(128) router_kernel(RouterParams p) {
  constexpr int WS = GEP + 8;            // padded Wr row (bf16), 16-byte multiple
  constexpr int NT = GEP / 8;            // n-tiles of 8 logits
  constexpr int WPT = kKC * GEP / 128;   // Wr elements per thread per chunk
  __shared__ __align__(128) uint16_t xs[kXStages][kTok * kKC];
  __shared__ __align__(16) uint16_t ws[2][kKC * WS];
  __shared__ float lg[kTok][GEP + 1];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tok0 = blockIdx.x * kTok;
  const int GE = p.G * p.E;
  const int nkc = p.D / kKC;
  // warp w: token rows (w & 1) * 16 .. +15, reduction half (w >> 1) of every chunk
  const int mrow = (warp & 1) * 16;
  const int khalf = warp >> 1;

  auto load_x = [&](int kc) {
    uint16_t* dst = xs[kc % kXStages];
#pragma unroll
    for (int i = 0; i < kTok * 8 / 128; ++i) {
      const int e = tid + 128 * i;     // kTok * 8 16-byte chunks
      const int r = e >> 3, c = e & 7;
      const int n = tok0 + r;
      const uint16_t* src = p.x + (size_t)(n < p.N ? n : 0) * p.D + kc * kKC + c * 8;
      cp_async_16(reinterpret_cast<uint8_t*>(dst) + r * 128 + ((c ^ (r & 7)) << 4), src, n < p.N);
    }
  };
  uint16_t wreg[WPT];
  auto fetch_w = [&](int kc) {
#pragma unroll
    for (int i = 0; i < WPT; ++i) {
      const int e = tid + 128 * i;
      const int r = e / GEP, c = e % GEP;
      wreg[i] = (c < GE) ? p.Wr[(size_t)(kc * kKC + r) * GE + c] : (uint16_t)0;
    }
  };
  auto store_w = [&](int buf) {
#pragma unroll
    for (int i = 0; i < WPT; ++i) {
      const int e = tid + 128 * i;
      ws[buf][(e / GEP) * WS + (e % GEP)] = wreg[i];
    }
  };

  float acc[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;

  for (int s = 0; s < kXStages - 1; ++s) {
    if (s < nkc) load_x(s);
    cp_async_commit();
  }
  fetch_w(0);
  store_w(0);

  for (int kc = 0; kc < nkc; ++kc) {
    if (kc + kXStages - 1 < nkc) load_x(kc + kXStages - 1);
    cp_async_commit();
    if (kc + 1 < nkc) fetch_w(kc + 1);
    cp_async_wait<kXStages - 1>();
    __syncthreads();
    const uint32_t xb = smem_u32(xs[kc % kXStages]);
    const uint32_t wb = smem_u32(ws[kc & 1]);
#pragma unroll
    for (int kh = 0; kh < kKC / 32; ++kh) {
      const int ks = khalf * (kKC / 32) + kh;
      const int mi = lane >> 3;
      const int ar = mrow + (mi & 1) * 8 + (lane & 7);
      const int ac = ks * 2 + (mi >> 1);
      uint32_t a0, a1, a2, a3;
      ldsm_x4(xb + ar * 128 + ((ac ^ (ar & 7)) << 4), a0, a1, a2, a3);
#pragma unroll
      for (int np = 0; np < NT / 2; ++np) {
        const int kr = ks * 16 + (mi & 1) * 8 + (lane & 7);
        const int nc = np * 16 + (mi >> 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(wb + (kr * WS + nc) * 2, b0, b1, b2, b3);
        mma_bf16_16816(acc[2 * np], a0, a1, a2, a3, b0, b1);
        mma_bf16_16816(acc[2 * np + 1], a0, a1, a2, a3, b2, b3);
      }
    }
    __syncthreads();
    if (kc + 1 < nkc) store_w((kc + 1) & 1);
  }
  cp_async_wait<0>();

  // the two reduction halves meet in shared memory
  if (khalf == 1) {
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const int r = mrow + (lane >> 2);
      const int c = t * 8 + (lane & 3) * 2;
      lg[r][c] = acc[t][0];
      lg[r][c + 1] = acc[t][1];
      lg[r + 8][c] = acc[t][2];
      lg[r + 8][c + 1] = acc[t][3];
    }
  }
  __syncthreads();
  if (khalf == 0) {
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const int r = mrow + (lane >> 2);
      const int c = t * 8 + (lane & 3) * 2;
      lg[r][c] += acc[t][0];
      lg[r][c + 1] += acc[t][1];
      lg[r + 8][c] += acc[t][2];
      lg[r + 8][c + 1] += acc[t][3];
    }
  }
  __syncthreads();

  if (tid >= kTok) return;
  const int n = tok0 + tid;
  if (n >= p.N) return;
  const int E = p.E, k = p.k;

  // pass 1 (token scope): sum of the selected probabilities over all groups
  float total = 0.f;
  for (int pass = (p.scope == 0 ? 0 : 1); pass < 2; ++pass) {
    for (int g = 0; g < p.G; ++g) {
      float s[8], pr[8];
      float mx = -INFINITY;
      for (int e = 0; e < E; ++e) {
        s[e] = lg[tid][g * E + e] + (p.bias ? p.bias[g * E + e] : 0.f);
        mx = fmaxf(mx, s[e]);
      }
      float Z = 0.f;
      for (int e = 0; e < E; ++e) {
        pr[e] = expf(s[e] - mx);
        Z += pr[e];
      }
      const float invZ = 1.f / Z;
      unsigned chosen = 0;
      for (int it = 0; it < k; ++it) {
        int best = -1;
        float bv = -INFINITY;
        for (int e = 0; e < E; ++e) {
          if ((chosen >> e) & 1u) continue;
          if (best < 0 || s[e] > bv) {
            best = e;
            bv = s[e];
          }
        }
        chosen |= 1u << best;
      }
      float gsum = 0.f;
      for (int e = 0; e < E; ++e)
        if ((chosen >> e) & 1u) gsum += pr[e] * invZ;
      if (pass == 0) {
        total += gsum;
        continue;
      }
      const float den = (p.scope == 0) ? total : gsum;
      const float inv_den = 1.f / den;
      const size_t o = ((size_t)n * p.G + g) * k;
      int j = 0;
      for (int e = 0; e < E; ++e) {
        if ((chosen >> e) & 1u) {
          p.topk_idx[o + j] = e;
          p.topk_w[o + j] = pr[e] * invZ * inv_den;
          ++j;
        }
      }
      if (p.probs)
        for (int e = 0; e < E; ++e) p.probs[((size_t)n * p.G + g) * E + e] = pr[e] * invZ;
    }
  }
}

}  // namespace

cudaError_t launch_router(const RouterParams& p, cudaStream_t stream) {
  const int GE = p.G * p.E;
  const int grid = (p.N + kTok - 1) / kTok;
  if (GE <= 16) router_kernel<16><<<grid, 128, 0, stream>>>(p);
  else if (GE <= 32) router_kernel<32><<<grid, 128, 0, stream>>>(p);
  else router_kernel<64><<<grid, 128, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace gqe
