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
// thread per (token, group) then runs that group's softmax and TopK in fp32
// registers, the token-scope denominator summed through shared memory.  Selection uses the fp32 logits (softmax is monotone within a
// group); ties go to the lower expert index; selected experts are emitted in
// ascending index order.
#include "route.cuh"
#include "launch.cuh"

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

// Softmax and TopK of one (token, group) from the token's fp32 logits.
// Returns the selected experts as a bit mask and the sum of their
// probabilities; pr receives the group's probabilities.
__device__ __forceinline__ unsigned route_group(const RouterParams& p, const float* logits, int g, float* pr,
                                                float* gsum) {
  const int E = p.E;
  float s[8];
  float mx = -INFINITY;
  for (int e = 0; e < E; ++e) {
    s[e] = logits[g * E + e] + (p.bias ? p.bias[g * E + e] : 0.f);
    mx = fmaxf(mx, s[e]);
  }
  float Z = 0.f;
  for (int e = 0; e < E; ++e) {
    pr[e] = expf(s[e] - mx);
    Z += pr[e];
  }
  const float invZ = 1.f / Z;
  for (int e = 0; e < E; ++e) pr[e] *= invZ;
  unsigned chosen = 0;
  for (int it = 0; it < p.k; ++it) {
    int best = -1;
    float bv = -INFINITY;
    for (int e = 0; e < E; ++e) {
      if ((chosen >> e) & 1u) continue;
      if (best < 0 || s[e] > bv) {   // strict: ties keep the lower index
        best = e;
        bv = s[e];
      }
    }
    chosen |= 1u << best;
  }
  float sum = 0.f;
  for (int e = 0; e < E; ++e)
    if ((chosen >> e) & 1u) sum += pr[e];
  *gsum = sum;
  return chosen;
}

// Routes the kTok tokens of a tile cooperatively, one (token, group) pair per
// thread: softmax and TopK per group, the token-scope denominator through
// shared memory, then the selected experts (ascending), their renormalised
// weights and optionally the probabilities.  `lg` holds the tile's logits
// with row stride `ls`; `gs` is kTok*G floats of shared scratch.
__device__ __forceinline__ void route_tile(const RouterParams& p, const float* lg, int ls, int tok0, float* gs) {
  const int G = p.G, E = p.E, k = p.k;
  const int npairs = kTok * G;
  for (int e = threadIdx.x; e < npairs; e += blockDim.x) {
    const int t = e / G, g = e % G;
    float pr[8], sum;
    route_group(p, lg + t * ls, g, pr, &sum);
    gs[e] = sum;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < npairs; e += blockDim.x) {
    const int t = e / G, g = e % G;
    const int n = tok0 + t;
    if (n >= p.N) continue;
    float pr[8], sum;
    const unsigned chosen = route_group(p, lg + t * ls, g, pr, &sum);
    float den = sum;
    if (p.scope == 0) {
      den = 0.f;
      for (int gg = 0; gg < G; ++gg) den += gs[t * G + gg];
    }
    const float inv_den = 1.f / den;
    const size_t o = ((size_t)n * G + g) * k;
    int j = 0;
    for (int ee = 0; ee < E; ++ee) {
      if ((chosen >> ee) & 1u) {
        p.topk_idx[o + j] = ee;
        p.topk_w[o + j] = pr[ee] * inv_den;
        ++j;
      }
    }
    if (p.probs)
      for (int ee = 0; ee < E; ++ee) p.probs[((size_t)n * G + g) * E + ee] = pr[ee];
  }
}

template <int GEP>
__global__ void __launch_bounds__(128) router_kernel(RouterParams p) {
  constexpr int WS = GEP + 8;            // padded Wr row (bf16), 16-byte multiple
  constexpr int NT = GEP / 8;            // n-tiles of 8 logits
  constexpr int WPT = kKC * GEP / 128;   // Wr elements per thread per chunk
  __shared__ __align__(128) uint16_t xs[kXStages][kTok * kKC];
  __shared__ __align__(16) uint16_t ws[2][kKC * WS];
  __shared__ float lg[kTok][GEP + 1];
  // the per-(token, group) sums reuse the x ring once the reduction is done
  float* gsum_s = reinterpret_cast<float*>(&xs[0][0]);
  static_assert(sizeof(float) * kTok * 64 <= sizeof(uint16_t) * kXStages * kTok * kKC, "group sums fit");

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tok0 = blockIdx.x * kTok;
  pdl_launch_dependents();
  pdl_wait();
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

  route_tile(p, &lg[0][0], GEP + 1, tok0, gsum_s);
}


// Wr resident in shared memory (when it fits); every warp streams its own
// 16-token tile through a private cp.async ring (no block barriers), so eight
// independent pipelines per CTA keep bytes in flight, then routes its tokens:
// two lanes per token, each taking every other group, the token-scope sum
// combined with one shuffle.
constexpr int kWarpTok = 16;
constexpr int kRouterWarps = 8;

template <int GEP, int STAGES>
__global__ void __launch_bounds__(kRouterWarps * 32, 1) router_resident_kernel(RouterParams p) {
  constexpr int WS = GEP + 8;
  constexpr int NT = GEP / 8;
  constexpr int kStageBytes = kWarpTok * kKC * 2;                           // 2 KB
  extern __shared__ __align__(128) uint8_t rsm[];
  uint16_t* wsm = reinterpret_cast<uint16_t*>(rsm);                           // [D][WS]
  uint8_t* xring = rsm + (((size_t)p.D * WS * 2 + 127) & ~size_t(127));       // [warps][STAGES][2 KB]
  float* lgw = reinterpret_cast<float*>(xring + (size_t)kRouterWarps * STAGES * kStageBytes);  // [warps][16][GEP+1]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int GE = p.G * p.E;
  const int nkc = p.D / kKC;
  const int n_tiles = (p.N + kWarpTok - 1) / kWarpTok;
  uint8_t* ring = xring + (size_t)warp * STAGES * kStageBytes;
  float* lg = lgw + (size_t)warp * kWarpTok * (GEP + 1);
  pdl_launch_dependents();
  pdl_wait();

  // Wr into shared memory once (padded columns zero)
  if ((GE & 7) == 0 && (reinterpret_cast<uintptr_t>(p.Wr) & 15) == 0) {
    const int n16 = p.D * GE / 8;
    for (int e = threadIdx.x; e < n16; e += blockDim.x) {
      const int r = (e * 8) / GE, c = (e * 8) % GE;
      cp_async_16(wsm + (size_t)r * WS + c, reinterpret_cast<const uint4*>(p.Wr) + e, true);
    }
    if (GE < GEP)
      for (int e = threadIdx.x; e < p.D * (GEP - GE); e += blockDim.x)
        wsm[(size_t)(e / (GEP - GE)) * WS + GE + e % (GEP - GE)] = 0;
  } else {
    for (int e = threadIdx.x; e < p.D * GEP; e += blockDim.x) {
      const int r = e / GEP, c = e % GEP;
      wsm[r * WS + c] = (c < GE) ? p.Wr[(size_t)r * GE + c] : (uint16_t)0;
    }
  }
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();

  for (int tile = blockIdx.x * kRouterWarps + warp; tile < n_tiles; tile += gridDim.x * kRouterWarps) {
    const int tok0 = tile * kWarpTok;
    auto load_x = [&](int kc) {
      uint8_t* dst = ring + (kc % STAGES) * kStageBytes;
#pragma unroll
      for (int i = 0; i < kWarpTok * 8 / 32; ++i) {       // 128 16-byte chunks, 4 per lane
        const int e = lane + 32 * i;
        const int r = e >> 3, c = e & 7;
        const int n = tok0 + r;
        const uint16_t* src = p.x + (size_t)(n < p.N ? n : 0) * p.D + kc * kKC + c * 8;
        cp_async_16(dst + r * 128 + ((c ^ (r & 7)) << 4), src, n < p.N);
      }
    };
    for (int kc = 0; kc < STAGES - 1; ++kc) {
      if (kc < nkc) load_x(kc);
      cp_async_commit();
    }
    float acc[NT][4];
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
    for (int kc = 0; kc < nkc; ++kc) {
      cp_async_wait<STAGES - 2>();
      __syncwarp();
      if (kc + STAGES - 1 < nkc) load_x(kc + STAGES - 1);
      cp_async_commit();
      const uint32_t xb = smem_u32(ring + (kc % STAGES) * kStageBytes);
      const uint32_t wb = smem_u32(wsm + (size_t)kc * kKC * WS);
#pragma unroll
      for (int ks = 0; ks < kKC / 16; ++ks) {
        const int mi = lane >> 3;
        const int ar = (mi & 1) * 8 + (lane & 7);
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
    }
    cp_async_wait<0>();
    // logits of the 16 tokens into the warp's scratch
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const int r = lane >> 2;
      const int c = t * 8 + (lane & 3) * 2;
      lg[r * (GEP + 1) + c] = acc[t][0];
      lg[r * (GEP + 1) + c + 1] = acc[t][1];
      lg[(r + 8) * (GEP + 1) + c] = acc[t][2];
      lg[(r + 8) * (GEP + 1) + c + 1] = acc[t][3];
    }
    __syncwarp();
    // routing: lanes 2i and 2i+1 share token i, each taking every other group
    {
      const int t = lane >> 1, half = lane & 1;
      const int n = tok0 + t;
      const float* row = lg + t * (GEP + 1);
      float part = 0.f;
      for (int g = half; g < p.G; g += 2) {
        float pr[8], sum;
        route_group(p, row, g, pr, &sum);
        part += sum;
      }
      const float total = part + __shfl_xor_sync(0xffffffffu, part, 1);
      if (n < p.N) {
        for (int g = half; g < p.G; g += 2) {
          float pr[8], sum;
          const unsigned chosen = route_group(p, row, g, pr, &sum);
          const float inv_den = 1.f / (p.scope == 0 ? total : sum);
          const size_t o = ((size_t)n * p.G + g) * p.k;
          int j = 0;
          for (int ee = 0; ee < p.E; ++ee) {
            if ((chosen >> ee) & 1u) {
              p.topk_idx[o + j] = ee;
              p.topk_w[o + j] = pr[ee] * inv_den;
              ++j;
            }
          }
          if (p.probs)
            for (int ee = 0; ee < p.E; ++ee) p.probs[((size_t)n * p.G + g) * p.E + ee] = pr[ee];
        }
      }
    }
    __syncwarp();
  }
}

template <int GEP>
size_t resident_smem(int D, int stages) {
  return (((size_t)D * (GEP + 8) * 2 + 127) & ~size_t(127)) + (size_t)kRouterWarps * stages * kWarpTok * kKC * 2 +
         (size_t)kRouterWarps * kWarpTok * (GEP + 1) * 4;
}

int router_num_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  }
  return n;
}

template <int GEP>
cudaError_t launch_router_gep(const RouterParams& p, cudaStream_t stream) {
  constexpr int STAGES = 8;
  const size_t smem = resident_smem<GEP>(p.D, STAGES);
  if (smem <= 200 * 1024) {
    auto kern = router_resident_kernel<GEP, STAGES>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kern), smem);
    if (e != cudaSuccess) return e;
    const int n_tiles = (p.N + kWarpTok - 1) / kWarpTok;
    int grid = router_num_sms();
    const int need = (n_tiles + kRouterWarps - 1) / kRouterWarps;
    if (grid > need) grid = need;
    return launch_kernel(kern, dim3(grid), dim3(kRouterWarps * 32), smem, stream, 1, p);
  }
  return launch_kernel(router_kernel<GEP>, dim3((p.N + kTok - 1) / kTok), dim3(128), 0, stream, 1, p);
}

}  // namespace

cudaError_t launch_router(const RouterParams& p, cudaStream_t stream) {
  const int GE = p.G * p.E;
  if (GE <= 16) return launch_router_gep<16>(p, stream);
  if (GE <= 32) return launch_router_gep<32>(p, stream);
  return launch_router_gep<64>(p, stream);
}

}  // namespace gqe
