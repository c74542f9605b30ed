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
    const float inv_den = p.scope == 2 ? 1.f : 1.f / den;
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
          const float inv_den = p.scope == 2 ? 1.f : 1.f / (p.scope == 0 ? total : sum);
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

// ---------------------------------------------------------------------------
// tcgen05 router.  A CTA takes R consecutive tokens at a time (R <= 128 and a
// multiple of 8, given by router_tc_tile_rows; the kernel streams x once and
// is HBM bound).  Every 64-dimension
// k-block of a tile arrives by TMA in one ring stage together with the same
// 64 rows of Wr, as Wr is stored ([D, G*E]): the MMA reads it as an MN-major B
// operand of 64 columns, the columns past G*E zero-filled by the TMA, so Wr
// is never rearranged in shared memory.  The logits accumulate in fp32 in
// tensor memory (two buffers, so one tile's routing overlaps the next tile's
// MMAs) and the epilogue routes one token per thread: per-group softmax and
// TopK on logit + bias, the renormalised weights of the selected experts.
namespace {

constexpr int kRtBM = 128;                    // MMA rows; rows R..127 of a tile are not routed
constexpr int kRtBK = 64;
constexpr int kRtN = 64;                      // MMA columns: G*E zero-padded by the TMA
constexpr int kRtX = kRtBM * kRtBK * 2;       // 16 KB of x rows per stage
constexpr int kRtW = kRtN * kRtBK * 2;        // 8 KB of Wr rows per stage
constexpr int kRtStage = kRtX + kRtW;
// Ring depth of the tcgen05 router.  With short x rows (d_model < 2048) a
// deeper ring makes the router alone faster but slows the layer, whose K/V
// projection reads x beside it (main layer step: 4 stages 196.5 us, 6 stages
// 197.4 us, 8 stages 198.4 us); with long rows the router needs the deeper
// ring to keep enough of x in flight (d_model 4096: 55 us at 4 stages, 42 us
// at 8).
// Ring depth below d_model 2048, and 128-token tiles per CTA.  The layer runs
// its K/V projection on a side stream beside the router, so the router is
// sized for the step, not for its own time: with four tiles per CTA (32 CTAs
// at 16384 tokens) each CTA's routing epilogue overlaps its next tile's x
// stream and the other SMs start the K/V GEMM at once.  Measured on B200,
// main-layer step 187.2 -> 178.9 us (one tile per CTA, 4 stages -> four, 8),
// wide/skewed 1326 -> 1268 us, T = 32768 1666 -> 1650 us; the router call
// alone 21.7 -> 28.6 us.  Two tiles per CTA, three and six or eight gave
// steps in between or slower.
#ifndef GQE_ROUTER_STAGES_SHORT
#define GQE_ROUTER_STAGES_SHORT 8
#endif
#ifndef GQE_ROUTER_TILES_PER_CTA
#define GQE_ROUTER_TILES_PER_CTA 4
#endif
constexpr int kRouterStagesShort = GQE_ROUTER_STAGES_SHORT;
constexpr int kRouterStagesLong = 8;

struct __align__(8) RouterTcBarriers {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint32_t tmem_base;
  int abort;
};

template <int GEP>
__device__ __forceinline__ void route_token(const RouterParams& p, const float* lg, int n) {
  const int G = p.G, E = p.E, k = p.k;
  float den_tok = 0.f;
  if (p.scope == 0) {
    for (int g = 0; g < G; ++g) {
      float pr[8], sum;
      route_group(p, lg, g, pr, &sum);
      den_tok += sum;
    }
  }
  for (int g = 0; g < G; ++g) {
    float pr[8], sum;
    const unsigned chosen = route_group(p, lg, g, pr, &sum);
    const float inv_den = p.scope == 2 ? 1.f : 1.f / (p.scope == 0 ? den_tok : sum);
    const size_t o = ((size_t)n * G + g) * k;
    int j = 0;
    for (int e = 0; e < E; ++e) {
      if ((chosen >> e) & 1u) {
        p.topk_idx[o + j] = e;
        p.topk_w[o + j] = pr[e] * inv_den;
        ++j;
      }
    }
    if (p.probs)
      for (int e = 0; e < E; ++e) p.probs[((size_t)n * G + g) * E + e] = pr[e];
  }
}

// One token's routing with the group width E fixed at compile time: every
// array index is static, the exponentials are ex2.approx on pre-scaled
// arguments, and each group is evaluated once.
template <int GEP, int E>
__device__ __forceinline__ void route_token_e(const RouterParams& p, const float* lg, const float* bias, int n) {
  constexpr int GM = GEP / E;          // groups that fit the padded width
  const int G = p.G, k = p.k;
  float pr[GEP];
  unsigned chosen[GM];
  float gsum[GM];
  float den_tok = 0.f;
#pragma unroll
  for (int g = 0; g < GM; ++g) {
    chosen[g] = 0;
    gsum[g] = 1.f;
    if (g < G) {
      float sv[E];
      float mx = -INFINITY;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        sv[e] = lg[g * E + e] + bias[g * E + e];
        mx = fmaxf(mx, sv[e]);
      }
      float Z = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        pr[g * E + e] = ex2((sv[e] - mx) * 1.4426950408889634f);
        Z += pr[g * E + e];
      }
      const float invZ = 1.f / Z;
#pragma unroll
      for (int e = 0; e < E; ++e) pr[g * E + e] *= invZ;
      unsigned ch = 0;
      for (int it = 0; it < k; ++it) {
        int best = 0;
        float bv = -INFINITY;
        bool found = false;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const bool free_e = !((ch >> e) & 1u);
          if (free_e && (!found || sv[e] > bv)) {   // strict: ties keep the lower index
            best = e;
            bv = sv[e];
            found = true;
          }
        }
        ch |= 1u << best;
      }
      float sum = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e)
        if ((ch >> e) & 1u) sum += pr[g * E + e];
      chosen[g] = ch;
      gsum[g] = sum;
      den_tok += sum;
    }
  }
  if (k == 1 && G == GM && GM % 4 == 0 && !p.probs &&
      ((reinterpret_cast<uintptr_t>(p.topk_idx) | reinterpret_cast<uintptr_t>(p.topk_w)) & 15u) == 0) {
    // one selection per group: the token's index and weight rows (G entries
    // each, 16-byte aligned) leave as 16-byte vectors
    int ri[GM];
    float rw[GM];
#pragma unroll
    for (int g = 0; g < GM; ++g) {
      int e1 = 0;
#pragma unroll
      for (int e = 1; e < E; ++e)
        if ((chosen[g] >> e) & 1u) e1 = e;
      ri[g] = e1;
      rw[g] = pr[g * E + e1] * (p.scope == 2 ? 1.f : 1.f / (p.scope == 0 ? den_tok : gsum[g]));
    }
    int4* di = reinterpret_cast<int4*>(p.topk_idx + (size_t)n * GM);
    float4* dw = reinterpret_cast<float4*>(p.topk_w + (size_t)n * GM);
#pragma unroll
    for (int q = 0; q < GM / 4; ++q) {
      di[q] = make_int4(ri[4 * q], ri[4 * q + 1], ri[4 * q + 2], ri[4 * q + 3]);
      dw[q] = make_float4(rw[4 * q], rw[4 * q + 1], rw[4 * q + 2], rw[4 * q + 3]);
    }
    return;
  }
#pragma unroll
  for (int g = 0; g < GM; ++g) {
    if (g < G) {
      const float inv_den = p.scope == 2 ? 1.f : 1.f / (p.scope == 0 ? den_tok : gsum[g]);
      const size_t o = ((size_t)n * G + g) * k;
      int j = 0;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        if ((chosen[g] >> e) & 1u) {
          p.topk_idx[o + j] = e;
          p.topk_w[o + j] = pr[g * E + e] * inv_den;
          ++j;
        }
      }
      if (p.probs) {
#pragma unroll
        for (int e = 0; e < E; ++e) p.probs[((size_t)n * G + g) * E + e] = pr[g * E + e];
      }
    }
  }
}

// CTA (224 threads): warp 0 TMA producer; warps 1 and 6 issue the MMAs of the
// even and odd k-blocks into two partial accumulators (a small-N MMA keeps the
// tensor pipe busy for less time than one thread needs to issue it); warps
// 2..5 sum the partials and route, one token per thread.
template <int GEP, int STAGES>
__global__ void __launch_bounds__(224, 1) router_tc_kernel(const __grid_constant__ CUtensorMap mapX,
                                                           const __grid_constant__ CUtensorMap mapW, RouterParams p,
                                                           int R) {
  constexpr uint32_t kTmemCols = 4 * kRtN;          // 2 buffers x 2 partial accumulators
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sS = smem;                                        // STAGES x [x 16 KB | Wr 8 KB]
  RouterTcBarriers* bar = reinterpret_cast<RouterTcBarriers*>(sS + STAGES * kRtStage);
  float* sBias = reinterpret_cast<float*>(bar + 1);          // GEP
  volatile int* abort = &bar->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int GE = p.G * p.E;
  const int nk = p.D / kRtBK;
  const int n_tiles = (p.N + R - 1) / R;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&bar->full[s], 1);
      mbar_init(&bar->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&bar->acc_full[a], 2);     // one commit from each MMA thread
      mbar_init(&bar->acc_empty[a], 4);
    }
    bar->abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&mapX);
    tma_prefetch_desc(&mapW);
  }
  if (warp == 1) tmem_alloc(&bar->tmem_base, kTmemCols);
  pdl_launch_dependents();
  pdl_wait();
  for (int e = threadIdx.x; e < GEP; e += blockDim.x) sBias[e] = (p.bias && e < GE) ? p.bias[e] : 0.f;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      const uint32_t stage_tx = (uint32_t)R * kRtBK * 2 + kRtW;
      int it = 0;
      for (int t = blockIdx.x; t < n_tiles && !*abort; t += gridDim.x) {
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % STAGES;
          if (it >= STAGES &&
              !mbar_wait(&bar->empty[s], ((it / STAGES) & 1) ^ 1, abort, p.err, kErrTimeoutRouter))
            break;
          mbar_arrive_expect_tx(&bar->full[s], stage_tx);
          tma_load_2d(sS + s * kRtStage, &mapX, &bar->full[s], kb * kRtBK, t * R);
          tma_load_2d(sS + s * kRtStage + kRtX, &mapW, &bar->full[s], 0, kb * kRtBK);
        }
      }
    }
  } else if (warp == 1 || warp == 6) {
    if (lane == 0) {
      // warp 1: k-blocks 0, 2, 4, ... into partial 0; warp 6: 1, 3, 5, ... into partial 1
      const int half = warp == 6 ? 1 : 0;
      constexpr uint32_t idesc = idesc_bf16_f32(kRtBM, kRtN, false, true);
      int tc = 0;
      for (int t = blockIdx.x; t < n_tiles && !*abort; t += gridDim.x, ++tc) {
        const int ab = tc & 1, use = tc >> 1;
        if (tc >= 2 && !mbar_wait(&bar->acc_empty[ab], (use & 1) ^ 1, abort, p.err, kErrTimeoutRouter)) break;
        tc_fence_after();
        const uint32_t acc = tmem + (uint32_t)((2 * ab + half) * kRtN);
        bool ok = true;
        for (int kb = half; kb < nk; kb += 2) {
          const int it = tc * nk + kb;
          const int s = it % STAGES;
          if (!mbar_wait(&bar->full[s], (it / STAGES) & 1, abort, p.err, kErrTimeoutRouter)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sS + s * kRtStage);
          const uint32_t b0 = a0 + kRtX;
#pragma unroll
          for (int kk = 0; kk < kRtBK / 16; ++kk)
            // A: x rows, K-major; B: Wr rows, MN-major (a 16-deep k-step is 16 rows of 128 bytes)
            umma_ss(acc, sdesc_sw128(a0 + kk * 32, 16, 1024), sdesc_sw128(b0 + kk * 2048, kRtW, 1024), idesc,
                    (kb != half) || kk != 0);
          umma_commit(&bar->empty[s]);
        }
        if (!ok) break;
        umma_commit(&bar->acc_full[ab]);
      }
    }
  } else {
    const int lg = warp & 3;
    const uint32_t lane_off = (uint32_t)(lg * 32) << 16;
    const int r = lg * 32 + lane;
    int tc = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++tc) {
      const int ab = tc & 1, use = tc >> 1;
      const bool ok = mbar_wait(&bar->acc_full[ab], use & 1, abort, p.err, kErrTimeoutRouter);
      tc_fence_after();
      float logit[GEP];
#pragma unroll
      for (int c0 = 0; c0 < GEP; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(tmem + lane_off + (uint32_t)(2 * ab * kRtN + c0), v);
#pragma unroll
        for (int i = 0; i < 16; ++i) logit[c0 + i] = __uint_as_float(v[i]);
        if (nk > 1) {   // the odd k-blocks' partial
          tmem_ld16(tmem + lane_off + (uint32_t)((2 * ab + 1) * kRtN + c0), v);
#pragma unroll
          for (int i = 0; i < 16; ++i) logit[c0 + i] += __uint_as_float(v[i]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar->acc_empty[ab]);
      const int n = t * R + r;
      if (ok && r < R && n < p.N) {
        if (p.E == 2 && GEP <= 32) route_token_e<GEP, 2>(p, logit, sBias, n);
        else if (p.E == 4) route_token_e<GEP, 4>(p, logit, sBias, n);
        else if (p.E == 8) route_token_e<GEP, 8>(p, logit, sBias, n);
        else route_token<GEP>(p, logit, n);
      }
      if (!ok) break;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  drain_after_abort(abort);
}

template <int GEP, int STAGES>
cudaError_t launch_router_tc_st(const CUtensorMap& mapX, const CUtensorMap& mapW, const RouterParams& p, int R,
                                cudaStream_t stream) {
  const size_t smem = 1024 + (size_t)STAGES * kRtStage + sizeof(RouterTcBarriers) + GEP * sizeof(float);
  auto kern = router_tc_kernel<GEP, STAGES>;
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  const int n_tiles = (p.N + R - 1) / R;
  const int sms = router_num_sms();
  const int want = (n_tiles + GQE_ROUTER_TILES_PER_CTA - 1) / GQE_ROUTER_TILES_PER_CTA;
  const int grid = want < sms ? want : sms;
  return launch_kernel(kern, dim3(grid), dim3(224), smem, stream, 1, mapX, mapW, p, R);
}

template <int GEP>
cudaError_t launch_router_tc_gep(const CUtensorMap& mapX, const CUtensorMap& mapW, const RouterParams& p, int R,
                                 cudaStream_t stream) {
  if (p.D / kRtBK >= 32) return launch_router_tc_st<GEP, kRouterStagesLong>(mapX, mapW, p, R, stream);
  return launch_router_tc_st<GEP, kRouterStagesShort>(mapX, mapW, p, R, stream);
}

}  // namespace

int router_tc_tile_rows(int N) {
  // 128-row tiles (tiles sized to cover every SM made the router alone faster
  // but the layer's step slower, 202 against 195.5 us on the main layer)
  (void)N;
  return kRtBM;
}

cudaError_t launch_router_tc(const CUtensorMap& mapX, const CUtensorMap& mapW, const RouterParams& p, int R,
                             cudaStream_t stream) {
  const int GE = p.G * p.E;
  if (p.D % kRtBK != 0 || p.E > 8 || GE > kRtN || GE % 8 != 0 || R < 8 || R > kRtBM || R % 8 != 0)
    return cudaErrorNotSupported;
  if (GE <= 16) return launch_router_tc_gep<16>(mapX, mapW, p, R, stream);
  if (GE <= 32) return launch_router_tc_gep<32>(mapX, mapW, p, R, stream);
  return launch_router_tc_gep<64>(mapX, mapW, p, R, stream);
}

// ---------------------------------------------------------------------------
// Router statistics: one thread per token adds its selections and in-group
// probabilities into shared-memory totals per (group, expert); each block then
// adds its totals into the outputs.
namespace {
__global__ void __launch_bounds__(256) router_stats_kernel(const float* __restrict__ probs,
                                                           const int* __restrict__ idx, int N, int G, int E,
                                                           int k, int* counts, float* prob_sum) {
  __shared__ int c_s[64];
  __shared__ float p_s[64];
  const int GE = G * E;
  for (int i = threadIdx.x; i < GE; i += blockDim.x) {
    c_s[i] = 0;
    p_s[i] = 0.f;
  }
  pdl_launch_dependents();
  pdl_wait();
  __syncthreads();
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n < N) {
    for (int s = 0; s < GE; ++s) atomicAdd(&p_s[s], probs[(size_t)n * GE + s]);
    for (int g = 0; g < G; ++g)
      for (int j = 0; j < k; ++j) {
        const int e = idx[((size_t)n * G + g) * k + j];
        if (e >= 0 && e < E) atomicAdd(&c_s[g * E + e], 1);
      }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < GE; i += blockDim.x) {
    if (c_s[i]) atomicAdd(&counts[i], c_s[i]);
    atomicAdd(&prob_sum[i], p_s[i]);
  }
}
}  // namespace

cudaError_t launch_router_stats(const float* probs, const int* topk_idx, int N, int G, int E, int k,
                                int* counts, float* prob_sum, cudaStream_t stream) {
  cudaError_t e = cudaMemsetAsync(counts, 0, sizeof(int) * G * E, stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(prob_sum, 0, sizeof(float) * G * E, stream);
  if (e != cudaSuccess) return e;
  return launch_kernel(router_stats_kernel, dim3((N + 255) / 256), dim3(256), 0, stream, 1, probs, topk_idx, N, G,
                       E, k, counts, prob_sum);
}

cudaError_t launch_router(const RouterParams& p, cudaStream_t stream) {
  const int GE = p.G * p.E;
  if (GE <= 16) return launch_router_gep<16>(p, stream);
  if (GE <= 32) return launch_router_gep<32>(p, stream);
  return launch_router_gep<64>(p, stream);
}

}  // namespace gqe
