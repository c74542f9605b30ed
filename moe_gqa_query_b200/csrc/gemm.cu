// gemm.cu -- tcgen05 GEMMs of the GQE layer: C = A W^T, bf16 operands, fp32
// accumulation in tensor memory.
//
//   * dense path: A and W tiles by TMA (128-byte swizzle), used for the dense
//     K/V projection (written straight into the [B, G, T, d] head layout or
//     into a decode cache row) and for the output projection over the kG+2
//     slots ("GQE" study note §3-2 7));
//   * routed path: the A rows are gathered per (group, expert) segment of the
//     token-to-expert permutation with 16-byte cp.async (one 128-row tile of
//     one expert per CTA), so only selected experts' query projections are
//     computed ("GQE" study note §3-2 2)); the shared head's projection rides
//     in the same launch as extra tiles.
//
// CTA layout (192 threads, one 128 x BN tile):
//   warp 0      TMA producer (lane 0)
//   warp 1      tensor-memory owner and MMA issuer (lane 0)
//   warps 2..5  routed path: A-row gather producers; then the epilogue
//               (tensor memory -> registers -> bf16 -> global), one row per thread.
#include "gemm.cuh"

namespace gqe {

namespace {

constexpr int kBM = 128;
constexpr int kBK = 64;                 // 64 bf16 = one 128-byte swizzle row
constexpr int kATileBytes = kBM * kBK * 2;
constexpr int kThreads = 192;

struct __align__(8) GemmSmemTail {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t accum;
  uint32_t tmem_base;
  int abort;
  int rowsrc[kBM];
  int rowdst[kBM];
};

template <int BN>
__device__ __forceinline__ void epilogue_store(const EpiParams& ep, int map_sel, int row,
                                               int grow_dst, int n0, uint32_t tmem_row,
                                               bool valid) {
  // grow_dst: row index in the destination (dense: the A row)
  for (int c0 = 0; c0 < BN; c0 += 32) {
    uint32_t v[32];
    tmem_ld32(tmem_row + c0, v);
    const int n = n0 + c0;
    if (!valid || n >= ep.n_limit) continue;
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
    gqe_bf16_t* dst = nullptr;
    gqe_bf16_t* base = map_sel ? ep.out1 : ep.out0;
    switch (ep.mode) {
      case kEpiRowMajor:
        dst = base + (size_t)grow_dst * ep.ldo + n;
        break;
      case kEpiHeads: {
        const int g = n / ep.d, dd = n % ep.d;
        const int b = grow_dst / ep.T, t = grow_dst % ep.T;
        dst = base + (((size_t)b * ep.G + g) * ep.T + t) * ep.d + dd;
        break;
      }
      case kEpiCacheRow: {
        const int g = n / ep.d, dd = n % ep.d;
        const int pos = ep.cache_len[grow_dst] - 1;
        dst = base + (((size_t)grow_dst * ep.G + g) * ep.L_max + pos) * ep.d + dd;
        break;
      }
      default:  // kEpiRows: destination row given per tile row
        dst = base + (size_t)grow_dst * ep.ldo + n;
        break;
    }
    uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int i = 0; i < 4; ++i) d4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
  }
}

// ---------------------------------------------------------------------------
// dense: A [M, K] and W [N, K] by TMA
template <int BN, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
gemm_dense_kernel(const __grid_constant__ CUtensorMap mapA,
                  const __grid_constant__ CUtensorMap mapB0,
                  const __grid_constant__ CUtensorMap mapB1, EpiParams ep, int M, int K,
                  int n_tiles_b0) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * kATileBytes;
  constexpr int kBTileBytes = BN * kBK * 2;
  GemmSmemTail* tail = reinterpret_cast<GemmSmemTail*>(sB + STAGES * kBTileBytes);
  volatile int* abort = &tail->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kBM;
  const int map_sel = (int)blockIdx.y >= n_tiles_b0 ? 1 : 0;
  const int n0 = (map_sel ? (int)blockIdx.y - n_tiles_b0 : (int)blockIdx.y) * BN;
  const CUtensorMap* mapB = map_sel ? &mapB1 : &mapB0;
  const int nk = K / kBK;
  constexpr uint32_t kTmemCols = BN < 32 ? 32 : BN;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&tail->full[s], 1);
      mbar_init(&tail->empty[s], 1);
    }
    mbar_init(&tail->accum, 1);
    tail->abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&mapA);
    tma_prefetch_desc(mapB);
  }
  if (warp == 1) tmem_alloc(&tail->tmem_base, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tail->tmem_base;

  if (warp == 0 && lane == 0) {
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % STAGES;
      const uint32_t ph = (kb / STAGES) & 1;
      if (kb >= STAGES && !mbar_wait(&tail->empty[s], ph ^ 1, abort, ep.err, kErrTimeoutGemm)) break;
      mbar_arrive_expect_tx(&tail->full[s], kATileBytes + kBTileBytes);
      tma_load_2d(sA + s * kATileBytes, &mapA, &tail->full[s], kb * kBK, m0);
      tma_load_2d(sB + s * kBTileBytes, mapB, &tail->full[s], kb * kBK, n0);
    }
  } else if (warp == 1 && lane == 0) {
    constexpr uint32_t idesc = idesc_bf16_f32(kBM, BN, false, false);
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % STAGES;
      const uint32_t ph = (kb / STAGES) & 1;
      if (!mbar_wait(&tail->full[s], ph, abort, ep.err, kErrTimeoutGemm)) break;
      tc_fence_after();
      const uint32_t a0 = smem_u32(sA + s * kATileBytes);
      const uint32_t b0 = smem_u32(sB + s * kBTileBytes);
#pragma unroll
      for (int kk = 0; kk < kBK / 16; ++kk) {
        umma_ss(tmem, sdesc_sw128(a0 + kk * 32, 16, 1024), sdesc_sw128(b0 + kk * 32, 16, 1024),
                idesc, (kb | kk) != 0);
      }
      umma_commit(&tail->empty[s]);
    }
    umma_commit(&tail->accum);
  } else if (warp >= 2) {
    const bool ok = mbar_wait(&tail->accum, 0, abort, ep.err, kErrTimeoutGemm);
    tc_fence_after();
    const int lg = warp & 3;
    const int row = m0 + lg * 32 + lane;
    const uint32_t trow = tmem + ((uint32_t)(lg * 32) << 16);
    epilogue_store<BN>(ep, map_sel, row, row, n0, trow, ok && row < M);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  drain_after_abort(abort);
}

// ---------------------------------------------------------------------------
// routed: A rows gathered per (group, expert) segment, W by TMA
template <int BN, int STAGES, int LAG>
__global__ void __launch_bounds__(kThreads, 1)
gemm_routed_kernel(const __grid_constant__ CUtensorMap mapWq,
                   const __grid_constant__ CUtensorMap mapWsh, const gqe_bf16_t* __restrict__ x,
                   RoutedParams rp, EpiParams ep_routed, EpiParams ep_shared) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * kATileBytes;
  constexpr int kBTileBytes = BN * kBK * 2;
  GemmSmemTail* tail = reinterpret_cast<GemmSmemTail*>(sB + STAGES * kBTileBytes);
  volatile int* abort = &tail->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x;
  const int K = rp.K;
  const int nk = K / kBK;

  // ---- which tile is this
  bool shared_tile = false;
  int seg = 0, row0 = 0, nrows = 0;
  if (tile < rp.max_routed_tiles) {
    const int total = rp.tile_start[rp.n_seg];
    if (tile >= total) return;            // unused upper-bound slot
    seg = 0;
    while (seg + 1 < rp.n_seg && rp.tile_start[seg + 1] <= tile) ++seg;
    const int local = tile - rp.tile_start[seg];
    row0 = rp.seg_off[seg] + local * kBM;
    nrows = min(kBM, rp.seg_cnt[seg] - local * kBM);
  } else {
    shared_tile = true;
    row0 = (tile - rp.max_routed_tiles) * kBM;
    nrows = min(kBM, rp.n_tokens - row0);
    if (nrows <= 0) return;
  }
  const CUtensorMap* mapB = shared_tile ? &mapWsh : &mapWq;
  const int nb0 = shared_tile ? 0 : seg * rp.d;

  constexpr uint32_t kTmemCols = BN < 32 ? 32 : BN;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&tail->full[s], 1 + 128);
      mbar_init(&tail->empty[s], 1);
    }
    mbar_init(&tail->accum, 1);
    tail->abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(mapB);
  }
  if (threadIdx.x < kBM) {
    const int r = threadIdx.x;
    int src = -1, dst = -1;
    if (r < nrows) {
      if (shared_tile) {
        src = row0 + r;
        dst = row0 + r;
      } else {
        src = rp.src_row[row0 + r];
        dst = rp.dst_row[row0 + r];
      }
    }
    tail->rowsrc[r] = src;
    tail->rowdst[r] = dst;
  }
  if (warp == 1) tmem_alloc(&tail->tmem_base, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tail->tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % STAGES;
        const uint32_t ph = (kb / STAGES) & 1;
        if (kb >= STAGES && !mbar_wait(&tail->empty[s], ph ^ 1, abort, ep_routed.err, kErrTimeoutGemm)) break;
        mbar_arrive_expect_tx(&tail->full[s], kBTileBytes);
        tma_load_2d(sB + s * kBTileBytes, mapB, &tail->full[s], kb * kBK, nb0);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kBM, BN, false, false);
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % STAGES;
        const uint32_t ph = (kb / STAGES) & 1;
        if (!mbar_wait(&tail->full[s], ph, abort, ep_routed.err, kErrTimeoutGemm)) break;
        tc_fence_after();
        const uint32_t a0 = smem_u32(sA + s * kATileBytes);
        const uint32_t b0 = smem_u32(sB + s * kBTileBytes);
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          umma_ss(tmem, sdesc_sw128(a0 + kk * 32, 16, 1024), sdesc_sw128(b0 + kk * 32, 16, 1024),
                  idesc, (kb | kk) != 0);
        }
        umma_commit(&tail->empty[s]);
      }
      umma_commit(&tail->accum);
    }
  } else {
    // ---- gather producers: 128 threads, 8 threads per 128-byte row segment
    const int t = threadIdx.x - 64;
    const int c = t & 7;
    const int rsub = t >> 3;
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % STAGES;
      const uint32_t ph = (kb / STAGES) & 1;
      if (kb >= STAGES && !mbar_wait(&tail->empty[s], ph ^ 1, abort, ep_routed.err, kErrTimeoutGemm)) break;
      uint8_t* st = sA + s * kATileBytes;
#pragma unroll
      for (int i = 0; i < kBM / 16; ++i) {
        const int r = rsub + 16 * i;
        const int src = tail->rowsrc[r];
        const gqe_bf16_t* g = x + (size_t)(src < 0 ? 0 : src) * K + kb * kBK + c * 8;
        cp_async_16(st + r * 128 + ((c ^ (r & 7)) << 4), g, src >= 0);
      }
      cp_async_commit();
      if (kb >= LAG) {
        cp_async_wait<LAG>();
        fence_proxy_async_smem();
        mbar_arrive(&tail->full[(kb - LAG) % STAGES]);
      }
    }
    cp_async_wait<0>();
    fence_proxy_async_smem();
    for (int kb = (nk > LAG ? nk - LAG : 0); kb < nk; ++kb) mbar_arrive(&tail->full[kb % STAGES]);

    // ---- epilogue
    const bool ok = mbar_wait(&tail->accum, 0, abort, ep_routed.err, kErrTimeoutGemm);
    tc_fence_after();
    const int lg = warp & 3;
    const int r = lg * 32 + lane;
    const int dst = tail->rowdst[r];
    const uint32_t trow = tmem + ((uint32_t)(lg * 32) << 16);
    epilogue_store<BN>(shared_tile ? ep_shared : ep_routed, 0, r, dst, 0, trow, ok && dst >= 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  drain_after_abort(abort);
}

}  // namespace

// ---------------------------------------------------------------------------
// host launchers

template <int BN, int STAGES>
static size_t dense_smem_bytes() {
  return 1024 + STAGES * (kATileBytes + BN * kBK * 2) + sizeof(GemmSmemTail);
}

cudaError_t launch_gemm_dense(const CUtensorMap& mapA, const CUtensorMap& mapB0,
                              const CUtensorMap& mapB1, const EpiParams& ep, int M, int K,
                              int n_tiles_b0, int n_tiles_total, cudaStream_t stream) {
  constexpr int BN = 128, STAGES = 4;
  const size_t smem = dense_smem_bytes<BN, STAGES>();
  auto kern = gemm_dense_kernel<BN, STAGES>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((M + kBM - 1) / kBM, n_tiles_total);
  kern<<<grid, kThreads, smem, stream>>>(mapA, mapB0, mapB1, ep, M, K, n_tiles_b0);
  return cudaGetLastError();
}

template <int BN>
static cudaError_t launch_routed_bn(const CUtensorMap& mapWq, const CUtensorMap& mapWsh,
                                    const gqe_bf16_t* x, const RoutedParams& rp,
                                    const EpiParams& epr, const EpiParams& eps, int grid,
                                    cudaStream_t stream) {
  constexpr int STAGES = 4, LAG = 2;
  const size_t smem = 1024 + STAGES * (kATileBytes + BN * kBK * 2) + sizeof(GemmSmemTail);
  auto kern = gemm_routed_kernel<BN, STAGES, LAG>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, smem, stream>>>(mapWq, mapWsh, x, rp, epr, eps);
  return cudaGetLastError();
}

cudaError_t launch_gemm_routed(const CUtensorMap& mapWq, const CUtensorMap& mapWsh,
                               const gqe_bf16_t* x, const RoutedParams& rp, const EpiParams& epr,
                               const EpiParams& eps, int grid, cudaStream_t stream) {
  if (rp.d == 64) return launch_routed_bn<64>(mapWq, mapWsh, x, rp, epr, eps, grid, stream);
  return launch_routed_bn<128>(mapWq, mapWsh, x, rp, epr, eps, grid, stream);
}

}  // namespace gqe
