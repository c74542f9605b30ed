// gemm.cu -- tcgen05 GEMMs of the GQE layer: C = A W^T, bf16 operands, fp32
// accumulation in tensor memory.
//
//   * dense path: A and W tiles by TMA (128-byte swizzle), used for the dense
//     K/V projection (written straight into the [B, G, T, d] head layout or
//     into a decode cache row) and for the output projection over the kG+2
//     slots ("GQE" study note §3-2 7));
//   * routed path: the A rows are gathered per (group, expert) segment of the
//     token-to-expert permutation with 16-byte cp.async (one 128-row tile of
//     one expert at a time), so only selected experts' query projections are
//     computed ("GQE" study note §3-2 2)); the shared head's projection rides
//     in the same launch as extra tiles.  (TMA tile::gather4 was measured 3.7x
//     slower here: 128-byte rows are too small a request for the TMA unit.)
//
// Both are persistent (one CTA per SM walks a static tile list) with two
// accumulators in tensor memory, so the epilogue of one tile overlaps the
// main loop of the next.
//
// Dense CTA (192 threads):  warp 0 TMA producer, warp 1 MMA issuer (and
//   tensor-memory owner), warps 2..5 epilogue (one output row per thread).
// Routed CTA (320 threads): warp 0 TMA producer of W, warp 1 MMA issuer,
//   warps 2..5 A-row gather producers, warps 6..9 epilogue.
#include "gemm.cuh"
#include "launch.cuh"

namespace gqe {

namespace {

constexpr int kBM = 128;
constexpr int kBK = 64;                 // 64 bf16 = one 128-byte swizzle row
constexpr int kATileBytes = kBM * kBK * 2;

struct __align__(8) GemmBarriers {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint32_t tmem_base;
  int abort;
};

// One 32-column chunk of an output row: fp32 from tensor memory -> bf16 -> global.
__device__ __forceinline__ void store_chunk(const EpiParams& ep, int map_sel, int row_dst, int n,
                                            const uint32_t* v) {
  uint32_t pk[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
  gqe_bf16_t* base = map_sel ? ep.out1 : ep.out0;
  gqe_bf16_t* dst;
  switch (ep.mode) {
    case kEpiHeads: {
      const int g = n / ep.d, dd = n % ep.d;
      const int b = row_dst / ep.T, t = row_dst % ep.T;
      dst = base + (((size_t)b * ep.G + g) * ep.T + t) * ep.d + dd;
      break;
    }
    case kEpiCacheRow: {
      const int g = n / ep.d, dd = n % ep.d;
      const int pos = ep.cache_len[row_dst] - 1;
      dst = base + (((size_t)row_dst * ep.G + g) * ep.L_max + pos) * ep.d + dd;
      break;
    }
    default:  // kEpiRowMajor, kEpiRows
      dst = base + (size_t)row_dst * ep.ldo + n;
      break;
  }
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i) d4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
}

template <int BN>
__device__ __forceinline__ void epilogue_tile(const EpiParams& ep, int map_sel, int row_dst, int n0,
                                              uint32_t tmem_row, bool valid) {
#pragma unroll 1
  for (int c0 = 0; c0 < BN; c0 += 32) {
    uint32_t v[32];
    tmem_ld32(tmem_row + c0, v);
    if (valid && n0 + c0 < ep.n_limit) store_chunk(ep, map_sel, row_dst, n0 + c0, v);
  }
}

// Coalesced epilogue: each 64-column chunk of the warp's 32 rows goes through
// a 4 KB 128-byte-swizzled staging buffer (two per warp, alternating) and out
// with one TMA store; rows past the output are clipped by the tensor map.
constexpr int kStageOutBytes = 32 * 64 * 2;
constexpr int kEpiStagingBytes = 4 * 2 * kStageOutBytes;   // four epilogue warps

// fp32 partial tiles (one K slice each) reduce-added into an fp32 [M, N]
// tensor: 32 columns of the warp's 32 rows per 4 KB staging buffer.
template <int BN>
__device__ __forceinline__ void epilogue_tile_reduce(const EpiParams& ep, const CUtensorMap* mo, int row0, int n0,
                                                     uint32_t tmem_row, uint8_t* stg, int& chunk, bool ok) {
  const int lane = threadIdx.x & 31;
#pragma unroll 1
  for (int c0 = 0; c0 < BN; c0 += 32) {
    if (n0 + c0 >= ep.n_limit) break;
    uint32_t v[32];
    tmem_ld32(tmem_row + c0, v);
    if (!ok) continue;
    uint8_t* buf = stg + (chunk & 1) * kStageOutBytes;
    if (chunk >= 2) {
      if (lane == 0) bulk_wait_read<1>();
      __syncwarp();
    }
#pragma unroll
    for (int j = 0; j < 8; ++j)
      st_shared_v4(buf + lane * 128 + ((j ^ (lane & 7)) << 4), v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_reduce_add_2d(mo, buf, n0 + c0, row0);
      bulk_commit();
    }
    ++chunk;
  }
}

template <int BN>
__device__ __forceinline__ void epilogue_tile_tma(const EpiParams& ep, const CUtensorMap* mo, int row0, int n0,
                                                  uint32_t tmem_row, uint8_t* stg, int& chunk, bool ok) {
  if (ep.store_mode == kStoreReduceF32) {
    epilogue_tile_reduce<BN>(ep, mo, row0, n0, tmem_row, stg, chunk, ok);
    return;
  }
  const int lane = threadIdx.x & 31;
#pragma unroll 1
  for (int c0 = 0; c0 < BN; c0 += 64) {
    if (n0 + c0 >= ep.n_limit) break;
    uint32_t v[64];
    tmem_ld64(tmem_row + c0, v);
    if (!ok) continue;
    uint8_t* buf = stg + (chunk & 1) * kStageOutBytes;
    if (chunk >= 2) {
      if (lane == 0) bulk_wait_read<1>();   // the store that used this buffer has read it
      __syncwarp();
    }
#pragma unroll
    for (int j = 0; j < 8; ++j)
      st_shared_v4(buf + lane * 128 + ((j ^ (lane & 7)) << 4), pack_bf16x2(__uint_as_float(v[8 * j]), __uint_as_float(v[8 * j + 1])),
                   pack_bf16x2(__uint_as_float(v[8 * j + 2]), __uint_as_float(v[8 * j + 3])),
                   pack_bf16x2(__uint_as_float(v[8 * j + 4]), __uint_as_float(v[8 * j + 5])),
                   pack_bf16x2(__uint_as_float(v[8 * j + 6]), __uint_as_float(v[8 * j + 7])));
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      const int n = n0 + c0;
      if (ep.store_mode == kStoreTma2d) {
        tma_store_2d(mo, buf, n, row0);
      } else {
        const int b = row0 / ep.T, t = row0 - b * ep.T;
        tma_store_3d(mo, buf, n % ep.d, t, b * ep.G + n / ep.d);
      }
      bulk_commit();
    }
    ++chunk;
  }
}

// ---------------------------------------------------------------------------
// Operand majorness.  K-major (the default): a tile of rows x 64 k, one 128-byte
// row per M (N) index.  MN-major (kMnA / kMnB): the operand is stored [K, M]
// ([K, N]) and comes in as 64-column boxes of 64 k rows, 8 KB each, so a
// 16-deep k-step is 16 rows (2 KB) further on and the 64-wide M (N) atoms are
// kMnBox apart.
constexpr int kMnA = 1, kMnB = 2;
constexpr int kMnBox = 64 * 64 * 2;

__device__ __forceinline__ uint64_t operand_desc(uint32_t base, int kk, int mn_major) {
  return mn_major ? sdesc_sw128(base + kk * 2048, kMnBox, 1024) : sdesc_sw128(base + kk * 32, 16, 1024);
}

// ---------------------------------------------------------------------------
// dense: A [M, K] and W [N, K] by TMA; persistent over (m-tile, n-tile)
template <int BN, int STAGES, int mn>
__global__ void __launch_bounds__(192, 1)
gemm_dense_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB0,
                  const __grid_constant__ CUtensorMap mapB1, const __grid_constant__ CUtensorMap mapO0,
                  const __grid_constant__ CUtensorMap mapO1, EpiParams ep, int M, int K, int n_tiles_b0,
                  int n_tiles_total) {
  constexpr int kBTileBytes = BN * kBK * 2;
  constexpr uint32_t kTmemCols = 2 * BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * kATileBytes;
  uint8_t* sOut = sB + STAGES * kBTileBytes;
  GemmBarriers* bar = reinterpret_cast<GemmBarriers*>(sOut + kEpiStagingBytes);
  volatile int* abort = &bar->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = K / kBK;
  const int m_tiles = (M + kBM - 1) / kBM;
  const int ks_n = ep.ksplit > 1 ? ep.ksplit : 1;   // K split (fp32 reduce-add epilogue)
  const int total = m_tiles * n_tiles_total * ks_n;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&bar->full[s], 1);
      mbar_init(&bar->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&bar->acc_full[a], 1);
      mbar_init(&bar->acc_empty[a], 4);
    }
    bar->abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&mapA);
    tma_prefetch_desc(&mapB0);
    tma_prefetch_desc(&mapB1);
  }
  if (warp == 1) tmem_alloc(&bar->tmem_base, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;
  pdl_launch_dependents();
  pdl_wait();

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;
      for (int t = blockIdx.x; t < total && !*abort; t += gridDim.x) {
        const int ks = t % ks_n, tt = t / ks_n;
        const int mt = tt / n_tiles_total, nt = tt % n_tiles_total;
        const int kb0 = (int)((long long)nk * ks / ks_n), kb1 = (int)((long long)nk * (ks + 1) / ks_n);
        const int sel = nt >= n_tiles_b0;
        const CUtensorMap* mB = sel ? &mapB1 : &mapB0;
        const int n0 = (sel ? nt - n_tiles_b0 : nt) * BN;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % STAGES;
          if (it >= STAGES && !mbar_wait(&bar->empty[s], ((it / STAGES) & 1) ^ 1, abort, ep.err, kErrTimeoutGemm))
            break;
          mbar_arrive_expect_tx(&bar->full[s], kATileBytes + kBTileBytes);
          if constexpr ((mn & kMnA) != 0) {
            for (int h = 0; h < kBM / 64; ++h)
              tma_load_2d(sA + s * kATileBytes + h * kMnBox, &mapA, &bar->full[s], mt * kBM + h * 64, kb * kBK);
          } else {
            tma_load_2d(sA + s * kATileBytes, &mapA, &bar->full[s], kb * kBK, mt * kBM);
          }
          if constexpr ((mn & kMnB) != 0) {
            for (int h = 0; h < BN / 64; ++h)
              tma_load_2d(sB + s * kBTileBytes + h * kMnBox, mB, &bar->full[s], n0 + h * 64, kb * kBK);
          } else {
            tma_load_2d(sB + s * kBTileBytes, mB, &bar->full[s], kb * kBK, n0);
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kBM, BN, (mn & kMnA) != 0, (mn & kMnB) != 0);
      int it = 0, tc = 0;
      for (int t = blockIdx.x; t < total && !*abort; t += gridDim.x, ++tc) {
        const int ab = tc & 1, use = tc >> 1;
        const int ks = t % ks_n;
        const int kb0 = (int)((long long)nk * ks / ks_n), kb1 = (int)((long long)nk * (ks + 1) / ks_n);
        if (tc >= 2 && !mbar_wait(&bar->acc_empty[ab], (use & 1) ^ 1, abort, ep.err, kErrTimeoutGemm)) break;
        tc_fence_after();
        const uint32_t acc = tmem + (uint32_t)(ab * BN);
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(&bar->full[s], (it / STAGES) & 1, abort, ep.err, kErrTimeoutGemm)) break;
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + s * kATileBytes);
          const uint32_t b0 = smem_u32(sB + s * kBTileBytes);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            umma_ss(acc, operand_desc(a0, kk, mn & kMnA), operand_desc(b0, kk, mn & kMnB), idesc, (kb != kb0 || kk != 0));
          umma_commit(&bar->empty[s]);
        }
        umma_commit(&bar->acc_full[ab]);
      }
    }
  } else {
    const int lg = warp & 3;
    const uint32_t lane_off = (uint32_t)(lg * 32) << 16;
    uint8_t* stg = sOut + lg * 2 * kStageOutBytes;
    int tc = 0, chunk = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++tc) {
      const int ab = tc & 1, use = tc >> 1;
      const bool ok = mbar_wait(&bar->acc_full[ab], use & 1, abort, ep.err, kErrTimeoutGemm);
      tc_fence_after();
      const int tt = t / ks_n;   // the K slice (t % ks_n) does not change where the tile goes
      const int mt = tt / n_tiles_total, nt = tt % n_tiles_total;
      const int sel = nt >= n_tiles_b0;
      const int n0 = (sel ? nt - n_tiles_b0 : nt) * BN;
      const int row = mt * kBM + lg * 32 + lane;
      const uint32_t tacc = tmem + lane_off + (uint32_t)(ab * BN);
      if (ep.store_mode != kStorePerThread)
        epilogue_tile_tma<BN>(ep, sel ? &mapO1 : &mapO0, mt * kBM + lg * 32, n0, tacc, stg, chunk, ok);
      else
        epilogue_tile<BN>(ep, sel, row, n0, tacc, ok && row < M);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar->acc_empty[ab]);
      if (!ok) break;
    }
    if (lane == 0) bulk_wait<0>();
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
// dense, CTA pairs: one 256 x 256 output tile per pair and step, issued as
// M = 256 tcgen05 MMAs over both SMs.  Each CTA loads 128 rows of A and 128
// rows of W per k-block (32 KB) where the single-CTA 128 x 256 tile loads
// 16 + 32 KB for the same MMA work: a third fewer bytes through L2 per FLOP.
// Both CTAs' loads count on the even CTA's `full` barrier; the even CTA's MMA
// thread releases stages and accumulators in both CTAs with one commit each.
template <int BN, int STAGES, int mn>
__global__ void __launch_bounds__(192, 1)
gemm_dense_pair_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapR,
                       const __grid_constant__ CUtensorMap mapS, ASource as,
                       const __grid_constant__ CUtensorMap mapB0,
                       const __grid_constant__ CUtensorMap mapB1, const __grid_constant__ CUtensorMap mapO0,
                       const __grid_constant__ CUtensorMap mapO1, EpiParams ep, int M, int K, int n_tiles_b0,
                       int n_tiles_total) {
  constexpr int kPM = 2 * kBM;                       // pair tile rows
  constexpr int kHalfB = (BN / 2) * kBK * 2;         // this CTA's half of the W k-block
  constexpr uint32_t kTmemCols = 2 * BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * kATileBytes;
  uint8_t* sOut = sB + STAGES * kHalfB;
  GemmBarriers* bar = reinterpret_cast<GemmBarriers*>(sOut + kEpiStagingBytes);
  volatile int* abort = &bar->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  const int nk = K / kBK;
  const int m_tiles = (M + kPM - 1) / kPM;
  const int ks_n = ep.ksplit > 1 ? ep.ksplit : 1;   // K split (fp32 reduce-add epilogue)
  const int total = m_tiles * n_tiles_total * ks_n;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&bar->full[s], 1);      // used in the even CTA only
      mbar_init(&bar->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&bar->acc_full[a], 1);
      mbar_init(&bar->acc_empty[a], 8);  // even CTA: 4 epilogue warps of each CTA
    }
    bar->abort = 0;
    fence_mbar_init_cluster();
    tma_prefetch_desc(&mapA);
    if (as.mode == kASlots) {
      tma_prefetch_desc(&mapR);
      tma_prefetch_desc(&mapS);
    }
    tma_prefetch_desc(&mapB0);
    tma_prefetch_desc(&mapB1);
  }
  if (warp == 1) tmem_alloc_pair(&bar->tmem_base, kTmemCols);
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;
  pdl_launch_dependents();
  pdl_wait();

  if (warp == 0) {
    if (lane == 0) {
      const uint32_t full0 = cluster_addr(&bar->full[0], 0);
      int it = 0;
      for (int t = pair; t < total && !*abort; t += n_pairs) {
        const int ks = t % ks_n, tt = t / ks_n;
        const int mt = tt / n_tiles_total, nt = tt % n_tiles_total;
        const int kb0 = (int)((long long)nk * ks / ks_n), kb1 = (int)((long long)nk * (ks + 1) / ks_n);
        const int sel = nt >= n_tiles_b0;
        const CUtensorMap* mB = sel ? &mapB1 : &mapB0;
        const int n0 = (sel ? nt - n_tiles_b0 : nt) * BN + (int)rank * (BN / 2);
        const int m0 = mt * kPM + (int)rank * kBM;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % STAGES;
          if (it >= STAGES && !mbar_wait(&bar->empty[s], ((it / STAGES) & 1) ^ 1, abort, ep.err, kErrTimeoutGemm))
            break;
          if (rank == 0) mbar_arrive_expect_tx(&bar->full[s], 2 * (kATileBytes + kHalfB));
          const uint32_t fb = full0 + (uint32_t)(s * sizeof(uint64_t));
          if ((mn & kMnA) != 0 && as.mode == kASingle) {
            for (int h = 0; h < kBM / 64; ++h)
              tma_load_2d_pair(sA + s * kATileBytes + h * kMnBox, &mapA, fb, m0 + h * 64, kb * kBK);
          } else if (as.mode == kASingle) {
            tma_load_2d_pair(sA + s * kATileBytes, &mapA, fb, kb * kBK, m0);
          } else {
            const int col = kb * kBK, slot = col / as.d, sub = col - slot * as.d;
            const int kG = as.k * as.G;
            if (slot < kG) {
              // o_routed as [B*G*T, k*d]: the 128 tokens of this box share (b, g)
              const int g = slot / as.k, kk = slot - g * as.k;
              const int b = m0 / as.T, t = m0 - b * as.T;
              tma_load_2d_pair(sA + s * kATileBytes, &mapA, fb, kk * as.d + sub, (b * as.G + g) * as.T + t);
            } else {
              tma_load_2d_pair(sA + s * kATileBytes, (slot == kG && as.route) ? &mapR : &mapS, fb, sub, m0);
            }
          }
          if constexpr ((mn & kMnB) != 0) {
            for (int h = 0; h < BN / 128; ++h)
              tma_load_2d_pair(sB + s * kHalfB + h * kMnBox, mB, fb, n0 + h * 64, kb * kBK);
          } else {
            tma_load_2d_pair(sB + s * kHalfB, mB, fb, kb * kBK, n0);
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kPM, BN, (mn & kMnA) != 0, (mn & kMnB) != 0);
      const uint32_t empty_peer0 = cluster_addr(&bar->empty[0], peer);
      const uint32_t accf_peer0 = cluster_addr(&bar->acc_full[0], peer);
      int it = 0, tc = 0;
      for (int t = pair; t < total && !*abort; t += n_pairs, ++tc) {
        const int ab = tc & 1, use = tc >> 1;
        const int ks = t % ks_n;
        const int kb0 = (int)((long long)nk * ks / ks_n), kb1 = (int)((long long)nk * (ks + 1) / ks_n);
        if (tc >= 2 && !mbar_wait(&bar->acc_empty[ab], (use & 1) ^ 1, abort, ep.err, kErrTimeoutGemm)) break;
        tc_fence_after();
        const uint32_t acc = tmem + (uint32_t)(ab * BN);
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(&bar->full[s], (it / STAGES) & 1, abort, ep.err, kErrTimeoutGemm)) break;
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + s * kATileBytes);
          const uint32_t b0 = smem_u32(sB + s * kHalfB);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            umma_ss_pair(acc, operand_desc(a0, kk, mn & kMnA), operand_desc(b0, kk, mn & kMnB), idesc,
                         (kb != kb0 || kk != 0));
          umma_commit_pair(smem_u32(&bar->empty[s]));
          umma_commit_pair(empty_peer0 + (uint32_t)(s * sizeof(uint64_t)));
        }
        umma_commit_pair(smem_u32(&bar->acc_full[ab]));
        umma_commit_pair(accf_peer0 + (uint32_t)(ab * sizeof(uint64_t)));
      }
    }
  } else {
    const int lg = warp & 3;
    const uint32_t lane_off = (uint32_t)(lg * 32) << 16;
    const uint32_t acce0 = cluster_addr(&bar->acc_empty[0], 0);
    uint8_t* stg = sOut + lg * 2 * kStageOutBytes;
    int tc = 0, chunk = 0;
    for (int t = pair; t < total; t += n_pairs, ++tc) {
      const int ab = tc & 1, use = tc >> 1;
      const bool ok = mbar_wait(&bar->acc_full[ab], use & 1, abort, ep.err, kErrTimeoutGemm);
      tc_fence_after();
      const int tt = t / ks_n;   // the K slice (t % ks_n) does not change where the tile goes
      const int mt = tt / n_tiles_total, nt = tt % n_tiles_total;
      const int sel = nt >= n_tiles_b0;
      const int n0 = (sel ? nt - n_tiles_b0 : nt) * BN;
      const int row0 = mt * kPM + (int)rank * kBM + lg * 32;
      const uint32_t tacc = tmem + lane_off + (uint32_t)(ab * BN);
      if (ep.store_mode != kStorePerThread)
        epilogue_tile_tma<BN>(ep, sel ? &mapO1 : &mapO0, row0, n0, tacc, stg, chunk, ok);
      else
        epilogue_tile<BN>(ep, sel, row0 + lane, n0, tacc, ok && row0 + lane < M);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acce0 + (uint32_t)(ab * sizeof(uint64_t)));
      if (!ok) break;
    }
    if (lane == 0) bulk_wait<0>();
  }
  // an aborted CTA lets copies in flight land before its pair partner may exit
  drain_after_abort(abort);
  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// routed: A rows gathered per (group, expert) segment, W by TMA; persistent
struct RoutedTile {
  int shared;   // 0 routed, 1 shared head
  int seg;
  int row0;     // first permutation entry (routed) or token row (shared)
  int nrows;
};

// Segment tables staged in shared memory once per CTA (a tile's segment is
// found by a scan that would otherwise cost one global load per step).
struct SegTables {
  int tile_start[65];
  int seg_off[64];
  int seg_cnt[64];
};

__device__ __forceinline__ RoutedTile routed_tile(const RoutedParams& rp, const SegTables& st, int t,
                                                  int n_routed) {
  RoutedTile r{};
  if (t < n_routed) {
    int s = 0;
    while (s + 1 < rp.n_seg && st.tile_start[s + 1] <= t) ++s;
    const int local = t - st.tile_start[s];
    r.shared = 0;
    r.seg = s;
    r.row0 = st.seg_off[s] + local * kBM;
    r.nrows = min(kBM, st.seg_cnt[s] - local * kBM);
  } else {
    r.shared = 1;
    r.seg = 0;
    r.row0 = (t - n_routed) * kBM;
    r.nrows = min(kBM, rp.n_tokens - r.row0);
  }
  return r;
}

template <int BN, int STAGES, int CPS>
__global__ void __launch_bounds__(320, CPS)
gemm_routed_kernel(const __grid_constant__ CUtensorMap mapWq, const __grid_constant__ CUtensorMap mapWsh,
                   const gqe_bf16_t* __restrict__ x, RoutedParams rp, EpiParams ep_routed, EpiParams ep_shared) {
  constexpr int kBTileBytes = BN * kBK * 2;
  constexpr uint32_t kTmemCols = 2 * BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * kATileBytes;
  GemmBarriers* bar = reinterpret_cast<GemmBarriers*>(sB + STAGES * kBTileBytes);
  SegTables* seg = reinterpret_cast<SegTables*>(bar + 1);
  volatile int* abort = &bar->abort;
  unsigned* err = ep_routed.err;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = rp.K;
  const int nk = K / kBK;
  pdl_launch_dependents();
  pdl_wait();
  for (int i = threadIdx.x; i < rp.n_seg; i += blockDim.x) {
    const int c = rp.seg_cnt[i];
    seg->seg_cnt[i] = c;
    seg->seg_off[i] = i * rp.seg_cap;
    if (blockIdx.x == 0 && rp.expert_counts) rp.expert_counts[i] = c;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int tiles = 0;
    for (int i = 0; i < rp.n_seg; ++i) {
      seg->tile_start[i] = tiles;
      tiles += (seg->seg_cnt[i] + kBM - 1) / kBM;
    }
    seg->tile_start[rp.n_seg] = tiles;
  }
  __syncthreads();
  const int n_routed = seg->tile_start[rp.n_seg];
  const int total = n_routed + rp.shared_tiles;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&bar->full[s], 1 + 128);
      mbar_init(&bar->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&bar->acc_full[a], 1);
      mbar_init(&bar->acc_empty[a], 4);
    }
    bar->abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&mapWq);
    tma_prefetch_desc(&mapWsh);
  }
  if (warp == 1) tmem_alloc(&bar->tmem_base, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;
      for (int t = blockIdx.x; t < total && !*abort; t += gridDim.x) {
        const RoutedTile tl = routed_tile(rp, *seg, t, n_routed);
        const CUtensorMap* mB = tl.shared ? &mapWsh : &mapWq;
        const int nb0 = tl.shared ? 0 : tl.seg * rp.d;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % STAGES;
          if (it >= STAGES && !mbar_wait(&bar->empty[s], ((it / STAGES) & 1) ^ 1, abort, err, kErrTimeoutGemm))
            break;
          mbar_arrive_expect_tx(&bar->full[s], kBTileBytes);
          tma_load_2d(sB + s * kBTileBytes, mB, &bar->full[s], kb * kBK, nb0);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kBM, BN, false, false);
      int it = 0, tc = 0;
      for (int t = blockIdx.x; t < total && !*abort; t += gridDim.x, ++tc) {
        const int ab = tc & 1, use = tc >> 1;
        if (tc >= 2 && !mbar_wait(&bar->acc_empty[ab], (use & 1) ^ 1, abort, err, kErrTimeoutGemm)) break;
        tc_fence_after();
        const uint32_t acc = tmem + (uint32_t)(ab * BN);
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(&bar->full[s], (it / STAGES) & 1, abort, err, kErrTimeoutGemm)) break;
          fence_proxy_async_smem();
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + s * kATileBytes);
          const uint32_t b0 = smem_u32(sB + s * kBTileBytes);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            umma_ss(acc, sdesc_sw128(a0 + kk * 32, 16, 1024), sdesc_sw128(b0 + kk * 32, 16, 1024), idesc,
                    (kb | kk) != 0);
          umma_commit(&bar->empty[s]);
        }
        umma_commit(&bar->acc_full[ab]);
      }
    }
  } else if (warp < 6) {
    // ---- gather producers: 128 threads, 8 threads per 128-byte row segment
    const int tg = threadIdx.x - 64;
    const int c = tg & 7;
    const int rsub = tg >> 3;
    int it = 0;
    for (int t = blockIdx.x; t < total && !*abort; t += gridDim.x) {
      const RoutedTile tl = routed_tile(rp, *seg, t, n_routed);
      int src[kBM / 16];
#pragma unroll
      for (int i = 0; i < kBM / 16; ++i) {
        const int r = rsub + 16 * i;
        src[i] = r < tl.nrows ? (tl.shared ? tl.row0 + r : rp.src_row[tl.row0 + r]) : -1;
      }
      for (int kb = 0; kb < nk; ++kb, ++it) {
        const int s = it % STAGES;
        if (it >= STAGES && !mbar_wait(&bar->empty[s], ((it / STAGES) & 1) ^ 1, abort, err, kErrTimeoutGemm))
          break;
        uint8_t* st = sA + s * kATileBytes;
#pragma unroll
        for (int i = 0; i < kBM / 16; ++i) {
          const int r = rsub + 16 * i;
          const gqe_bf16_t* g = x + (size_t)(src[i] < 0 ? 0 : src[i]) * K + kb * kBK + c * 8;
          cp_async_16(st + r * 128 + ((c ^ (r & 7)) << 4), g, src[i] >= 0);
        }
        // the stage's barrier hears from this thread once its copies land; the
        // MMA thread makes them visible to the tensor core's (async) proxy
        cp_async_arrive_noinc(&bar->full[s]);
      }
    }
    cp_async_wait<0>();
  } else {
    // ---- epilogue: warps 6..9, tensor-memory lane quarters 2, 3, 0, 1
    const int lg = warp & 3;
    const uint32_t lane_off = (uint32_t)(lg * 32) << 16;
    int tc = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++tc) {
      const RoutedTile tl = routed_tile(rp, *seg, t, n_routed);
      const int ab = tc & 1, use = tc >> 1;
      const int r = lg * 32 + lane;
      int dst = -1;
      if (r < tl.nrows) dst = tl.shared ? tl.row0 + r : rp.dst_row[tl.row0 + r];
      const bool ok = mbar_wait(&bar->acc_full[ab], use & 1, abort, err, kErrTimeoutGemm);
      tc_fence_after();
      epilogue_tile<BN>(tl.shared ? ep_shared : ep_routed, 0, dst, 0, tmem + lane_off + (uint32_t)(ab * BN),
                        ok && dst >= 0);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar->acc_empty[ab]);
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

}  // namespace

// ---------------------------------------------------------------------------
// host launchers

template <int BN, int STAGES>
static cudaError_t launch_dense_bn(const CUtensorMap& mapA, const CUtensorMap& mapB0, const CUtensorMap& mapB1,
                                   const CUtensorMap& mapO0, const CUtensorMap& mapO1, const EpiParams& ep, int M,
                                   int K, int n_tiles_b0, int n_tiles_total, cudaStream_t stream, int mn) {
  const size_t smem = 1024 + STAGES * (kATileBytes + BN * kBK * 2) + kEpiStagingBytes + sizeof(GemmBarriers);
  auto kern = mn == 3   ? gemm_dense_kernel<BN, STAGES, 3>
              : mn == 2 ? gemm_dense_kernel<BN, STAGES, 2>
              : mn == 1 ? gemm_dense_kernel<BN, STAGES, 1>
                        : gemm_dense_kernel<BN, STAGES, 0>;
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  const int tiles = ((M + kBM - 1) / kBM) * n_tiles_total * (ep.ksplit > 1 ? ep.ksplit : 1);
  const int grid = tiles < num_sms() ? tiles : num_sms();
  return launch_kernel(kern, dim3(grid), dim3(192), smem, stream, 1, mapA, mapB0, mapB1, mapO0, mapO1, ep, M, K,
                       n_tiles_b0, n_tiles_total);
}

template <int BN, int STAGES>
static cudaError_t launch_dense_pair_st(const CUtensorMap& mapA, const CUtensorMap& mapR, const CUtensorMap& mapS,
                                        const ASource& as, const CUtensorMap& mapB0, const CUtensorMap& mapB1,
                                        const CUtensorMap& mapO0, const CUtensorMap& mapO1, const EpiParams& ep,
                                        int M, int K, int n_tiles_b0, int n_tiles_total, cudaStream_t stream,
                                        int mn) {
  const size_t smem = 1024 + STAGES * (kATileBytes + (BN / 2) * kBK * 2) + kEpiStagingBytes + sizeof(GemmBarriers);
  auto kern = mn == 3   ? gemm_dense_pair_kernel<BN, STAGES, 3>
              : mn == 2 ? gemm_dense_pair_kernel<BN, STAGES, 2>
              : mn == 1 ? gemm_dense_pair_kernel<BN, STAGES, 1>
                        : gemm_dense_pair_kernel<BN, STAGES, 0>;
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(192, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // co-resident pairs on this device (a cluster needs both SMs in one GPC)
  static int max_pairs[64] = {0};   // per instantiation (static in the template)
  int dev = 0;
  cudaGetDevice(&dev);
  int& mp = max_pairs[dev & 63];
  if (mp <= 0) {
    cfg.gridDim = dim3(2 * (num_sms() / 2), 1, 1);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, reinterpret_cast<const void*>(kern), &cfg) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = num_sms() / 2;
    }
    mp = n;
  }
  const int total = ((M + 255) / 256) * n_tiles_total * (ep.ksplit > 1 ? ep.ksplit : 1);
  const int pairs = total < mp ? total : mp;
  return launch_kernel(kern, dim3(2 * pairs), dim3(192), smem, stream, 2, mapA, mapR, mapS, as, mapB0, mapB1,
                       mapO0, mapO1, ep, M, K, n_tiles_b0, n_tiles_total);
}

cudaError_t launch_gemm_dense_pair(const CUtensorMap& mapA, const CUtensorMap& mapR, const CUtensorMap& mapS,
                                   const ASource& as, const CUtensorMap& mapB0, const CUtensorMap& mapB1,
                                   const CUtensorMap& mapO0, const CUtensorMap& mapO1, const EpiParams& ep, int M,
                                   int K, int n_tiles_b0, int n_tiles_total, int bn, cudaStream_t stream, int mn) {
  if (bn != 256) return cudaErrorInvalidValue;
  return launch_dense_pair_st<256, 6>(mapA, mapR, mapS, as, mapB0, mapB1, mapO0, mapO1, ep, M, K, n_tiles_b0,
                                      n_tiles_total, stream, mn);
}

int num_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  }
  return n;
}

// Output tile width of the single-CTA dense GEMM.  With all rows in one
// 128-row tile (the decode step's M = batch), 64-column tiles put four times
// as many CTAs on the weight stream as 256-column ones.
int dense_tile_n(int n_per_weight, int M) {
  if (M <= kBM && n_per_weight % 64 == 0) return 64;
  return (n_per_weight % 256 == 0) ? 256 : 128;
}

cudaError_t launch_gemm_dense(const CUtensorMap& mapA, const CUtensorMap& mapB0, const CUtensorMap& mapB1,
                              const CUtensorMap& mapO0, const CUtensorMap& mapO1, const EpiParams& ep, int M, int K,
                              int n_tiles_b0, int n_tiles_total, int bn, cudaStream_t stream, int mn) {
  if (bn == 256)
    return launch_dense_bn<256, 4>(mapA, mapB0, mapB1, mapO0, mapO1, ep, M, K, n_tiles_b0, n_tiles_total, stream, mn);
  if (bn == 64)
    return launch_dense_bn<64, 7>(mapA, mapB0, mapB1, mapO0, mapO1, ep, M, K, n_tiles_b0, n_tiles_total, stream, mn);
  return launch_dense_bn<128, 6>(mapA, mapB0, mapB1, mapO0, mapO1, ep, M, K, n_tiles_b0, n_tiles_total, stream, mn);
}

template <int BN, int STAGES, int CPS>
static cudaError_t launch_routed_bn(const CUtensorMap& mapWq, const CUtensorMap& mapWsh, const gqe_bf16_t* x,
                                    const RoutedParams& rp, const EpiParams& epr, const EpiParams& eps,
                                    cudaStream_t stream) {
  const size_t smem = 1024 + STAGES * (kATileBytes + BN * kBK * 2) + sizeof(GemmBarriers) + sizeof(SegTables);
  auto kern = gemm_routed_kernel<BN, STAGES, CPS>;
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  const int max_tiles = rp.max_routed_tiles + rp.shared_tiles;
  const int slots = CPS * num_sms();
  const int grid = max_tiles < slots ? max_tiles : slots;
  return launch_kernel(kern, dim3(grid), dim3(320), smem, stream, 1, mapWq, mapWsh, x, rp, epr, eps);
}

// Ring depth and CTAs per SM of the routed GEMM.  A tcgen05.mma of N = 64 or
// 128 keeps the tensor pipe busy for less time than one issuing thread needs
// per instruction (about 100 cycles), so several CTAs per SM, each with its
// own MMA thread, feed the pipe where one cannot (measured on B200, d = 64:
// 1 CTA x 8 stages 73 us, 2 x 4 54 us, 3 x 3 49 us, 4 x 2 49 us).
#ifndef GQE_ROUTED64_ST
#define GQE_ROUTED64_ST 3
#endif
#ifndef GQE_ROUTED64_CPS
#define GQE_ROUTED64_CPS 3
#endif
// d = 128 (wide/skewed, routed call alone): 3 stages x 2 CTAs 341 us; 2 x 3
// 484, 6 x 1 410, 4 x 1 444 us.
#ifndef GQE_ROUTED128_ST
#define GQE_ROUTED128_ST 3
#endif
#ifndef GQE_ROUTED128_CPS
#define GQE_ROUTED128_CPS 2
#endif

cudaError_t launch_gemm_routed(const CUtensorMap& mapWq, const CUtensorMap& mapWsh, const gqe_bf16_t* x,
                               const RoutedParams& rp, const EpiParams& epr, const EpiParams& eps,
                               cudaStream_t stream) {
  if (rp.d == 64) return launch_routed_bn<64, GQE_ROUTED64_ST, GQE_ROUTED64_CPS>(mapWq, mapWsh, x, rp, epr, eps, stream);
  return launch_routed_bn<128, GQE_ROUTED128_ST, GQE_ROUTED128_CPS>(mapWq, mapWsh, x, rp, epr, eps, stream);
}

}  // namespace gqe
