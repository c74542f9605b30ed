// attn_bwd.cu -- backward of the routed causal attention on tcgen05.
//
// The forward is o = softmax(q K^T * scale) V per selected (token, expert) row
// of a KV group and per shared-head row of group sg ("GQE" study note §1-1 and
// §3-2 2), 5)).  With P the softmax, dO the upstream gradient and
// Delta_r = sum_c dO_rc O_rc:
//   dV = P^T dO,  dP = dO V^T,  dS = scale * P o (dP - Delta),
//   dK = dS^T q,  dq = dS K.
//
// Work item: one 128-key tile j of one KV sequence (b, g).  The CTA keeps K_j,
// V_j in shared memory and dK_j, dV_j in tensor memory, and walks every query
// tile that sees key tile j: the packed rows of (b, g) from token 128 j on and,
// when g is the shared head's group, the shared head's rows too.  For each
// query tile i (128 packed rows, TMA-loaded with dO_i, its LSE and Delta):
//   S^T  = K_j Q_i^T          (tensor memory, keys in lanes)
//   dP^T = V_j dO_i^T
//   P^T  = exp2(S^T * scale*log2e - LSE2_i), causal mask  -> bf16 over S^T
//   dV  += P^T dO_i            (A operand from tensor memory)
//   dS^T = scale * P^T o (dP^T - Delta_i)                 -> bf16 over dP^T,
//                                                            and into smem
//   dK  += dS^T Q_i            (A operand from tensor memory)
//   dQ_i = dS K_j              (A = dS^T read MN-major from smem)
// dQ_i leaves through a TMA reduce-add into an fp32 workspace (several key
// tiles add to the same query tile); a last kernel rounds it to bf16.
//
// CTA: 512 threads.  warp 0 TMA producer; warp 1 issues S, dP, dV (and owns
// tensor memory); warp 2 issues dK, dQ; warp 3 idle; warps 4-7 and 8-11 are
// two warpgroups computing P and dS, one key row per thread, warpgroup w on
// query columns [64 w, 64 w + 64) (two warps per SM sub-partition hide each
// other's latency); warps 12-15 drain dQ and write dK, dV at the end.
// Tensor memory (d = 64): S^T 0 | dP^T 128 | dV 256 | dK 320 | dQ 384 | P^T 448.
// P^T has columns of its own, so S^T(i+1) is issued as soon as both
// warpgroups hold S^T(i) in registers (s_free), before dV(i) has read P^T(i);
// warpgroup w writes its dS^T into the first half of its own dP^T columns (the
// MMAs read that K = 128 query operand as two 64-query halves).  dK(i)
// signals as soon as it has read dS^T(i), ahead of dQ(i), so dP^T(i+1) follows.
// Tensor memory (d = 128): S^T 0 | dP^T 128 | dV 256 | dK 384, all 512 columns.
// P^T goes to S^T's columns 0-63 and dS^T to its columns 64-127 (the two
// warpgroups meet at a named barrier once both hold their S^T in registers);
// dQ_i accumulates over dP^T's columns once the warpgroups have read them, so
// dP^T(i+1) waits for dQ_i to be drained and S^T(i+1) for dK_i.  dO has a
// one-stage ring here (shared memory holds K, V, two Q stages, dO and dS).
#include "attn.cuh"
#include "launch.cuh"

namespace gqe {

namespace {

constexpr int kBwdThreads = 512;
constexpr int kTileB = 128;
constexpr int kBoxB = 128 * 64 * 2;   // one 128-row x 64-column bf16 TMA box

struct __align__(8) BwdBarriers {
  uint64_t kv_full;
  uint64_t q_full[2], q_empty[2], o_full[2], o_empty[2];
  uint64_t s_full, s_free, p_full, pv_done, dp_full, ds_full, dk_done;
  uint64_t dq_full[2], dq_free[2];
  uint32_t tmem_base;
  int abort;
};

template <int D>
struct BwdCfg {
  static constexpr int NB = D / 64;
  static constexpr int TileBytes = NB * kBoxB;        // one 128-row tile of Q, dO, K or V
  static constexpr bool kWide = D == 128;
  static constexpr int OST = kWide ? 1 : 2;           // dO ring depth
  static constexpr int EpiCh = kWide ? 1 : D / 32;    // 32-column dQ chunks staged per warp at once
  static constexpr uint32_t kS = 0, kDP = 128, kDV = 256, kDK = 256 + D;
  static constexpr uint32_t kDQ = kWide ? 128 : 384;
  static constexpr uint32_t kPT = 448;                // d = 64: P^T
  // shared memory, every operand region 1024-byte aligned
  static constexpr int OffK = 0;
  static constexpr int OffV = OffK + TileBytes;
  static constexpr int OffQ = OffV + TileBytes;                 // [2] stages
  static constexpr int OffDO = OffQ + 2 * TileBytes;            // [OST]
  static constexpr int OffDS = OffDO + OST * TileBytes;         // 128 x 128 bf16, MN-major
  static constexpr int OffEpi = OffDS + 2 * kBoxB;              // 4 warps x EpiCh x 4 KB
  static constexpr int OffLse = OffEpi + 4 * EpiCh * 4096;      // [2][128] f32
  static constexpr int OffDelta = OffLse + 2 * 512;             // [2][128] f32
  static constexpr int OffBar = OffDelta + 2 * 512;
  static constexpr size_t Smem = 1024 + OffBar + sizeof(BwdBarriers);
};

// One query tile of the item's walk.
struct QTile {
  bool shared;
  int i;         // tile index within its sequence
  int kk;        // packed rows per token (k for routed rows, 1 for the shared head)
  int row_pad;   // first row in the padded LSE / Delta / dQ workspace
};

__device__ __forceinline__ QTile qtile(const AttnBwdParams& p, int s, int jt, int n_r, int n) {
  QTile q;
  if (n < n_r) {
    q.shared = false;
    q.i = jt * p.k + n;
    q.kk = p.k;
    q.row_pad = s * p.rows_pad + q.i * kTileB;
  } else {
    q.shared = true;
    q.i = jt + (n - n_r);
    q.kk = 1;
    q.row_pad = p.B * p.G * p.rows_pad + (s / p.G) * p.rows_pad_sh + q.i * kTileB;
  }
  return q;
}

// Tensor-memory column of a bf16 query operand's k-step ks (16 queries).
// P^T: contiguous, in columns of its own (d = 64) or S^T's columns 0-63
// (d = 128).  dS^T: d = 64, queries [0, 64) packed at dP^T + [0, 32) and
// [64, 128) at dP^T + 64 + [0, 32) (each warpgroup inside its own fp32
// columns); d = 128, contiguous at S^T's columns 64-127.
__device__ __forceinline__ uint32_t half_col(uint32_t base, int ks) {
  return base + (ks >> 2) * 64 + (ks & 3) * 8;
}
template <int D>
__device__ __forceinline__ uint32_t pt_col(int ks) {
  return D == 64 ? BwdCfg<D>::kPT + ks * 8 : BwdCfg<D>::kS + ks * 8;
}
template <int D>
__device__ __forceinline__ uint32_t dst_col(int ks) {
  return D == 64 ? half_col(BwdCfg<D>::kDP, ks) : BwdCfg<D>::kS + 64 + ks * 8;
}
// Where warpgroup w writes its 32 packed columns of P^T and dS^T.
template <int D>
__device__ __forceinline__ uint32_t pt_wcol(int w) {
  return D == 64 ? BwdCfg<D>::kPT + 32 * w : BwdCfg<D>::kS + 32 * w;
}
template <int D>
__device__ __forceinline__ uint32_t dst_wcol(int w) {
  return D == 64 ? BwdCfg<D>::kDP + 64 * w : BwdCfg<D>::kS + 64 + 32 * w;
}

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
attn_bwd_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapQs,
                const __grid_constant__ CUtensorMap mapdO, const __grid_constant__ CUtensorMap mapdOs,
                const __grid_constant__ CUtensorMap mapK, const __grid_constant__ CUtensorMap mapV,
                const __grid_constant__ CUtensorMap mapdQ, AttnBwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem + C::OffK;
  uint8_t* sV = smem + C::OffV;
  uint8_t* sDS = smem + C::OffDS;
  float* sLse = reinterpret_cast<float*>(smem + C::OffLse);
  float* sDelta = reinterpret_cast<float*>(smem + C::OffDelta);
  BwdBarriers* bar = reinterpret_cast<BwdBarriers*>(smem + C::OffBar);
  volatile int* abort = &bar->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work item: key tile jt of sequence s, key tiles in ascending order
  // (tile 0 sees the most query tiles: heaviest first)
  const int BG = p.B * p.G;
  const int jt = (int)blockIdx.x / BG;
  const int s = (int)blockIdx.x % BG;
  const int g = s % p.G;
  const int nq_r = (p.T * p.k + kTileB - 1) / kTileB;
  const int n_r = nq_r - jt * p.k;
  const int n_s = (p.n_shared && g == p.sg) ? (p.T + kTileB - 1) / kTileB - jt : 0;
  const int cnt = n_r + n_s;
  const float sl2 = p.scale_log2;

  if (threadIdx.x == 0) {
    mbar_init(&bar->kv_full, 1);
    for (int st = 0; st < 2; ++st) {
      mbar_init(&bar->q_full[st], 1);
      mbar_init(&bar->q_empty[st], 2 + 256);
      mbar_init(&bar->o_full[st], 1);
      mbar_init(&bar->o_empty[st], 1);
      mbar_init(&bar->dq_full[st], 1);
      mbar_init(&bar->dq_free[st], 128);
    }
    mbar_init(&bar->s_full, 1);
    mbar_init(&bar->s_free, 256);
    mbar_init(&bar->p_full, 256);
    mbar_init(&bar->pv_done, 1);
    mbar_init(&bar->dp_full, 1);
    mbar_init(&bar->ds_full, 256);
    mbar_init(&bar->dk_done, 1);
    bar->abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&mapQ);
    tma_prefetch_desc(&mapdO);
    tma_prefetch_desc(&mapK);
    tma_prefetch_desc(&mapV);
    tma_prefetch_desc(&mapdQ);
  }
  if (warp == 1) tmem_alloc(&bar->tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;
  pdl_launch_dependents();
  pdl_wait();

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- producer: K_j, V_j once; Q_i, dO_i, LSE2_i, Delta_i per tile
      mbar_arrive_expect_tx(&bar->kv_full, 2 * C::TileBytes);
      for (int bx = 0; bx < C::NB; ++bx) {
        tma_load_3d(sK + bx * kBoxB, &mapK, &bar->kv_full, bx * 64, jt * kTileB, s);
        tma_load_3d(sV + bx * kBoxB, &mapV, &bar->kv_full, bx * 64, jt * kTileB, s);
      }
      for (int n = 0; n < cnt; ++n) {
        const int st = n & 1;
        if (n >= 2 && !mbar_wait(&bar->q_empty[st], ((n >> 1) - 1) & 1, abort, p.err, kErrTimeoutAttnBwd)) break;
        const QTile q = qtile(p, s, jt, n_r, n);
        const CUtensorMap* mq = q.shared ? &mapQs : &mapQ;
        const CUtensorMap* mo = q.shared ? &mapdOs : &mapdO;
        const int seq = q.shared ? s / p.G : s;
        mbar_arrive_expect_tx(&bar->q_full[st], C::TileBytes + 2 * 512);
        for (int bx = 0; bx < C::NB; ++bx)
          tma_load_3d(smem + C::OffQ + st * C::TileBytes + bx * kBoxB, mq, &bar->q_full[st], bx * 64,
                      q.i * kTileB, seq);
        bulk_load(sLse + st * 128, p.lse2 + q.row_pad, 512, &bar->q_full[st]);
        bulk_load(sDelta + st * 128, p.delta + q.row_pad, 512, &bar->q_full[st]);
        const int so = n % C::OST;
        if (n >= C::OST &&
            !mbar_wait(&bar->o_empty[so], ((n / C::OST) - 1) & 1, abort, p.err, kErrTimeoutAttnBwd))
          break;
        mbar_arrive_expect_tx(&bar->o_full[so], C::TileBytes);
        for (int bx = 0; bx < C::NB; ++bx)
          tma_load_3d(smem + C::OffDO + so * C::TileBytes + bx * kBoxB, mo, &bar->o_full[so], bx * 64,
                      q.i * kTileB, seq);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer A: S^T, dP^T, dV
      constexpr uint32_t idesc_s = idesc_bf16_f32(kTileB, kTileB, false, false);
      constexpr uint32_t idesc_v = idesc_bf16_f32(kTileB, D, false, true);
      const uint32_t k0 = smem_u32(sK), v0 = smem_u32(sV);
      auto issue_s = [&](int n) {
        const int st = n & 1;
        if (!mbar_wait(&bar->q_full[st], (n >> 1) & 1, abort, p.err, kErrTimeoutAttnBwd)) return false;
        tc_fence_after();
        const uint32_t q0 = smem_u32(smem + C::OffQ + st * C::TileBytes);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (ks >> 2) * kBoxB + (ks & 3) * 32;
          umma_ss(tmem + C::kS, sdesc_sw128(k0 + off, 16, 1024), sdesc_sw128(q0 + off, 16, 1024), idesc_s, ks > 0);
        }
        umma_commit(&bar->s_full);
        return true;
      };
      auto issue_dp = [&](int n) {
        const int so = n % C::OST;
        if (!mbar_wait(&bar->o_full[so], (n / C::OST) & 1, abort, p.err, kErrTimeoutAttnBwd)) return false;
        tc_fence_after();
        const uint32_t o0 = smem_u32(smem + C::OffDO + so * C::TileBytes);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (ks >> 2) * kBoxB + (ks & 3) * 32;
          umma_ss(tmem + C::kDP, sdesc_sw128(v0 + off, 16, 1024), sdesc_sw128(o0 + off, 16, 1024), idesc_s, ks > 0);
        }
        umma_commit(&bar->dp_full);
        return true;
      };
      bool ok = mbar_wait(&bar->kv_full, 0, abort, p.err, kErrTimeoutAttnBwd);
      if (ok) ok = issue_s(0);
      if (ok) ok = issue_dp(0);
      for (int n = 0; ok && n < cnt; ++n) {
        // d = 64: S^T(n+1) as soon as the warpgroups hold S^T(n) in registers
        if (!C::kWide && n + 1 < cnt) {
          if (!mbar_wait(&bar->s_free, n & 1, abort, p.err, kErrTimeoutAttnBwd)) break;
          if (!issue_s(n + 1)) break;
        }
        // dV += P^T dO_i once P^T is in tensor memory
        if (!mbar_wait(&bar->p_full, n & 1, abort, p.err, kErrTimeoutAttnBwd)) break;
        tc_fence_after();
        const uint32_t o0 = smem_u32(smem + C::OffDO + (n % C::OST) * C::TileBytes);
#pragma unroll
        for (int ks = 0; ks < kTileB / 16; ++ks)
          umma_ts(tmem + C::kDV, tmem + pt_col<D>(ks), sdesc_sw128(o0 + ks * 2048, kBoxB, 1024), idesc_v,
                  (n > 0 || ks > 0));
        umma_commit(&bar->pv_done);
        umma_commit(&bar->q_empty[n & 1]);
        umma_commit(&bar->o_empty[n % C::OST]);
        if (n + 1 < cnt) {
          // d = 128: S^T(n+1) overwrites P^T(n) and dS^T(n): wait for dV and dK
          // to have read them
          if (C::kWide) {
            if (!mbar_wait(&bar->pv_done, n & 1, abort, p.err, kErrTimeoutAttnBwd)) break;
            if (!mbar_wait(&bar->dk_done, n & 1, abort, p.err, kErrTimeoutAttnBwd)) break;
            if (!issue_s(n + 1)) break;
          }
          // dP^T(n+1) overwrites dS^T(n) (d = 64) or dQ(n) (d = 128)
          if (C::kWide) {
            if (!mbar_wait(&bar->dq_free[0], n & 1, abort, p.err, kErrTimeoutAttnBwd)) break;
          } else {
            if (!mbar_wait(&bar->dk_done, n & 1, abort, p.err, kErrTimeoutAttnBwd)) break;
          }
          tc_fence_after();
          if (!issue_dp(n + 1)) break;
        }
      }
    }
  } else if (warp == 2) {
    if (lane == 0) {
      // ---------------- MMA issuer B: dK += dS^T Q_i, dQ_i = dS K_j (dQ double-buffered)
      constexpr uint32_t idesc_k = idesc_bf16_f32(kTileB, D, false, true);
      constexpr uint32_t idesc_q = idesc_bf16_f32(kTileB, D, true, true);
      const uint32_t k0 = smem_u32(sK), ds0 = smem_u32(sDS);
      for (int n = 0; n < cnt; ++n) {
        if (!mbar_wait(&bar->ds_full, n & 1, abort, p.err, kErrTimeoutAttnBwd)) break;
        tc_fence_after();
        const uint32_t q0 = smem_u32(smem + C::OffQ + (n & 1) * C::TileBytes);
#pragma unroll
        for (int ks = 0; ks < kTileB / 16; ++ks)
          umma_ts(tmem + C::kDK, tmem + dst_col<D>(ks), sdesc_sw128(q0 + ks * 2048, kBoxB, 1024), idesc_k,
                  (n > 0 || ks > 0));
        umma_commit(&bar->q_empty[n & 1]);
        // dK(n) has read dS^T(n) (d = 64: from dP^T's columns, d = 128: from
        // S^T's): signal before dQ(n), so dP^T(n+1) / S^T(n+1) may follow
        umma_commit(&bar->dk_done);
        // dQ(n) over dQ(n-1): wait for the drain (d = 128: dQ sits over dP^T's
        // columns, which the warpgroups have read, ds_full)
        if (!C::kWide && n >= 1 &&
            !mbar_wait(&bar->dq_free[0], (n - 1) & 1, abort, p.err, kErrTimeoutAttnBwd))
          break;
        tc_fence_after();
        const uint32_t dq_col = C::kDQ;
#pragma unroll
        for (int ks = 0; ks < kTileB / 16; ++ks)
          umma_ss(tmem + dq_col, sdesc_sw128(ds0 + ks * 2048, kBoxB, 1024),
                  sdesc_sw128(k0 + ks * 2048, kBoxB, 1024), idesc_q, ks > 0);
        umma_commit(&bar->dq_full[0]);
      }
    }
  } else if (warp >= 4 && warp < 12) {
    // ---------------- P and dS: one key row per thread, 64 query columns per warpgroup
    const int qd = warp & 3;
    const int wg = (warp - 4) >> 2;
    const int r = qd * 32 + lane;
    const int kv_pos = jt * kTileB + r;
    const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
    const uint32_t col0 = (uint32_t)(wg * 64);
    const float scale = p.scale;
    bool ok = true;
    for (int n = 0; n < cnt && ok; ++n) {
      const int st = n & 1;
      const QTile q = qtile(p, s, jt, n_r, n);
      ok = mbar_wait(&bar->q_full[st], (n >> 1) & 1, abort, p.err, kErrTimeoutAttnBwd);
      ok = ok && mbar_wait(&bar->s_full, n & 1, abort, p.err, kErrTimeoutAttnBwd);
      if (!C::kWide && !ok) break;
      tc_fence_after();
      const float* lse2 = sLse + st * 128 + col0;
      const float* dlt = sDelta + st * 128 + col0;
      // query columns c < cmin belong to tokens before this key: masked
      const int cmin = kv_pos * q.kk - q.i * kTileB - (int)col0;
      float pf[64];
#pragma unroll
      for (int h = 0; h < 2 && ok; ++h) {
        uint32_t sv[32];
        tmem_ld32(tmem + lane_off + C::kS + col0 + h * 32, sv);
        if (!C::kWide && h == 1) {
          // S^T(n) is in registers: S^T(n+1) may be computed into its columns
          tc_fence_before();
          mbar_arrive(&bar->s_free);
        }
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4) {
          const float4 l4 = *reinterpret_cast<const float4*>(lse2 + h * 32 + c4 * 4);
          const int c = h * 32 + c4 * 4;
          pf[c + 0] = ex2(fmaf(__uint_as_float(sv[c4 * 4 + 0]), sl2, -l4.x));
          pf[c + 1] = ex2(fmaf(__uint_as_float(sv[c4 * 4 + 1]), sl2, -l4.y));
          pf[c + 2] = ex2(fmaf(__uint_as_float(sv[c4 * 4 + 2]), sl2, -l4.z));
          pf[c + 3] = ex2(fmaf(__uint_as_float(sv[c4 * 4 + 3]), sl2, -l4.w));
        }
      }
      if (cmin > 0) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c < cmin) pf[c] = 0.f;
      }
      if (!C::kWide) {
        // P^T(n-1) must have been read by dV(n-1) before P^T(n) replaces it
        if (n > 0) ok = mbar_wait(&bar->pv_done, (n - 1) & 1, abort, p.err, kErrTimeoutAttnBwd);
        if (!ok) break;
        tc_fence_after();
      }
      if (C::kWide) {
        // both warpgroups hold their S^T columns in registers before warpgroup 1
        // writes P^T over warpgroup 0's; every thread of the two warpgroups
        // passes here each tile and they leave together if any wait failed
        int any_fail;
        asm volatile(
            "{\n\t.reg .pred q, r;\n\tsetp.ne.b32 q, %1, 0;\n\t"
            "bar.red.or.pred r, 1, 256, q;\n\tselp.b32 %0, 1, 0, r;\n\t}"
            : "=r"(any_fail)
            : "r"((int)!ok)
            : "memory");
        if (any_fail) break;
      }
      {
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) pk[c] = pack_bf16x2(pf[2 * c], pf[2 * c + 1]);
        tmem_st32(tmem + lane_off + pt_wcol<D>(wg), pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar->p_full);

      ok = mbar_wait(&bar->dp_full, n & 1, abort, p.err, kErrTimeoutAttnBwd);
      if (!ok) break;
      tc_fence_after();
      // dP^T chunks of 16 columns.  d = 128: the next chunk's load in flight
      // while this one is used (measured faster there, slower at d = 64)
      constexpr bool kPipe = C::kWide;
      uint32_t dpb[2][16];
      if (kPipe) {
        tmem_ld16_async(tmem + lane_off + C::kDP + col0, dpb[0]);
        tmem_wait_ld16(dpb[0]);
      }
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t* dp = dpb[ch & 1];
        if (!kPipe)
          tmem_ld16(tmem + lane_off + C::kDP + col0 + ch * 16, dp);
        else if (ch < 3)
          tmem_ld16_async(tmem + lane_off + C::kDP + col0 + (ch + 1) * 16, dpb[(ch + 1) & 1]);
        uint32_t dsk[8];
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          const float4 d4 = *reinterpret_cast<const float4*>(dlt + ch * 16 + c4 * 4);
          const int c = ch * 16 + c4 * 4;
          const float a0 = scale * pf[c + 0] * (__uint_as_float(dp[c4 * 4 + 0]) - d4.x);
          const float a1 = scale * pf[c + 1] * (__uint_as_float(dp[c4 * 4 + 1]) - d4.y);
          const float a2 = scale * pf[c + 2] * (__uint_as_float(dp[c4 * 4 + 2]) - d4.z);
          const float a3 = scale * pf[c + 3] * (__uint_as_float(dp[c4 * 4 + 3]) - d4.w);
          dsk[c4 * 2] = pack_bf16x2(a0, a1);
          dsk[c4 * 2 + 1] = pack_bf16x2(a2, a3);
        }
        // dS^T row r: into the first half of this warpgroup's dP^T columns (the
        // dK operand) ...
        tmem_st8(tmem + lane_off + dst_wcol<D>(wg) + ch * 8, dsk);
        // ... and into the MN-major smem operand of dQ: the 64-query atom of
        // this warpgroup, [128 keys x 128 B], 16-byte pieces swizzled by key row
        // (d = 64: once dQ(n-1) has read the previous tile's)
        if (!C::kWide && ch == 0 && n > 0) {
          ok = mbar_wait(&bar->dq_full[0], (n - 1) & 1, abort, p.err, kErrTimeoutAttnBwd);
          if (!ok) break;
        }
        uint8_t* atom = sDS + wg * kBoxB + r * 128;
#pragma unroll
        for (int j2 = 0; j2 < 2; ++j2) {
          const int piece = ch * 2 + j2;
          st_shared_v4(atom + ((piece ^ (r & 7)) << 4), dsk[j2 * 4], dsk[j2 * 4 + 1], dsk[j2 * 4 + 2],
                       dsk[j2 * 4 + 3]);
        }
        if (kPipe && ch < 3) tmem_wait_ld16(dpb[(ch + 1) & 1]);
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bar->ds_full);
      mbar_arrive(&bar->q_empty[st]);
    }
  } else if (warp >= 12) {
    // ---------------- dQ drain (TMA reduce-add into fp32), then dK, dV
    const int qd = warp & 3;
    const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
    uint8_t* stage = smem + C::OffEpi + qd * C::EpiCh * 4096;
    bool ok = true;
    for (int n = 0; n < cnt && ok; ++n) {
      const int b = 0;
      const int ph = n & 1;
      const QTile q = qtile(p, s, jt, n_r, n);
      ok = mbar_wait(&bar->dq_full[b], ph, abort, p.err, kErrTimeoutAttnBwd);
      if (!ok) break;
      tc_fence_after();
      const uint32_t dq_col = C::kDQ;
#pragma unroll
      for (int g0 = 0; g0 < D / 32; g0 += C::EpiCh) {
        // staging free: every earlier reduce of this warp has read it
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
#pragma unroll
        for (int c = 0; c < C::EpiCh; ++c) {
          const int c0 = g0 + c;
          uint32_t v[32];
          tmem_ld32(tmem + lane_off + dq_col + c0 * 32, v);
          if (c0 == D / 32 - 1) {
            tc_fence_before();
            mbar_arrive(&bar->dq_free[b]);
          }
          uint8_t* rowp = stage + c * 4096 + lane * 128;
#pragma unroll
          for (int j = 0; j < 8; ++j)
            st_shared_v4(rowp + ((j ^ (lane & 7)) << 4), v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
#pragma unroll
          for (int c = 0; c < C::EpiCh; ++c)
            tma_reduce_add_2d(&mapdQ, stage + c * 4096, (g0 + c) * 32, q.row_pad + qd * 32);
          bulk_commit();
        }
      }
    }
    // dK, dV of the key tile
    if (ok) ok = mbar_wait(&bar->pv_done, (cnt - 1) & 1, abort, p.err, kErrTimeoutAttnBwd);
    if (ok) ok = mbar_wait(&bar->dk_done, (cnt - 1) & 1, abort, p.err, kErrTimeoutAttnBwd);
    tc_fence_after();
    const int kv_pos = jt * kTileB + qd * 32 + lane;
    const size_t orow = ((size_t)s * p.T + kv_pos) * D;
#pragma unroll
    for (int which = 0; which < 2; ++which) {
      gqe_bf16_t* dst = (which ? p.dV : p.dK) + orow;
      const uint32_t col = which ? C::kDV : C::kDK;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_off + col + c0, v);
        if (ok && kv_pos < p.T) {
          uint32_t pkv[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) pkv[c] = pack_bf16x2(__uint_as_float(v[2 * c]), __uint_as_float(v[2 * c + 1]));
          uint4* d4 = reinterpret_cast<uint4*>(dst + c0);
#pragma unroll
          for (int c = 0; c < 4; ++c) d4[c] = make_uint4(pkv[4 * c], pkv[4 * c + 1], pkv[4 * c + 2], pkv[4 * c + 3]);
        }
      }
    }
    if (lane == 0) bulk_wait<0>();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  drain_after_abort(abort);
}

// Delta_r = sum_c dO_rc O_rc and LSE2_r = LSE_r * log2(e) into the padded row
// space (+inf LSE2 and 0 Delta on padding rows, so their P is 0), and the dQ
// accumulator zeroed.  d/8 threads per row, 16 bytes each.
__global__ void __launch_bounds__(256) attn_bwd_prep_kernel(AttnBwdParams p) {
  pdl_launch_dependents();
  pdl_wait();
  const int tpr = p.d / 8;
  const long long gt = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long pr = gt / tpr;
  const int part = (int)(gt % tpr);
  if (pr >= p.n_rows_pad) return;
  const int BG = p.B * p.G;
  const long long routed_rows = (long long)BG * p.rows_pad;
  bool valid;
  long long src;   // row of o / dO / lse
  if (pr < routed_rows) {
    const int sq = (int)(pr / p.rows_pad), r = (int)(pr % p.rows_pad);
    valid = r < p.T * p.k;
    src = (long long)sq * p.T * p.k + r;
  } else {
    const long long q2 = pr - routed_rows;
    const int b = (int)(q2 / p.rows_pad_sh), r = (int)(q2 % p.rows_pad_sh);
    valid = r < p.T;
    src = (long long)BG * p.T * p.k + (long long)b * p.T + r;
  }
  float dot = 0.f;
  if (valid) {
    const gqe_bf16_t* o = (pr < routed_rows) ? p.o_routed + src * p.d
                                             : p.o_sh + (src - (long long)BG * p.T * p.k) * p.d;
    const gqe_bf16_t* dO = (pr < routed_rows) ? p.do_routed + src * p.d
                                              : p.do_sh + (src - (long long)BG * p.T * p.k) * p.d;
    const uint4 a = reinterpret_cast<const uint4*>(o)[part];
    const uint4 b = reinterpret_cast<const uint4*>(dO)[part];
    const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) dot += bf16_lo(av[e]) * bf16_lo(bv[e]) + bf16_hi(av[e]) * bf16_hi(bv[e]);
  }
  for (int off = tpr >> 1; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
  float4* acc = reinterpret_cast<float4*>(p.dq_acc + pr * p.d + part * 8);
  acc[0] = make_float4(0.f, 0.f, 0.f, 0.f);
  acc[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  if (part == 0) {
    p.delta[pr] = valid ? dot : 0.f;
    p.lse2[pr] = valid ? p.lse[src] * 1.4426950408889634f : INFINITY;
  }
}

// dq (bf16) from the fp32 accumulator, valid rows only.
__global__ void __launch_bounds__(256) attn_bwd_post_kernel(AttnBwdParams p) {
  pdl_launch_dependents();
  pdl_wait();
  const int tpr = p.d / 8;
  const long long gt = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long pr = gt / tpr;
  const int part = (int)(gt % tpr);
  if (pr >= p.n_rows_pad) return;
  const int BG = p.B * p.G;
  const long long routed_rows = (long long)BG * p.rows_pad;
  gqe_bf16_t* dst;
  if (pr < routed_rows) {
    const int sq = (int)(pr / p.rows_pad), r = (int)(pr % p.rows_pad);
    if (r >= p.T * p.k) return;
    dst = p.dq_routed + ((long long)sq * p.T * p.k + r) * p.d;
  } else {
    const long long q2 = pr - routed_rows;
    const int b = (int)(q2 / p.rows_pad_sh), r = (int)(q2 % p.rows_pad_sh);
    if (r >= p.T) return;
    dst = p.dq_sh + ((long long)b * p.T + r) * p.d;
  }
  const float4* a = reinterpret_cast<const float4*>(p.dq_acc + pr * p.d + part * 8);
  const float4 x = a[0], y = a[1];
  reinterpret_cast<uint4*>(dst)[part] =
      make_uint4(pack_bf16x2(x.x, x.y), pack_bf16x2(x.z, x.w), pack_bf16x2(y.x, y.y), pack_bf16x2(y.z, y.w));
}

}  // namespace

void attn_bwd_layout(int B, int T, int G, int k, int n_shared, int d, AttnBwdLayout* L) {
  L->rows_pad = (T * k + kTileB - 1) / kTileB * kTileB;
  L->rows_pad_sh = (T + kTileB - 1) / kTileB * kTileB;
  L->n_rows_pad = (long long)B * G * L->rows_pad + (n_shared ? (long long)B * L->rows_pad_sh : 0);
  size_t o = 0;
  L->off_lse2 = o;
  o += ((size_t)L->n_rows_pad * 4 + 255) & ~size_t(255);
  L->off_delta = o;
  o += ((size_t)L->n_rows_pad * 4 + 255) & ~size_t(255);
  L->off_dq = o;
  o += (size_t)L->n_rows_pad * d * 4;
  L->bytes = o;
}

cudaError_t launch_attn_bwd(const CUtensorMap& mQ, const CUtensorMap& mQs, const CUtensorMap& mdO,
                            const CUtensorMap& mdOs, const CUtensorMap& mK, const CUtensorMap& mV,
                            const CUtensorMap& mdQ, const AttnBwdParams& p, cudaStream_t stream) {
  if (p.d != 64 && p.d != 128) return cudaErrorNotSupported;
  const long long threads = p.n_rows_pad * (p.d / 8);
  const int blocks = (int)((threads + 255) / 256);
  cudaError_t e = launch_kernel(attn_bwd_prep_kernel, dim3(blocks), dim3(256), 0, stream, 1, p);
  if (e != cudaSuccess) return e;
  auto kern = p.d == 64 ? attn_bwd_kernel<64> : attn_bwd_kernel<128>;
  const size_t smem = p.d == 64 ? BwdCfg<64>::Smem : BwdCfg<128>::Smem;
  e = ensure_smem(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  const int n_kvt = (p.T + kTileB - 1) / kTileB;
  e = launch_kernel(kern, dim3(n_kvt * p.B * p.G), dim3(kBwdThreads), smem, stream, 1, mQ, mQs, mdO, mdOs, mK, mV,
                    mdQ, p);
  if (e != cudaSuccess) return e;
  return launch_kernel(attn_bwd_post_kernel, dim3(blocks), dim3(256), 0, stream, 1, p);
}

}  // namespace gqe
