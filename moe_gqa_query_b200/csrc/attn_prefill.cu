// attn_prefill.cu -- routed causal attention for the GQE prefill on tcgen05.
//
// Every selected (token, expert) query row of one KV group attends causally to
// that group's dense K/V ("GQE" study note §3-2 2) and §1-1 attention
// equation); the shared head does the same against KV group sg (§3-2 5)).
//
// Work item = one 128-row tile of packed query rows of one sequence:
//   routed: rows (t, j) of group (b, g), row = t*k + j, so one tile spans
//           128/k tokens and every K/V tile loaded for it serves all of the
//           group's selected experts at once;
//   shared: 128 tokens of the shared head of sequence b.
// Items are launched heaviest first (descending 128-token level), so the
// causal triangle's long tiles start early.
//
// Per item: TMA brings Q once and K/V tiles (128 keys) through a ring of
// shared-memory stages; tcgen05 computes S = Q K^T into one of three tensor-
// memory S buffers; 4 softmax warps (one row per thread) apply the causal
// mask, keep the running max in the base-2 domain, write P (bf16) over the S
// columns, and rescale the O accumulator in tensor memory only when the max
// grows by more than 2^8 (exact: l and O share the stale max); tcgen05 then
// adds P V (A operand from tensor memory) into O.
//
// CTA: 192 threads.  warp 0 TMA producer, warp 1 MMA issuer (and tensor-memory
// owner), warps 2..5 softmax + epilogue.  Tensor memory: S0|S1|S2|O at columns
// 0|128|256|384.
#include "attn.cuh"

namespace gqe {

namespace {

constexpr int kThreads = 192;
constexpr int kTile = 128;          // query rows and keys per tile
constexpr int kBox = 128 * 64 * 2;  // one TMA box: 128 rows x 64 bf16, 16 KB
constexpr float kRescaleLog2 = 8.0f;

struct __align__(8) AttnBarriers {
  uint64_t q_full;
  uint64_t k_full[4], k_empty[4], v_full[4], v_empty[4];
  uint64_t s_full[3], p_full[3], pv_done[3];
  uint32_t tmem_base;
  int abort;
};

template <int D>
struct AttnCfg {
  static constexpr int NB = D / 64;                  // 64-column boxes per tile
  static constexpr int ST = (D == 64) ? 3 : 2;       // K/V ring depth
  static constexpr int QBytes = NB * kBox;
  static constexpr int KVBytes = NB * kBox;
  static constexpr size_t Smem = 1024 + QBytes + 2 * ST * KVBytes + sizeof(AttnBarriers);
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
attn_prefill_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapQs,
                    const __grid_constant__ CUtensorMap mapK, const __grid_constant__ CUtensorMap mapV,
                    AttnParams p) {
  using C = AttnCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + C::QBytes;
  uint8_t* sV = sK + C::ST * C::KVBytes;
  AttnBarriers* bar = reinterpret_cast<AttnBarriers*>(sV + C::ST * C::KVBytes);
  volatile int* abort = &bar->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work item
  const int BG = p.B * p.G;
  const int per_level = BG * p.k + p.B * p.n_shared;
  const int ntq_sh = (p.T + kTile - 1) / kTile;
  const int level = blockIdx.x / per_level;
  const int i = blockIdx.x % per_level;
  const int qt_sh = ntq_sh - 1 - level;
  bool routed;
  int seq, qt, kvseq, kk, rows_total;
  if (i < BG * p.k) {
    routed = true;
    const int r = i / BG;
    seq = i % BG;
    qt = qt_sh * p.k + r;
    kvseq = seq;
    kk = p.k;
    rows_total = p.T * p.k;
  } else {
    routed = false;
    seq = i - BG * p.k;
    qt = qt_sh;
    kvseq = seq * p.G + p.sg;
    kk = 1;
    rows_total = p.T;
  }
  const int row0 = qt * kTile;
  if (row0 >= rows_total) return;
  const int t_first = row0 / kk;
  const int t_last = min(p.T - 1, (row0 + kTile - 1) / kk);
  const int n_kv = t_last / kTile + 1;
  const CUtensorMap* mq = routed ? &mapQ : &mapQs;

  if (threadIdx.x == 0) {
    mbar_init(&bar->q_full, 1);
    for (int s = 0; s < C::ST; ++s) {
      mbar_init(&bar->k_full[s], 1);
      mbar_init(&bar->k_empty[s], 1);
      mbar_init(&bar->v_full[s], 1);
      mbar_init(&bar->v_empty[s], 1);
    }
    for (int s = 0; s < 3; ++s) {
      mbar_init(&bar->s_full[s], 1);
      mbar_init(&bar->p_full[s], 128);
      mbar_init(&bar->pv_done[s], 1);
    }
    bar->abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(mq);
    tma_prefetch_desc(&mapK);
    tma_prefetch_desc(&mapV);
  }
  if (warp == 1) tmem_alloc(&bar->tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;
  constexpr uint32_t kOcol = 384;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- producer: Q once, then K_0, K_1, V_0, K_2, V_1, ...
      mbar_arrive_expect_tx(&bar->q_full, C::QBytes);
      for (int bx = 0; bx < C::NB; ++bx)
        tma_load_3d(sQ + bx * kBox, mq, &bar->q_full, bx * 64, row0, seq);
      auto load_k = [&](int j) -> bool {
        const int s = j % C::ST;
        if (j >= C::ST && !mbar_wait(&bar->k_empty[s], ((j / C::ST) & 1) ^ 1, abort, p.err, kErrTimeoutAttn))
          return false;
        mbar_arrive_expect_tx(&bar->k_full[s], C::KVBytes);
        for (int bx = 0; bx < C::NB; ++bx)
          tma_load_3d(sK + s * C::KVBytes + bx * kBox, &mapK, &bar->k_full[s], bx * 64, j * kTile, kvseq);
        return true;
      };
      auto load_v = [&](int j) -> bool {
        const int s = j % C::ST;
        if (j >= C::ST && !mbar_wait(&bar->v_empty[s], ((j / C::ST) & 1) ^ 1, abort, p.err, kErrTimeoutAttn))
          return false;
        mbar_arrive_expect_tx(&bar->v_full[s], C::KVBytes);
        for (int bx = 0; bx < C::NB; ++bx)
          tma_load_3d(sV + s * C::KVBytes + bx * kBox, &mapV, &bar->v_full[s], bx * 64, j * kTile, kvseq);
        return true;
      };
      for (int j = 0; j < n_kv; ++j) {
        if (!load_k(j)) break;
        if (j >= 1 && !load_v(j - 1)) break;
      }
      if (!*abort) load_v(n_kv - 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer: S_0, S_1, PV_0, S_2, PV_1, ...
      constexpr uint32_t idesc_s = idesc_bf16_f32(kTile, kTile, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(kTile, D, false, true);
      const uint32_t q0 = smem_u32(sQ);
      auto issue_s = [&](int j) -> bool {
        const int s = j % C::ST;
        if (!mbar_wait(&bar->k_full[s], (j / C::ST) & 1, abort, p.err, kErrTimeoutAttn)) return false;
        tc_fence_after();
        const uint32_t k0 = smem_u32(sK + s * C::KVBytes);
        const uint32_t dst = tmem + (uint32_t)((j % 3) * kTile);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (ks >> 2) * kBox + (ks & 3) * 32;
          umma_ss(dst, sdesc_sw128(q0 + off, 16, 1024), sdesc_sw128(k0 + off, 16, 1024), idesc_s,
                  ks > 0);
        }
        umma_commit(&bar->s_full[j % 3]);
        umma_commit(&bar->k_empty[s]);
        return true;
      };
      auto issue_pv = [&](int j) -> bool {
        const int s = j % C::ST;
        if (!mbar_wait(&bar->v_full[s], (j / C::ST) & 1, abort, p.err, kErrTimeoutAttn)) return false;
        tc_fence_after();
        const uint32_t v0 = smem_u32(sV + s * C::KVBytes);
        const uint32_t pcol = tmem + (uint32_t)((j % 3) * kTile);
#pragma unroll
        for (int ks = 0; ks < kTile / 16; ++ks) {
          // V rows 16*ks .. 16*ks+15 (K dim), all D columns (MN-major, 64-col boxes 16 KB apart)
          umma_ts(tmem + kOcol, pcol + ks * 8, sdesc_sw128(v0 + ks * 2048, kBox, 1024), idesc_o,
                  (j > 0 || ks > 0));
        }
        umma_commit(&bar->pv_done[j % 3]);
        umma_commit(&bar->v_empty[s]);
        return true;
      };
      if (mbar_wait(&bar->q_full, 0, abort, p.err, kErrTimeoutAttn)) {
        bool ok = issue_s(0);
        if (ok && n_kv > 1) ok = issue_s(1);
        for (int j = 0; ok && j < n_kv; ++j) {
          if (!mbar_wait(&bar->p_full[j % 3], (j / 3) & 1, abort, p.err, kErrTimeoutAttn)) break;
          tc_fence_after();
          if (!issue_pv(j)) break;
          if (j + 2 < n_kv) {
            if (j >= 1 && !mbar_wait(&bar->pv_done[(j - 1) % 3], ((j - 1) / 3) & 1, abort, p.err, kErrTimeoutAttn))
              break;
            if (!issue_s(j + 2)) break;
          }
        }
      }
    }
  } else {
    // ---------------- softmax warps: one query row per thread
    const int lg = warp & 3;
    const int r = lg * 32 + lane;
    const int prow = row0 + r;
    const bool valid = prow < rows_total;
    const int t_r = prow / kk;
    const uint32_t lane_off = (uint32_t)(lg * 32) << 16;
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv && ok; ++j) {
      ok = mbar_wait(&bar->s_full[j % 3], (j / 3) & 1, abort, p.err, kErrTimeoutAttn);
      tc_fence_after();
      const uint32_t sbase = tmem + lane_off + (uint32_t)((j % 3) * kTile);
      uint32_t s[128];
      tmem_ld32(sbase + 0, s);
      tmem_ld32(sbase + 32, s + 32);
      tmem_ld32(sbase + 64, s + 64);
      tmem_ld32(sbase + 96, s + 96);
      float mx = -INFINITY;
      if (j * kTile + kTile - 1 > t_first) {
        const int lim = t_r - j * kTile;   // columns > lim are in the future
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          if (c > lim) s[c] = __float_as_uint(-INFINITY);
          mx = fmaxf(mx, __uint_as_float(s[c]));
        }
      } else {
#pragma unroll
        for (int c = 0; c < 128; ++c) mx = fmaxf(mx, __uint_as_float(s[c]));
      }
      const float m_new = fmaxf(m_run, mx * sl2);
      if (j == 0) {
        m_run = m_new;
      } else {
        const bool need = m_new > m_run + kRescaleLog2;
        if (__any_sync(0xffffffffu, need)) {
          const float alpha = need ? ex2(m_run - m_new) : 1.f;
          if (need) {
            l_run *= alpha;
            m_run = m_new;
          }
          ok = mbar_wait(&bar->pv_done[(j - 1) % 3], ((j - 1) / 3) & 1, abort, p.err, kErrTimeoutAttn) && ok;
          tc_fence_after();
#pragma unroll
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t o[32];
            tmem_ld32(tmem + lane_off + kOcol + c0, o);
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st32(tmem + lane_off + kOcol + c0, o);
          }
          tmem_wait_st();
        }
      }
      float sum = 0.f;
      const float neg_m = -m_run;
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const float p0 = ex2(fmaf(__uint_as_float(s[2 * c]), sl2, neg_m));
        const float p1 = ex2(fmaf(__uint_as_float(s[2 * c + 1]), sl2, neg_m));
        sum += p0 + p1;
        s[c] = pack_bf16x2(p0, p1);
      }
      l_run += sum;
      tmem_st32(sbase + 0, s);
      tmem_st32(sbase + 32, s + 32);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar->p_full[j % 3]);
    }
    // ---------------- epilogue: O / l -> bf16
    ok = mbar_wait(&bar->pv_done[(n_kv - 1) % 3], ((n_kv - 1) / 3) & 1, abort, p.err, kErrTimeoutAttn) && ok;
    tc_fence_after();
    const float inv_l = 1.f / l_run;
    gqe_bf16_t* orow = routed ? p.o_routed + ((size_t)seq * rows_total + prow) * D
                              : p.o_sh + ((size_t)seq * p.T + prow) * D;
#pragma unroll
    for (int c0 = 0; c0 < D; c0 += 32) {
      uint32_t o[32];
      tmem_ld32(tmem + lane_off + kOcol + c0, o);
      if (valid && ok) {
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 16; ++c)
          pk[c] = pack_bf16x2(__uint_as_float(o[2 * c]) * inv_l, __uint_as_float(o[2 * c + 1]) * inv_l);
        uint4* d4 = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
        for (int c = 0; c < 4; ++c) d4[c] = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      }
    }
    if (p.lse && valid && ok) {
      const size_t li = routed ? (size_t)seq * rows_total + prow
                               : (size_t)BG * p.T * p.k + (size_t)seq * p.T + prow;
      p.lse[li] = (m_run + __log2f(l_run)) * 0.69314718055994531f;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  drain_after_abort(abort);
}

}  // namespace

template <int D>
static cudaError_t launch_d(const CUtensorMap& mQ, const CUtensorMap& mQs, const CUtensorMap& mK,
                            const CUtensorMap& mV, const AttnParams& p, cudaStream_t stream) {
  const size_t smem = AttnCfg<D>::Smem;
  auto kern = attn_prefill_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int ntq_sh = (p.T + kTile - 1) / kTile;
  const int per_level = p.B * p.G * p.k + p.B * p.n_shared;
  kern<<<ntq_sh * per_level, kThreads, smem, stream>>>(mQ, mQs, mK, mV, p);
  return cudaGetLastError();
}

cudaError_t launch_attn_prefill(const CUtensorMap& mQ, const CUtensorMap& mQs, const CUtensorMap& mK,
                                const CUtensorMap& mV, const AttnParams& p, int d,
                                cudaStream_t stream) {
  if (d == 64) return launch_d<64>(mQ, mQs, mK, mV, p, stream);
  return launch_d<128>(mQ, mQs, mK, mV, p, stream);
}

}  // namespace gqe
