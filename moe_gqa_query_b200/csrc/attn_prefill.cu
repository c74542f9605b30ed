// attn_prefill.cu -- routed causal attention for the GQE prefill on tcgen05.
//
// Every selected (token, expert) query row of one KV group attends causally to
// that group's dense K/V ("GQE" study note §3-2 2) and §1-1 attention
// equation); the shared head does the same against KV group sg (§3-2 5)).
//
// Packing: the rows (t, j) of group (b, g) are contiguous (row = t*k + j), so
// one 128-row query tile holds 128/k tokens x k selected experts and every
// K/V tile loaded for it serves all of them at once.
//
// Work item = two consecutive 128-row query tiles A and B of one sequence
// (routed: one (b, g); shared: one b).  They share every K/V tile load and run
// in ping-pong: while the softmax warpgroup of A works on S_A, the tensor core
// computes P_B V and Q_B K^T, and the other way round.  Items are launched
// heaviest first (descending 256-token level); the hardware block scheduler
// hands each SM the next item when it frees up, which balances the causal
// triangle's unequal items better than a static per-SM list.
//
// Per item: TMA brings Q_A, Q_B once and K/V tiles (128 keys) through rings of
// shared-memory stages.  tcgen05 computes S = Q K^T into tensor memory; the
// softmax warps (one query row per thread) load their S row once (row max,
// then exponentials from registers), apply the causal mask on diagonal tiles, keep
// the running max in the base-2 domain, write P (bf16) to tensor memory, and
// rescale the O accumulator only when the max grows by more than 2^8 (exact:
// l and O share the stale max); tcgen05 then adds P V (A operand from tensor
// memory) into O.
//
// CTA: 320 threads.  warps 0-3 softmax + epilogue of tile A, warps 4-7 of tile
// B, warp 8 TMA producer, warp 9 MMA issuer and tensor-memory owner.  Tensor
// memory (512 columns):
//   d=64 : S_A 0 | S_B 128 | O_A 256 | O_B 320 | P_A 384 | P_B 448
//   d=128: S_A 0 | S_B 128 | O_A 256 | O_B 384, P_X written over S_X's first
//          64 columns (the next S_X waits for P_X V to finish).
#include "attn.cuh"
#include "launch.cuh"

namespace gqe {

// Per-CTA timeline of the d = 64 kernel, built only into the diagnostic
// library (GQE_ATTN_TRACE; read by gqe_debug_attn_trace, include/gqe_trace.h):
// 12 values per CTA, globaltimer nanoseconds unless noted.
#ifdef GQE_ATTN_TRACE
constexpr int kTraceCtas = 16384;
__device__ unsigned long long g_attn_trace[kTraceCtas * 12];
#define ATTN_TRACE(...) __VA_ARGS__
#else
#define ATTN_TRACE(...)
#endif

namespace {

constexpr int kThreads = 320;
constexpr int kTile = 128;          // query rows and keys per tile
constexpr int kBox = 128 * 64 * 2;  // one TMA box: 128 rows x 64 bf16, 16 KB
constexpr float kRescaleLog2 = 8.0f;
// Single-tile kernel (d = 64): GQE_ATTN1_F2 computes the scaled logits and the
// row sums with packed f32x2 FMA/ADD (half the instructions), and POLY column
// pairs of every 16 (a template parameter) take the FMA-pipe polynomial 2^x
// instead of MUFU ex2.  Measured on B200: 2 of 16 is 3-5 % faster than 0 at
// T = 2048, where 3 of 16 is 2 % slower; at T = 32768, where the steady
// per-tile loop dominates, 3 of 16 is 1 % faster than 2 and 4 of 16 slower
// than both.  The launcher takes 3 from T = 16384 on.
#ifndef GQE_ATTN1_F2
#define GQE_ATTN1_F2 1
#endif
constexpr int kPolyShortT = 2, kPolyLongT = 3, kPolyLongFromT = 16384;
#ifndef GQE_ATTN_POLY_PAIRS
#define GQE_ATTN_POLY_PAIRS 0
#endif
// Paired kernel (d = 128): column pairs (of every 16) whose exponentials run as
// the polynomial.  There the softmax is bound by instruction issue, not by MUFU
// throughput (measured: 0, 3, 5 and 8 of 16 within 3 % of each other), so the
// default keeps every exponential on MUFU.
constexpr int kPolyPairs = GQE_ATTN_POLY_PAIRS;

struct __align__(8) AttnBarriers {
  uint64_t q_full;
  uint64_t k_full[4], k_empty[4], v_full[4], v_empty[4];
  uint64_t s_full[2], p_full[2], pv_done[2];
  uint32_t tmem_base;
  int abort;
};

template <int D>
struct AttnCfg {
  static constexpr int NB = D / 64;                  // 64-column boxes per tile
  static constexpr int ST = (D == 64) ? 3 : 2;       // K/V ring depth
  static constexpr int QBytes = NB * kBox;           // one Q tile
  static constexpr int KVBytes = NB * kBox;
  static constexpr bool kPAliasS = (D != 64);
  // tensor-memory columns of tile x's S, O and P
  __host__ __device__ static constexpr uint32_t scol(int x) { return x ? 128u : 0u; }
  __host__ __device__ static constexpr uint32_t ocol(int x) { return x ? (uint32_t)(256 + D) : 256u; }
  __host__ __device__ static constexpr uint32_t pcol(int x) {
    return kPAliasS ? scol(x) : (x ? 448u : 384u);
  }
  static constexpr size_t Smem = 1024 + 2 * QBytes + 2 * ST * KVBytes + sizeof(AttnBarriers);
};

struct TileInfo {
  int row0;      // first packed row
  int n_kv;      // key tiles 0..n_kv-1 (0: tile absent)
  int t_first;   // first token of the tile
};

__device__ __forceinline__ TileInfo tile_info(int qt, int rows_total, int kk, int T) {
  TileInfo ti;
  ti.row0 = qt * kTile;
  if (ti.row0 >= rows_total) {
    ti.n_kv = 0;
    ti.t_first = 0;
    return ti;
  }
  ti.t_first = ti.row0 / kk;
  const int t_last = min(T - 1, (ti.row0 + kTile - 1) / kk);
  ti.n_kv = t_last / kTile + 1;
  return ti;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
attn_prefill_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapQs,
                    const __grid_constant__ CUtensorMap mapK, const __grid_constant__ CUtensorMap mapV,
                    AttnParams p) {
  using C = AttnCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                                 // [2][QBytes]
  uint8_t* sK = sQ + 2 * C::QBytes;
  uint8_t* sV = sK + C::ST * C::KVBytes;
  AttnBarriers* bar = reinterpret_cast<AttnBarriers*>(sV + C::ST * C::KVBytes);
  volatile int* abort = &bar->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work item: level-major (heaviest first), then routed pairs, then shared
  const int BG = p.B * p.G;
  const int per_level = BG * p.k + p.B * p.n_shared;
  const int n_levels = (p.T + 2 * kTile - 1) / (2 * kTile);
  const int level = n_levels - 1 - (int)blockIdx.x / per_level;
  const int i = blockIdx.x % per_level;
  bool routed;
  int seq, pair, kvseq, kk, rows_total;
  if (i < BG * p.k) {
    routed = true;
    seq = i % BG;
    pair = level * p.k + i / BG;
    kvseq = seq;
    kk = p.k;
    rows_total = p.T * p.k;
  } else {
    routed = false;
    seq = i - BG * p.k;
    pair = level;
    kvseq = seq * p.G + p.sg;
    kk = 1;
    rows_total = p.T;
  }
  const TileInfo tA = tile_info(2 * pair, rows_total, kk, p.T);
  const TileInfo tB = tile_info(2 * pair + 1, rows_total, kk, p.T);
  if (tA.n_kv == 0) return;
  const int n_kv = max(tA.n_kv, tB.n_kv);
  const CUtensorMap* mq = routed ? &mapQ : &mapQs;

  if (threadIdx.x == 0) {
    mbar_init(&bar->q_full, 1);
    for (int s = 0; s < C::ST; ++s) {
      mbar_init(&bar->k_full[s], 1);
      mbar_init(&bar->k_empty[s], 1);
      mbar_init(&bar->v_full[s], 1);
      mbar_init(&bar->v_empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bar->s_full[x], 1);
      mbar_init(&bar->p_full[x], 128);
      mbar_init(&bar->pv_done[x], 1);
    }
    bar->abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(mq);
    tma_prefetch_desc(&mapK);
    tma_prefetch_desc(&mapV);
  }
  if (warp == 9) tmem_alloc(&bar->tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;
  pdl_launch_dependents();
  pdl_wait();

  if (warp == 8) {
    if (lane == 0) {
      // ---------------- producer: Q_A, Q_B once; then K_0, V_0, K_1, V_1, ...
      const int nq = tB.n_kv > 0 ? 2 : 1;
      mbar_arrive_expect_tx(&bar->q_full, nq * C::QBytes);
      for (int x = 0; x < nq; ++x)
        for (int bx = 0; bx < C::NB; ++bx)
          tma_load_3d(sQ + x * C::QBytes + bx * kBox, mq, &bar->q_full, bx * 64, (x ? tB : tA).row0, seq);
      for (int j = 0; j < n_kv; ++j) {
        const int s = j % C::ST;
        const uint32_t ph = ((j / C::ST) & 1) ^ 1;
        if (j >= C::ST && !mbar_wait(&bar->k_empty[s], ph, abort, p.err, kErrTimeoutAttn)) break;
        mbar_arrive_expect_tx(&bar->k_full[s], C::KVBytes);
        for (int bx = 0; bx < C::NB; ++bx)
          tma_load_3d(sK + s * C::KVBytes + bx * kBox, &mapK, &bar->k_full[s], bx * 64, j * kTile, kvseq);
        if (j >= C::ST && !mbar_wait(&bar->v_empty[s], ph, abort, p.err, kErrTimeoutAttn)) break;
        mbar_arrive_expect_tx(&bar->v_full[s], C::KVBytes);
        for (int bx = 0; bx < C::NB; ++bx)
          tma_load_3d(sV + s * C::KVBytes + bx * kBox, &mapV, &bar->v_full[s], bx * 64, j * kTile, kvseq);
      }
    }
  } else if (warp == 9) {
    if (lane == 0) {
      // ---------------- MMA issuer
      constexpr uint32_t idesc_s = idesc_bf16_f32(kTile, kTile, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(kTile, D, false, true);
      const int nA = tA.n_kv, nB = tB.n_kv;
      bool ok = true;
      auto issue_s = [&](int x, int j) {
        const int s = j % C::ST;
        if (!mbar_wait(&bar->k_full[s], (j / C::ST) & 1, abort, p.err, kErrTimeoutAttn)) return false;
        tc_fence_after();
        const uint32_t q0 = smem_u32(sQ + x * C::QBytes);
        const uint32_t k0 = smem_u32(sK + s * C::KVBytes);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (ks >> 2) * kBox + (ks & 3) * 32;
          umma_ss(tmem + C::scol(x), sdesc_sw128(q0 + off, 16, 1024), sdesc_sw128(k0 + off, 16, 1024),
                  idesc_s, ks > 0);
        }
        umma_commit(&bar->s_full[x]);
        // K_j's last reader is tile B when it reaches j, else tile A
        if (x == 1 || nB <= j) umma_commit(&bar->k_empty[s]);
        return true;
      };
      auto issue_pv = [&](int x, int j) {
        const int s = j % C::ST;
        if (!mbar_wait(&bar->v_full[s], (j / C::ST) & 1, abort, p.err, kErrTimeoutAttn)) return false;
        tc_fence_after();
        const uint32_t v0 = smem_u32(sV + s * C::KVBytes);
#pragma unroll
        for (int ks = 0; ks < kTile / 16; ++ks)
          umma_ts(tmem + C::ocol(x), tmem + C::pcol(x) + ks * 8, sdesc_sw128(v0 + ks * 2048, kBox, 1024),
                  idesc_o, (j > 0 || ks > 0));
        umma_commit(&bar->pv_done[x]);
        if (x == 1 || nB <= j) umma_commit(&bar->v_empty[s]);
        return true;
      };
      if (mbar_wait(&bar->q_full, 0, abort, p.err, kErrTimeoutAttn)) {
        ok = issue_s(0, 0);
        if (ok && nB > 0) ok = issue_s(1, 0);
        for (int j = 0; ok && j < n_kv; ++j) {
          for (int x = 0; x < 2 && ok; ++x) {
            const int nx = x ? nB : nA;
            if (j >= nx) continue;
            ok = mbar_wait(&bar->p_full[x], j & 1, abort, p.err, kErrTimeoutAttn);
            tc_fence_after();
            ok = ok && issue_pv(x, j);
            if (ok && j + 1 < nx) {
              if (C::kPAliasS) ok = mbar_wait(&bar->pv_done[x], j & 1, abort, p.err, kErrTimeoutAttn);
              ok = ok && issue_s(x, j + 1);
            }
          }
        }
      }
    }
  } else {
    // ---------------- softmax warpgroups: one query row per thread
    const int x = warp >> 2;                 // 0: tile A, 1: tile B
    const TileInfo ti = x ? tB : tA;
    if (ti.n_kv > 0) {
      const int lg = warp & 3;
      const int r = lg * 32 + lane;
      const int prow = ti.row0 + r;
      const bool valid = prow < rows_total;
      const int t_r = prow / kk;
      const uint32_t lane_off = (uint32_t)(lg * 32) << 16;
      const uint32_t s_base = tmem + lane_off + C::scol(x);
      const uint32_t p_base = tmem + lane_off + C::pcol(x);
      const uint32_t o_base = tmem + lane_off + C::ocol(x);
      const float sl2 = p.scale_log2;
      float m_run = -INFINITY, l_run = 0.f;
      bool ok = true;
      for (int j = 0; j < ti.n_kv && ok; ++j) {
        ok = mbar_wait(&bar->s_full[x], j & 1, abort, p.err, kErrTimeoutAttn);
        tc_fence_after();
        const bool diag = j * kTile + kTile - 1 > ti.t_first;
        const int lim = t_r - j * kTile;     // columns > lim are in the future
        // the whole S row, once (two loads, one wait), then the row max with
        // 8 independent partial maxima
        uint32_t s[128];
        tmem_ld128(s_base, s);
        if (diag) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c > lim) s[c] = __float_as_uint(-INFINITY);
        }
        float m8[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) m8[q] = -INFINITY;
#pragma unroll
        for (int c = 0; c < 64; ++c)
          m8[c & 7] = fmax3(m8[c & 7], __uint_as_float(s[2 * c]), __uint_as_float(s[2 * c + 1]));
        const float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                               fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
        const float m_new = fmaxf(m_run, mx * sl2);
        // lazy rescale: only when some row's max grew by more than 2^8; O itself
        // is rescaled after the exponentials (S registers are dead by then) and
        // before P is released to the MMA
        bool rescale = false;
        float alpha = 1.f;
        if (j == 0) {
          m_run = m_new;
        } else {
          const bool need = m_new > m_run + kRescaleLog2;
          rescale = __any_sync(0xffffffffu, need);
          if (need) {
            alpha = ex2(m_run - m_new);
            l_run *= alpha;
            m_run = m_new;
          }
        }
        // exponentials (MUFU, or the FMA-pipe polynomial for kPolyPairs of every
        // 16 pairs), row sum, P (bf16) into tensor memory
        const float neg_m = -m_run;
        float sum4[4] = {0.f, 0.f, 0.f, 0.f};   // independent partial sums
#pragma unroll
        for (int c0 = 0; c0 < 64; c0 += 16) {
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int q = c0 + c;          // column pair
            const float x0 = fmaf(__uint_as_float(s[2 * q]), sl2, neg_m);
            const float x1 = fmaf(__uint_as_float(s[2 * q + 1]), sl2, neg_m);
            float p0, p1;
            if ((q & 15) < kPolyPairs) {
              p0 = exp2_poly(x0);
              p1 = exp2_poly(x1);
            } else {
              p0 = ex2(x0);
              p1 = ex2(x1);
            }
            sum4[(c & 1) * 2] += p0;
            sum4[(c & 1) * 2 + 1] += p1;
            pk[c] = pack_bf16x2(p0, p1);
          }
          tmem_st16(p_base + c0, pk);
        }
        l_run += (sum4[0] + sum4[1]) + (sum4[2] + sum4[3]);
        if (rescale) {
          ok = mbar_wait(&bar->pv_done[x], (j - 1) & 1, abort, p.err, kErrTimeoutAttn) && ok;
          tc_fence_after();
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t o[32];
            tmem_ld32(o_base + c0, o);
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st32(o_base + c0, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bar->p_full[x]);
      }
      // ---------------- epilogue: O / l -> bf16
      ok = mbar_wait(&bar->pv_done[x], (ti.n_kv - 1) & 1, abort, p.err, kErrTimeoutAttn) && ok;
      tc_fence_after();
      const float inv_l = 1.f / l_run;
      gqe_bf16_t* orow = routed ? p.o_routed + ((size_t)seq * rows_total + prow) * D
                                : p.o_sh + ((size_t)seq * p.T + prow) * D;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o[32];
        tmem_ld32(o_base + c0, o);
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
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  drain_after_abort(abort);
}

// ---------------------------------------------------------------------------
// d = 64: one 128-row query tile per CTA in 256 tensor-memory columns
// (S 0-127 | P 128-191 | O 192-255), so two CTAs share an SM.  The hardware
// block scheduler then overlaps one item's set-up and epilogue with another
// item's work, which matters when causal rows are short.
//
// The softmax warps copy S(j) into registers and release its columns at once
// (s_free), so the MMA warp computes S(j+1) = Q K_{j+1}^T while the
// exponentials of tile j run.  Before writing P(j+1) (and rescaling O) the
// softmax waits for P(j) V to finish (pv_done).  P(j) is announced in two
// halves: the V-side thread issues the first four 16-key steps of P(j) V once
// keys 0-63 of P(j) (and the rescaled O) are in tensor memory (p_half), while
// the softmax computes keys 64-127, and the last four at p_full.  One thread
// issues every P V step in order, so the result does not depend on timing.
// Measured on B200 (same box, interleaved): 75.8 -> 73.7 us at T = 2048,
// 1.487 -> 1.464 ms at T = 32768.
struct __align__(8) Attn1Barriers {
  uint64_t q_full;
  uint64_t k_full[4], k_empty[4], v_full[4], v_empty[4];
  uint64_t s_full, s_free, p_half, p_full, pv_done;
  uint32_t tmem_base;
  int abort;
};

constexpr int kSingleST = 2;   // two CTAs per SM must fit in 228 KB of shared memory
constexpr size_t kSingleSmem = 1024 + kBox + 2 * kSingleST * kBox + sizeof(Attn1Barriers);

template <int POLY>
__global__ void __launch_bounds__(192, 2)
attn_prefill_single_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapQs,
                           const __grid_constant__ CUtensorMap mapK, const __grid_constant__ CUtensorMap mapV,
                           AttnParams p) {
  constexpr int D = 64;
  ATTN_TRACE(const unsigned long long tr_entry = globaltimer();
             unsigned long long* TR = blockIdx.x < kTraceCtas ? g_attn_trace + (size_t)blockIdx.x * 12 : nullptr;
             unsigned long long tr_ws = 0, tr_wpv = 0;)
  constexpr int ST = kSingleST;
  constexpr uint32_t kS = 0, kP = 128, kO = 192;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + kBox;
  uint8_t* sV = sK + ST * kBox;
  Attn1Barriers* bar = reinterpret_cast<Attn1Barriers*>(sV + ST * kBox);
  volatile int* abort = &bar->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work item: one q-tile, level-major (heaviest first)
  const int BG = p.B * p.G;
  const int per_level = BG * p.k + p.B * p.n_shared;
  const int n_levels = (p.T + kTile - 1) / kTile;
  const int level = n_levels - 1 - (int)blockIdx.x / per_level;
  const int i = blockIdx.x % per_level;
  bool routed;
  int seq, qt, kvseq, kk, rows_total;
  if (i < BG * p.k) {
    routed = true;
    seq = i % BG;
    qt = level * p.k + i / BG;
    kvseq = seq;
    kk = p.k;
    rows_total = p.T * p.k;
  } else {
    routed = false;
    seq = i - BG * p.k;
    qt = level;
    kvseq = seq * p.G + p.sg;
    kk = 1;
    rows_total = p.T;
  }
  const TileInfo ti = tile_info(qt, rows_total, kk, p.T);
  if (ti.n_kv == 0) return;
  const int n_kv = ti.n_kv;
  const CUtensorMap* mq = routed ? &mapQ : &mapQs;

  // The K-side thread sets up the barriers and puts Q and the first K and V
  // tiles in flight before the CTA-wide barrier, so they load while tensor
  // memory is allocated.
  if (warp == 4 && lane == 0) {
    mbar_init(&bar->q_full, 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(&bar->k_full[s], 1);
      mbar_init(&bar->k_empty[s], 1);
      mbar_init(&bar->v_full[s], 1);
      mbar_init(&bar->v_empty[s], 1);
    }
    mbar_init(&bar->s_full, 1);
    mbar_init(&bar->s_free, 128);
    mbar_init(&bar->p_half, 128);
    mbar_init(&bar->p_full, 128);
    mbar_init(&bar->pv_done, 1);
    bar->abort = 0;
    fence_mbar_init();
    pdl_wait();
    mbar_arrive_expect_tx(&bar->q_full, kBox);
    tma_load_3d(sQ, mq, &bar->q_full, 0, ti.row0, seq);
    for (int j = 0; j < ST && j < n_kv; ++j) {
      mbar_arrive_expect_tx(&bar->k_full[j], kBox);
      tma_load_3d(sK + j * kBox, &mapK, &bar->k_full[j], 0, j * kTile, kvseq);
      mbar_arrive_expect_tx(&bar->v_full[j], kBox);
      tma_load_3d(sV + j * kBox, &mapV, &bar->v_full[j], 0, j * kTile, kvseq);
    }
  }
  if (warp == 5) tmem_alloc(&bar->tmem_base, 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;
  pdl_launch_dependents();
  pdl_wait();
  ATTN_TRACE(if (TR && threadIdx.x == 0) {
    unsigned sm;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(sm));
    TR[0] = sm | ((unsigned long long)n_kv << 16) | ((unsigned long long)routed << 31);
    TR[1] = tr_entry;
    TR[2] = globaltimer();
  })

  if (warp == 4) {
    if (lane == 0) {
      // ---------------- K side: Q and K tiles by TMA, S(j) = Q K_j^T.  S(j+1)
      // is issued as soon as the softmax holds S(j) in registers (s_free), so
      // it runs while the exponentials of tile j do.
      constexpr uint32_t idesc_s = idesc_bf16_f32(kTile, kTile, false, false);
      const uint32_t q0 = smem_u32(sQ);
      bool ok = mbar_wait(&bar->q_full, 0, abort, p.err, kErrTimeoutAttn);
      ATTN_TRACE(if (TR) TR[3] = globaltimer();)
      for (int j = 0; ok && j < n_kv; ++j) {
        const int s = j % ST;
        if (j > 0) ok = mbar_wait(&bar->s_free, (j - 1) & 1, abort, p.err, kErrTimeoutAttn);
        ok = ok && mbar_wait(&bar->k_full[s], (j / ST) & 1, abort, p.err, kErrTimeoutAttn);
        if (!ok) break;
        tc_fence_after();
        const uint32_t k0 = smem_u32(sK + s * kBox);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          umma_ss(tmem + kS, sdesc_sw128(q0 + ks * 32, 16, 1024), sdesc_sw128(k0 + ks * 32, 16, 1024), idesc_s,
                  ks > 0);
        umma_commit(&bar->s_full);
        umma_commit(&bar->k_empty[s]);
        if (j + ST < n_kv) {
          // refill this stage with K_{j+ST} once S(j) has read it
          ok = mbar_wait(&bar->k_empty[s], (j / ST) & 1, abort, p.err, kErrTimeoutAttn);
          if (!ok) break;
          mbar_arrive_expect_tx(&bar->k_full[s], kBox);
          tma_load_3d(sK + s * kBox, &mapK, &bar->k_full[s], 0, (j + ST) * kTile, kvseq);
        }
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      // ---------------- V side: V tiles by TMA, O += P(j) V_j once P(j) is in
      // tensor memory (a second issuing thread: an MMA of N = 64 takes the
      // tensor pipe for less time than one thread needs to issue it)
      constexpr uint32_t idesc_o = idesc_bf16_f32(kTile, D, false, true);
      bool ok = true;
      for (int j = 0; ok && j < n_kv; ++j) {
        const int s = j % ST;
        // keys 0-63 of P(j) V as soon as the softmax has stored that half of
        // P(j) (p_half), keys 64-127 once all of it is in (p_full)
        ok = mbar_wait(&bar->p_half, j & 1, abort, p.err, kErrTimeoutAttn);
        ok = ok && mbar_wait(&bar->v_full[s], (j / ST) & 1, abort, p.err, kErrTimeoutAttn);
        if (!ok) break;
        tc_fence_after();
        const uint32_t v0 = smem_u32(sV + s * kBox);
#pragma unroll
        for (int ks = 0; ks < kTile / 32; ++ks)
          umma_ts(tmem + kO, tmem + kP + ks * 8, sdesc_sw128(v0 + ks * 2048, kBox, 1024), idesc_o,
                  (j > 0 || ks > 0));
        ok = mbar_wait(&bar->p_full, j & 1, abort, p.err, kErrTimeoutAttn);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int ks = kTile / 32; ks < kTile / 16; ++ks)
          umma_ts(tmem + kO, tmem + kP + ks * 8, sdesc_sw128(v0 + ks * 2048, kBox, 1024), idesc_o, 1u);
        umma_commit(&bar->pv_done);
        umma_commit(&bar->v_empty[s]);
        if (j + ST < n_kv) {
          ok = mbar_wait(&bar->v_empty[s], (j / ST) & 1, abort, p.err, kErrTimeoutAttn);
          if (!ok) break;
          mbar_arrive_expect_tx(&bar->v_full[s], kBox);
          tma_load_3d(sV + s * kBox, &mapV, &bar->v_full[s], 0, (j + ST) * kTile, kvseq);
        }
      }
    }
  } else {
    // ---------------- softmax: warps 0-3, one query row per thread
    const int lg = warp;
    const int r = lg * 32 + lane;
    const int prow = ti.row0 + r;
    const bool valid = prow < rows_total;
    const int t_r = prow / kk;
    const uint32_t lane_off = (uint32_t)(lg * 32) << 16;
    const uint32_t s_base = tmem + lane_off + kS;
    const uint32_t p_base = tmem + lane_off + kP;
    const uint32_t o_base = tmem + lane_off + kO;
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv && ok; ++j) {
      ATTN_TRACE(const unsigned long long tw0 = threadIdx.x == 0 ? globaltimer() : 0ull;)
      ok = mbar_wait(&bar->s_full, j & 1, abort, p.err, kErrTimeoutAttn);
      ATTN_TRACE(if (TR && threadIdx.x == 0) {
        const unsigned long long tw1 = globaltimer();
        if (j == 0) TR[4] = tw1;
        else tr_ws += tw1 - tw0;
      })
      tc_fence_after();
      const bool diag = j * kTile + kTile - 1 > ti.t_first;
      const int lim = t_r - j * kTile;
      uint32_t s[128];
      tmem_ld128(s_base, s);
      tc_fence_before();
      mbar_arrive(&bar->s_free);     // S(j) is in registers; the MMA warp may overwrite it
      if (diag) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c > lim) s[c] = __float_as_uint(-INFINITY);
      }
      float m8[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) m8[q] = -INFINITY;
#pragma unroll
      for (int c = 0; c < 64; ++c)
        m8[c & 7] = fmax3(m8[c & 7], __uint_as_float(s[2 * c]), __uint_as_float(s[2 * c + 1]));
      const float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                             fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      const float m_new = fmaxf(m_run, mx * sl2);
      bool rescale = false;
      float alpha = 1.f;
      if (j == 0) {
        m_run = m_new;
      } else {
        const bool need = m_new > m_run + kRescaleLog2;
        rescale = __any_sync(0xffffffffu, need);
        if (need) {
          alpha = ex2(m_run - m_new);
          l_run *= alpha;
          m_run = m_new;
        }
      }
      const float neg_m = -m_run;
#if GQE_ATTN1_F2
      const unsigned long long sl2x2 = f2_pack(sl2, sl2), negm2 = f2_pack(neg_m, neg_m);
      unsigned long long sum2[2] = {0ull, 0ull};
#else
      float sum4[4] = {0.f, 0.f, 0.f, 0.f};
#endif
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const int q = h * 32 + c;
#if GQE_ATTN1_F2
          const unsigned long long x =
              f2_fma(f2_pack(__uint_as_float(s[2 * q]), __uint_as_float(s[2 * q + 1])), sl2x2, negm2);
          float p0, p1;
          if ((c & 15) < POLY) {
            exp2_poly2(x, p0, p1);
          } else {
            float x0, x1;
            f2_unpack(x, x0, x1);
            p0 = ex2(x0);
            p1 = ex2(x1);
          }
          sum2[c & 1] = f2_add(sum2[c & 1], f2_pack(p0, p1));
#else
          const float x0 = fmaf(__uint_as_float(s[2 * q]), sl2, neg_m);
          const float x1 = fmaf(__uint_as_float(s[2 * q + 1]), sl2, neg_m);
          const float p0 = ex2(x0), p1 = ex2(x1);
          sum4[(c & 1) * 2] += p0;
          sum4[(c & 1) * 2 + 1] += p1;
#endif
          pk[c] = pack_bf16x2(p0, p1);
        }
        // P(j-1) V must be done before P is overwritten and O rescaled; the
        // rescaled O and the first half of P(j) are announced together
        if (h == 0 && j > 0) {
          ATTN_TRACE(const unsigned long long tp0 = threadIdx.x == 0 ? globaltimer() : 0ull;)
          ok = mbar_wait(&bar->pv_done, (j - 1) & 1, abort, p.err, kErrTimeoutAttn) && ok;
          ATTN_TRACE(if (threadIdx.x == 0) tr_wpv += globaltimer() - tp0;)
          tc_fence_after();
          if (rescale) {
#pragma unroll 1
            for (int c0 = 0; c0 < D; c0 += 32) {
              uint32_t o[32];
              tmem_ld32(o_base + c0, o);
#pragma unroll
              for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
              tmem_st32(o_base + c0, o);
            }
          }
        }
        tmem_st32(p_base + h * 32, pk);
        if (h == 0) {
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(&bar->p_half);
        }
      }
#if GQE_ATTN1_F2
      {
        float a0, a1, b0, b1;
        f2_unpack(sum2[0], a0, a1);
        f2_unpack(sum2[1], b0, b1);
        l_run += (a0 + a1) + (b0 + b1);
      }
#else
      l_run += (sum4[0] + sum4[1]) + (sum4[2] + sum4[3]);
#endif
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar->p_full);
      ATTN_TRACE(if (TR && threadIdx.x == 0 && j == 0) TR[5] = globaltimer();)
    }
    ATTN_TRACE(if (TR && threadIdx.x == 0) {
      TR[6] = globaltimer();
      TR[10] = tr_ws;
      TR[11] = tr_wpv;
    })
    // ---------------- epilogue: O / l -> bf16
    ok = mbar_wait(&bar->pv_done, (n_kv - 1) & 1, abort, p.err, kErrTimeoutAttn) && ok;
    ATTN_TRACE(if (TR && threadIdx.x == 0) TR[7] = globaltimer();)
    tc_fence_after();
    const float inv_l = 1.f / l_run;
    gqe_bf16_t* orow = routed ? p.o_routed + ((size_t)seq * rows_total + prow) * D
                              : p.o_sh + ((size_t)seq * p.T + prow) * D;
    {
      uint32_t o[64];
      tmem_ld64(o_base, o);
      if (valid && ok) {
        uint4* d4 = reinterpret_cast<uint4*>(orow);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            pk[e] = pack_bf16x2(__uint_as_float(o[8 * c + 2 * e]) * inv_l, __uint_as_float(o[8 * c + 2 * e + 1]) * inv_l);
          d4[c] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      }
    }
    if (p.lse && valid && ok) {
      const size_t li = routed ? (size_t)seq * rows_total + prow
                               : (size_t)BG * p.T * p.k + (size_t)seq * p.T + prow;
      p.lse[li] = (m_run + __log2f(l_run)) * 0.69314718055994531f;
    }
    ATTN_TRACE(if (TR && threadIdx.x == 0) TR[8] = globaltimer();)
  }
  tc_fence_before();
  __syncthreads();
  ATTN_TRACE(if (TR && threadIdx.x == 0) TR[9] = globaltimer();)
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
  drain_after_abort(abort);
}

}  // namespace

template <int D>
static cudaError_t launch_d(const CUtensorMap& mQ, const CUtensorMap& mQs, const CUtensorMap& mK,
                            const CUtensorMap& mV, const AttnParams& p, cudaStream_t stream) {
  const size_t smem = AttnCfg<D>::Smem;
  auto kern = attn_prefill_kernel<D>;
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  const int n_levels = (p.T + 2 * kTile - 1) / (2 * kTile);
  const int per_level = p.B * p.G * p.k + p.B * p.n_shared;
  return launch_kernel(kern, dim3(n_levels * per_level), dim3(kThreads), smem, stream, 1, mQ, mQs, mK, mV, p);
}

static cudaError_t launch_single(const CUtensorMap& mQ, const CUtensorMap& mQs, const CUtensorMap& mK,
                                 const CUtensorMap& mV, const AttnParams& p, cudaStream_t stream) {
  auto kern = p.T >= kPolyLongFromT ? attn_prefill_single_kernel<kPolyLongT> : attn_prefill_single_kernel<kPolyShortT>;
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kern), kSingleSmem);
  if (e != cudaSuccess) return e;
  const int n_levels = (p.T + kTile - 1) / kTile;
  const int per_level = p.B * p.G * p.k + p.B * p.n_shared;
  return launch_kernel(kern, dim3(n_levels * per_level), dim3(192), kSingleSmem, stream, 1, mQ, mQs, mK, mV, p);
}

cudaError_t launch_attn_prefill(const CUtensorMap& mQ, const CUtensorMap& mQs, const CUtensorMap& mK,
                                const CUtensorMap& mV, const AttnParams& p, int d, cudaStream_t stream) {
#ifndef GQE_ATTN_PAIRED_D64
  if (d == 64) return launch_single(mQ, mQs, mK, mV, p, stream);
#endif
  if (d == 64) return launch_d<64>(mQ, mQs, mK, mV, p, stream);
  return launch_d<128>(mQ, mQs, mK, mV, p, stream);
}

}  // namespace gqe

#ifdef GQE_ATTN_TRACE
extern "C" int gqe_debug_attn_trace(void* host, size_t bytes) {
  if (!host || bytes > sizeof(gqe::g_attn_trace)) return 1;
  return cudaMemcpyFromSymbol(host, gqe::g_attn_trace, bytes) == cudaSuccess ? 0 : 4;
}
#endif
