// gemm.cuh -- parameters and launchers of the tcgen05 GEMMs (gemm.cu).
#pragma once

#include "sm100.cuh"

namespace gqe {

typedef uint16_t gqe_bf16_t;

enum EpiMode : int {
  kEpiRowMajor = 0,   // out[row * ldo + n]
  kEpiHeads = 1,      // out[b, g, t, dd] with row = b*T + t, n = g*d + dd
  kEpiCacheRow = 2,   // out[b, g, cache_len[b]-1, dd] with row = b
  kEpiRows = 3,       // out[dst_row * ldo + n], dst_row given per tile row
};

struct EpiParams {
  gqe_bf16_t* out0;
  gqe_bf16_t* out1;      // second weight's output (K / V pair)
  const int* cache_len;
  int mode;
  int ldo;
  int n_limit;           // columns >= n_limit are not written
  int T, G, d, L_max;
  unsigned* err;         // device error word
  int store_mode;        // dense kernels: kStorePerThread or a TMA store layout
  int ksplit;            // kStoreReduceF32: K split into this many slices (<= 1: none)
};

// How the dense kernels write their output.
enum StoreMode : int {
  kStorePerThread = 0,   // each thread stores its row (any EpiMode)
  kStoreTma2d = 1,       // kEpiRowMajor through maps over [M, N], box 64 cols x 32 rows
  kStoreTmaHeads = 2,    // kEpiHeads through maps over [B*G, T, d], box 64 x 32 x 1 (T % 32 == 0)
  kStoreReduceF32 = 3,   // fp32 tiles reduce-added into an fp32 [M, N] map, box 32 cols x 32 rows
};

// Token-to-expert permutation produced by perm.cu, consumed by the routed GEMM.
// Segment s = g*E + e holds its entries at [s*seg_cap, s*seg_cap + seg_cnt[s]).
struct RoutedParams {
  const int* src_row;     // [n_seg * seg_cap] token row of x
  const int* dst_row;     // [n_seg * seg_cap] row of q_routed [B, G, T, k]
  const int* seg_cnt;     // [n_seg]
  int* expert_counts;     // [n_seg] copy of seg_cnt for the caller, or null
  int seg_cap;            // entries reserved per segment (= tokens)
  int n_seg;              // G * E
  int max_routed_tiles;   // upper bound on the routed 128-row tiles
  int shared_tiles;       // 128-row tiles of the shared head (0 without one)
  int n_tokens;           // B * T (shared-head tiles)
  int K;                  // d_model
  int d;                  // head width (= tile N)
};

// Output tile width for a weight with n_per_weight rows: 256 when it divides, else 128.
int dense_tile_n(int n_per_weight, int M);
int num_sms();

// mapO0 / mapO1: output maps for ep.store_mode != kStorePerThread.
// mn: bit 0 -> A is stored [K, M] (map over [K rows, M cols], box 64 x 64),
// bit 1 -> B is stored [K, N] (same); otherwise [M, K] / [N, K].  K may then
// be rounded up to a multiple of 64 (the maps' zero fill covers the tail).
cudaError_t launch_gemm_dense(const CUtensorMap& mapA, const CUtensorMap& mapB0,
                              const CUtensorMap& mapB1, const CUtensorMap& mapO0,
                              const CUtensorMap& mapO1, const EpiParams& ep, int M, int K,
                              int n_tiles_b0, int n_tiles_total, int bn, cudaStream_t stream, int mn = 0);

// Where the pair GEMM's A operand comes from.  kASingle: one map over A [M, K]
// (box 64 x 128).  kASlots: the output projection's h = [hard slots, weighted
// sum, shared] read without h: k-block kb (64 columns of slot kb*64/d) comes
// from o_routed through a map over [B*G*T, k*d] (box 64 x 128; needs
// T % 128 == 0 so a box stays inside one (b, g)), from the weighted-sum buffer
// [M, d] or from o_sh [M, d].
enum ASourceMode : int { kASingle = 0, kASlots = 1 };
struct ASource {
  int mode;
  int k, G, T, d;
  int route;    // kASlots: 1 when slot k*G is the weighted-sum slot, 0 when the shared slot follows the hard ones
};

// 256 x 256 tiles over CTA pairs (bn must be 256); W maps with 128-row boxes,
// weights' rows a multiple of 256.  mapR / mapS: the weighted-sum and shared
// slot maps of kASlots (ignored for kASingle).
cudaError_t launch_gemm_dense_pair(const CUtensorMap& mapA, const CUtensorMap& mapR, const CUtensorMap& mapS,
                                   const ASource& as, const CUtensorMap& mapB0,
                                   const CUtensorMap& mapB1, const CUtensorMap& mapO0,
                                   const CUtensorMap& mapO1, const EpiParams& ep, int M, int K,
                                   int n_tiles_b0, int n_tiles_total, int bn, cudaStream_t stream, int mn = 0);

cudaError_t launch_gemm_routed(const CUtensorMap& mapWq, const CUtensorMap& mapWsh,
                               const gqe_bf16_t* x, const RoutedParams& rp, const EpiParams& epr,
                               const EpiParams& eps, cudaStream_t stream);

}  // namespace gqe
