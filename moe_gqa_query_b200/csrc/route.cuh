// route.cuh -- parameters and launchers of the router, the token-to-expert
// permutation and the output-construction kernels.
#pragma once

#include "sm100.cuh"

namespace gqe {

struct RouterParams {
  const uint16_t* x;      // [N, D] bf16
  const uint16_t* Wr;     // [D, G*E] bf16
  const float* bias;      // [G*E] or null
  int* topk_idx;          // [N, G, k]
  float* topk_w;          // [N, G, k]
  float* probs;           // [N, G, E] or null
  int N, D, G, E, k, scope;   // scope: 0 token, 1 group, 2 none (w = p)
  unsigned* err;          // device error word (bounded waits of the tcgen05 router)
};
cudaError_t launch_router(const RouterParams& p, cudaStream_t stream);
// tcgen05 router streaming x and Wr by TMA: mapX over x [N, D] with a box of
// 64 columns x R rows, R = router_tc_tile_rows(N); mapW over Wr [D, G*E] with
// a box of 64 x 64 (G*E a multiple of 8).  Returns cudaErrorNotSupported for
// shapes it does not take (the caller falls back to the CUDA-core routers).
int router_tc_tile_rows(int N);
cudaError_t launch_router_tc(const CUtensorMap& mapX, const CUtensorMap& mapW, const RouterParams& p, int R,
                             cudaStream_t stream);

// Token-to-expert permutation workspace (int32 arrays, see perm.cu): segment
// counters, then per segment `cap` slots of source and destination rows.
struct PermLayout {
  int n_seg;         // G*E
  int cap;           // slots per segment (= tokens: a token enters a segment at most once)
  size_t off_seg_cnt, off_src_row, off_dst_row;
  size_t bytes;
};
PermLayout perm_layout(int N, int G, int E, int k);
// Zeroes the counters and fills the segments in one kernel.
cudaError_t launch_permutation(const int* topk_idx, int N, int T, int G, int E, int k, void* ws,
                               const PermLayout& L, cudaStream_t stream);

cudaError_t launch_router_stats(const float* probs, const int* topk_idx, int N, int G, int E, int k,
                                int* counts, float* prob_sum, cudaStream_t stream);

struct CombineParams {
  const uint16_t* o_routed;   // [B, G, T, k, d]
  const uint16_t* o_sh;       // [B, T, d]
  const float* w;             // [N, G, k]
  uint16_t* h;                // [N, slots*d], or the weighted-sum slot alone [N, d] when route_only
  int B, T, G, k, d, n_shared;
  int route_only;
  int output_mode;            // 0 GQE, 1 hard slots only, 2 weighted hard slots (no weighted-sum slot)
};
cudaError_t launch_combine(const CombineParams& p, cudaStream_t stream);

}  // namespace gqe
