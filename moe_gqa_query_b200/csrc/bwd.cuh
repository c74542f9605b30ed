// bwd.cuh -- parameters and launchers of the layer backward outside attention.
#pragma once

#include "sm100.cuh"

namespace gqe {

typedef uint16_t gqe_bf16_t;

struct CombineBwdParams {
  const gqe_bf16_t* o_routed;   // [B, G, T, k, d]
  const float* w;               // [N, G, k] router weights p~
  const gqe_bf16_t* dh;         // [N, slots * d]
  gqe_bf16_t* do_routed;        // [B, G, T, k, d]
  gqe_bf16_t* do_sh;            // [B, T, d]
  float* dw;                    // [N, G, k]
  int B, T, G, k, d, n_shared, output_mode, slots;
};

constexpr int kMaxBwdRouterCols = 64;

struct RouterBwdParams {
  const float* probs;   // [N, G, E]
  const int* idx;       // [N, G, k]
  const float* w;       // [N, G, k] p~
  const float* dw;      // [N, G, k]
  float* dlogits;       // [N, G, E]
  float* dbias;         // [G * E] or null
  int N, G, E, k, scope;
};

struct PackParams {
  const int* idx;            // [N, G, k]
  const gqe_bf16_t* dq;      // [B, G, T, k, d]
  const gqe_bf16_t* dq_sh;   // [B, T, d]
  const gqe_bf16_t* dK;      // [B, G, T, d]
  const gqe_bf16_t* dV;
  const float* dlogits;      // [N, G * E]
  gqe_bf16_t* A;             // [N, Kc]
  int B, T, G, E, k, d, n_shared, Kc;
};

// Columns of the packed projection-gradient matrix.
inline int bwd_pack_cols(int G, int E, int d, int n_shared) {
  return G * E * d + n_shared * d + 2 * G * d + 64 * ((G * E + 63) / 64);
}

cudaError_t launch_combine_bwd(const CombineBwdParams& p, cudaStream_t stream);
cudaError_t launch_router_bwd(const RouterBwdParams& p, cudaStream_t stream);
cudaError_t launch_bwd_pack(const PackParams& p, cudaStream_t stream);
cudaError_t launch_transpose(const uint16_t* src, uint16_t* dst, int rows, int cols, int ld_dst,
                             cudaStream_t stream);
cudaError_t launch_transpose_f32(const float* src, float* dst, int rows, int cols, int ld_dst, cudaStream_t stream);

}  // namespace gqe
