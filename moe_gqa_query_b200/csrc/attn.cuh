// attn.cuh -- parameters and launchers of the GQE attention kernels.
#pragma once

#include "sm100.cuh"

namespace gqe {

typedef uint16_t gqe_bf16_t;

struct AttnParams {
  gqe_bf16_t* o_routed;   // [B, G, T, k, d]
  gqe_bf16_t* o_sh;       // [B, T, d]
  float* lse;             // optional
  int B, T, G, k, n_shared, sg;
  float scale_log2;       // scale * log2(e)
  unsigned* err;          // device error word
};

cudaError_t launch_attn_prefill(const CUtensorMap& mQ, const CUtensorMap& mQs, const CUtensorMap& mK,
                                const CUtensorMap& mV, const AttnParams& p, int d,
                                cudaStream_t stream);

struct DecodeParams {
  const gqe_bf16_t* q_routed;   // [B, G, k, d]
  const gqe_bf16_t* q_sh;       // [B, d]
  const gqe_bf16_t* Kc;         // [B, G, L_max, d]
  const gqe_bf16_t* Vc;
  const int* cache_len;         // [B]
  gqe_bf16_t* o_routed;         // [B, G, k, d]
  gqe_bf16_t* o_sh;             // [B, d]
  float* part;                  // [B, G, n_chunks, nq_max, d + 2]
  int B, G, k, d, n_shared, sg, L_max;
  int chunk;                    // keys per split
  int n_chunks;
  int nq_max;                   // k + n_shared
  float scale_log2;
  unsigned* err;                // device error word
};

size_t decode_workspace_bytes(int B, int G, int k, int d, int n_shared, int L_max);
cudaError_t launch_attn_decode_maps(const CUtensorMap& mK, const CUtensorMap& mV, const DecodeParams& p,
                                   cudaStream_t stream);
void decode_split_plan(int L_max, int* chunk, int* n_chunks);

}  // namespace gqe
