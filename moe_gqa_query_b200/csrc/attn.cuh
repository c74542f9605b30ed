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

// diag.cu: a bounded wait that runs out (failure-path test)
cudaError_t launch_debug_wait(unsigned* err, cudaStream_t stream);

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

// Backward of the prefill attention.  Query rows live in a padded row space:
// routed sequence s (= b*G + g) owns rows [s*rows_pad, (s+1)*rows_pad), the
// shared head of sequence b owns B*G*rows_pad + [b*rows_pad_sh, ...); rows
// past a sequence's T*k (or T) are padding.
struct AttnBwdParams {
  const float* lse;                 // forward LSE (natural log), routed rows then shared rows
  const gqe_bf16_t* o_routed;       // [B, G, T, k, d]
  const gqe_bf16_t* o_sh;           // [B, T, d]
  const gqe_bf16_t* do_routed;
  const gqe_bf16_t* do_sh;
  float* lse2;                      // [n_rows_pad] LSE * log2(e), +inf on padding
  float* delta;                     // [n_rows_pad] sum_c dO * O
  float* dq_acc;                    // [n_rows_pad, d] fp32
  gqe_bf16_t* dq_routed;            // [B, G, T, k, d]
  gqe_bf16_t* dq_sh;                // [B, T, d]
  gqe_bf16_t* dK;                   // [B, G, T, d]
  gqe_bf16_t* dV;
  int B, T, G, k, n_shared, sg, d;
  int rows_pad, rows_pad_sh;
  long long n_rows_pad;
  float scale, scale_log2;
  unsigned* err;
};

struct AttnBwdLayout {
  int rows_pad, rows_pad_sh;
  long long n_rows_pad;
  size_t off_lse2, off_delta, off_dq, bytes;
};

void attn_bwd_layout(int B, int T, int G, int k, int n_shared, int d, AttnBwdLayout* L);
cudaError_t launch_attn_bwd(const CUtensorMap& mQ, const CUtensorMap& mQs, const CUtensorMap& mdO,
                            const CUtensorMap& mdOs, const CUtensorMap& mK, const CUtensorMap& mV,
                            const CUtensorMap& mdQ, const AttnBwdParams& p, cudaStream_t stream);

size_t decode_workspace_bytes(int B, int G, int k, int d, int n_shared, int L_max);
cudaError_t launch_attn_decode_maps(const CUtensorMap& mK, const CUtensorMap& mV, const DecodeParams& p,
                                   cudaStream_t stream);
void decode_split_plan(int L_max, int* chunk, int* n_chunks);

}  // namespace gqe
