/*
 * gqe.h -- C ABI of the Grouped Query Experts (GQE) attention forward for
 * NVIDIA B200 (sm_100a).
 *
 * GQE (as described in the "GQE" study note at dimensionstp.github.io, §3-2,
 * and the chatpaper abstract "Experts de requêtes groupées") keeps the dense
 * K/V heads of grouped-query attention and turns the E query heads of every
 * KV group into experts: a per-group router picks k experts per token, only
 * those query heads are projected and attend, and the layer output
 * concatenates the hard-selected expert outputs, one router-weighted sum of
 * them and one always-on shared query head.
 *
 * Conventions shared by every entry point
 *   - Every tensor pointer is DEVICE memory owned by the caller, contiguous,
 *     row-major, 16-byte aligned.  bf16 tensors are passed as pointers to
 *     uint16_t bit patterns (gqe_bf16).
 *   - Weights use the [out, in] layout of a linear layer, except Wr, which is
 *     [d_model, G*E].
 *   - No entry point allocates or frees device memory or synchronises the
 *     device; work is enqueued on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream).  Scratch memory, where a call needs it, is the
 *     caller's `ws` buffer of at least gqe_workspace_size() bytes.
 *   - Argument errors return GQE_ERR_INVALID_ARG / GQE_ERR_UNSUPPORTED /
 *     GQE_ERR_WORKSPACE before anything is launched; a failed launch returns
 *     GQE_ERR_CUDA.  Errors inside a kernel surface at the caller's next
 *     synchronisation; a kernel whose internal wait runs out of time, or a
 *     decode that meets a cache length outside its range, records a code
 *     that gqe_device_error() returns.
 *   - Supported shapes: d_head in {64, 128}; 1 <= k <= E <= 8; G*E <= 64;
 *     d_model a multiple of 64; n_shared in {0, 1}; 0 <= shared_kv_group < G.
 */
#ifndef GQE_H_
#define GQE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t gqe_bf16;     /* bfloat16 bit pattern */
typedef void* gqe_stream;      /* cudaStream_t */

typedef enum {
  GQE_OK = 0,
  GQE_ERR_INVALID_ARG = 1,
  GQE_ERR_UNSUPPORTED = 2,
  GQE_ERR_WORKSPACE = 3,
  GQE_ERR_CUDA = 4,
  GQE_ERR_DEVICE_CHECK = 5
} gqe_status;

/* Shape of one layer call.  B sequences of T tokens (T = 1 for decode),
 * model width d_model, G KV groups with E query experts each, k experts
 * routed per (token, group), head width d_head.  renorm_scope 0 normalises
 * the selected router probabilities over all k*G selections of a token, 1
 * within each group, 2 not at all (the weights are the in-group softmax
 * probabilities).  scale 0 means 1/sqrt(d_head).  output_mode selects the
 * output construction ("GQE" study note §3-2 3)-5) and the ablation rows of
 * §5-1's accuracy table): 0 GQE, h = [hard slots, weighted-sum slot,
 * shared]; 1 "hard concat only", h = [hard slots, shared]; 2 "weighted
 * concat, no renormalised slot", h = [weight * hard slot each, shared].  The
 * number of slots of h is k*G + (output_mode == 0) + n_shared. */
typedef struct {
  int B, T, d_model, G, E, k, d_head;
  int n_shared;          /* 0 or 1 always-on shared query heads */
  int shared_kv_group;   /* KV group the shared head reads */
  int renorm_scope;      /* 0 token, 1 group, 2 none */
  float scale;
  int output_mode;       /* 0 GQE, 1 hard concat only, 2 weighted concat */
} gqe_dims;

enum {
  GQE_OP_ROUTED_QPROJ = 1,
  GQE_OP_ATTN_DECODE = 2,
  GQE_OP_COMBINE_OUT_PROJ = 3,
  GQE_OP_ATTN_BWD = 4,
  GQE_OP_LAYER_FORWARD = 5,       /* gqe_layer_forward */
  GQE_OP_LAYER_FORWARD_HOST = 6   /* gqe_layer_forward_host; dims->B = sequences per chunk */
};

/* Bytes of scratch the call `op` needs for these dims (L_max: the decode
 * cache length, used by GQE_OP_ATTN_DECODE only).  For
 * GQE_OP_LAYER_FORWARD_HOST, dims->B is the number of sequences per chunk,
 * not the batch.  Returns GQE_ERR_INVALID_ARG for bad dims or op. */
gqe_status gqe_workspace_size(const gqe_dims* dims, int op, int L_max, size_t* bytes);

/* Router: "GQE" study note §3-2 2) (score, in-group softmax, TopK) and 4)
 * (renormalised weights p~).
 *   x [B*T, d_model] bf16, Wr [d_model, G*E] bf16, bias [G*E] fp32 or NULL.
 *   topk_idx [B*T, G, k] int32: the selected experts of each (token, group)
 *     in ascending expert order (ties in the logits go to the lower index).
 *   topk_w   [B*T, G, k] fp32: p~ aligned with topk_idx.
 *   probs    [B*T, G, E] fp32 softmax probabilities, or NULL.
 * Logits are accumulated in fp32 from the bf16 inputs. */
gqe_status gqe_router_topk(const gqe_dims* dims, const gqe_bf16* x, const gqe_bf16* Wr,
                           const float* bias, int32_t* topk_idx, float* topk_w, float* probs,
                           gqe_stream stream);

/* Router statistics for collapse monitoring and a load-balancing loss
 * ("GQE" study note §4-3 routing auxiliary loss, §4-4 "router collapse
 * should be monitored"; ai-feeds summary, 局限: a loss on the tokens'
 * allocation proportions).  The loss itself is not specified by the pages;
 * this returns its inputs, per (group g, expert e), s = g*E + e:
 *   counts[s]   tokens whose selection in group g includes e   (int32 [G*E])
 *   prob_sum[s] sum over tokens of the in-group probability p (fp32 [G*E])
 * from probs [B*T, G, E] fp32 and topk_idx [B*T, G, k] int32 as
 * gqe_router_topk writes them.  Fractions and means are these over B*T.
 * The outputs are zeroed and accumulated on `stream` (fp32 sums in an order
 * that may differ between runs).  Errors: GQE_ERR_INVALID_ARG. */
gqe_status gqe_router_stats(const gqe_dims* dims, const float* probs, const int32_t* topk_idx,
                            int32_t* counts, float* prob_sum, gqe_stream stream);

/* Routed and shared query projection: "GQE" study note §3-2 2) (only the
 * selected experts compute their query) and 5) (shared head); ai-feeds
 * summary, 方法 (unselected query heads are skipped).
 *   x [B*T, d_model], Wq [G, E, d_head, d_model], Wsh [n_shared*d_head, d_model],
 *   topk_idx [B*T, G, k] as written by gqe_router_topk.
 *   q_routed [B, G, T, k, d_head]: slot j of (b, g, t) holds x_t Wq[g, topk_idx[t,g,j]]^T.
 *   q_sh [B, T, d_head] (ignored when n_shared == 0).
 *   expert_counts [G*E] int32 tokens per expert, or NULL.
 *   ws: scratch of gqe_workspace_size(GQE_OP_ROUTED_QPROJ) bytes (the
 *   token-to-expert permutation lives there). */
gqe_status gqe_routed_qproj(const gqe_dims* dims, const gqe_bf16* x, const gqe_bf16* Wq,
                            const gqe_bf16* Wsh, const int32_t* topk_idx, gqe_bf16* q_routed,
                            gqe_bf16* q_sh, int32_t* expert_counts, void* ws, size_t ws_bytes,
                            gqe_stream stream);

/* Dense, unchanged K/V projection ("GQE" study note §1-2 3) and §3-2 1)):
 *   K[b, g, t, :] = x[b*T+t] Wk[g*d:(g+1)*d]^T, likewise V.
 *   x [B*T, d_model]; Wk, Wv [G*d_head, d_model]; K, V [B, G, T, d_head]. */
gqe_status gqe_kv_proj(const gqe_dims* dims, const gqe_bf16* x, const gqe_bf16* Wk,
                       const gqe_bf16* Wv, gqe_bf16* K, gqe_bf16* V, gqe_stream stream);

/* Decode-step K/V append: projects the B new tokens (T must be 1) and writes
 * their rows at index cache_len[b]-1 of the caches Kc, Vc [B, G, L_max, d_head].
 * cache_len [B] int32 device array, each value in [1, L_max]. */
gqe_status gqe_kv_append(const gqe_dims* dims, const gqe_bf16* x, const gqe_bf16* Wk,
                         const gqe_bf16* Wv, gqe_bf16* Kc, gqe_bf16* Vc, int L_max,
                         const int32_t* cache_len, gqe_stream stream);

/* Routed causal attention, prefill ("GQE" study note §1-1 attention
 * equation; §3-2 2) every selected expert attends to its group's dense K/V;
 * §3-2 5) the shared head, which reads KV group shared_kv_group).
 *   q_routed [B, G, T, k, d], q_sh [B, T, d], K, V [B, G, T, d] (bf16).
 *   o_routed [B, G, T, k, d], o_sh [B, T, d] (bf16).
 *   lse: NULL, or fp32 [B*G*T*k + B*T*n_shared]: natural-log sum of
 *   exp(scaled scores) per query row, routed rows first.
 * Row (t, j) of a group attends to keys 0..t.  fp32 softmax and accumulation. */
gqe_status gqe_attn_prefill(const gqe_dims* dims, const gqe_bf16* q_routed,
                            const gqe_bf16* q_sh, const gqe_bf16* K, const gqe_bf16* V,
                            gqe_bf16* o_routed, gqe_bf16* o_sh, float* lse, gqe_stream stream);

/* Backward of gqe_attn_prefill ("GQE" study note §1-1 attention equation,
 * differentiated; §3-2 2) and 5): the gradients of every selected expert's
 * rows and of the shared head's rows flow into the K/V of the group they
 * read).  With P the causal softmax and Delta_r = sum_c dO_rc O_rc:
 *   dV = P^T dO,  dS = scale * P o (dO V^T - Delta),  dK = dS^T q,  dq = dS K.
 *   q_routed, q_sh, K, V: the forward's inputs; o_routed, o_sh: its outputs;
 *   lse: its fp32 LSE output (required here; the layout gqe_attn_prefill
 *   writes).  do_routed [B, G, T, k, d], do_sh [B, T, d]: upstream gradients.
 *   dq_routed, dq_sh (shapes of q), dK, dV [B, G, T, d]: bf16 outputs,
 *   overwritten.  fp32 accumulation; dq is summed over key tiles in an fp32
 *   workspace, in an order that may differ between runs.
 *   ws: scratch of gqe_workspace_size(GQE_OP_ATTN_BWD) bytes, 256-byte
 *   aligned. */
gqe_status gqe_attn_prefill_bwd(const gqe_dims* dims, const gqe_bf16* q_routed, const gqe_bf16* q_sh,
                                const gqe_bf16* K, const gqe_bf16* V, const gqe_bf16* o_routed,
                                const gqe_bf16* o_sh, const float* lse, const gqe_bf16* do_routed,
                                const gqe_bf16* do_sh, gqe_bf16* dq_routed, gqe_bf16* dq_sh, gqe_bf16* dK,
                                gqe_bf16* dV, void* ws, size_t ws_bytes, gqe_stream stream);

/* C [M, N] = sum_k A(m, k) B(n, k), bf16 in and out, fp32 accumulation on
 * tcgen05 (the projections of the backward pass).  Operand layouts:
 *   a_kn = 0: A stored [M, K] row-major;  a_kn = 1: A stored [K, M] (A^T).
 *   b_kn = 0: B stored [N, K] (nn.Linear weight); b_kn = 1: B stored [K, N].
 * C row-major [M, N].  N % 64 == 0; the contiguous dimension of each operand
 * a multiple of 8 elements; any K (the tail is zero-filled).  Errors:
 * GQE_ERR_UNSUPPORTED for other shapes, GQE_ERR_INVALID_ARG for null or
 * misaligned pointers. */
gqe_status gqe_gemm(int M, int N, int K, const gqe_bf16* A, int a_kn, const gqe_bf16* B, int b_kn, gqe_bf16* C,
                    gqe_stream stream);

/* C [M, N] (fp32) = (accumulate ? C : 0) + sum_k A(m, k) B(n, k): gqe_gemm's
 * operand layouts with an fp32 result added into C by reduce-add (weight
 * gradients; accumulate = 1 sums over micro-batches).  The K range is split
 * over several CTAs when the output alone has too few tiles to fill the GPU,
 * so the fp32 sums are taken in an order that may differ between runs.  Same
 * shape rules as gqe_gemm. */
gqe_status gqe_gemm_acc(int M, int N, int K, const gqe_bf16* A, int a_kn, const gqe_bf16* B, int b_kn, float* C,
                        int accumulate, gqe_stream stream);

/* Backward of the output construction ("GQE" study note §3-2 3) hard slots,
 * 4) weighted-sum slot, 5) shared head; §4-1: the weighted-sum slot is the
 * router's gradient path).  Per token, for selected (g, j) with weight w:
 *   output_mode 0: do = dh_hard + w dh_route,  dw = <dh_route, o>;
 *   output_mode 1: do = dh_hard,               dw = 0;
 *   output_mode 2: do = w dh_hard,             dw = <dh_hard, o>;
 *   do_sh = the shared slot of dh.
 *   o_routed [B, G, T, k, d], topk_w [B*T, G, k] fp32 (the forward's),
 *   dh [B*T, slots*d] bf16 -> do_routed [B, G, T, k, d], do_sh [B, T, d] bf16,
 *   dtopk_w [B*T, G, k] fp32.  o_sh is not read (may be NULL). */
gqe_status gqe_combine_bwd(const gqe_dims* dims, const gqe_bf16* o_routed, const gqe_bf16* o_sh,
                           const float* topk_w, const gqe_bf16* dh, gqe_bf16* do_routed, gqe_bf16* do_sh,
                           float* dtopk_w, gqe_stream stream);

/* Backward of the router ("GQE" study note §3-2 2) in-group softmax, 4)
 * renormalisation; TopK is a selection and passes no gradient):
 *   dp~ -> dp on the selected experts (dp_i = (dw_i - sum_j dw_j p~_j) / Z
 *   over the renorm scope, or dw_i for scope 2) -> ds_e = p_e (dp_e -
 *   sum_e' p_e' dp_e') per group.
 *   probs [B*T, G, E], topk_idx, topk_w [B*T, G, k] as gqe_router_topk wrote
 *   them; dtopk_w [B*T, G, k] -> dlogits [B*T, G*E] fp32; dbias [G*E] fp32 (the
 *   column sums of dlogits, accumulated with atomics in an order that may
 *   differ between runs) or NULL. */
gqe_status gqe_router_bwd(const gqe_dims* dims, const float* probs, const int32_t* topk_idx, const float* topk_w,
                          const float* dtopk_w, float* dlogits, float* dbias, gqe_stream stream);

/* Columns Kc of the packed projection-gradient matrix of gqe_bwd_pack:
 * G*E*d + n_shared*d + 2*G*d + 64*ceil(G*E/64). */
gqe_status gqe_bwd_pack_cols(const gqe_dims* dims, int* cols);

/* The projection gradients as one bf16 matrix A [B*T, Kc], row = token:
 * [dq scattered to its expert's d columns, block g*E+e, zeros for experts the
 * token did not select | dq_sh | dK of groups 0..G-1 | dV | dlogits (bf16),
 * zero padding].  With W_cat = [Wq; Wsh; Wk; Wv; Wr^T] stacked by rows,
 * dx = A W_cat and dW_cat = A^T x ("GQE" study note §3-2 2): only selected
 * experts receive query gradient).
 *   dq_routed [B, G, T, k, d], dq_sh [B, T, d], dK, dV [B, G, T, d] bf16,
 *   dlogits [B*T, G*E] fp32. */
gqe_status gqe_bwd_pack(const gqe_dims* dims, const int32_t* topk_idx, const gqe_bf16* dq_routed,
                        const gqe_bf16* dq_sh, const gqe_bf16* dK, const gqe_bf16* dV, const float* dlogits,
                        gqe_bf16* A, gqe_stream stream);

/* W_cat [Kc, d_model] bf16 = [Wq; Wsh; Wk; Wv; Wr^T; zero rows] stacked by rows
 * from the layer's weights (Wr [d_model, G*E], Wq [G, E, d, d_model],
 * Wsh [d, d_model], Wk, Wv [G*d, d_model]): the B operand (stored [K, N]) of
 * dx = A W_cat in gqe_gemm. */
gqe_status gqe_bwd_pack_weights(const gqe_dims* dims, const gqe_bf16* Wr, const gqe_bf16* Wq, const gqe_bf16* Wsh,
                                const gqe_bf16* Wk, const gqe_bf16* Wv, gqe_bf16* Wcat, gqe_stream stream);

/* dst[c * ld_dst + r] = src[r * cols + c] for a row-major bf16 src [rows, cols];
 * dst columns r in [rows, ld_dst) are zeroed (a K padded to a multiple of 64
 * for gqe_linear). */
gqe_status gqe_transpose(int rows, int cols, const gqe_bf16* src, gqe_bf16* dst, int ld_dst, gqe_stream stream);

/* gqe_transpose for fp32 (e.g. a weight gradient into its weight's layout). */
gqe_status gqe_transpose_f32(int rows, int cols, const float* src, float* dst, int ld_dst, gqe_stream stream);

/* Decode attention: one new token per sequence (dims->T must be 1) against a
 * dense cache (freeguideonline GQA tutorial, "自回归推理中的内存带宽优势": a
 * decode step reads the whole KV cache).
 *   q_routed [B, G, k, d], q_sh [B, d]; Kc, Vc [B, G, L_max, d];
 *   cache_len [B] int32 device array, each value in [1, L_max]: rows
 *   [0, cache_len[b]) are attended.  A value outside that range is a caller
 *   error the device detects: the kernel records code 0x302 in the device
 *   error word (gqe_device_error) and clamps the value to [0, L_max]; a
 *   sequence clamped to 0 gets zero outputs.
 *   o_routed [B, G, k, d], o_sh [B, d].
 *   ws: scratch of gqe_workspace_size(GQE_OP_ATTN_DECODE) bytes (split-L
 *   partial softmax states). */
gqe_status gqe_attn_decode(const gqe_dims* dims, const gqe_bf16* q_routed,
                           const gqe_bf16* q_sh, const gqe_bf16* Kc, const gqe_bf16* Vc,
                           int L_max, const int32_t* cache_len, gqe_bf16* o_routed,
                           gqe_bf16* o_sh, void* ws, size_t ws_bytes, gqe_stream stream);

/* Decode attention that allocates nothing and takes no scratch buffer.  The
 * GQE pages have no counterpart to this call: it exists for callers that
 * cannot allocate device memory when they decode, such as a serving engine
 * that reserved all device memory for its own pool at start-up (a
 * library-side allocation would fail or bypass its accounting), or a
 * latency-bound decode loop that cannot afford cudaMalloc's implicit device
 * synchronisation.
 *   Arguments and results are those of gqe_attn_decode without ws/ws_bytes.
 *   The split-L partial states live in one array inside the library,
 *   GQE_DECODE_NOALLOC_MAX_BYTES (8 MiB) of device memory that every GPU that
 *   loads the library holds until the process exits.  Dims and L_max whose
 *   partial states need more (gqe_workspace_size(GQE_OP_ATTN_DECODE) larger
 *   than the maximum) are rejected with GQE_ERR_WORKSPACE before anything is
 *   launched.  The 64-sequence, 8-group, 32768-key main-layer decode needs 4.3 MB.
 *   A call looks up the array's device address with the current device,
 *   and a call made under stream capture reuses the address that the last
 *   uncaptured call on that device found: make the first call on a device
 *   before any stream capture, and again after a reset of the device's
 *   primary context (cudaDeviceReset), which reloads the array elsewhere.
 *   Every call shares the array and it keeps the last call's contents (each
 *   slot a call reads is written earlier in the same call, so nothing needs
 *   clearing).  Calls that can overlap on the GPU, e.g. on two streams with no
 *   ordering between them, race on the array and corrupt each other's
 *   results: serialise them. */
#define GQE_DECODE_NOALLOC_MAX_BYTES (8u << 20)
gqe_status gqe_attn_decode_noalloc(const gqe_dims* dims, const gqe_bf16* q_routed,
                                   const gqe_bf16* q_sh, const gqe_bf16* Kc, const gqe_bf16* Vc,
                                   int L_max, const int32_t* cache_len, gqe_bf16* o_routed,
                                   gqe_bf16* o_sh, gqe_stream stream);

/* Output construction ("GQE" study note §3-2 3) hard slots, 4) weighted-sum
 * slot, 5) final concat):
 *   h[n] = [o(g=0, slot 0..k-1), ..., o(g=G-1, ...), sum_g sum_j w[n,g,j] o(g,j), o_sh]
 *   o_routed [B, G, T, k, d], o_sh [B, T, d], topk_w [B*T, G, k] fp32
 *   -> h [B*T, (k*G + 1 + n_shared) * d] bf16 (the weighted sum in fp32). */
gqe_status gqe_combine(const gqe_dims* dims, const gqe_bf16* o_routed, const gqe_bf16* o_sh,
                       const float* topk_w, gqe_bf16* h, gqe_stream stream);

/* Output projection and general linear map ("GQE" study note §3-2 7)):
 *   C [M, N] = A [M, K] W^T with W [N, K]; bf16 in and out, fp32 accumulation.
 *   K must be a multiple of 64 and N a multiple of 64. */
gqe_status gqe_linear(int M, int N, int K, const gqe_bf16* A, const gqe_bf16* W, gqe_bf16* C,
                      gqe_stream stream);

/* Output construction and projection in one call ("GQE" study note §3-2
 * 3)-5) and 7)): y [B*T, d_model] = h W_o^T with h as gqe_combine builds it,
 * without writing h.  When T is a multiple of 128 and d_model a multiple of
 * 256 (and B*T >= 2048) only the weighted-sum slot is materialised (in `ws`)
 * and the projection reads the hard slots from o_routed and the shared slot
 * from o_sh directly; otherwise h is built in `ws` and projected.
 *   o_routed [B, G, T, k, d], o_sh [B, T, d] (NULL without a shared head),
 *   topk_w [B*T, G, k] fp32, Wo [d_model, (k*G + 1 + n_shared) * d] bf16,
 *   y [B*T, d_model] bf16; all device pointers, 16-byte aligned.
 *   ws: scratch of gqe_workspace_size(GQE_OP_COMBINE_OUT_PROJ) bytes.
 * Errors: GQE_ERR_INVALID_ARG (null/misaligned pointers, bad dims),
 * GQE_ERR_WORKSPACE (ws too small), GQE_ERR_CUDA (launch failure). */
gqe_status gqe_combine_out_proj(const gqe_dims* dims, const gqe_bf16* o_routed, const gqe_bf16* o_sh,
                                const float* topk_w, const gqe_bf16* Wo, gqe_bf16* y, void* ws,
                                size_t ws_bytes, gqe_stream stream);

/* The weights of one layer, device pointers in the layouts the calls above
 * take: Wr [d_model, G*E], bias [G*E] fp32 or NULL, Wq [G, E, d_head,
 * d_model], Wsh [n_shared*d_head, d_model] (NULL when n_shared == 0), Wk and
 * Wv [G*d_head, d_model], Wo [d_model, slots*d_head].  All but Wr and bias
 * 16-byte aligned. */
typedef struct {
  const gqe_bf16* Wr;
  const float* bias;
  const gqe_bf16* Wq;
  const gqe_bf16* Wsh;
  const gqe_bf16* Wk;
  const gqe_bf16* Wv;
  const gqe_bf16* Wo;
} gqe_layer_weights;

/* Prefill forward of a whole GQE layer in one call ("GQE" study note §3-2
 * 1)-7): router and renormalised weights, routed and shared query
 * projection, dense K/V projection, routed causal attention, output
 * construction and projection).  Enqueues on `stream`, in this order,
 * gqe_router_topk, gqe_routed_qproj, gqe_kv_proj, gqe_attn_prefill and
 * gqe_combine_out_proj, the same kernels as those calls; the intermediates
 * (top-k indices and weights, q, K, V, the attention outputs and the calls'
 * own scratch) live in `ws`.
 *   x [B, T, d_model] bf16 -> y [B, T, d_model] bf16, device, 16-byte aligned.
 *   ws: gqe_workspace_size(GQE_OP_LAYER_FORWARD) bytes, 16-byte aligned.
 * Errors: GQE_ERR_INVALID_ARG (null or misaligned pointers, bad dims) and
 * GQE_ERR_WORKSPACE are returned before anything is launched; a failed
 * launch returns GQE_ERR_CUDA, possibly after earlier steps were enqueued. */
gqe_status gqe_layer_forward(const gqe_dims* dims, const gqe_layer_weights* w, const gqe_bf16* x,
                             gqe_bf16* y, void* ws, size_t ws_bytes, gqe_stream stream);

/* The same forward on HOST buffers: x_host and y_host [B, T, d_model] bf16
 * in host memory (page-locked, e.g. from cudaHostAlloc, for the copies to
 * run asynchronously; pageable memory works but the copies then block the
 * calling thread).  The batch is cut into chunks of chunk_seqs sequences
 * (the last one may be shorter); chunk i is copied in on stream_in, run
 * through the layer on stream_compute and copied back on stream_out, with
 * two device buffers for each direction, so the copies of neighbouring
 * chunks overlap each other and the compute.  The three streams may be the
 * same stream (nothing overlaps then).  The call orders the streams with
 * CUDA events that it creates and releases itself; it allocates no device
 * memory and does not synchronise.  It returns once everything is enqueued;
 * y_host is written when the work this call left on stream_compute (or on
 * stream_out) has completed.  It also leaves stream_in behind its last
 * compute step and stream_compute behind its last copy-back.  So calls in a
 * row on the same streams may share ws without further synchronisation
 * when their dims agree apart from B and they pass the same chunk_seqs (the
 * layout of ws depends on those alone).  Before ws serves a call with other
 * dims or another chunk_seqs, let stream_out's work complete.
 *   chunk_seqs >= 1; a batch of fewer sequences runs as one chunk.
 *   ws: device, 16-byte aligned, gqe_workspace_size(GQE_OP_LAYER_FORWARD_HOST)
 *   bytes for dims with B = chunk_seqs.
 * Errors as gqe_layer_forward; GQE_ERR_INVALID_ARG also for chunk_seqs < 1
 * or a null host pointer. */
gqe_status gqe_layer_forward_host(const gqe_dims* dims, const gqe_layer_weights* w,
                                  const gqe_bf16* x_host, gqe_bf16* y_host, int chunk_seqs, void* ws,
                                  size_t ws_bytes, gqe_stream stream_in, gqe_stream stream_compute,
                                  gqe_stream stream_out);

/* Reads and clears the device error word (0 = none).  Kernels set it when one
 * of their internal waits runs out of time (0x101 GEMM, 0x201 attention,
 * 0x202 attention backward, 0x301 decode, 0x401 router, 0x7F1 the failure
 * check below) and when gqe_attn_decode meets a cache_len outside
 * [1, L_max] (0x302).  The first code recorded is kept.  Synchronises
 * `stream`. */
gqe_status gqe_device_error(int* code, gqe_stream stream);

/* Failure-path check: launches one thread that waits, through the kernels'
 * own bounded wait (about one second of GPU time), on a barrier nothing ever
 * completes.  When the limit passes it records code 0x7F1 in the device error
 * word (read and cleared by gqe_device_error) and returns: the context stays
 * usable.  No fault, no trap. */
gqe_status gqe_debug_wait_timeout(gqe_stream stream);

/* Diagnostics.  Evaluates the attention kernel's exponential helpers on n
 * fp32 inputs (device arrays): y_poly the polynomial exp2 used on the FMA
 * pipe, y_pair its packed two-lane form, y_hw the hardware exp2 (MUFU).  For
 * tests; not part of the layer. */
gqe_status gqe_debug_exp2(const float* x, float* y_poly, float* y_pair, float* y_hw, int n,
                          gqe_stream stream);

const char* gqe_status_string(gqe_status status);

#ifdef __cplusplus
}
#endif

#endif  /* GQE_H_ */
