// perm.cu -- token-to-expert permutation for the routed query projection.
//
// Only the experts in S_{t,g} compute a query ("GQE" study note §3-2 2);
// ai-feeds summary, 方法: unselected query heads are skipped).  The routing
// entries (token n, group g, slot j) with expert e = topk_idx[n, g, j] are
// grouped into segments s = g*E + e so the routed GEMM can run one expert's
// weight against a gathered 128-row tile.  A token enters a segment at most
// once (its k experts in a group are distinct, groups own disjoint
// segments), so segment s owns N slots from s*N on and no prefix over the
// segments is needed before filling it.
//
// One thread per token, 256 tokens per block: warp ballots count the block's
// tokens per segment and rank them inside each warp, a scan over the block's
// warps gives each warp its offset, and one atomicAdd per (block, segment)
// reserves the block's slots.  Blocks land in a segment in any order; the
// GEMM computes every row on its own, so the result does not depend on it.

#include "launch.cuh"
#include "route.cuh"

namespace gqe {

namespace {

constexpr int kThreads = 256;     // tokens per block
constexpr int kWarps = kThreads / 32;
constexpr int kMaxSeg = 64;

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Bit s set when this token routes to segment s (out-of-range experts skipped).
__device__ __forceinline__ unsigned long long token_segments(const int* __restrict__ idx, int n, int N, int G,
                                                             int E, int k) {
  unsigned long long bits = 0;
  if (n < N) {
    const int* row = idx + (size_t)n * G * k;
    for (int g = 0; g < G; ++g)
      for (int j = 0; j < k; ++j) {
        const int e = row[g * k + j];
        if (e >= 0 && e < E) bits |= 1ull << (g * E + e);
      }
  }
  return bits;
}

__global__ void __launch_bounds__(kThreads) perm_fill_kernel(const int* __restrict__ idx, int N, int T, int G, int E,
                                                             int k, int cap, int* seg_cnt, int* src_row,
                                                             int* dst_row) {
  __shared__ int wcnt[kWarps][kMaxSeg];   // per-warp counts, then each warp's offset in the block
  __shared__ int bbase[kMaxSeg];          // the block's first slot in each segment
  const int nseg = G * E;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = blockIdx.x * kThreads + threadIdx.x;
  pdl_launch_dependents();
  pdl_wait();
  const unsigned long long bits = token_segments(idx, n, N, G, E, k);
  for (int s = 0; s < nseg; ++s) {
    const unsigned m = __ballot_sync(0xffffffffu, (bits >> s) & 1ull);
    if (lane == 0) wcnt[warp][s] = __popc(m);
  }
  __syncthreads();
  for (int s = threadIdx.x; s < nseg; s += kThreads) {
    int run = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const int c = wcnt[w][s];
      wcnt[w][s] = run;
      run += c;
    }
    bbase[s] = run ? atomicAdd(&seg_cnt[s], run) : 0;
  }
  __syncthreads();
  const int b = n / T, t = n % T;
  const int* row = idx + (size_t)(n < N ? n : 0) * G * k;
  const unsigned lt = lanemask_lt();
  for (int s = 0; s < nseg; ++s) {
    const bool mine = (bits >> s) & 1ull;
    const unsigned m = __ballot_sync(0xffffffffu, mine);
    if (!mine) continue;
    const int g = s / E, e = s % E;
    int j = 0;
    while (j < k - 1 && row[g * k + j] != e) ++j;
    const size_t pos = (size_t)s * cap + bbase[s] + wcnt[warp][s] + __popc(m & lt);
    src_row[pos] = n;
    dst_row[pos] = ((b * G + g) * T + t) * k + j;
  }
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

PermLayout perm_layout(int N, int G, int E, int k) {
  (void)k;
  PermLayout L{};
  L.n_seg = G * E;
  L.cap = N;
  size_t o = 0;
  L.off_seg_cnt = o; o = align256(o + sizeof(int) * L.n_seg);
  L.off_src_row = o; o = align256(o + sizeof(int) * (size_t)L.n_seg * L.cap);
  L.off_dst_row = o; o = align256(o + sizeof(int) * (size_t)L.n_seg * L.cap);
  L.bytes = o;
  return L;
}

cudaError_t launch_permutation(const int* topk_idx, int N, int T, int G, int E, int k, void* ws,
                               const PermLayout& L, cudaStream_t stream) {
  uint8_t* w = static_cast<uint8_t*>(ws);
  int* seg_cnt = reinterpret_cast<int*>(w + L.off_seg_cnt);
  int* src_row = reinterpret_cast<int*>(w + L.off_src_row);
  int* dst_row = reinterpret_cast<int*>(w + L.off_dst_row);
  cudaError_t e = cudaMemsetAsync(seg_cnt, 0, sizeof(int) * L.n_seg, stream);
  if (e != cudaSuccess) return e;
  return launch_kernel(perm_fill_kernel, dim3((N + kThreads - 1) / kThreads), dim3(kThreads), 0, stream, 1,
                       topk_idx, N, T, G, E, k, L.cap, seg_cnt, src_row, dst_row);
}

}  // namespace gqe
