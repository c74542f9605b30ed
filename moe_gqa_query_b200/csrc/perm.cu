// perm.cu -- token-to-expert permutation for the routed query projection.
//
// Only the experts in S_{t,g} compute a query ("GQE" study note §3-2 2);
// ai-feeds summary, 方法: unselected query heads are skipped).  The routing
// entries (token n, group g, slot j) with expert e = topk_idx[n, g, j] are
// grouped into segments s = g*E + e, stably (token order kept inside a
// segment), so the routed GEMM can run one expert's weight against a gathered
// 128-row tile.
//
// A token contributes at most one entry to any segment (its k experts in a
// group are distinct, and groups own disjoint segments).  So with one thread
// per token, the rank of a token inside a segment is a prefix count of one
// bit per token: a warp ballot per segment gives the in-warp rank, a scan over
// the block's warps and over the preceding blocks gives the rest.
//
//   count:   per block of 256 tokens, tokens per segment (ballot + popc);
//   scatter: each block sums the counts of the blocks before it (and of all
//            blocks, for the segment offsets), ranks its tokens with ballots
//            and writes (source token row, destination row of
//            q_routed [B, G, T, k]).  Block 0 also writes the segment counts,
//            offsets and 128-row tile offsets the GEMM reads.
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

__global__ void __launch_bounds__(kThreads) perm_count_kernel(const int* __restrict__ idx, int N, int G, int E,
                                                              int k, int* block_counts) {
  __shared__ int wcnt[kWarps][kMaxSeg];
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
    int c = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) c += wcnt[w][s];
    block_counts[blockIdx.x * nseg + s] = c;
  }
}

__global__ void __launch_bounds__(kThreads) perm_scatter_kernel(const int* __restrict__ idx, int N, int T, int G,
                                                                int E, int k, int n_blocks,
                                                                const int* __restrict__ block_counts, int* seg_cnt,
                                                                int* seg_off, int* tile_start, int* expert_counts,
                                                                int* src_row, int* dst_row) {
  __shared__ int wcnt[kWarps][kMaxSeg];
  __shared__ int base[kMaxSeg];    // this block's first position inside each segment
  __shared__ int off[kMaxSeg];     // segment offsets
  const int nseg = G * E;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = blockIdx.x * kThreads + threadIdx.x;
  pdl_launch_dependents();
  pdl_wait();
  const unsigned long long bits = token_segments(idx, n, N, G, E, k);

  // ---- preceding blocks and totals: 4 threads per segment share the block loop
  {
    const int s = threadIdx.x >> 2, part = threadIdx.x & 3;
    int before = 0, total = 0;
    if (s < nseg) {
      for (int b = part; b < n_blocks; b += 4) {
        const int c = block_counts[b * nseg + s];
        total += c;
        before += (b < (int)blockIdx.x) ? c : 0;
      }
    }
    before += __shfl_xor_sync(0xffffffffu, before, 1);
    before += __shfl_xor_sync(0xffffffffu, before, 2);
    total += __shfl_xor_sync(0xffffffffu, total, 1);
    total += __shfl_xor_sync(0xffffffffu, total, 2);
    if (s < nseg && part == 0) {
      base[s] = before;
      off[s] = total;     // totals for now; turned into offsets below
    }
  }
  // ---- in-warp ranks: one ballot per segment
  for (int s = 0; s < nseg; ++s) {
    const unsigned m = __ballot_sync(0xffffffffu, (bits >> s) & 1ull);
    if (lane == 0) wcnt[warp][s] = __popc(m);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int o = 0, tiles = 0;
    for (int s = 0; s < nseg; ++s) {
      const int c = off[s];
      if (blockIdx.x == 0) {
        seg_cnt[s] = c;
        tile_start[s] = tiles;
        if (expert_counts) expert_counts[s] = c;
      }
      off[s] = o;
      o += c;
      tiles += (c + 127) / 128;
    }
    if (blockIdx.x == 0) {
      for (int s = 0; s < nseg; ++s) seg_off[s] = off[s];
      tile_start[nseg] = tiles;
    }
  }
  // ---- ranks of this warp's first token in each segment: scan over the block's warps
  for (int s2 = threadIdx.x; s2 < nseg; s2 += kThreads) {
    int run = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const int c = wcnt[w][s2];
      wcnt[w][s2] = run;
      run += c;
    }
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
    const int pos = off[s] + base[s] + wcnt[warp][s] + __popc(m & lt);
    src_row[pos] = n;
    dst_row[pos] = ((b * G + g) * T + t) * k + j;
  }
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

PermLayout perm_layout(int N, int G, int E, int k) {
  PermLayout L{};
  L.n_entries = N * G * k;
  L.n_seg = G * E;
  L.n_blocks = (N + kThreads - 1) / kThreads;
  size_t o = 0;
  L.off_block_counts = o; o = align256(o + sizeof(int) * (size_t)L.n_blocks * L.n_seg);
  L.off_block_base = o;   // unused: the scatter kernel derives block bases from the counts
  L.off_seg_cnt = o;      o = align256(o + sizeof(int) * L.n_seg);
  L.off_seg_off = o;      o = align256(o + sizeof(int) * L.n_seg);
  L.off_tile_start = o;   o = align256(o + sizeof(int) * (L.n_seg + 1));
  L.off_src_row = o;      o = align256(o + sizeof(int) * (size_t)L.n_entries);
  L.off_dst_row = o;      o = align256(o + sizeof(int) * (size_t)L.n_entries);
  L.bytes = o;
  return L;
}

cudaError_t launch_permutation(const int* topk_idx, int N, int T, int G, int E, int k, void* ws,
                               const PermLayout& L, int* expert_counts, cudaStream_t stream) {
  uint8_t* w = static_cast<uint8_t*>(ws);
  int* block_counts = reinterpret_cast<int*>(w + L.off_block_counts);
  int* seg_cnt = reinterpret_cast<int*>(w + L.off_seg_cnt);
  int* seg_off = reinterpret_cast<int*>(w + L.off_seg_off);
  int* tile_start = reinterpret_cast<int*>(w + L.off_tile_start);
  int* src_row = reinterpret_cast<int*>(w + L.off_src_row);
  int* dst_row = reinterpret_cast<int*>(w + L.off_dst_row);
  cudaError_t e = launch_kernel(perm_count_kernel, dim3(L.n_blocks), dim3(kThreads), 0, stream, 1, topk_idx, N, G,
                                E, k, block_counts);
  if (e != cudaSuccess) return e;
  return launch_kernel(perm_scatter_kernel, dim3(L.n_blocks), dim3(kThreads), 0, stream, 1, topk_idx, N, T, G, E, k,
                       L.n_blocks, static_cast<const int*>(block_counts), seg_cnt, seg_off, tile_start,
                       expert_counts, src_row, dst_row);
}

}  // namespace gqe
