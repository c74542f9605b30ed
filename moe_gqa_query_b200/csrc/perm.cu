// perm.cu -- token-to-expert permutation for the routed query projection.
//
// Only the experts in S_{t,g} compute a query ("GQE" study note §3-2 2);
// ai-feeds summary, 方法: unselected query heads are skipped).  The routing
// entries (token n, group g, slot j) with expert e = topk_idx[n, g, j] are
// grouped into segments s = g*E + e, stably (token order kept inside a
// segment), so the routed GEMM can run one expert's weight against a gathered
// 128-row tile.
//
//   count:   each block counts its chunk of entries per segment with a
//            warp-level histogram (__match_any_sync + one shared atomic per
//            distinct key);
//   scan:    per segment, an exclusive scan over blocks; segment offsets and
//            128-row tile offsets;
//   scatter: each block ranks its entries with the same warp histogram plus
//            a scan over warps and writes (source token row, destination row
//            of q_routed [B, G, T, k]).
#include "route.cuh"

namespace gqe {

namespace {

constexpr int kChunk = 4096;      // entries per block
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

__global__ void __launch_bounds__(kThreads) perm_count_kernel(const int* __restrict__ idx, int n_entries,
                                                              int G, int E, int k, int* block_counts) {
  __shared__ int hist[64];
  const int nseg = G * E;
  for (int s = threadIdx.x; s < nseg; s += kThreads) hist[s] = 0;
  __syncthreads();
  const int base = blockIdx.x * kChunk;
  const int end = min(base + kChunk, n_entries);
  for (int e0 = base; e0 < end; e0 += kThreads) {
    const int e = e0 + threadIdx.x;
    int key = -1;
    if (e < end) {
      const int ev = idx[e];   // out-of-range experts are skipped
      if (ev >= 0 && ev < E) key = ((e / k) % G) * E + ev;
    }
    const unsigned peers = __match_any_sync(0xffffffffu, key);
    if (key >= 0 && (threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&hist[key], __popc(peers));
  }
  __syncthreads();
  for (int s = threadIdx.x; s < nseg; s += kThreads) block_counts[blockIdx.x * nseg + s] = hist[s];
}

__global__ void __launch_bounds__(64) perm_scan_kernel(const int* block_counts, int n_blocks, int nseg,
                                                       int* block_base, int* seg_cnt, int* seg_off,
                                                       int* tile_start, int* expert_counts) {
  __shared__ int cnt[64];
  const int s = threadIdx.x;
  if (s < nseg) {
    int run = 0;
    for (int b = 0; b < n_blocks; ++b) {
      block_base[b * nseg + s] = run;
      run += block_counts[b * nseg + s];
    }
    cnt[s] = run;
    seg_cnt[s] = run;
    if (expert_counts) expert_counts[s] = run;
  }
  __syncthreads();
  if (s == 0) {
    int off = 0, tiles = 0;
    for (int i = 0; i < nseg; ++i) {
      seg_off[i] = off;
      tile_start[i] = tiles;
      off += cnt[i];
      tiles += (cnt[i] + 127) / 128;
    }
    tile_start[nseg] = tiles;
  }
}

__global__ void __launch_bounds__(kThreads) perm_scatter_kernel(const int* __restrict__ idx, int n_entries,
                                                                int T, int G, int E, int k,
                                                                const int* block_base, const int* seg_off,
                                                                int* src_row, int* dst_row) {
  __shared__ int wcnt[kWarps][64];
  __shared__ int run[64];
  const int nseg = G * E;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int s = threadIdx.x; s < nseg; s += kThreads) run[s] = 0;
  const int base = blockIdx.x * kChunk;
  const int end = min(base + kChunk, n_entries);
  for (int e0 = base; e0 < end; e0 += kThreads) {
    for (int i = threadIdx.x; i < kWarps * 64; i += kThreads) (&wcnt[0][0])[i] = 0;
    __syncthreads();
    const int e = e0 + threadIdx.x;
    int key = -1;
    if (e < end) {
      const int ev = idx[e];   // out-of-range experts are skipped
      if (ev >= 0 && ev < E) key = ((e / k) % G) * E + ev;
    }
    const unsigned peers = __match_any_sync(0xffffffffu, key);
    const int rank = __popc(peers & lanemask_lt());
    if (key >= 0 && rank == 0) wcnt[warp][key] = __popc(peers);
    __syncthreads();
    if (key >= 0) {
      int pos = seg_off[key] + block_base[blockIdx.x * nseg + key] + run[key] + rank;
      for (int w = 0; w < warp; ++w) pos += wcnt[w][key];
      const int n = e / (G * k);
      const int g = (e / k) % G;
      const int j = e % k;
      const int b = n / T, t = n % T;
      src_row[pos] = n;
      dst_row[pos] = ((b * G + g) * T + t) * k + j;
    }
    __syncthreads();
    for (int s = threadIdx.x; s < nseg; s += kThreads) {
      int add = 0;
      for (int w = 0; w < kWarps; ++w) add += wcnt[w][s];
      run[s] += add;
    }
    __syncthreads();
  }
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

PermLayout perm_layout(int N, int G, int E, int k) {
  PermLayout L{};
  L.n_entries = N * G * k;
  L.n_seg = G * E;
  L.n_blocks = (L.n_entries + kChunk - 1) / kChunk;
  size_t o = 0;
  L.off_block_counts = o; o = align256(o + sizeof(int) * (size_t)L.n_blocks * L.n_seg);
  L.off_block_base = o;   o = align256(o + sizeof(int) * (size_t)L.n_blocks * L.n_seg);
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
  int* block_base = reinterpret_cast<int*>(w + L.off_block_base);
  int* seg_cnt = reinterpret_cast<int*>(w + L.off_seg_cnt);
  int* seg_off = reinterpret_cast<int*>(w + L.off_seg_off);
  int* tile_start = reinterpret_cast<int*>(w + L.off_tile_start);
  int* src_row = reinterpret_cast<int*>(w + L.off_src_row);
  int* dst_row = reinterpret_cast<int*>(w + L.off_dst_row);
  if (L.n_entries == 0) return cudaSuccess;
  perm_count_kernel<<<L.n_blocks, kThreads, 0, stream>>>(topk_idx, L.n_entries, G, E, k, block_counts);
  perm_scan_kernel<<<1, 64, 0, stream>>>(block_counts, L.n_blocks, L.n_seg, block_base, seg_cnt, seg_off,
                                         tile_start, expert_counts);
  perm_scatter_kernel<<<L.n_blocks, kThreads, 0, stream>>>(topk_idx, L.n_entries, T, G, E, k, block_base,
                                                           seg_off, src_row, dst_row);
  return cudaGetLastError();
}

}  // namespace gqe
