// Dispatch: stable counting sort of the routed slots by expert.
//
// DS4Server issue #112, "Current upstream route": sort_rows takes the argsort
// of the flattened expert ids, inv_order = argsort(order) and row_map =
// order // top_k (uint32), without copying token rows; "Kernel contract":
// per-expert tile and row prefix tables, expert found by binary search.
// "5.5 real sparse MoE kernels (Metal)", Scope -- in: expert dispatch
// (tokens, expert_indices) -> grouped tokens, "the hard part".
//
// The argsort is realised as a counting sort, which is stable by
// construction and needs no comparison sort:
//   1. count   -- one block per chunk of 1024 slots counts ids per expert
//   2. scan    -- one block: counts, row_off, tile_off, and each chunk's
//                 starting position per expert (chunks in slot order)
//   3. scatter -- one block per chunk: per-warp counts of every id, a scan of
//                 each id's counts over the chunk's 32 warps, and the rank
//                 among equal ids inside a warp (__match_any_sync) place each
//                 slot at once, in slot order.
// When all slots fit one chunk the three steps run in a single block
// (decode), so a whole dispatch is one launch there.
#include <mutex>

#include "common.cuh"
#include "launch.h"

namespace moe {

constexpr int kChunk = 1024;   // slots per block (32 warps x 32 lanes)
constexpr size_t kScanSmemMax = 160 * 1024;   // dynamic shared memory of the scan block

static inline int num_chunks(long long R) { return (int)((R + kChunk - 1) / kChunk); }

size_t sort_workspace_bytes(int R, int E) {
  // per-chunk counts and per-chunk bases, int32 [chunks][E] each
  return (size_t)2 * num_chunks(R) * E * sizeof(int32_t) + 256;
}

__device__ __forceinline__ int clamp_id(int e, int E) { return e < 0 ? 0 : (e >= E ? E - 1 : e); }

// Exclusive scan of v[0..n) in shared memory by one block of 1024 threads,
// writes the total to *total. Every thread owns a contiguous run.
__device__ void block_exclusive_scan(int* v, int n, int* total, int* warp_tmp) {
  const int tid = threadIdx.x, nt = blockDim.x;
  const int per = (n + nt - 1) / nt;
  const int lo = min(n, tid * per), hi = min(n, lo + per);
  int run = 0;
  for (int i = lo; i < hi; ++i) run += v[i];
  // inclusive warp scan of run
  const int lane = tid & 31, warp = tid >> 5;
  int inc = run;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) warp_tmp[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int w = (lane < (nt >> 5)) ? warp_tmp[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    if (lane < (nt >> 5)) warp_tmp[lane] = wi - w;   // exclusive warp offsets
    if (lane == 31) *total = wi;
  }
  __syncthreads();
  int base = warp_tmp[warp] + inc - run;
  for (int i = lo; i < hi; ++i) {
    int c = v[i];
    v[i] = base;
    base += c;
  }
  __syncthreads();
}

// Scatter the slots of one chunk in slot order. cursor[e] holds the first
// sorted position of expert e for this chunk. wtab is a [32][E] uint16
// table in shared memory: each warp's count of every id, then (in place)
// the number of equal ids in the earlier warps of the chunk; with the rank
// among equal ids inside the warp (__match_any_sync) that gives every slot
// its position at once, in slot order.
__device__ void scatter_chunk(const int32_t* __restrict__ idx, long long r0, long long R, int k,
                              int E, const int* cursor, uint16_t* wtab,
                              uint32_t* __restrict__ order, uint32_t* __restrict__ inv_order,
                              uint32_t* __restrict__ row_map) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < 32 * E; i += blockDim.x) wtab[i] = 0;
  __syncthreads();
  const long long r = r0 + warp * 32 + lane;
  const int e = (r < R) ? clamp_id(idx[r], E) : -1;
  const unsigned peers = __match_any_sync(0xffffffffu, e);
  const int rank = __popc(peers & ((1u << lane) - 1u));
  if (e >= 0 && rank == 0) wtab[warp * E + e] = (uint16_t)__popc(peers);
  __syncthreads();
  for (int x = threadIdx.x; x < E; x += blockDim.x) {     // exclusive scan over warps
    int run = 0;
    for (int w = 0; w < 32; ++w) {
      const int c = wtab[w * E + x];
      wtab[w * E + x] = (uint16_t)run;
      run += c;
    }
  }
  __syncthreads();
  if (e >= 0) {
    const int pos = cursor[e] + wtab[warp * E + e] + rank;
    order[pos] = (uint32_t)r;
    inv_order[r] = (uint32_t)pos;
    row_map[pos] = (uint32_t)(r / k);
  }
}

// Whole sort in one block (R <= kChunk).
__global__ void __launch_bounds__(1024) sort_single_kernel(
    const int32_t* __restrict__ idx, int R, int k, int E, int BM, uint32_t* __restrict__ order,
    uint32_t* __restrict__ inv_order, uint32_t* __restrict__ row_map, int32_t* __restrict__ counts,
    int32_t* __restrict__ row_off, int32_t* __restrict__ tile_off) {
  pdl_wait();
  pdl_launch();
  extern __shared__ int sm[];
  int* cnt = sm;            // [E]
  int* tiles = sm + E;      // [E]
  uint16_t* wtab = reinterpret_cast<uint16_t*>(sm + 2 * E);   // [32][E]
  __shared__ int warp_tmp[32];
  __shared__ int totals[2];
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  for (int r = threadIdx.x; r < R; r += blockDim.x) atomicAdd(&cnt[clamp_id(idx[r], E)], 1);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    counts[e] = cnt[e];
    tiles[e] = (cnt[e] + BM - 1) / BM;
  }
  __syncthreads();
  block_exclusive_scan(cnt, E, &totals[0], warp_tmp);
  block_exclusive_scan(tiles, E, &totals[1], warp_tmp);
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    row_off[e] = cnt[e];
    tile_off[e] = tiles[e];
  }
  if (threadIdx.x == 0) {
    row_off[E] = totals[0];
    tile_off[E] = totals[1];
  }
  __syncthreads();
  scatter_chunk(idx, 0, R, k, E, cnt, wtab, order, inv_order, row_map);
}

__global__ void __launch_bounds__(1024) sort_count_kernel(const int32_t* __restrict__ idx, long long R,
                                                          int E, int32_t* __restrict__ chunk_cnt) {
  pdl_wait();
  pdl_launch();
  extern __shared__ int cnt[];
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  const long long r = (long long)blockIdx.x * kChunk + threadIdx.x;
  if (r < R) atomicAdd(&cnt[clamp_id(idx[r], E)], 1);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) chunk_cnt[(size_t)blockIdx.x * E + e] = cnt[e];
}

__global__ void __launch_bounds__(1024) sort_scan_kernel(const int32_t* __restrict__ chunk_cnt,
                                                         int nchunks, int E, int BM, bool stage_fits,
                                                         int32_t* __restrict__ chunk_base,
                                                         int32_t* __restrict__ counts,
                                                         int32_t* __restrict__ row_off,
                                                         int32_t* __restrict__ tile_off) {
  pdl_wait();
  pdl_launch();
  extern __shared__ int sm[];
  int* cnt = sm;
  int* tiles = sm + E;
  // the chunk counts, staged in shared memory by all threads at once when
  // they fit (one round of independent loads instead of a chain of
  // nchunks dependent ones per expert), else read from global memory
  int* stage = sm + 2 * E;
  const bool staged = stage_fits;
  __shared__ int warp_tmp[32];
  __shared__ int totals[2];
  if (staged)
    for (int i = threadIdx.x; i < nchunks * E; i += blockDim.x) stage[i] = chunk_cnt[i];
  __syncthreads();
  const int32_t* cc = staged ? stage : chunk_cnt;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int c = 0;
    for (int b = 0; b < nchunks; ++b) c += cc[(size_t)b * E + e];
    cnt[e] = c;
    counts[e] = c;
    tiles[e] = (c + BM - 1) / BM;
  }
  __syncthreads();
  block_exclusive_scan(cnt, E, &totals[0], warp_tmp);
  block_exclusive_scan(tiles, E, &totals[1], warp_tmp);
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    row_off[e] = cnt[e];
    tile_off[e] = tiles[e];
    int base = cnt[e];
    for (int b = 0; b < nchunks; ++b) {
      chunk_base[(size_t)b * E + e] = base;
      base += cc[(size_t)b * E + e];
    }
  }
  if (threadIdx.x == 0) {
    row_off[E] = totals[0];
    tile_off[E] = totals[1];
  }
}

__global__ void __launch_bounds__(1024) sort_scatter_kernel(
    const int32_t* __restrict__ idx, long long R, int k, int E,
    const int32_t* __restrict__ chunk_base, uint32_t* __restrict__ order,
    uint32_t* __restrict__ inv_order, uint32_t* __restrict__ row_map) {
  pdl_wait();
  pdl_launch();
  extern __shared__ int cursor[];
  uint16_t* wtab = reinterpret_cast<uint16_t*>(cursor + E);   // [32][E]
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    cursor[e] = chunk_base[(size_t)blockIdx.x * E + e];
  __syncthreads();
  scatter_chunk(idx, (long long)blockIdx.x * kChunk, R, k, E, cursor, wtab, order, inv_order,
                row_map);
}

cudaError_t launch_sort_rows(const int32_t* idx, int T, int k, int E, int BM, uint32_t* order,
                             uint32_t* inv_order, uint32_t* row_map, int32_t* counts,
                             int32_t* row_off, int32_t* tile_off, void* ws, cudaStream_t s) {
  const long long R = (long long)T * k;
  const size_t smem2 = (size_t)2 * E * sizeof(int);
  const size_t wtab = (size_t)32 * E * sizeof(uint16_t);
  if (R <= kChunk) {
    cudaFuncSetAttribute(sort_single_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)(smem2 + wtab));
    launch_pdl(sort_single_kernel, 1, 1024, smem2 + wtab, s, idx, (int)R, k, E, BM, order, inv_order,
                                                     row_map, counts, row_off, tile_off);
    return cudaGetLastError();
  }
  const int nch = num_chunks(R);
  int32_t* chunk_cnt = reinterpret_cast<int32_t*>(ws);
  int32_t* chunk_base = chunk_cnt + (size_t)nch * E;
  launch_pdl(sort_count_kernel, nch, 1024, E * sizeof(int), s, idx, R, E, chunk_cnt);
  // the scan stages the chunk counts in shared memory when they fit
  const size_t stage_bytes = (size_t)nch * E * sizeof(int);
  const bool fits = smem2 + stage_bytes <= kScanSmemMax;
  const size_t smem_scan = smem2 + (fits ? stage_bytes : 0);
  cudaFuncSetAttribute(sort_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_scan);
  launch_pdl(sort_scan_kernel, 1, 1024, smem_scan, s, chunk_cnt, nch, E, BM, fits, chunk_base, counts,
                                          row_off, tile_off);
  cudaFuncSetAttribute(sort_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)(E * sizeof(int) + wtab));
  launch_pdl(sort_scatter_kernel, nch, 1024, E * sizeof(int) + wtab, s, idx, R, k, E, chunk_base, order,
                                                                inv_order, row_map);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ no-alloc

// Scratch for moe_sort_rows_noalloc: the per-chunk counts and bases of the
// multi-block sort, sized for up to kNoAllocMaxRows routed rows and
// kNoAllocMaxExperts experts (2 * 32 * 1024 int32 = 256 KiB). It is a
// file-scope device array, so every GPU that loads this library holds it for
// the life of the process. Host code must not pass the symbol itself to a
// kernel (on the host it only names a stand-in); it passes the device address
// looked up once per device below.
constexpr int kNoAllocMaxRows = 32768;
constexpr int kNoAllocMaxExperts = 1024;
constexpr int kNoAllocChunks = (kNoAllocMaxRows + kChunk - 1) / kChunk;
static __device__ __align__(256) int32_t g_noalloc_sort_scratch[2 * kNoAllocChunks *
                                                                kNoAllocMaxExperts];

// Device address of the scratch on the current device, looked up on first use
// with that device current; nullptr when the lookup fails.
static int32_t* noalloc_scratch_ptr() {
  static std::mutex mu;
  static int32_t* ptrs[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (!ptrs[dev]) {
    int32_t* p = nullptr;
    if (cudaGetSymbolAddress((void**)&p, g_noalloc_sort_scratch) != cudaSuccess) return nullptr;
    ptrs[dev] = p;
  }
  return ptrs[dev];
}

bool noalloc_sort_fits(long long R, int E) {
  return R <= kNoAllocMaxRows && E <= kNoAllocMaxExperts;
}

cudaError_t launch_sort_rows_noalloc(const int32_t* idx, int T, int k, int E, int BM,
                                     uint32_t* order, uint32_t* inv_order, uint32_t* row_map,
                                     int32_t* counts, int32_t* row_off, int32_t* tile_off,
                                     cudaStream_t s) {
  int32_t* scratch = noalloc_scratch_ptr();
  if (!scratch) return cudaErrorUnknown;
  // every chunk count and base the sort reads is written by the same call
  // first, so the scratch needs no clearing between calls
  return launch_sort_rows(idx, T, k, E, BM, order, inv_order, row_map, counts, row_off, tile_off,
                          scratch, s);
}

}  // namespace moe
