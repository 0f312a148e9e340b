// scan.cu -- device exclusive prefix sum over int32 (reduce-then-scan).
//
// Used for the "prefix sum to get offsets" step of the CSR preallocation
// (page "Locality-Aware Automatic Differentiation on the GPU for Mesh-Based
// Computations", section 方法, key design 3) and for the dynamic pair
// insertion.  Three passes per level (tile sums, scan of the tile sums,
// tile scans with offsets) and recursion over the tile sums; no kernel waits
// on another block, so nothing can spin.
#include "mad_internal.h"

namespace mad {
namespace {

constexpr int kThreads = 256;
constexpr int kItems = 8;
constexpr int kTile = kThreads * kItems;

__device__ __forceinline__ int warp_incl_scan(int v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  return v;
}

// Exclusive scan of one value per thread across the block; returns the
// thread's exclusive prefix and writes the block total to *total.
__device__ __forceinline__ int block_excl_scan(int v, int* total) {
  __shared__ int warp_sums[kThreads / 32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int incl = warp_incl_scan(v);
  if (lane == 31) warp_sums[w] = incl;
  __syncthreads();
  if (w == 0) {
    int s = lane < kThreads / 32 ? warp_sums[lane] : 0;
    s = warp_incl_scan(s);
    if (lane < kThreads / 32) warp_sums[lane] = s;
  }
  __syncthreads();
  int base = w > 0 ? warp_sums[w - 1] : 0;
  *total = warp_sums[kThreads / 32 - 1];
  __syncthreads();
  return base + incl - v;
}

__global__ void __launch_bounds__(kThreads) k_tile_sums(const int32_t* __restrict__ in,
                                                        int64_t n,
                                                        int32_t* __restrict__ sums) {
  const int64_t base = (int64_t)blockIdx.x * kTile;
  int s = 0;
#pragma unroll
  for (int i = 0; i < kItems; ++i) {
    int64_t idx = base + (int64_t)i * kThreads + threadIdx.x;
    if (idx < n) s += in[idx];
  }
  int total;
  block_excl_scan(s, &total);
  if (threadIdx.x == 0) sums[blockIdx.x] = total;
}

// Scans one tile per block; adds offs[blockIdx.x] (if offs) and writes
// out[n] = grand total from the last block.
__global__ void __launch_bounds__(kThreads) k_tile_scan(const int32_t* __restrict__ in,
                                                        int32_t* __restrict__ out,
                                                        int64_t n,
                                                        const int32_t* __restrict__ offs) {
  const int64_t base = (int64_t)blockIdx.x * kTile + (int64_t)threadIdx.x * kItems;
  int v[kItems];
  int s = 0;
#pragma unroll
  for (int i = 0; i < kItems; ++i) {
    int64_t idx = base + i;
    v[i] = idx < n ? in[idx] : 0;
    s += v[i];
  }
  int total;
  int pre = block_excl_scan(s, &total);
  int off = offs ? offs[blockIdx.x] : 0;
  pre += off;
#pragma unroll
  for (int i = 0; i < kItems; ++i) {
    int64_t idx = base + i;
    if (idx < n) out[idx] = pre;
    pre += v[i];
  }
  if (blockIdx.x == gridDim.x - 1 && threadIdx.x == 0) out[n] = off + total;
}

}  // namespace

size_t scan_tmp_elems(int64_t n) {
  size_t t = 0;
  while (n > kTile) {
    int64_t tiles = (n + kTile - 1) / kTile;
    t += 2 * (size_t)(tiles + 1);
    n = tiles;
  }
  return t + 1;
}

cudaError_t scan_exclusive(const int32_t* in, int32_t* out, int64_t n, int32_t* tmp,
                           cudaStream_t s) {
  if (n <= 0) {
    return cudaMemsetAsync(out, 0, sizeof(int32_t), s);
  }
  if (n <= kTile) {
    k_tile_scan<<<1, kThreads, 0, s>>>(in, out, n, nullptr);
    return cudaGetLastError();
  }
  int64_t tiles = (n + kTile - 1) / kTile;
  int32_t* sums = tmp;
  int32_t* sums_scan = tmp + (tiles + 1);
  k_tile_sums<<<(unsigned)tiles, kThreads, 0, s>>>(in, n, sums);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = scan_exclusive(sums, sums_scan, tiles, tmp + 2 * (tiles + 1), s);
  if (e != cudaSuccess) return e;
  k_tile_scan<<<(unsigned)tiles, kThreads, 0, s>>>(in, out, n, sums_scan);
  return cudaGetLastError();
}

}  // namespace mad
