// Shared device/host helpers of libsa (sm_100a). Internal header.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sa.h"

namespace sa {

constexpr int kTile = SA_TILE;  // query/key tile height of every list and kernel

// Workspace header: the first 256 bytes of every workspace.
struct DeviceStatus {
  int32_t code;    // 0 = ok, else an sa_status value
  int32_t where;   // kernel-specific location of the first problem
  int32_t aux[62];
};
constexpr size_t kStatusBytes = 256;
static_assert(sizeof(DeviceStatus) == kStatusBytes, "status header is 256 bytes");

// Tile counters of the instrumented build (compiled with -DSA_COUNT_TILES into
// a separate library; the product build has none): 64-bit counters in the
// status header from aux[8] on, cleared with it by every call. Units:
//  FWD_VISITS   128 x 128 tiles the forward loads and multiplies
//  FWD_DENSE    tiles of the dense causal lower triangle of the same items
//               (one per key tile at or below the query tile; not in pair mode)
//  PAIR_BLOCKS  pair mode: b x b block pairs of the mask among the visits
//  PAIR_DENSE   pair mode: block pairs of the dense causal triangle of the
//               items' query blocks
//  DQ_VISITS    tiles of the query-major dQ pass (every query head)
//  DKDV_VISITS  tiles of the key-major dK/dV pass (every query head)
enum {
  CNT_FWD_VISITS = 0, CNT_FWD_DENSE, CNT_PAIR_BLOCKS, CNT_PAIR_DENSE, CNT_DQ_VISITS,
  CNT_DKDV_VISITS, kNumTileCounters
};
constexpr int kTileCounterWord = 8;  // first aux word (8-byte aligned in the header)
// item counters of the run-time queues of the backward passes (aux words)
constexpr int kQueueWordDq = 24, kQueueWordDkdv = 25;

__device__ __forceinline__ void count_tiles(DeviceStatus* st, int which, long long v) {
#ifdef SA_COUNT_TILES
  atomicAdd(reinterpret_cast<unsigned long long*>(st->aux + kTileCounterWord) + which,
            (unsigned long long)v);
#else
  (void)st, (void)which, (void)v;
#endif
}

// Records the first device-side problem; later ones are dropped.
__device__ __forceinline__ void report(DeviceStatus* st, int code, int where) {
  if (st != nullptr && atomicCAS(&st->code, 0, code) == 0) st->where = where;
}

__device__ __forceinline__ float load_as_float(const float* p) { return *p; }
__device__ __forceinline__ float load_as_float(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}
__device__ __forceinline__ void store_from_float(float* p, float v) { *p = v; }
__device__ __forceinline__ void store_from_float(__nv_bfloat16* p, float v) {
  *p = __float2bfloat16_rn(v);
}

// Block-wide in-place inclusive scan of a[0..n) (int32, global or shared),
// then a[i] += base. Every thread of the block must call it.
__device__ inline void block_inclusive_scan(int32_t* a, int n, int32_t base) {
  __shared__ int32_t warp_sums[32];
  __shared__ int32_t carry;
  if (threadIdx.x == 0) carry = base;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = (blockDim.x + 31) >> 5;
  for (int start = 0; start < n; start += blockDim.x) {
    const int i = start + threadIdx.x;
    int32_t v = (i < n) ? a[i] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int32_t t = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += t;
    }
    if (lane == 31) warp_sums[warp] = v;
    __syncthreads();
    if (warp == 0) {
      int32_t s = (lane < nwarps) ? warp_sums[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int32_t t = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += t;
      }
      warp_sums[lane] = s;
    }
    __syncthreads();
    const int32_t prefix = carry + (warp > 0 ? warp_sums[warp - 1] : 0);
    if (i < n) a[i] = v + prefix;
    __syncthreads();
    if (threadIdx.x == 0) carry += warp_sums[nwarps - 1];
    __syncthreads();
  }
}

}  // namespace sa
