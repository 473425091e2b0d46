// Work list of the tensor-core attention forward kernels: items of
// (sequence, head, 128-query tile), sorted by descending number of visible
// key tiles ("Ragged kernels": only real lengths are scheduled) by a device
// counting sort, then dealt round-robin to one persistent CTA per SM.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"

namespace hstu {

struct AttnItem {
  int32_t b;
  int16_t qt;
  int16_t h;
};

constexpr int kTile = 128;
constexpr int kMaxCost = 514;  // key tiles per item, 65536 / 128 + 2

struct SchedWs {
  int32_t* hist;     // [kMaxCost]
  int32_t* cursor;   // [kMaxCost]
  int32_t* total;    // [1]
  AttnItem* items;   // [max_items]
};

// Threads of the one-block scan kernels of the counting sorts: at least one
// per cost bin, whole warps.
constexpr int kScanThreads = (kMaxCost + 31) / 32 * 32;

// Exclusive scan of hist[0, n) in descending bin order, by one block of
// blockDim.x >= n threads (whole warps, at most 1024): cursor[c] = sum of
// hist[c'] over c' > c, and *total = the sum of all bins.
__device__ __forceinline__ void scan_descending(const int32_t* hist, int32_t* cursor,
                                                int32_t* total, int n) {
  __shared__ int32_t warp_sum[32];
  const int t = threadIdx.x, lane = t & 31, wid = t >> 5, nw = blockDim.x >> 5;
  const int c = n - 1 - t;                       // thread t holds the t-th largest bin
  const int v = c >= 0 ? hist[c] : 0;
  int x = v;                                     // inclusive scan within the warp
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sum[wid] = x;
  __syncthreads();
  if (wid == 0) {
    int sw = lane < nw ? warp_sum[lane] : 0;     // inclusive scan of the warp sums
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, sw, o);
      if (lane >= o) sw += y;
    }
    if (lane < nw) warp_sum[lane] = sw;
  }
  __syncthreads();
  if (c >= 0) cursor[c] = (wid > 0 ? warp_sum[wid - 1] : 0) + x - v;
  if (t == 0) *total = warp_sum[nw - 1];
}

SchedWs sched_ws(void* ws);
// Fills the work list in `ws` (attn_sched_bytes of it) on stream s.
cudaError_t build_schedule(const AttnArgs& a, void* ws, cudaStream_t s);

// Key tiles an item needs, and the item's geometry.
struct SeqGeom {
  int64_t qs, ks;   // first query row, first key row
  int nq, hlen;     // queries; keys visible to candidates (= history length)
  int qbase;        // position of query 0
};

__device__ __forceinline__ SeqGeom seq_geom(const AttnArgs& a, int b) {
  SeqGeom g;
  g.qs = a.q_offsets[b];
  g.nq = (int)(a.q_offsets[b + 1] - g.qs);
  g.ks = a.kv_offsets[b];
  const int nkv = (int)(a.kv_offsets[b + 1] - g.ks);
  if (a.cached) {
    g.hlen = nkv;
    g.qbase = nkv;
  } else {
    const int m = a.num_targets ? a.num_targets[b] : 0;
    g.hlen = min(max(g.nq - m, 0), g.nq);
    g.qbase = 0;
  }
  return g;
}

__device__ __forceinline__ int item_kend(const SeqGeom& g, int qt) {
  const int rows = min(kTile, g.nq - qt * kTile);
  return min(g.hlen, g.qbase + qt * kTile + rows);
}

}  // namespace hstu
