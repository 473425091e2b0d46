// Stochastic Length sampler: per-sequence subsequence selection over a jagged
// batch, and the row gather that builds the sampled batch.
//
// HSTU walkthrough (chenhuiyu.github.io, "generative-recommendation-16-hstu"),
// section "Three more scaling components / Stochastic Length": training
// usually replaces a long history by a shorter subsequence of it and now and
// then keeps it whole; alpha = 1.6 maps a length of 4,096 to 776.  Readings
// taken: L = floor(N^(alpha/2)) for maximum length N; only the history
// (n - num_targets positions) is sampled, targets are always kept; a history
// with h <= L is kept whole, a longer one with probability L^2 / h^2; the
// subsequence is the L history positions with the smallest (key, position)
// pairs, kept in their original order.
//
// Three launches, no host synchronisation:
//   sl_offsets_kernel  one CTA: output lengths and their exclusive scan
//   sl_select_kernel   one CTA per sequence: radix select of the L-th
//                      smallest key (four 8-bit digit passes over the keys,
//                      which stay in L2), then an order-preserving compaction
//                      written straight into the gather index
//   gather_rows_*      warps (wide rows) or lane groups (narrow rows) copy
//                      rows in 16/8/4/2/1-byte vectors; the row count is
//                      read on the device
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace hstu {
namespace {

constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;

// Keep-whole decision in fp64: L*L and h*h are exact integers, one correctly
// rounded division, then an exact scaling by 2^32.
__device__ __forceinline__ bool sl_keep_whole(int64_t h, int64_t L, uint32_t draw) {
  if (h <= L) return true;
  const double p = (double)(L * L) / (double)(h * h);
  return (double)draw < p * 4294967296.0;
}

// Rows [s, s + n) of sequence b with both ends clamped into [0, T], so that
// malformed offsets (decreasing, negative or past T) never move a read or a
// write outside the T rows of keys and of the gather index.
__device__ __forceinline__ void sl_rows(const int64_t* __restrict__ offs, int64_t b, int64_t T,
                                        int64_t& s, int64_t& n) {
  s = min(max(offs[b], (int64_t)0), T);
  const int64_t e = min(max(offs[b + 1], s), T);
  n = e - s;
}

__global__ void __launch_bounds__(1024) sl_offsets_kernel(const int64_t* __restrict__ offs,
                                                          const int32_t* __restrict__ nt, int B,
                                                          int64_t T, int64_t L,
                                                          const uint32_t* __restrict__ keep,
                                                          int64_t* __restrict__ new_offs) {
  __shared__ int64_t warp_tot[32];
  __shared__ int64_t carry;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    carry = 0;
    new_offs[0] = 0;
  }
  __syncthreads();
  for (int64_t base = 0; base < B; base += 1024) {
    const int64_t b = base + (int64_t)threadIdx.x;
    int64_t len = 0;
    if (b < B) {
      int64_t s0, n;
      sl_rows(offs, b, T, s0, n);
      const int64_t m = nt ? min(max((int64_t)nt[b], (int64_t)0), n) : 0;  // in [0, n]
      len = sl_keep_whole(n - m, L, keep[b]) ? n : L + m;
    }
    int64_t v = len;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t t = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += t;
    }
    if (lane == 31) warp_tot[warp] = v;
    __syncthreads();
    if (warp == 0) {
      int64_t w = warp_tot[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int64_t t = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += t;
      }
      warp_tot[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    const int64_t before = carry + (warp ? warp_tot[warp - 1] : 0);
    if (b < B) new_offs[b + 1] = before + v;
    __syncthreads();
    if (threadIdx.x == 0) carry += warp_tot[31];
    __syncthreads();
  }
}

// Exclusive block scan of a 32-bit value over kSelThreads threads; returns the
// exclusive prefix and writes the block total to *total.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t x, uint32_t* red, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t v = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  if (lane == 31) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = lane < kSelWarps ? red[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += t;
    }
    if (lane < kSelWarps) red[lane] = w;
  }
  __syncthreads();
  const uint32_t excl = (warp ? red[warp - 1] : 0u) + v - x;
  *total = red[kSelWarps - 1];
  __syncthreads();  // red is reused by the next call
  return excl;
}

__global__ void __launch_bounds__(kSelThreads) sl_select_kernel(
    const int64_t* __restrict__ offs, const int32_t* __restrict__ nt,
    const uint32_t* __restrict__ keys, const int64_t* __restrict__ new_offs, int64_t T, int64_t L,
    int64_t* __restrict__ gidx) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t red[kSelWarps];
  __shared__ uint32_t s_digit;
  __shared__ int64_t s_below;
  const int b = blockIdx.x;
  const int tid = threadIdx.x;
  int64_t s, n;
  sl_rows(offs, b, T, s, n);
  const int64_t m = nt ? min(max((int64_t)nt[b], (int64_t)0), n) : 0;  // in [0, n]
  const int64_t h = n - m;
  const int64_t o = new_offs[b];
  const int64_t out_n = new_offs[b + 1] - o;
  // the gather index holds T entries; with well-formed offsets every write
  // lands inside it, and the check keeps malformed ones from writing past it
  auto put = [&](int64_t at, int64_t row) {
    if (at >= 0 && at < T) gidx[at] = row;
  };

  if (out_n == n) {  // kept whole (always so when h <= L)
    for (int64_t j = tid; j < n; j += kSelThreads) put(o + j, s + j);
    return;
  }
  // Sampled: out_n == L + m with L < h.  Targets go after the L history rows.
  for (int64_t j = tid; j < m; j += kSelThreads) put(o + L + j, s + h + j);
  if (L == 0) return;

  const uint32_t* kb = keys + s;
  // Radix select, most significant digit first.  `rank` is the 0-based rank
  // of the wanted element (the L-th smallest) among keys matching `prefix`
  // on the digits fixed so far.
  uint32_t prefix = 0, mask = 0;
  int64_t rank = L - 1;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0u;
    __syncthreads();
    for (int64_t j = tid; j < h; j += kSelThreads) {
      const uint32_t k = kb[j];
      if ((k & mask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (tid < 32) {
      // Lane l owns bins [8l, 8l + 8).
      uint32_t c[8], sum = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        c[i] = hist[tid * 8 + i];
        sum += c[i];
      }
      uint32_t incl = sum;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, incl, d);
        if (tid >= d) incl += t;
      }
      const int64_t excl = (int64_t)(incl - sum);
      if (rank >= excl && rank < (int64_t)incl) {  // exactly one lane
        // First bin whose cumulative count passes rank.
        int64_t acc = excl;
        int bin = 7;
        bool found = false;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (!found) {
            if (rank < acc + (int64_t)c[i]) {
              bin = i;
              found = true;
            } else {
              acc += c[i];
            }
          }
        }
        s_digit = (uint32_t)(tid * 8 + bin);
        s_below = acc;
      }
    }
    __syncthreads();
    prefix |= s_digit << shift;
    mask |= 255u << shift;
    rank -= s_below;
    __syncthreads();
  }
  // prefix is the threshold key K; the first rank + 1 positions holding K
  // (in position order) are selected along with every key below K.
  const uint32_t K = prefix;
  const int64_t take_eq = rank + 1;
  int64_t run_lt = 0, run_eq = 0;
  for (int64_t base = 0; base < h; base += kSelThreads) {
    const int64_t j = base + tid;
    const uint32_t k = j < h ? kb[j] : 0xffffffffu;
    const uint32_t lt = (j < h && k < K) ? 1u : 0u;
    const uint32_t eq = (j < h && k == K) ? 1u : 0u;
    uint32_t total;
    const uint32_t before = block_excl_scan(lt | (eq << 16), red, &total);
    const int64_t eq_rank = run_eq + (before >> 16);
    const bool sel = lt || (eq && eq_rank < take_eq);
    if (sel) {
      const int64_t pos = run_lt + (before & 0xffffu) + (eq_rank < take_eq ? eq_rank : take_eq);
      put(o + pos, s + j);
    }
    run_lt += total & 0xffffu;
    run_eq += total >> 16;
  }
}

// Copies row r (r < min(*n_rows, max_rows)) of dst from row index[r] of src,
// in vectors of V; G lanes per row.  Rows whose index lies outside
// [0, src_rows) are left unwritten.
template <typename V, int G>
__global__ void __launch_bounds__(256) gather_rows_kernel(
    const unsigned char* __restrict__ src, int64_t src_ld, int64_t src_rows,
    const int64_t* __restrict__ index, const int64_t* __restrict__ n_rows, int64_t max_rows,
    int64_t vecs_per_row, unsigned char* __restrict__ dst, int64_t dst_ld) {
  int64_t rows = *n_rows;
  if (rows > max_rows) rows = max_rows;
  const int64_t groups = (int64_t)gridDim.x * (blockDim.x / G);
  const int sub = threadIdx.x % G;
  for (int64_t r = (int64_t)blockIdx.x * (blockDim.x / G) + threadIdx.x / G; r < rows;
       r += groups) {
    const int64_t sr = index[r];
    if (sr < 0 || sr >= src_rows) continue;
    const V* sp = reinterpret_cast<const V*>(src + sr * src_ld);
    V* dp = reinterpret_cast<V*>(dst + r * dst_ld);
#pragma unroll 4
    for (int64_t q = sub; q < vecs_per_row; q += G) dp[q] = sp[q];
  }
}

// Wide rows (at least 32 vectors): the work is split into units of one
// 32-vector segment of a row, dealt to warps round-robin (unit u = row * segs
// + seg goes to warp u mod warps), so that the last round leaves at most one
// unit per warp idle instead of one row.  Each warp keeps four units' loads
// in flight before storing; (row, seg) advance incrementally, with no
// division in the loop.
template <typename V>
__global__ void __launch_bounds__(256) gather_rows_wide_kernel(
    const unsigned char* __restrict__ src, int64_t src_ld, int64_t src_rows,
    const int64_t* __restrict__ index, const int64_t* __restrict__ n_rows, int64_t max_rows,
    int64_t vecs_per_row, int64_t segs, unsigned char* __restrict__ dst, int64_t dst_ld) {
  constexpr int kInFlight = 4;
  int64_t rows = *n_rows;
  if (rows > max_rows) rows = max_rows;
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  int64_t row = warp0 / segs, seg = warp0 - (warp0 / segs) * segs;
  const int64_t drow = nwarps / segs, dseg = nwarps - drow * segs;
  while (row < rows) {
    V v[kInFlight];
    V* dp[kInFlight];
#pragma unroll
    for (int k = 0; k < kInFlight; ++k) {
      dp[k] = nullptr;
      if (row < rows) {
        const int64_t q = seg * 32 + lane;
        const int64_t sr = index[row];
        if (q < vecs_per_row && sr >= 0 && sr < src_rows) {
          v[k] = reinterpret_cast<const V*>(src + sr * src_ld)[q];
          dp[k] = reinterpret_cast<V*>(dst + row * dst_ld) + q;
        }
      }
      seg += dseg;
      row += drow;
      if (seg >= segs) {
        seg -= segs;
        ++row;
      }
    }
#pragma unroll
    for (int k = 0; k < kInFlight; ++k)
      if (dp[k]) *dp[k] = v[k];
  }
}

template <typename V>
cudaError_t launch_gather(const void* src, int64_t src_ld, int64_t src_rows, const int64_t* index,
                          const int64_t* n_rows, int64_t max_rows, int64_t row_bytes, void* dst,
                          int64_t dst_ld, cudaStream_t s) {
  const int64_t vecs = row_bytes / (int64_t)sizeof(V);
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  auto grid = [&](int rows_per_cta) {
    int64_t g = (max_rows + rows_per_cta - 1) / rows_per_cta;
    const int64_t cap = (int64_t)sms * 8;
    return (unsigned)(g < 1 ? 1 : (g > cap ? cap : g));
  };
  const auto* sp = static_cast<const unsigned char*>(src);
  auto* dp = static_cast<unsigned char*>(dst);
  if (vecs >= 32) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, gather_rows_wide_kernel<V>, 256,
                                                      0) != cudaSuccess || per_sm < 1)
      per_sm = 1;
    const int64_t segs = (vecs + 31) / 32;
    const int64_t units_cap = max_rows * segs;            // warps beyond this have no work
    int64_t g = (units_cap + 7) / 8;
    const int64_t cap = (int64_t)sms * per_sm;
    g = g < 1 ? 1 : (g > cap ? cap : g);
    gather_rows_wide_kernel<V><<<(unsigned)g, 256, 0, s>>>(sp, src_ld, src_rows, index, n_rows,
                                                            max_rows, vecs, segs, dp, dst_ld);
  } else if (vecs >= 8)
    gather_rows_kernel<V, 8><<<grid(32), 256, 0, s>>>(sp, src_ld, src_rows, index, n_rows,
                                                      max_rows, vecs, dp, dst_ld);
  else
    gather_rows_kernel<V, 1><<<grid(256), 256, 0, s>>>(sp, src_ld, src_rows, index, n_rows,
                                                       max_rows, vecs, dp, dst_ld);
  count_launch();
  return cudaGetLastError();
}

bool multiple_of(int64_t v, int64_t a) { return v % a == 0; }
bool addr_multiple_of(const void* p, int64_t a) {
  return reinterpret_cast<uintptr_t>(p) % (uintptr_t)a == 0;
}

}  // namespace
}  // namespace hstu

using namespace hstu;

extern "C" {

int64_t hstu_sl_subsequence_length(int64_t max_len, double alpha) {
  if (max_len < 0 || !(alpha >= 0.0) || alpha > 64.0) return -1;
  if (max_len == 0) return 0;
  const double v = floor(pow((double)max_len, alpha / 2.0));
  if (!(v < 9.0e18)) return -1;
  return (int64_t)v;
}

hstu_status hstu_stochastic_length(const int64_t* seq_offsets, const int32_t* num_targets,
                                   int32_t B, int64_t T, int64_t sub_len,
                                   const uint32_t* keep_draw, const uint32_t* keys,
                                   int64_t* new_offsets, int64_t* gather_index,
                                   cudaStream_t stream) {
  if (B < 0 || T < 0 || sub_len < 0) return HSTU_ERR_INVALID;
  if (T >= ((int64_t)1 << 31)) return HSTU_ERR_UNSUPPORTED;
  if (!seq_offsets || !new_offsets) return HSTU_ERR_INVALID;
  if (!addr_multiple_of(seq_offsets, 8) || !addr_multiple_of(new_offsets, 8))
    return HSTU_ERR_UNSUPPORTED;
  if (B > 0 && !keep_draw) return HSTU_ERR_INVALID;
  if (T > 0 && (!keys || !gather_index)) return HSTU_ERR_INVALID;
  if ((keep_draw && !addr_multiple_of(keep_draw, 4)) || (keys && !addr_multiple_of(keys, 4)) ||
      (num_targets && !addr_multiple_of(num_targets, 4)) ||
      (gather_index && !addr_multiple_of(gather_index, 8)))
    return HSTU_ERR_UNSUPPORTED;
  prof_begin(HSTU_K_MISC, stream);
  sl_offsets_kernel<<<1, 1024, 0, stream>>>(seq_offsets, num_targets, B, T, sub_len, keep_draw,
                                            new_offsets);
  count_launch();
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess && B > 0) {
    sl_select_kernel<<<(unsigned)B, kSelThreads, 0, stream>>>(seq_offsets, num_targets, keys,
                                                               new_offsets, T, sub_len, gather_index);
    count_launch();
    e = cudaGetLastError();
  }
  prof_end(HSTU_K_MISC, stream);
  return e == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

hstu_status hstu_gather_rows(const void* src, int64_t src_stride_bytes, int64_t src_rows,
                             const int64_t* gather_index, const int64_t* d_num_rows,
                             int64_t max_rows, int64_t row_bytes, void* dst,
                             int64_t dst_stride_bytes, cudaStream_t stream) {
  if (max_rows < 0 || row_bytes < 0 || src_rows < 0) return HSTU_ERR_INVALID;
  if (max_rows == 0 || row_bytes == 0) return HSTU_OK;
  if (!src || !gather_index || !d_num_rows || !dst) return HSTU_ERR_INVALID;
  if (src_stride_bytes < row_bytes || dst_stride_bytes < row_bytes) return HSTU_ERR_INVALID;
  if (!addr_multiple_of(gather_index, 8) || !addr_multiple_of(d_num_rows, 8))
    return HSTU_ERR_UNSUPPORTED;
  int64_t v = 16;
  while (v > 1 && !(multiple_of(row_bytes, v) && multiple_of(src_stride_bytes, v) &&
                    multiple_of(dst_stride_bytes, v) && addr_multiple_of(src, v) &&
                    addr_multiple_of(dst, v)))
    v >>= 1;
  prof_begin(HSTU_K_MISC, stream);
  cudaError_t e;
  switch (v) {
    case 16:
      e = launch_gather<uint4>(src, src_stride_bytes, src_rows, gather_index, d_num_rows, max_rows,
                               row_bytes, dst, dst_stride_bytes, stream);
      break;
    case 8:
      e = launch_gather<uint2>(src, src_stride_bytes, src_rows, gather_index, d_num_rows, max_rows,
                               row_bytes, dst, dst_stride_bytes, stream);
      break;
    case 4:
      e = launch_gather<uint32_t>(src, src_stride_bytes, src_rows, gather_index, d_num_rows,
                                  max_rows, row_bytes, dst, dst_stride_bytes, stream);
      break;
    case 2:
      e = launch_gather<uint16_t>(src, src_stride_bytes, src_rows, gather_index, d_num_rows,
                                  max_rows, row_bytes, dst, dst_stride_bytes, stream);
      break;
    default:
      e = launch_gather<unsigned char>(src, src_stride_bytes, src_rows, gather_index, d_num_rows,
                                       max_rows, row_bytes, dst, dst_stride_bytes, stream);
  }
  prof_end(HSTU_K_MISC, stream);
  return e == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

}  // extern "C"
