// Small kernels of the HSTU path: bias-gradient column sums, the dQ
// finalisation (fp32 accumulator times SiLU'(Pre_Q)), strided column copies
// (M-FALCON history K/V cache) and the jagged-metadata validator.
#include "common.cuh"
#include "internal.h"

namespace hstu {
namespace {

// out[c] += sum_r x[r][c]; CTA = 32 columns x 8 row-groups
template <typename T>
__global__ void colsum_kernel(const T* __restrict__ x, int64_t rows, int64_t cols, int64_t ld,
                              float* __restrict__ out) {
  __shared__ float red[8][33];
  const int tx = threadIdx.x % 32, ty = threadIdx.x / 32;
  const int64_t c = (int64_t)blockIdx.x * 32 + tx;
  float s = 0.f;
  if (c < cols)
    for (int64_t r = (int64_t)blockIdx.y * 8 + ty; r < rows; r += (int64_t)gridDim.y * 8)
      s += to_f(x[r * ld + c]);
  red[ty][tx] = s;
  __syncthreads();
  if (ty == 0 && c < cols) {
    float t = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) t += red[k][tx];
    atomicAdd(out + c, t);
  }
}

template <typename T>
__global__ void dq_finalize_kernel(const float* __restrict__ dq, const T* __restrict__ pre_q,
                                   int64_t pre_stride, T* __restrict__ dpre_q, int64_t rows, int d) {
  const int64_t n = rows * d;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / d;
    const int c = (int)(i % d);
    dpre_q[r * pre_stride + c] = from_f<T>(dq[i] * silu_grad_acc(to_f(pre_q[r * pre_stride + c])));
  }
}

// bf16, d and the Pre stride multiples of 8, 16-byte aligned rows: eight
// columns per thread and step (two fp32 vectors of dQ, one bf16 vector of Pre)
__global__ void dq_finalize_bf16x8_kernel(const float* __restrict__ dq, const bf16* __restrict__ pre_q,
                                          int64_t pre_stride, bf16* __restrict__ dpre_q, int64_t rows,
                                          int d) {
  const int dv = d / 8;
  const int64_t n = rows * dv;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / dv;
    const int c = (int)(i - r * dv) * 8;
    const float4 a = *reinterpret_cast<const float4*>(dq + r * d + c);
    const float4 b = *reinterpret_cast<const float4*>(dq + r * d + c + 4);
    const uint4 pu = *reinterpret_cast<const uint4*>(pre_q + r * pre_stride + c);
    const __nv_bfloat162* ph = reinterpret_cast<const __nv_bfloat162*>(&pu);
    const float g[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint4 o;
    __nv_bfloat162* oh = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 pf = __bfloat1622float2(ph[k]);
      oh[k] = __floats2bfloat162_rn(g[2 * k] * silu_grad_fast(pf.x), g[2 * k + 1] * silu_grad_fast(pf.y));
    }
    *reinterpret_cast<uint4*>(dpre_q + r * pre_stride + c) = o;
  }
}

template <typename T>
__global__ void copy_columns_kernel(const T* __restrict__ src, int64_t ss, T* __restrict__ dst,
                                    int64_t ds, int64_t rows, int64_t cols) {
  const int64_t n = rows * cols;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / cols, c = i % cols;
    dst[r * ds + c] = src[r * ss + c];
  }
}

// One warp per token row, one 16-byte chunk per lane and pass: chunks 0-3 of
// a head hold its 32 values, chunks 4-7 zeros.
__global__ void pad_heads32_kernel(const bf16* __restrict__ b0, const bf16* __restrict__ b1,
                                   const bf16* __restrict__ b2, int nblk, int64_t ss,
                                   uint4* __restrict__ dst, int64_t T, int H) {
  const int per_row = nblk * H * 8;
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < T;
       r += nwarps) {
    uint4* drow = dst + r * per_row;
    for (int c = lane; c < per_row; c += 32) {
      const int q = c >> 3, j = c & 7;
      const int blk = q / H, h = q - blk * H;
      uint4 val = make_uint4(0u, 0u, 0u, 0u);
      if (j < 4) {
        const bf16* src = blk == 0 ? b0 : (blk == 1 ? b1 : b2);
        val = *reinterpret_cast<const uint4*>(src + r * ss + h * 32 + j * 8);
      }
      drow[c] = val;
    }
  }
}

__global__ void convert_kernel(const float* __restrict__ src, bf16* __restrict__ dst, int64_t n) {
  const int64_t n8 = n / 8;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float4 a = reinterpret_cast<const float4*>(src)[2 * i];
    const float4 b = reinterpret_cast<const float4*>(src)[2 * i + 1];
    uint4 o;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&o);
    h[0] = __floats2bfloat162_rn(a.x, a.y);
    h[1] = __floats2bfloat162_rn(a.z, a.w);
    h[2] = __floats2bfloat162_rn(b.x, b.y);
    h[3] = __floats2bfloat162_rn(b.z, b.w);
    reinterpret_cast<uint4*>(dst)[i] = o;
  }
  for (int64_t i = n8 * 8 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    dst[i] = __float2bfloat16_rn(src[i]);
}

__global__ void validate_seq_kernel(const int64_t* __restrict__ offs, int B, int64_t T,
                                    const int32_t* __restrict__ nt, int max_len,
                                    uint32_t* __restrict__ flags) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b > B) return;
  uint32_t f = 0;
  if (b == 0 && offs[0] != 0) f |= HSTU_FLAG_OFFSETS_START;
  if (b == B && offs[B] != T) f |= HSTU_FLAG_OFFSETS_END;
  if (b < B) {
    const int64_t len = offs[b + 1] - offs[b];
    if (len < 0) f |= HSTU_FLAG_OFFSETS_ORDER;
    if (len > max_len) f |= HSTU_FLAG_SEQ_TOO_LONG;
    if (nt && (nt[b] < 0 || (int64_t)nt[b] > len)) f |= HSTU_FLAG_TARGETS_RANGE;
  }
  if (f) atomicOr(flags, f);
}

// A token whose timestamp is below its predecessor's inside one sequence.
// Sequences whose offsets fall outside [0, T] are skipped (already flagged).
__global__ void validate_time_kernel(const int64_t* __restrict__ offs, int B, int64_t T,
                                     const int64_t* __restrict__ ts, uint32_t* __restrict__ flags) {
  for (int b = blockIdx.y; b < B; b += gridDim.y) {
    const int64_t s = offs[b], e = offs[b + 1];
    if (s < 0 || e > T || e - s <= 1) continue;
    for (int64_t i = s + 1 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < e;
         i += (int64_t)gridDim.x * blockDim.x)
      if (ts[i] < ts[i - 1]) {
        atomicOr(flags, HSTU_FLAG_TIME_ORDER);
        break;
      }
  }
}

unsigned grid_for(int64_t n, int threads) {
  int64_t g = (n + threads - 1) / threads;
  if (g > 148 * 16) g = 148 * 16;
  return (unsigned)(g < 1 ? 1 : g);
}

}  // namespace

cudaError_t colsum_accumulate(int dtype, const void* x, int64_t rows, int64_t cols, int64_t ld,
                              float* out, cudaStream_t s) {
  if (rows == 0 || cols == 0) return cudaSuccess;
  dim3 grid((unsigned)((cols + 31) / 32), 1);
  int64_t gy = (rows + 255) / 256;
  const int64_t want = (4 * 148 + grid.x - 1) / grid.x;
  grid.y = (unsigned)(gy < want ? (gy < 1 ? 1 : gy) : want);
  if (dtype == HSTU_BF16)
    colsum_kernel<bf16><<<grid, 256, 0, s>>>((const bf16*)x, rows, cols, ld, out);
  else
    colsum_kernel<float><<<grid, 256, 0, s>>>((const float*)x, rows, cols, ld, out);
  count_launch();
  return cudaGetLastError();
}

cudaError_t dq_finalize(int dtype, const float* dq, const void* pre_q, int64_t ps, void* dpre_q,
                        int64_t T, int d, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const unsigned g = grid_for(T * d, 256);
  const bool vec = d % 8 == 0 && ps % 8 == 0 && ((uintptr_t)dq & 15) == 0 && ((uintptr_t)pre_q & 15) == 0 &&
                   ((uintptr_t)dpre_q & 15) == 0;
  if (dtype == HSTU_BF16 && vec)
    dq_finalize_bf16x8_kernel<<<grid_for(T * (d / 8), 256), 256, 0, s>>>(dq, (const bf16*)pre_q, ps,
                                                                        (bf16*)dpre_q, T, d);
  else if (dtype == HSTU_BF16)
    dq_finalize_kernel<bf16><<<g, 256, 0, s>>>(dq, (const bf16*)pre_q, ps, (bf16*)dpre_q, T, d);
  else
    dq_finalize_kernel<float><<<g, 256, 0, s>>>(dq, (const float*)pre_q, ps, (float*)dpre_q, T, d);
  count_launch();
  return cudaGetLastError();
}

cudaError_t copy_columns(int dtype, const void* src, int64_t ss, void* dst, int64_t ds,
                         int64_t rows, int64_t cols, cudaStream_t s) {
  if (rows == 0 || cols == 0) return cudaSuccess;
  const unsigned g = grid_for(rows * cols, 256);
  if (dtype == HSTU_BF16)
    copy_columns_kernel<bf16><<<g, 256, 0, s>>>((const bf16*)src, ss, (bf16*)dst, ds, rows, cols);
  else
    copy_columns_kernel<float><<<g, 256, 0, s>>>((const float*)src, ss, (float*)dst, ds, rows, cols);
  count_launch();
  return cudaGetLastError();
}

cudaError_t pad_heads32(const void* b0, const void* b1, const void* b2, int nblk, int64_t ss,
                        void* dst, int64_t T, int H, cudaStream_t s) {
  if (T == 0 || H == 0) return cudaSuccess;
  if (nblk < 1 || nblk > 3) return cudaErrorInvalidValue;
  const unsigned g = grid_for(T, 8);            // eight rows (warps) per block
  pad_heads32_kernel<<<g, 256, 0, s>>>((const bf16*)b0, (const bf16*)b1, (const bf16*)b2, nblk,
                                       ss, (uint4*)dst, T, H);
  count_launch();
  return cudaGetLastError();
}

cudaError_t convert_f32_to_bf16(const float* src, void* dst, int64_t n, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  convert_kernel<<<grid_for(n / 8 + 1, 256), 256, 0, s>>>(src, (bf16*)dst, n);
  count_launch();
  return cudaGetLastError();
}

cudaError_t validate_inputs(const int64_t* offs, int B, int64_t T, const int64_t* ts,
                            const int32_t* nt, int max_len, uint32_t* flags, cudaStream_t s) {
  validate_seq_kernel<<<(B + 1 + 255) / 256, 256, 0, s>>>(offs, B, T, nt, max_len, flags);
  count_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || B == 0 || ts == nullptr) return e;
  dim3 grid(8, (unsigned)(B < 65535 ? B : 65535));
  validate_time_kernel<<<grid, 256, 0, s>>>(offs, B, T, ts, flags);
  count_launch();
  return cudaGetLastError();
}

}  // namespace hstu
