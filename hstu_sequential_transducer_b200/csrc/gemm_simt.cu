// CUDA-core GEMM with the projection epilogues of the HSTU layer.
//
// Used for the fp32 layer (where tensor-core TF32 would not meet the fp32
// tolerance) and for shapes the tcgen05 GEMM does not take.  64x64 output
// tile, K slab of 16, 256 threads computing 4x4 outputs each, fp32 FMA.
#include "common.cuh"
#include "internal.h"

namespace hstu {
namespace {

constexpr int TM = 64, TN = 64, TK = 16;

template <typename T, bool AK, bool BK, int EPI, typename TIO>
__global__ void __launch_bounds__(256) gemm_simt_kernel(GemmArgs g, int64_t k_per_split) {
  __shared__ float As[TK][TM + 4];
  __shared__ float Bs[TK][TN + 4];
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
  const int64_t m0 = (int64_t)blockIdx.y * TM, n0 = (int64_t)blockIdx.x * TN;
  const int64_t kb = (int64_t)blockIdx.z * k_per_split;
  const int64_t ke = min(g.K, kb + k_per_split);
  const T* A = static_cast<const T*>(g.A);
  const T* B = static_cast<const T*>(g.B);
  float acc[4][4] = {};

  for (int64_t k0 = kb; k0 < ke; k0 += TK) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      int idx = tid + r * 256;
      int mm, kk;
      if (AK) { mm = idx / TK; kk = idx % TK; } else { kk = idx / TM; mm = idx % TM; }
      int64_t gm = m0 + mm, gk = k0 + kk;
      float v = 0.f;
      if (gm < g.M && gk < ke) v = to_f(AK ? A[gm * g.lda + gk] : A[gk * g.lda + gm]);
      As[kk][mm] = v;
      int nn;
      if (BK) { nn = idx / TK; kk = idx % TK; } else { kk = idx / TN; nn = idx % TN; }
      int64_t gn = n0 + nn;
      gk = k0 + kk;
      v = 0.f;
      if (gn < g.N && gk < ke) v = to_f(BK ? B[gn * g.ldb + gk] : B[gk * g.ldb + gn]);
      Bs[kk][nn] = v;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }

#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int64_t m = m0 + ty * 4 + i;
    if (m >= g.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int64_t n = n0 + tx + 16 * j;
      if (n >= g.N) continue;
      float v = acc[i][j];
      if (EPI == EPI_ATOMIC_F32) {
        atomicAdd(g.Cf + m * g.ldc + n, v);
        continue;
      }
      if (g.bias) v += to_f(static_cast<const T*>(g.bias)[n]);
      if (EPI == EPI_SILU_SPLIT) {
        if (g.C) static_cast<T*>(g.C)[m * g.ldc + n] = from_f<T>(v);
        static_cast<T*>(g.C2)[m * g.ldc + n] = from_f<T>(silu_acc(v));
      } else {
        if (EPI == EPI_RESID) v += to_f(static_cast<const TIO*>(g.R)[m * g.ldr + n]);
        static_cast<TIO*>(g.C)[m * g.ldc + n] = from_f<TIO>(v);
      }
    }
  }
}

template <typename T, bool AK, bool BK>
cudaError_t launch_epi(const GemmArgs& g, cudaStream_t s) {
  dim3 grid((unsigned)((g.N + TN - 1) / TN), (unsigned)((g.M + TM - 1) / TM), 1);
  int64_t kps = g.K;
  if (g.epi == EPI_ATOMIC_F32) {
    // split K so that the grid covers the GPU several times
    int64_t tiles = (int64_t)grid.x * grid.y;
    int64_t splits = (4 * 148 + tiles - 1) / tiles;
    int64_t max_splits = (g.K + 255) / 256;
    if (splits > max_splits) splits = max_splits;
    if (splits < 1) splits = 1;
    kps = (g.K + splits - 1) / splits;
    kps = (kps + TK - 1) / TK * TK;
    grid.z = (unsigned)((g.K + kps - 1) / kps);
  }
  if (grid.x == 0 || grid.y == 0 || grid.z == 0) return cudaSuccess;
  switch (g.epi) {
    case EPI_STORE:
      if (g.io_f32) gemm_simt_kernel<T, AK, BK, EPI_STORE, float><<<grid, 256, 0, s>>>(g, kps);
      else gemm_simt_kernel<T, AK, BK, EPI_STORE, T><<<grid, 256, 0, s>>>(g, kps);
      break;
    case EPI_SILU_SPLIT: gemm_simt_kernel<T, AK, BK, EPI_SILU_SPLIT, T><<<grid, 256, 0, s>>>(g, kps); break;
    case EPI_RESID:
      if (g.io_f32) gemm_simt_kernel<T, AK, BK, EPI_RESID, float><<<grid, 256, 0, s>>>(g, kps);
      else gemm_simt_kernel<T, AK, BK, EPI_RESID, T><<<grid, 256, 0, s>>>(g, kps);
      break;
    case EPI_ATOMIC_F32: gemm_simt_kernel<T, AK, BK, EPI_ATOMIC_F32, T><<<grid, 256, 0, s>>>(g, kps); break;
    default: return cudaErrorInvalidValue;
  }
  count_launch();
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_t(const GemmArgs& g, cudaStream_t s) {
  if (g.a_kmajor && g.b_kmajor) return launch_epi<T, true, true>(g, s);
  if (g.a_kmajor && !g.b_kmajor) return launch_epi<T, true, false>(g, s);
  if (!g.a_kmajor && g.b_kmajor) return launch_epi<T, false, true>(g, s);
  return launch_epi<T, false, false>(g, s);
}

}  // namespace

cudaError_t gemm_simt(int dtype, const GemmArgs& g, cudaStream_t s) {
  if (g.M == 0 || g.N == 0) return cudaSuccess;
  if (g.K == 0 && g.epi == EPI_ATOMIC_F32) return cudaSuccess;
  return dtype == HSTU_BF16 ? launch_t<bf16>(g, s) : launch_t<float>(g, s);
}

}  // namespace hstu
