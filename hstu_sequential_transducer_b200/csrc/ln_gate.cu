// LayerNorm (.) U gating epilogue, forward and backward.
//
// Equation (3) of the HSTU walkthrough ("What an HSTU layer changes") and
// "Gating instead of a separate FFN": Z = Norm(O) (.) U, the LayerNorm taken
// over all d = H*dh features of a token (biased variance, eps), with an
// optional affine gamma/beta.
//
// Memory-bound: one warp per row, 16-byte vector loads and stores, fp32
// statistics with warp-shuffle reductions, a grid of a few CTAs per SM that
// strides over rows.  The backward keeps the per-column dgamma/dbeta partial
// sums in registers (each lane owns fixed columns) and flushes them once per
// CTA.
#include "common.cuh"
#include "internal.h"

namespace hstu {
namespace {

template <typename T> struct Vec;
template <> struct Vec<bf16> {
  static constexpr int N = 8;
  using U = uint4;
  __device__ static void load(const bf16* p, float* f) {
    uint4 u = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 t = __bfloat1622float2(h[i]);
      f[2 * i] = t.x;
      f[2 * i + 1] = t.y;
    }
  }
  __device__ static void store(bf16* p, const float* f) {
    uint4 u;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    *reinterpret_cast<uint4*>(p) = u;
  }
};
template <> struct Vec<float> {
  static constexpr int N = 4;
  __device__ static void load(const float* p, float* f) {
    float4 u = *reinterpret_cast<const float4*>(p);
    f[0] = u.x; f[1] = u.y; f[2] = u.z; f[3] = u.w;
  }
  __device__ static void store(float* p, const float* f) {
    *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]);
  }
};

template <int N>
__device__ __forceinline__ void load_f32(const float* p, float* f) {
#pragma unroll
  for (int i = 0; i < N; i += 4) {
    const float4 u = *reinterpret_cast<const float4*>(p + i);
    f[i] = u.x; f[i + 1] = u.y; f[i + 2] = u.z; f[i + 3] = u.w;
  }
}

// CH = vector chunks per lane (d <= 32 * CH * VEC)
// AFF: gamma/beta given, kept in shared memory (dynamic, 2 * d floats);
// otherwise the identity affine
template <typename T, int CH, bool AFF>
__global__ void __launch_bounds__(256) ln_gate_fwd_kernel(int d, float eps, const T* __restrict__ gamma,
                                                          const T* __restrict__ beta,
                                                          const float* __restrict__ o,
                                                          const T* __restrict__ g, int64_t g_stride,
                                                          int64_t rows, T* __restrict__ z,
                                                          float* __restrict__ mean_out,
                                                          float* __restrict__ rstd_out) {
  constexpr int VN = Vec<T>::N;
  extern __shared__ __align__(16) float shf[];     // gm[d], bt[d]
  const int lane = threadIdx.x % 32;
  const int nchunk = d / VN;
  if (AFF) {
    for (int i = threadIdx.x; i < d; i += blockDim.x) {
      shf[i] = gamma ? to_f(gamma[i]) : 1.f;
      shf[d + i] = beta ? to_f(beta[i]) : 0.f;
    }
    __syncthreads();
  }
  const int64_t warp = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int64_t nw = (int64_t)gridDim.x * (blockDim.x / 32);
  const float inv_d = 1.f / (float)d;
  for (int64_t r = warp; r < rows; r += nw) {
    float x[CH][VN], uu[CH][VN];
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int ch = lane + 32 * c;
      if (ch < nchunk) {
        load_f32<VN>(o + r * d + ch * VN, x[c]);
        Vec<T>::load(g + r * g_stride + ch * VN, uu[c]);   // in flight during the reductions
#pragma unroll
        for (int k = 0; k < VN; ++k) s += x[c][k];
      } else {
#pragma unroll
        for (int k = 0; k < VN; ++k) x[c][k] = 0.f;
      }
    }
    const float mu = warp_sum(s) * inv_d;
    float v = 0.f;
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int ch = lane + 32 * c;
      if (ch < nchunk)
#pragma unroll
        for (int k = 0; k < VN; ++k) { const float t = x[c][k] - mu; v += t * t; }
    }
    const float rs = rsqrtf(warp_sum(v) * inv_d + eps);
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int ch = lane + 32 * c;
      if (ch < nchunk) {
        float out[VN], gm[VN], bt[VN];
        if (AFF) {
          load_f32<VN>(shf + ch * VN, gm);
          load_f32<VN>(shf + d + ch * VN, bt);
        }
#pragma unroll
        for (int k = 0; k < VN; ++k)
          out[k] = AFF ? ((x[c][k] - mu) * rs * gm[k] + bt[k]) * uu[c][k] : (x[c][k] - mu) * rs * uu[c][k];
        Vec<T>::store(z + r * d + ch * VN, out);
      }
    }
    if (lane == 0) {
      if (mean_out) mean_out[r] = mu;
      if (rstd_out) rstd_out[r] = rs;
    }
  }
}

// AFF: gamma/beta and their gradients live in shared memory (gamma, beta
// once per CTA; dgamma/dbeta partials per warp, each lane updating only the
// columns it owns, so no atomics until the CTA's final flush), which keeps the
// kernel at two CTAs per SM.  Dynamic shared memory: (2 + 2 * warps) * d floats.
template <typename T, int CH, bool AFF>
__global__ void __launch_bounds__(256, CH <= 4 ? 2 : 1) ln_gate_bwd_kernel(
    int d, const T* __restrict__ gamma, const T* __restrict__ beta, const T* __restrict__ dz,
    const float* __restrict__ o, const T* __restrict__ g, const T* __restrict__ pre, int64_t g_stride,
    const float* __restrict__ mean, const float* __restrict__ rstd, int64_t rows,
    T* __restrict__ dout, T* __restrict__ dpre, float* __restrict__ dgamma,
    float* __restrict__ dbeta) {
  constexpr int VN = Vec<T>::N;
  extern __shared__ __align__(16) float sh[];   // gm[d], bt[d], then [warps][2][d] partials
  const int lane = threadIdx.x % 32, wid = threadIdx.x / 32;
  const int nwarps = blockDim.x / 32;
  const int nchunk = d / VN;
  float* const sgm = sh;
  float* const sbt = sh + d;
  float* const sacc = sh + 2 * d + wid * 2 * d;       // this warp's dgamma, dbeta partials
  if (AFF) {
    for (int i = threadIdx.x; i < d; i += blockDim.x) {
      sgm[i] = gamma ? to_f(gamma[i]) : 1.f;
      sbt[i] = beta ? to_f(beta[i]) : 0.f;
    }
    for (int i = threadIdx.x; i < 2 * d * nwarps; i += blockDim.x) sh[2 * d + i] = 0.f;
    __syncthreads();
  }
  const int64_t warp = (int64_t)blockIdx.x * nwarps + wid;
  const int64_t nw = (int64_t)gridDim.x * nwarps;
  const float inv_d = 1.f / (float)d;
  for (int64_t r = warp; r < rows; r += nw) {
    const float mu = mean[r], rs = rstd[r];
    float oh[CH][VN], dh[CH][VN];
    float sa = 0.f, sb = 0.f;
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int ch = lane + 32 * c;
      if (ch < nchunk) {
        float x[VN], gz[VN], u[VN], pu[VN], du[VN];
        load_f32<VN>(o + r * d + ch * VN, x);
        Vec<T>::load(dz + r * d + ch * VN, gz);
        Vec<T>::load(g + r * g_stride + ch * VN, u);
        Vec<T>::load(pre + r * g_stride + ch * VN, pu);
        float gm[VN], bt[VN], ag[VN], ab[VN];
        if (AFF) {
          load_f32<VN>(sgm + ch * VN, gm);
          load_f32<VN>(sbt + ch * VN, bt);
          load_f32<VN>(sacc + ch * VN, ag);
          load_f32<VN>(sacc + d + ch * VN, ab);
        }
#pragma unroll
        for (int k = 0; k < VN; ++k) {
          oh[c][k] = (x[k] - mu) * rs;
          const float ln = AFF ? oh[c][k] * gm[k] + bt[k] : oh[c][k];
          const float dln = gz[k] * u[k];
          du[k] = gz[k] * ln * silu_grad_t<T>(pu[k]);
          if (AFF) {
            ag[k] += dln * oh[c][k];
            ab[k] += dln;
          }
          dh[c][k] = AFF ? dln * gm[k] : dln;
          sa += dh[c][k];
          sb += dh[c][k] * oh[c][k];
        }
        if (AFF) {
#pragma unroll
          for (int k = 0; k < VN; k += 4) {
            *reinterpret_cast<float4*>(sacc + ch * VN + k) = make_float4(ag[k], ag[k + 1], ag[k + 2], ag[k + 3]);
            *reinterpret_cast<float4*>(sacc + d + ch * VN + k) = make_float4(ab[k], ab[k + 1], ab[k + 2], ab[k + 3]);
          }
        }
        Vec<T>::store(dpre + r * g_stride + ch * VN, du);
      } else {
#pragma unroll
        for (int k = 0; k < VN; ++k) { oh[c][k] = 0.f; dh[c][k] = 0.f; }
      }
    }
    sa = warp_sum(sa) * inv_d;
    sb = warp_sum(sb) * inv_d;
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int ch = lane + 32 * c;
      if (ch < nchunk) {
        float out[VN];
#pragma unroll
        for (int k = 0; k < VN; ++k) out[k] = rs * (dh[c][k] - sa - oh[c][k] * sb);
        Vec<T>::store(dout + r * d + ch * VN, out);
      }
    }
  }
  if (AFF && (dgamma || dbeta)) {
    __syncthreads();
    for (int i = threadIdx.x; i < d; i += blockDim.x) {
      float vg = 0.f, vb = 0.f;
      for (int w = 0; w < nwarps; ++w) {
        vg += sh[2 * d + w * 2 * d + i];
        vb += sh[2 * d + w * 2 * d + d + i];
      }
      if (dgamma) atomicAdd(dgamma + i, vg);
      if (dbeta) atomicAdd(dbeta + i, vb);
    }
  }
}

int num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

template <typename T, int CH, bool AFF>
cudaError_t fwd_ch(int d, float eps, const void* gamma, const void* beta, const float* o,
                   const void* g, int64_t gs, int64_t T_, void* z, float* mean, float* rstd,
                   cudaStream_t s) {
  int64_t blocks = (T_ + 7) / 8;
  const int64_t cap = (int64_t)num_sms() * 8;
  if (blocks > cap) blocks = cap;
  if (blocks == 0) return cudaSuccess;
  ln_gate_fwd_kernel<T, CH, AFF><<<(unsigned)blocks, 256, AFF ? 2 * d * sizeof(float) : 0, s>>>(
      d, eps, (const T*)gamma, (const T*)beta, o, (const T*)g, gs, T_, (T*)z, mean, rstd);
  count_launch();
  return cudaGetLastError();
}

template <typename T, int CH, bool AFF>
cudaError_t bwd_ch(int d, const void* gamma, const void* beta, const void* dz, const float* o,
                   const void* g, const void* pre, int64_t gs, const float* mean, const float* rstd,
                   int64_t T_, void* dout, void* dpre, float* dgamma, float* dbeta, cudaStream_t s) {
  int64_t blocks = (T_ + 7) / 8;
  const int64_t cap = (int64_t)num_sms() * 4;
  if (blocks > cap) blocks = cap;
  if (blocks == 0) return cudaSuccess;
  const size_t smem = AFF ? (size_t)(2 + 2 * 8) * d * sizeof(float) : 0;
  if (smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(ln_gate_bwd_kernel<T, CH, AFF>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  ln_gate_bwd_kernel<T, CH, AFF><<<(unsigned)blocks, 256, smem, s>>>(
      d, (const T*)gamma, (const T*)beta, (const T*)dz, o, (const T*)g, (const T*)pre, gs,
      mean, rstd, T_, (T*)dout, (T*)dpre, dgamma, dbeta);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

cudaError_t ln_gate_fwd(int dtype, int d, float eps, const void* gamma, const void* beta,
                        const float* o, const void* g, int64_t gs, int64_t T_, void* z, float* mean,
                        float* rstd, cudaStream_t s) {
  const int vn = dtype == HSTU_BF16 ? 8 : 4;
  const int ch = (d / vn + 31) / 32;
  const bool aff = gamma || beta;
  if (dtype == HSTU_BF16) {
    if (ch <= 1) return aff ? fwd_ch<bf16, 1, true>(d, eps, gamma, beta, o, g, gs, T_, z, mean, rstd, s)
                        : fwd_ch<bf16, 1, false>(d, eps, gamma, beta, o, g, gs, T_, z, mean, rstd, s);
    if (ch <= 2) return aff ? fwd_ch<bf16, 2, true>(d, eps, gamma, beta, o, g, gs, T_, z, mean, rstd, s)
                        : fwd_ch<bf16, 2, false>(d, eps, gamma, beta, o, g, gs, T_, z, mean, rstd, s);
    if (ch <= 4) return aff ? fwd_ch<bf16, 4, true>(d, eps, gamma, beta, o, g, gs, T_, z, mean, rstd, s)
                        : fwd_ch<bf16, 4, false>(d, eps, gamma, beta, o, g, gs, T_, z, mean, rstd, s);
    if (ch <= 8) return aff ? fwd_ch<bf16, 8, true>(d, eps, gamma, beta, o, g, gs, T_, z, mean, rstd, s)
                        : fwd_ch<bf16, 8, false>(d, eps, gamma, beta, o, g, gs, T_, z, mean, rstd, s);
  } else {
    if (ch <= 1) return aff ? fwd_ch<float, 1, true>(d, eps, gamma, beta, o, g, gs, T_, z, mean, rstd, s)
                        : fwd_ch<float, 1, false>(d, eps, gamma, beta, o, g, gs, T_, z, mean, rstd, s);
    if (ch <= 2) return aff ? fwd_ch<float, 2, true>(d, eps, gamma, beta, o, g, gs, T_, z, mean, rstd, s)
                        : fwd_ch<float, 2, false>(d, eps, gamma, beta, o, g, gs, T_, z, mean, rstd, s);
    if (ch <= 4) return aff ? fwd_ch<float, 4, true>(d, eps, gamma, beta, o, g, gs, T_, z, mean, rstd, s)
                        : fwd_ch<float, 4, false>(d, eps, gamma, beta, o, g, gs, T_, z, mean, rstd, s);
    if (ch <= 8) return aff ? fwd_ch<float, 8, true>(d, eps, gamma, beta, o, g, gs, T_, z, mean, rstd, s)
                        : fwd_ch<float, 8, false>(d, eps, gamma, beta, o, g, gs, T_, z, mean, rstd, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t ln_gate_bwd(int dtype, int d, const void* gamma, const void* beta, const void* dz,
                        const float* o, const void* g, const void* pre, int64_t gs,
                        const float* mean, const float* rstd, int64_t T_, void* dout, void* dpre,
                        float* dgamma, float* dbeta, cudaStream_t s) {
  const int vn = dtype == HSTU_BF16 ? 8 : 4;
  const int ch = (d / vn + 31) / 32;
  const bool aff = gamma || beta || dgamma || dbeta;
#define HSTU_LNB(TT, C)                                                                                     \
  return aff ? bwd_ch<TT, C, true>(d, gamma, beta, dz, o, g, pre, gs, mean, rstd, T_, dout, dpre, dgamma,  \
                                   dbeta, s)                                                                \
             : bwd_ch<TT, C, false>(d, gamma, beta, dz, o, g, pre, gs, mean, rstd, T_, dout, dpre, dgamma, \
                                    dbeta, s)
  if (dtype == HSTU_BF16) {
    if (ch <= 1) HSTU_LNB(bf16, 1);
    if (ch <= 2) HSTU_LNB(bf16, 2);
    if (ch <= 4) HSTU_LNB(bf16, 4);
    if (ch <= 8) HSTU_LNB(bf16, 8);
  } else {
    if (ch <= 1) HSTU_LNB(float, 1);
    if (ch <= 2) HSTU_LNB(float, 2);
    if (ch <= 4) HSTU_LNB(float, 4);
    if (ch <= 8) HSTU_LNB(float, 8);
  }
#undef HSTU_LNB
  return cudaErrorInvalidValue;
}

}  // namespace hstu
