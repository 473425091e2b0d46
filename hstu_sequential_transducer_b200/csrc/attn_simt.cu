// CUDA-core pointwise aggregated attention (forward and backward).
//
// Equation (2) of the HSTU walkthrough ("What an HSTU layer changes"):
//   O_h = (1/N) [M (.) SiLU(Q_h K_h^T + rab^{p,t}_h)] V_h
// with no softmax ("No sequence-wise softmax"), the causal / M-FALCON mask
// and ragged execution: one CTA per (query tile, head, sequence); tiles past a
// sequence's end exit at once and key tiles stop at the mask boundary, so no
// padded pair is computed.
//
// This is the fp32 path (and the reference CUDA-core path for shapes the
// tensor-core kernels do not take): 64x64 tiles, fp32 operands in shared
// memory, accurate expf-based SiLU.
#include "common.cuh"
#include "internal.h"

namespace hstu {
namespace {

constexpr int BQ = 64, BK = 64;

// Mask and position bookkeeping shared by both directions.  For a sequence
// with history length hlen, a query at position qpos and a key at index j
// (j < hlen always holds for keys visited by the tile loops):
//   allowed  <=>  qpos >= hlen (a candidate sees all history) || j <= qpos
__device__ __forceinline__ bool pair_allowed(int qpos, int hlen, int j) {
  return qpos >= hlen || j <= qpos;
}

template <typename T, int DH>
__global__ void __launch_bounds__(256) attn_fwd_simt_kernel(AttnArgs a) {
  constexpr int QP = DH + 1;
  extern __shared__ __align__(16) float sm[];
  float* Qs = sm;
  float* Ks = Qs + BQ * QP;
  float* Vs = Ks + BK * QP;
  float* Ps = Vs + BK * DH;
  float* rp = Ps + BQ * (BK + 1);
  float* rt = rp + 32;
  long long* kts = reinterpret_cast<long long*>(rt + 32);

  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  const int b = blockIdx.z, h = blockIdx.y, r0 = blockIdx.x * BQ;
  const int64_t qs = a.q_offsets[b];
  const int nq = (int)(a.q_offsets[b + 1] - qs);
  if (r0 >= nq) return;
  const int64_t ks = a.kv_offsets[b];
  const int nkv = (int)(a.kv_offsets[b + 1] - ks);
  int hlen, qbase;
  if (a.cached) {
    hlen = nkv;
    qbase = nkv;
  } else {
    const int m = a.num_targets ? a.num_targets[b] : 0;
    hlen = min(max(nq - m, 0), nq);  // clamped: malformed counts never index out of range
    qbase = 0;
  }
  const int rows = min(BQ, nq - r0);
  const int kend = min(hlen, qbase + r0 + rows);  // keys [0, kend)

  if (tid < 32) {
    rp[tid] = (a.rab_pos && tid < a.P) ? a.rab_pos[h * a.P + tid] : 0.f;
    rt[tid] = (a.rab_time && tid < a.Bt) ? a.rab_time[h * a.Bt + tid] : 0.f;
  }
  const T* Q = static_cast<const T*>(a.q);
  const T* Kg = static_cast<const T*>(a.k);
  const T* Vg = static_cast<const T*>(a.v);
  for (int idx = tid; idx < BQ * DH; idx += 256) {
    int r = idx / DH, e = idx % DH;
    Qs[r * QP + e] = r < rows ? to_f(Q[(qs + r0 + r) * a.q_stride + h * DH + e]) : 0.f;
  }
  int qpos[4];
  long long tq[4];
  bool rvalid[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int r = ty * 4 + i;
    rvalid[i] = r < rows;
    qpos[i] = qbase + r0 + r;
    tq[i] = rvalid[i] ? a.q_ts[qs + r0 + r] : 0;
  }
  float acc[4][DH / 16];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < DH / 16; ++j) acc[i][j] = 0.f;
  __syncthreads();

  for (int k0 = 0; k0 < kend; k0 += BK) {
    const int kn = min(BK, kend - k0);
    for (int idx = tid; idx < BK * DH; idx += 256) {
      int c = idx / DH, e = idx % DH;
      float kv = 0.f, vv = 0.f;
      if (c < kn) {
        kv = to_f(Kg[(ks + k0 + c) * a.kv_stride + h * DH + e]);
        vv = to_f(Vg[(ks + k0 + c) * a.kv_stride + h * DH + e]);
      }
      Ks[c * QP + e] = kv;
      Vs[c * DH + e] = vv;
    }
    if (tid < BK) kts[tid] = tid < kn ? a.kv_ts[ks + k0 + tid] : 0;
    __syncthreads();

    float s[4][4] = {};
#pragma unroll 4
    for (int e = 0; e < DH; ++e) {
      float qv[4], kv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) qv[i] = Qs[(ty * 4 + i) * QP + e];
#pragma unroll
      for (int j = 0; j < 4; ++j) kv[j] = Ks[(tx + 16 * j) * QP + e];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) s[i][j] = fmaf(qv[i], kv[j], s[i][j]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = tx + 16 * j, jk = k0 + c;
        float p = 0.f;
        if (rvalid[i] && c < kn && pair_allowed(qpos[i], hlen, jk)) {
          const int bp = pos_bucket(min(qpos[i], hlen) - jk, a.P);
          const int bt = time_bucket(tq[i] - kts[c], a.Bt);
          p = silu_acc(s[i][j] + rp[bp] + rt[bt]);
        }
        Ps[(ty * 4 + i) * (BK + 1) + c] = p;
      }
    __syncthreads();
    for (int c = 0; c < kn; ++c) {
      float pv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) pv[i] = Ps[(ty * 4 + i) * (BK + 1) + c];
#pragma unroll
      for (int j = 0; j < DH / 16; ++j) {
        const float vv = Vs[c * DH + tx + 16 * j];
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[i][j] = fmaf(pv[i], vv, acc[i][j]);
      }
    }
    __syncthreads();
  }

  // Self term of candidates (position >= history length): they attend to
  // themselves through their own K and V (bucket 0 for position and time).
  const T* SK = static_cast<const T*>(a.self_k);
  const T* SV = static_cast<const T*>(a.self_v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = ty * 4 + i;
    const bool cand = rvalid[i] && qpos[i] >= hlen;
    float part = 0.f;
    if (cand) {
      for (int e = tx; e < DH; e += 16)
        part += Qs[r * QP + e] * to_f(SK[(qs + r0 + r) * a.q_stride + h * DH + e]);
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (cand) {
      const float pa = silu_acc(part + rp[0] + rt[0]);
#pragma unroll
      for (int j = 0; j < DH / 16; ++j)
        acc[i][j] = fmaf(pa, to_f(SV[(qs + r0 + r) * a.q_stride + h * DH + tx + 16 * j]), acc[i][j]);
    }
  }

  float* O = static_cast<float*>(a.o);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (!rvalid[i]) continue;
    const int r = ty * 4 + i;
#pragma unroll
    for (int j = 0; j < DH / 16; ++j)
      O[(qs + r0 + r) * a.o_stride + h * DH + tx + 16 * j] = acc[i][j] * a.inv_N;
  }
}

// Backward over key tiles: one CTA per (key tile, head, sequence) owns dK and
// dV of its 64 history keys, walks every query tile that can see them,
// recomputes S, and scatters dQ into an fp32 accumulator.
template <typename T, int DH>
__global__ void __launch_bounds__(256) attn_bwd_simt_kernel(AttnBwdArgs A) {
  constexpr int QP = DH + 1;
  const AttnArgs& a = A.f;
  extern __shared__ __align__(16) float sm[];
  float* Ks = sm;
  float* Vs = Ks + BK * QP;
  float* Qs = Vs + BK * QP;
  float* dOs = Qs + BQ * QP;
  float* Ps = dOs + BQ * QP;
  float* dSs = Ps + BK * (BQ + 1);
  float* rp = dSs + BK * (BQ + 1);
  float* rt = rp + 32;
  float* drp = rt + 32;
  float* drt = drp + 32;
  long long* qts = reinterpret_cast<long long*>(drt + 32);

  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  const int b = blockIdx.z, h = blockIdx.y, k0 = blockIdx.x * BK;
  const int64_t s0 = a.q_offsets[b];
  const int n = (int)(a.q_offsets[b + 1] - s0);
  const int m = a.num_targets ? a.num_targets[b] : 0;
  const int hlen = min(max(n - m, 0), n);
  if (k0 >= hlen) return;
  const int kn = min(BK, hlen - k0);

  if (tid < 32) {
    rp[tid] = (a.rab_pos && tid < a.P) ? a.rab_pos[h * a.P + tid] : 0.f;
    rt[tid] = (a.rab_time && tid < a.Bt) ? a.rab_time[h * a.Bt + tid] : 0.f;
    drp[tid] = 0.f;
    drt[tid] = 0.f;
  }
  const T* Qg = static_cast<const T*>(a.q);
  const T* Kg = static_cast<const T*>(a.k);
  const T* Vg = static_cast<const T*>(a.v);
  const T* dOg = static_cast<const T*>(A.dout);
  for (int idx = tid; idx < BK * DH; idx += 256) {
    int c = idx / DH, e = idx % DH;
    float kv = 0.f, vv = 0.f;
    if (c < kn) {
      kv = to_f(Kg[(s0 + k0 + c) * a.kv_stride + h * DH + e]);
      vv = to_f(Vg[(s0 + k0 + c) * a.kv_stride + h * DH + e]);
    }
    Ks[c * QP + e] = kv;
    Vs[c * QP + e] = vv;
  }
  long long tk[4];
  bool kvalid[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int c = ty * 4 + i;
    kvalid[i] = c < kn;
    tk[i] = kvalid[i] ? a.kv_ts[s0 + k0 + c] : 0;
  }
  float dK[4][DH / 16], dV[4][DH / 16];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < DH / 16; ++j) dK[i][j] = dV[i][j] = 0.f;

  for (int q0 = k0; q0 < n; q0 += BQ) {
    const int qn = min(BQ, n - q0);
    __syncthreads();
    for (int idx = tid; idx < BQ * DH; idx += 256) {
      int r = idx / DH, e = idx % DH;
      float qv = 0.f, dv = 0.f;
      if (r < qn) {
        qv = to_f(Qg[(s0 + q0 + r) * a.q_stride + h * DH + e]);
        dv = to_f(dOg[(s0 + q0 + r) * a.o_stride + h * DH + e]);
      }
      Qs[r * QP + e] = qv;
      dOs[r * QP + e] = dv;
    }
    if (tid < BQ) qts[tid] = tid < qn ? a.q_ts[s0 + q0 + tid] : 0;
    __syncthreads();

    float s[4][4] = {}, dp[4][4] = {};
#pragma unroll 2
    for (int e = 0; e < DH; ++e) {
      float kq[4], vq[4], qv[4], dv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        kq[i] = Ks[(ty * 4 + i) * QP + e];
        vq[i] = Vs[(ty * 4 + i) * QP + e];
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        qv[j] = Qs[(tx + 16 * j) * QP + e];
        dv[j] = dOs[(tx + 16 * j) * QP + e];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          s[i][j] = fmaf(kq[i], qv[j], s[i][j]);
          dp[i][j] = fmaf(vq[i], dv[j], dp[i][j]);
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = ty * 4 + i, r = tx + 16 * j;
        const int jk = k0 + c, qi = q0 + r;
        float pa = 0.f, ds = 0.f;
        if (kvalid[i] && r < qn && pair_allowed(qi, hlen, jk)) {
          const int bp = pos_bucket(min(qi, hlen) - jk, a.P);
          const int bt = time_bucket(qts[r] - tk[i], a.Bt);
          const float x = s[i][j] + rp[bp] + rt[bt];
          const float sg = sigmoid_acc(x);
          pa = x * sg * a.inv_N;
          ds = dp[i][j] * sg * (1.f + x * (1.f - sg)) * a.inv_N;
          atomicAdd(&drp[bp], ds);
          atomicAdd(&drt[bt], ds);
        }
        Ps[c * (BQ + 1) + r] = pa;
        dSs[c * (BQ + 1) + r] = ds;
      }
    __syncthreads();
    for (int r = 0; r < qn; ++r) {
      float pv[4], dsv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        pv[i] = Ps[(ty * 4 + i) * (BQ + 1) + r];
        dsv[i] = dSs[(ty * 4 + i) * (BQ + 1) + r];
      }
#pragma unroll
      for (int j = 0; j < DH / 16; ++j) {
        const float dov = dOs[r * QP + tx + 16 * j];
        const float qv = Qs[r * QP + tx + 16 * j];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          dV[i][j] = fmaf(pv[i], dov, dV[i][j]);
          dK[i][j] = fmaf(dsv[i], qv, dK[i][j]);
        }
      }
    }
    // dQ rows of this query tile: rows ty*4+i, columns tx+16j
    {
      float dq[4][DH / 16];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < DH / 16; ++j) dq[i][j] = 0.f;
      for (int c = 0; c < kn; ++c) {
        float dsv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) dsv[i] = dSs[c * (BQ + 1) + ty * 4 + i];
#pragma unroll
        for (int j = 0; j < DH / 16; ++j) {
          const float kv = Ks[c * QP + tx + 16 * j];
#pragma unroll
          for (int i = 0; i < 4; ++i) dq[i][j] = fmaf(dsv[i], kv, dq[i][j]);
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = ty * 4 + i;
        if (r >= qn) continue;
        float* dst = A.dq_acc + (s0 + q0 + r) * (int64_t)A.d + h * DH;
#pragma unroll
        for (int j = 0; j < DH / 16; ++j) atomicAdd(dst + tx + 16 * j, dq[i][j]);
      }
    }
  }

  // dPre_K, dPre_V of the tile's keys
  const T* pre = static_cast<const T*>(A.pre);
  T* dpre = static_cast<T*>(A.dpre);
  const int d = A.d;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (!kvalid[i]) continue;
    const int64_t row = (s0 + k0 + ty * 4 + i) * A.pre_stride;
#pragma unroll
    for (int j = 0; j < DH / 16; ++j) {
      const int col = h * DH + tx + 16 * j;
      dpre[row + 3 * d + col] = from_f<T>(dK[i][j] * silu_grad_acc(to_f(pre[row + 3 * d + col])));
      dpre[row + d + col] = from_f<T>(dV[i][j] * silu_grad_acc(to_f(pre[row + d + col])));
    }
  }
  __syncthreads();
  if (tid < 32) {
    if (A.drab_pos && tid < a.P && drp[tid] != 0.f) atomicAdd(A.drab_pos + h * a.P + tid, drp[tid]);
    if (A.drab_time && tid < a.Bt && drt[tid] != 0.f)
      atomicAdd(A.drab_time + h * a.Bt + tid, drt[tid]);
  }
}

// Self term of the candidates in the backward: candidate i is the only query
// that sees key i, so this kernel alone owns dK_i and dV_i of candidates, and
// adds dS_ii K_i to dQ_i.  One warp per (candidate, head).
template <typename T, int DH>
__global__ void __launch_bounds__(256) attn_bwd_self_kernel(AttnBwdArgs A) {
  const AttnArgs& a = A.f;
  const int b = blockIdx.y, h = blockIdx.z;
  const int64_t s0 = a.q_offsets[b];
  const int n = (int)(a.q_offsets[b + 1] - s0);
  const int m = a.num_targets ? a.num_targets[b] : 0;
  const int hlen = min(max(n - m, 0), n);
  const int lane = threadIdx.x % 32;
  const int warp = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int nw = gridDim.x * (blockDim.x / 32);
  const T* Qg = static_cast<const T*>(a.q);
  const T* Kg = static_cast<const T*>(a.k);
  const T* Vg = static_cast<const T*>(a.v);
  const T* dOg = static_cast<const T*>(A.dout);
  const T* pre = static_cast<const T*>(A.pre);
  T* dpre = static_cast<T*>(A.dpre);
  const int d = A.d;
  const float rp0 = a.rab_pos ? a.rab_pos[h * a.P] : 0.f;
  const float rt0 = a.rab_time ? a.rab_time[h * a.Bt] : 0.f;
  float dsum = 0.f;
  for (int i = hlen + warp; i < n; i += nw) {
    const int64_t t = s0 + i;
    float qv[DH / 32], kv[DH / 32], vv[DH / 32], dov[DH / 32];
    float sq = 0.f, sa = 0.f;
#pragma unroll
    for (int k = 0; k < DH / 32; ++k) {
      const int col = h * DH + lane + 32 * k;
      qv[k] = to_f(Qg[t * a.q_stride + col]);
      kv[k] = to_f(Kg[t * a.kv_stride + col]);
      vv[k] = to_f(Vg[t * a.kv_stride + col]);
      dov[k] = to_f(dOg[t * a.o_stride + col]);
      sq += qv[k] * kv[k];
      sa += dov[k] * vv[k];
    }
    sq = warp_sum(sq) + rp0 + rt0;
    sa = warp_sum(sa);
    const float sg = sigmoid_acc(sq);
    const float pa = sq * sg * a.inv_N;
    const float ds = sa * sg * (1.f + sq * (1.f - sg)) * a.inv_N;
    dsum += ds;
#pragma unroll
    for (int k = 0; k < DH / 32; ++k) {
      const int col = h * DH + lane + 32 * k;
      A.dq_acc[t * d + col] += ds * kv[k];
      const int64_t row = t * A.pre_stride;
      dpre[row + 3 * d + col] = from_f<T>(ds * qv[k] * silu_grad_acc(to_f(pre[row + 3 * d + col])));
      dpre[row + d + col] = from_f<T>(pa * dov[k] * silu_grad_acc(to_f(pre[row + d + col])));
    }
  }
  if (lane == 0 && dsum != 0.f) {
    if (A.drab_pos) atomicAdd(A.drab_pos + h * a.P, dsum);
    if (A.drab_time) atomicAdd(A.drab_time + h * a.Bt, dsum);
  }
}

template <typename T, int DH>
size_t fwd_smem() {
  return (size_t)(2 * BQ * (DH + 1) + BK * DH + BQ * (BK + 1) + 64) * 4 + BK * 8;
}
template <typename T, int DH>
size_t bwd_smem() {
  return (size_t)(4 * BQ * (DH + 1) + 2 * BK * (BQ + 1) + 128) * 4 + BQ * 8;
}

template <typename T, int DH>
cudaError_t fwd_launch(const AttnArgs& a, cudaStream_t s) {
  const size_t smem = fwd_smem<T, DH>();
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_simt_kernel<T, DH>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((a.max_q_len + BQ - 1) / BQ), (unsigned)a.H, (unsigned)a.B);
  if (grid.x == 0 || grid.z == 0) return cudaSuccess;
  attn_fwd_simt_kernel<T, DH><<<grid, 256, smem, s>>>(a);
  count_launch();
  return cudaGetLastError();
}

template <typename T, int DH>
cudaError_t bwd_launch(const AttnBwdArgs& a, cudaStream_t s) {
  const size_t smem = bwd_smem<T, DH>();
  cudaError_t e = cudaFuncSetAttribute(attn_bwd_simt_kernel<T, DH>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((a.f.max_q_len + BK - 1) / BK), (unsigned)a.f.H, (unsigned)a.f.B);
  if (grid.x == 0 || grid.z == 0) return cudaSuccess;
  attn_bwd_simt_kernel<T, DH><<<grid, 256, smem, s>>>(a);
  count_launch();
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (a.f.num_targets) {
    dim3 g2(4, (unsigned)a.f.B, (unsigned)a.f.H);
    attn_bwd_self_kernel<T, DH><<<g2, 256, 0, s>>>(a);
    count_launch();
    e = cudaGetLastError();
  }
  return e;
}

template <typename T>
cudaError_t fwd_dh(const AttnArgs& a, cudaStream_t s) {
  switch (a.dh) {
    case 32: return fwd_launch<T, 32>(a, s);
    case 64: return fwd_launch<T, 64>(a, s);
    case 128: return fwd_launch<T, 128>(a, s);
  }
  return cudaErrorInvalidValue;
}
template <typename T>
cudaError_t bwd_dh(const AttnBwdArgs& a, cudaStream_t s) {
  switch (a.f.dh) {
    case 32: return bwd_launch<T, 32>(a, s);
    case 64: return bwd_launch<T, 64>(a, s);
    case 128: return bwd_launch<T, 128>(a, s);
  }
  return cudaErrorInvalidValue;
}

template <typename T>
cudaError_t self_dh(const AttnBwdArgs& a, cudaStream_t s) {
  dim3 g2(4, (unsigned)a.f.B, (unsigned)a.f.H);
  switch (a.f.dh) {
    case 32: attn_bwd_self_kernel<T, 32><<<g2, 256, 0, s>>>(a); break;
    case 64: attn_bwd_self_kernel<T, 64><<<g2, 256, 0, s>>>(a); break;
    case 128: attn_bwd_self_kernel<T, 128><<<g2, 256, 0, s>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  count_launch();
  return cudaGetLastError();
}

}  // namespace

// Candidate keys' dK, dV and their dQ contribution (the self term).
cudaError_t attention_bwd_self_simt(int dtype, const AttnBwdArgs& a, cudaStream_t s) {
  if (!a.f.num_targets || a.f.B == 0) return cudaSuccess;
  return dtype == HSTU_BF16 ? self_dh<bf16>(a, s) : self_dh<float>(a, s);
}

cudaError_t attention_fwd_simt(int dtype, const AttnArgs& a, cudaStream_t s) {
  return dtype == HSTU_BF16 ? fwd_dh<bf16>(a, s) : fwd_dh<float>(a, s);
}
cudaError_t attention_bwd_simt(int dtype, const AttnBwdArgs& a, cudaStream_t s) {
  return dtype == HSTU_BF16 ? bwd_dh<bf16>(a, s) : bwd_dh<float>(a, s);
}

}  // namespace hstu
