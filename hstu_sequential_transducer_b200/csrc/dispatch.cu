// Routes each step to its kernel family: tensor-core (tcgen05) kernels for
// bf16 shapes they take, CUDA-core kernels for fp32 and everything else.
#include "common.cuh"
#include "internal.h"

namespace hstu {

cudaError_t attention_fwd_simt(int dtype, const AttnArgs& a, cudaStream_t s);
cudaError_t attention_bwd_simt(int dtype, const AttnBwdArgs& a, cudaStream_t s);

cudaError_t gemm(int dtype, const GemmArgs& g, cudaStream_t s) {
  if (gemm_tc_supported(dtype, g)) return gemm_tc(g, device_status(), s);
  if (g.epi == EPI_RESID && g.io_f32 && g.C2) {
    // the CUDA-core GEMM writes C only; its bf16 copy follows
    GemmArgs h = g;
    h.C2 = nullptr;
    cudaError_t e = gemm_simt(dtype, h, s);
    if (e != cudaSuccess) return e;
    if (g.ldc != g.N) return cudaErrorInvalidValue;   // the layers' rows are dense
    return convert_f32_to_bf16(static_cast<const float*>(g.C), g.C2, g.M * g.N, s);
  }
  return gemm_simt(dtype, g, s);
}

namespace {

// Heads of 32 columns (bf16) run on the head_dim-64 tensor-core kernels:
// V|Q|K are copied to gp [T][3*H*64] with each head zero-padded to 64
// columns (the zeros add nothing to any dot product), and the kernels store
// only the first o_dh = 32 columns of each head's outputs.
AttnArgs padded_heads32(const AttnArgs& a, bf16* gp) {
  const int64_t w = (int64_t)a.H * 64;
  AttnArgs p = a;
  p.self_v = p.v = gp;
  p.q = gp + w;
  p.self_k = p.k = gp + 2 * w;
  p.q_stride = p.kv_stride = 3 * w;
  p.dh = 64;
  p.o_dh = 32;
  return p;
}

size_t pad32_bytes(int dtype, int64_t T, int H, int dh, int blocks) {
  if (dtype != HSTU_BF16 || dh != 32) return 0;
  return (size_t)T * blocks * H * 64 * 2;
}

}  // namespace

cudaError_t attention_fwd(int dtype, const AttnArgs& a, void* ws, size_t ws_bytes, cudaStream_t s) {
  const size_t sched = attn_sched_bytes(a.B, a.q_rows, a.H);
  if (ws_bytes >= sched) {
    if (attention_fwd_tc_supported(dtype, a)) return attention_fwd_tc(a, ws, device_status(), s);
    const size_t pad_at = align_up(sched, 256);
    const size_t pad = attention_fwd_pad_bytes(dtype, a.q_rows, a.H, a.dh);
    if (pad > 0 && !a.cached && ws_bytes >= pad_at + pad) {
      bf16* gp = reinterpret_cast<bf16*>(static_cast<char*>(ws) + pad_at);
      const AttnArgs p = padded_heads32(a, gp);
      if (attention_fwd_tc_supported(dtype, p)) {
        cudaError_t e = pad_heads32(a.self_v, a.q, a.self_k, 3, a.q_stride, gp, a.q_rows, a.H, s);
        if (e != cudaSuccess) return e;
        return attention_fwd_tc(p, ws, device_status(), s);
      }
    }
  }
  return attention_fwd_simt(dtype, a, s);
}

cudaError_t attention_bwd(int dtype, const AttnBwdArgs& a, void* ws, size_t ws_bytes,
                          cudaStream_t s) {
  const AttnArgs& f = a.f;
  const size_t sched = attn_bwd_sched_bytes(f.B, f.q_rows, f.H);
  if (ws_bytes >= sched) {
    if (attention_bwd_tc_supported(dtype, a)) {
      cudaError_t e = attention_bwd_tc(a, ws, device_status(), s);
      if (e != cudaSuccess) return e;
      return attention_bwd_self_simt(dtype, a, s);
    }
    const size_t pad_at = align_up(sched, 256);
    const size_t pad = pad32_bytes(dtype, f.q_rows, f.H, f.dh, 4);
    if (pad > 0 && !f.cached && ws_bytes >= pad_at + pad) {
      bf16* gp = reinterpret_cast<bf16*>(static_cast<char*>(ws) + pad_at);
      bf16* dop = gp + (int64_t)f.q_rows * 3 * f.H * 64;
      AttnBwdArgs p = a;
      p.f = padded_heads32(f, gp);
      p.dout = dop;
      p.f.o_stride = (int64_t)f.H * 64;
      if (attention_bwd_tc_supported(dtype, p)) {
        cudaError_t e = pad_heads32(f.self_v, f.q, f.self_k, 3, f.q_stride, gp, f.q_rows, f.H, s);
        if (e == cudaSuccess)
          e = pad_heads32(a.dout, nullptr, nullptr, 1, f.o_stride, dop, f.q_rows, f.H, s);
        if (e == cudaSuccess) e = attention_bwd_tc(p, ws, device_status(), s);
        if (e != cudaSuccess) return e;
        return attention_bwd_self_simt(dtype, a, s);
      }
    }
  }
  return attention_bwd_simt(dtype, a, s);
}

size_t attention_fwd_ws(int B, int64_t T, int H) { return attn_sched_bytes(B, T, H); }
size_t attention_fwd_pad_bytes(int dtype, int64_t T, int H, int dh) {
  return pad32_bytes(dtype, T, H, dh, 3);
}
size_t attention_fwd_ws_full(int dtype, int B, int64_t T, int H, int dh) {
  const size_t pad = attention_fwd_pad_bytes(dtype, T, H, dh);
  const size_t sched = attention_fwd_ws(B, T, H);
  return pad > 0 ? align_up(sched, 256) + pad : sched;
}
size_t attention_bwd_ws(int dtype, int B, int64_t T, int H, int dh) {
  const size_t pad = pad32_bytes(dtype, T, H, dh, 4);
  const size_t sched = attn_bwd_sched_bytes(B, T, H);
  return pad > 0 ? align_up(sched, 256) + pad : sched;
}

}  // namespace hstu
