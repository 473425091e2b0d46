// Routes each step to its kernel family: tensor-core (tcgen05) kernels for
// bf16 shapes they take, CUDA-core kernels for fp32 and everything else.
#include "common.cuh"
#include "internal.h"

namespace hstu {

cudaError_t attention_fwd_simt(int dtype, const AttnArgs& a, cudaStream_t s);
cudaError_t attention_bwd_simt(int dtype, const AttnBwdArgs& a, cudaStream_t s);

cudaError_t gemm(int dtype, const GemmArgs& g, cudaStream_t s) {
  if (gemm_tc_supported(dtype, g)) return gemm_tc(g, device_status(), s);
  return gemm_simt(dtype, g, s);
}

cudaError_t attention_fwd(int dtype, const AttnArgs& a, void* ws, size_t ws_bytes, cudaStream_t s) {
  if (attention_fwd_tc_supported(dtype, a) &&
      ws_bytes >= attn_sched_bytes(a.B, a.q_rows, a.H))
    return attention_fwd_tc(a, ws, device_status(), s);
  return attention_fwd_simt(dtype, a, s);
}

cudaError_t attention_bwd(int dtype, const AttnBwdArgs& a, void* ws, size_t ws_bytes,
                          cudaStream_t s) {
  if (attention_bwd_tc_supported(dtype, a) &&
      ws_bytes >= attn_bwd_sched_bytes(a.f.B, a.f.q_rows, a.f.H)) {
    cudaError_t e = attention_bwd_tc(a, ws, device_status(), s);
    if (e != cudaSuccess) return e;
    return attention_bwd_self_simt(dtype, a, s);
  }
  return attention_bwd_simt(dtype, a, s);
}

size_t attention_fwd_ws(int B, int64_t T, int H, int max_len) {
  (void)max_len;
  return attn_sched_bytes(B, T, H);
}
size_t attention_bwd_ws(int B, int64_t T, int H, int d, int max_len) {
  (void)d;
  (void)max_len;
  return attn_bwd_sched_bytes(B, T, H);
}

}  // namespace hstu
