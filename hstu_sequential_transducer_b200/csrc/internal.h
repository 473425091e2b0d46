// Internal launcher interfaces shared by the .cu files of the HSTU library.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "hstu.h"

namespace hstu {

// ---------------------------------------------------------------------------
// GEMM: C[M][N] = sum_k A(m,k) B(k,n), fp32 accumulation.
//   a_kmajor: A(m,k) = A[m*lda + k]   else A(m,k) = A[k*lda + m]
//   b_kmajor: B(k,n) = B[n*ldb + k]   else B(k,n) = B[k*ldb + n]
// ---------------------------------------------------------------------------
enum GemmEpilogue {
  EPI_STORE = 0,       // C = acc (+ bias)
  EPI_SILU_SPLIT = 1,  // C = acc + bias (Pre, optional), C2 = SiLU(acc + bias)
  EPI_RESID = 2,       // C = acc (+ bias) + R
  EPI_ATOMIC_F32 = 3,  // Cf += acc  (fp32, split-K safe)
};

struct GemmArgs {
  const void* A = nullptr;
  int64_t lda = 0;
  bool a_kmajor = true;
  const void* B = nullptr;
  int64_t ldb = 0;
  bool b_kmajor = true;
  int64_t M = 0, N = 0, K = 0;
  int epi = EPI_STORE;
  void* C = nullptr;        // dtype output (row-major, ldc)
  void* C2 = nullptr;       // second output: G (EPI_SILU_SPLIT); a bf16 copy of the fp32 C
                            // (EPI_RESID with io_f32; row stride ldc)
  int64_t ldc = 0;
  const void* bias = nullptr;  // [N] dtype
  const void* R = nullptr;     // residual, row-major ldr (EPI_RESID)
  int64_t ldr = 0;
  bool io_f32 = false;         // C (EPI_STORE / EPI_RESID) and R are fp32 whatever the operands
  float* Cf = nullptr;      // fp32 accumulation target, row-major ldc (EPI_ATOMIC_F32)
};

cudaError_t gemm(int dtype, const GemmArgs& g, cudaStream_t s);
cudaError_t gemm_simt(int dtype, const GemmArgs& g, cudaStream_t s);
bool gemm_tc_supported(int dtype, const GemmArgs& g);
cudaError_t gemm_tc(const GemmArgs& g, uint32_t* status, cudaStream_t s);

// ---------------------------------------------------------------------------
// Attention
// ---------------------------------------------------------------------------
struct AttnArgs {
  // query side: rows [q_offsets[b], q_offsets[b+1]) of sequence b
  const void* q = nullptr;       // Q block of the query rows' G (row stride q_stride)
  const void* self_k = nullptr;  // the query rows' own K (row stride q_stride)
  const void* self_v = nullptr;  // the query rows' own V (row stride q_stride)
  int64_t q_stride = 0;
  // key side: rows [kv_offsets[b], kv_offsets[b+1])
  const void* k = nullptr;
  const void* v = nullptr;
  int64_t kv_stride = 0;
  void* o = nullptr;             // [T_q][d] fp32
  int64_t o_stride = 0;
  const int64_t* q_offsets = nullptr;
  const int64_t* kv_offsets = nullptr;
  const int64_t* q_ts = nullptr;
  const int64_t* kv_ts = nullptr;
  const int32_t* num_targets = nullptr;  // full mode only
  int cached = 0;                // 0: queries and keys are the same sequence; 1: M-FALCON cache
  int B = 0, H = 0, dh = 0, P = 32, Bt = 32;
  int max_q_len = 0;             // upper bound of any query sequence length
  int64_t q_rows = 0;            // rows of the query-side tensor (T or Tc)
  int64_t kv_rows = 0;           // rows of the key-side tensor (T or T_hist)
  const float* rab_pos = nullptr;
  const float* rab_time = nullptr;
  float inv_N = 1.0f;
  // Columns of O per head when they differ from dh: heads of 32 zero-padded
  // to 64 run with dh = 64 and store only their first o_dh columns.
  int o_dh = 0;
};

struct AttnBwdArgs {
  AttnArgs f;                    // forward arguments (full mode)
  const void* dout = nullptr;    // dO [T][d] (row stride o_stride)
  const void* pre = nullptr;     // Pre [T][4d] (for SiLU')
  void* dpre = nullptr;          // dPre [T][4d]
  int64_t pre_stride = 0;        // 4d
  int d = 0;
  float* dq_acc = nullptr;       // fp32 [T][d] workspace, zeroed by the caller
  float* drab_pos = nullptr;
  float* drab_time = nullptr;
};

cudaError_t attention_fwd(int dtype, const AttnArgs& a, void* ws, size_t ws_bytes, cudaStream_t s);
cudaError_t attention_bwd(int dtype, const AttnBwdArgs& a, void* ws, size_t ws_bytes,
                          cudaStream_t s);
// Workspace of the attention forward: the work list (required) and, for bf16
// head_dim 32, a zero-padded copy of V|Q|K (optional: with it those heads run
// on the tensor-core kernel, without it on the CUDA-core one).
size_t attention_fwd_ws(int B, int64_t T, int H);
size_t attention_fwd_pad_bytes(int dtype, int64_t T, int H, int dh);
size_t attention_fwd_ws_full(int dtype, int B, int64_t T, int H, int dh);
size_t attn_sched_bytes(int B, int64_t Tq, int H);
bool attention_fwd_tc_supported(int dtype, const AttnArgs& a);
cudaError_t attention_fwd_tc(const AttnArgs& a, void* ws, uint32_t* status, cudaStream_t s);
// Backward workspace: the work list and, for bf16 head_dim 32, zero-padded
// copies of V|Q|K and dO (the head_dim-64 tensor-core kernel runs on them).
size_t attention_bwd_ws(int dtype, int B, int64_t T, int H, int dh);
size_t attn_bwd_sched_bytes(int B, int64_t T, int H);
bool attention_bwd_tc_supported(int dtype, const AttnBwdArgs& a);
cudaError_t attention_bwd_tc(const AttnBwdArgs& a, void* ws, uint32_t* status, cudaStream_t s);
cudaError_t attention_bwd_self_simt(int dtype, const AttnBwdArgs& a, cudaStream_t s);
// Softmax comparison attention (same score, buckets and mask; bf16, dh 64/128).
bool softmax_fwd_tc_supported(int dtype, const AttnArgs& a);
cudaError_t softmax_fwd_tc(const AttnArgs& a, void* ws, uint32_t* status, cudaStream_t s);

// ---------------------------------------------------------------------------
// LayerNorm (.) U epilogue
// ---------------------------------------------------------------------------
cudaError_t ln_gate_fwd(int dtype, int d, float eps, const void* gamma, const void* beta,
                        const float* o, const void* g, int64_t g_stride, int64_t T, void* z,
                        float* mean, float* rstd, cudaStream_t s);
cudaError_t ln_gate_bwd(int dtype, int d, const void* gamma, const void* beta, const void* dz,
                        const float* o, const void* g, const void* pre, int64_t g_stride,
                        const float* mean, const float* rstd, int64_t T, void* dout, void* dpre,
                        float* dgamma, float* dbeta, cudaStream_t s);

// ---------------------------------------------------------------------------
// Small kernels
// ---------------------------------------------------------------------------
cudaError_t colsum_accumulate(int dtype, const void* x, int64_t rows, int64_t cols, int64_t ld,
                              float* out, cudaStream_t s);
cudaError_t dq_finalize(int dtype, const float* dq_acc, const void* pre_q, int64_t pre_stride,
                        void* dpre_q, int64_t T, int d, cudaStream_t s);
cudaError_t copy_columns(int dtype, const void* src, int64_t src_stride, void* dst,
                         int64_t dst_stride, int64_t rows, int64_t cols, cudaStream_t s);
// dst [T][nblk*H*64] = blocks b0 (, b1, b2) of every token, bf16, each head's
// 32 values followed by 32 zeros; source rows ss elements apart, 16-byte
// aligned; nblk in 1..3.
cudaError_t pad_heads32(const void* b0, const void* b1, const void* b2, int nblk, int64_t ss,
                        void* dst, int64_t T, int H, cudaStream_t s);
cudaError_t convert_f32_to_bf16(const float* src, void* dst, int64_t n, cudaStream_t s);
cudaError_t validate_inputs(const int64_t* offs, int B, int64_t T, const int64_t* ts,
                            const int32_t* nt, int max_len, uint32_t* flags, cudaStream_t s);

// ---------------------------------------------------------------------------
// Launch accounting and the kernel-level profiler
// ---------------------------------------------------------------------------
// 2-D TMA tensor map over a row-major [outer][inner] bf16 (or fp32) array
// with rows `row_stride_elems` apart; 128-byte swizzle unless told otherwise.
bool encode_tmap_2d(CUtensorMap* m, bool f32, const void* ptr, uint64_t inner, uint64_t outer,
                    uint64_t row_stride_elems, uint32_t box_inner, uint32_t box_outer,
                    bool swizzle128 = true);

// The library's device status word (timeouts of bounded device waits); the
// address belongs to the current device.
uint32_t* device_status();

void prof_begin(int id, cudaStream_t s);
void prof_end(int id, cudaStream_t s);
void count_launch(int n = 1);

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
inline int dtype_size(int dtype) { return dtype == HSTU_BF16 ? 2 : 4; }

}  // namespace hstu
