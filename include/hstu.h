/*
 * hstu.h -- C ABI of the HSTU layer hot path on NVIDIA B200 (sm_100a).
 *
 * One HSTU layer over jagged (ragged, concatenated) user-action sequences, as
 * described by the HSTU walkthrough (chenhuiyu.github.io,
 * "generative-recommendation-16-hstu"), section "What an HSTU layer changes",
 * equations (1)-(3):
 *
 *     U, V, Q, K = Split(SiLU(X W1 + b1))                                (1)
 *     O_h        = (1/N) * [M (.) SiLU(Q_h K_h^T + rab^{p,t}_h)] V_h     (2)
 *     Y          = (LayerNorm(O) (.) U) W2 + b2 + X                      (3)
 *
 * with no softmax and no row normalisation ("No sequence-wise softmax" on the
 * same page), ragged execution ("Three more scaling components / Ragged
 * kernels"), and the M-FALCON target mask and history caching
 * ("Sequential Transduction for Recommendation", praveentn.live, "What HSTU
 * actually changed"; "Actions speak louder than words" course,
 * yonasstephen.com, "Serving it: M-FALCON").
 *
 * Readings taken where the pages are silent:
 *   - N is a configuration constant (norm_N); Q K^T has no 1/sqrt(dh) factor;
 *   - Y adds the residual X;
 *   - mask M: key j is allowed for query i iff j <= i and (j < h or j == i),
 *     h = n - num_targets (candidates see the history and themselves only);
 *   - position bucket min(P-1, min(i,h) - min(j,h)); time bucket 0 for a zero
 *     gap, else min(Bt-1, floor(log2(t_i - t_j)) + 1), timestamps in seconds;
 *   - rab tables are per head, fp32: rab_pos[H][P], rab_time[H][Bt];
 *   - LayerNorm over all d = H*dh features of a token, biased variance,
 *     eps = ln_eps, optional affine gamma/beta;
 *   - split order U, V, Q, K; head k of a block is columns [k*dh, (k+1)*dh).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers unless stated otherwise, owned by
 *     the caller.  The library never allocates device memory and keeps no
 *     state between calls except cached device attributes and the optional
 *     profiler's events.
 *   - Every call is asynchronous on `stream` and never synchronises (except
 *     hstu_profiler_collect).
 *   - Host-checkable errors (null pointers, unsupported sizes, misalignment,
 *     workspace too small) return a status before any launch, with no writes.
 *     Launch failures return HSTU_ERR_CUDA.  Malformed *data* (offsets,
 *     timestamps, num_targets) is only detected by hstu_validate_inputs; the
 *     compute kernels assume validated data and never trap.
 *   - Internal activations (Pre, G, O, Z, dO, ...) are row-major [T][width]
 *     in cfg->dtype (fp32 or bf16).  The layer boundary tensors x, y, dy, dx
 *     (the residual stream) are in cfg->io_dtype, which may be fp32 while
 *     cfg->dtype is bf16: the stream then keeps fp32 precision across a stack
 *     of layers and only the operands of the contractions are bf16.
 *     Jagged sequences are concatenated: sequence b owns rows
 *     [seq_offsets[b], seq_offsets[b+1]); seq_offsets is int64 [B+1] with
 *     seq_offsets[0] = 0 and seq_offsets[B] = T.  timestamps is int64 [T]
 *     (seconds), non-decreasing within a sequence.  num_targets is int32 [B]
 *     or NULL (no candidates).
 *   - Weights: W1 [d][4d] (X W1), W2 [d][d], b1 [4d], b2 [d], gamma/beta [d]
 *     in cfg->dtype; b1, b2, gamma, beta, rab_pos, rab_time may be NULL
 *     (NULL means 0, or 1 for gamma).
 *   - Gradients are fp32 and ACCUMULATED (+=) into caller buffers.
 *   - Pointers must be 16-byte aligned; d_model a multiple of 16;
 *     head_dim in {32, 64, 128}; num_pos_buckets, num_time_buckets in [1, 32].
 *     Anything else returns HSTU_ERR_UNSUPPORTED.
 *   - No C++ exception crosses this ABI.
 */
#ifndef HSTU_H_
#define HSTU_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HSTU_OK = 0,
  HSTU_ERR_INVALID = 1,          /* null pointer, negative size, bad enum     */
  HSTU_ERR_UNSUPPORTED = 2,      /* shape / alignment outside what is built   */
  HSTU_ERR_CUDA = 3,             /* a CUDA launch or API call failed          */
  HSTU_ERR_WORKSPACE = 4,        /* workspace smaller than required           */
  HSTU_ERR_DEVICE_TIMEOUT = 5,   /* a bounded device-side wait ran out        */
  HSTU_ERR_BAD_INPUT_DATA = 6    /* reported through validation flags only    */
} hstu_status;

typedef enum { HSTU_F32 = 0, HSTU_BF16 = 1 } hstu_dtype;

/* Layer shape and constants. */
typedef struct {
  int32_t d_model;          /* d = num_heads * head_dim                        */
  int32_t num_heads;        /* H                                               */
  int32_t head_dim;         /* dh in {32, 64, 128}                             */
  int32_t num_pos_buckets;  /* P  (<= 32)                                      */
  int32_t num_time_buckets; /* Bt (<= 32)                                      */
  int32_t max_seq_len;      /* upper bound on any sequence length (<= 65536)   */
  float norm_N;             /* the 1/N normaliser of equation (2)              */
  float ln_eps;             /* LayerNorm epsilon                               */
  int32_t dtype;            /* hstu_dtype of weights, internal activations and
                               contraction operands                            */
  int32_t io_dtype;         /* hstu_dtype of x, y, dy, dx; must equal dtype
                               unless dtype is bf16 and io_dtype fp32         */
} hstu_config;

/* One layer's parameters (device pointers; see conventions for NULLs). */
typedef struct {
  const void* W1;
  const void* b1;
  const void* W2;
  const void* b2;
  const void* ln_gamma;
  const void* ln_beta;
  const float* rab_pos;     /* [H][P]  fp32 */
  const float* rab_time;    /* [H][Bt] fp32 */
} hstu_weights;

/* Parameter gradients, fp32, accumulated (+=).  A NULL member is skipped. */
typedef struct {
  float* dW1;
  float* db1;
  float* dW2;
  float* db2;
  float* dgamma;
  float* dbeta;
  float* drab_pos;
  float* drab_time;
} hstu_grads;

/* Activations a training forward keeps for the backward (see
 * hstu_saved_layout): Pre = X W1 + b1 [T][4d], G = SiLU(Pre) [T][4d] (U|V|Q|K)
 * in cfg->dtype, O [T][d] in fp32, Z = LN(O) (.) U [T][d] in cfg->dtype, then
 * mean [T] and rstd [T] in fp32, then (only when io_dtype differs from dtype)
 * X rounded to cfg->dtype [T][d].
 *
 * O is always fp32: LayerNorm subtracts each row's mean, and the rows of O
 * have a mean many times their spread (SiLU weights and values are mostly
 * positive), so a bf16 O would lose the deviations LayerNorm keeps. */
typedef enum {
  HSTU_SAVED_PRE = 0, HSTU_SAVED_G = 1, HSTU_SAVED_O = 2, HSTU_SAVED_Z = 3,
  HSTU_SAVED_MEAN = 4, HSTU_SAVED_RSTD = 5, HSTU_SAVED_XLOW = 6, HSTU_SAVED_COUNT = 7
} hstu_saved_part;

/* ------------------------------------------------------------------------ */
/* Sizes                                                                     */
/* ------------------------------------------------------------------------ */

/* Workspace bytes needed by hstu_fwd / hstu_bwd / hstu_fwd_cached for B
 * sequences and T tokens (the maximum of the three), and bytes of the saved
 * block of one layer.  Either output pointer may be NULL.  Host only. */
hstu_status hstu_workspace_size(const hstu_config* cfg, int32_t B, int64_t T,
                                size_t* ws_bytes, size_t* saved_bytes);

/* Byte offsets of each hstu_saved_part inside one layer's saved block
 * (offsets[HSTU_SAVED_COUNT] = total bytes).  Host only. */
hstu_status hstu_saved_layout(const hstu_config* cfg, int64_t T,
                              size_t offsets[HSTU_SAVED_COUNT + 1]);

/* ------------------------------------------------------------------------ */
/* Step-level entry points (one per step of the hot path)                    */
/* ------------------------------------------------------------------------ */

/* Equation (1): Pre = X W1 + b1 and G = SiLU(Pre), split as U|V|Q|K.
 * x [T][d] in cfg->dtype (the contraction operand); pre_out [T][4d] may be
 * NULL (inference); g_out [T][4d]. */
hstu_status hstu_proj_in_fwd(const hstu_config* cfg, const hstu_weights* w,
                             const void* x, int64_t T, void* pre_out, void* g_out,
                             cudaStream_t stream);

/* Equation (2) for every head, with rab^{p,t} bucketing, the causal or
 * M-FALCON mask, and ragged work partitioning (sequences are not padded).
 * g [T][4d] holds U|V|Q|K of every token; o_out [T][d] fp32.
 * workspace: hstu_attention_workspace_size(B, T) bytes; less than its
 * work-list part returns HSTU_ERR_WORKSPACE. */
hstu_status hstu_attention_fwd(const hstu_config* cfg, const float* rab_pos,
                               const float* rab_time, const void* g,
                               const int64_t* seq_offsets, int32_t B, int64_t T,
                               const int64_t* timestamps, const int32_t* num_targets,
                               void* o_out, void* workspace, size_t ws_bytes,
                               cudaStream_t stream);

/* M-FALCON cached attention ("Serving it: M-FALCON"): candidate queries of
 * user b (rows [cand_offsets[b], cand_offsets[b+1]) of cand_g [Tc][4d]) attend
 * to every cached history token of that user (hist_kv rows
 * [hist_offsets[b], hist_offsets[b+1]), layout [T_hist][2d] = V|K) and to
 * themselves, never to other candidates.  A candidate's position is the
 * user's history length.  o_out [Tc][d] fp32. */
hstu_status hstu_attention_fwd_cached(const hstu_config* cfg, const float* rab_pos,
                                      const float* rab_time, const void* cand_g,
                                      const int64_t* cand_offsets, int32_t B, int64_t Tc,
                                      const int64_t* cand_timestamps, const void* hist_kv,
                                      const int64_t* hist_offsets, int64_t T_hist,
                                      const int64_t* hist_timestamps, void* o_out,
                                      void* workspace, size_t ws_bytes, cudaStream_t stream);

/* hstu_attention_fwd for callers that cannot allocate device memory (the
 * paper has no counterpart: this is a property of this library's interface).
 * Same arguments and result as hstu_attention_fwd, without the workspace: the
 * scratch (the work list of the tensor-core kernel, and for bf16 head_dim 32
 * the zero-padded copy of V|Q|K when it fits after it) lives in a 2 MiB
 * static device array that every GPU loading the library keeps until process
 * exit.
 * Meant for processes held to a device-memory budget fixed at start-up, which
 * may not allocate while serving, and for C hosts that own only their input
 * and output buffers.
 *   - Capacity: (floor(T / 128) + B + 1) * H <= 261,344 (128-query tile,
 *     head) items; larger inputs return HSTU_ERR_WORKSPACE and nothing is
 *     launched.  Empty inputs (B == 0 or T == 0) return HSTU_OK at once.
 *   - The first call on a device looks up the array's device address (with
 *     that device current); make that first call before any stream capture.
 *     The address is kept for the life of the device's primary context: do
 *     not call this entry point after cudaDeviceReset in the same process.
 *   - It never calls cudaMalloc, cudaFree or any allocating routine.
 *   - Every call on a device shares the same array and rebuilds (and clears)
 *     its contents; calls that can overlap on the GPU (other streams, other
 *     host threads) race on it and must be serialised by the caller. */
hstu_status hstu_attention_fwd_noalloc(const hstu_config* cfg, const float* rab_pos,
                                       const float* rab_time, const void* g,
                                       const int64_t* seq_offsets, int32_t B, int64_t T,
                                       const int64_t* timestamps, const int32_t* num_targets,
                                       void* o_out, cudaStream_t stream);

/* Softmax comparison attention (HSTU walkthrough, "No sequence-wise
 * softmax": HSTU's pointwise SiLU aggregation against the softmax attention of
 * a standard Transformer, which the paper's speed claim at length 8,192 is
 * measured against).  Same arguments, layouts, workspace and errors as
 * hstu_attention_fwd, and the same score S_h(i, j) = Q_h(i).K_h(j) +
 * rab_pos[h][bp] + rab_time[h][bt] (no 1/sqrt(dh)) and mask; the weights are
 * softmax_j(S_h(i, j)) over each query's allowed keys instead of
 * SiLU(S_h(i, j)) / N (norm_N is not used).  o_out [T][d] fp32.  Tensor cores
 * only: bf16 with head_dim 64 or 128, else HSTU_ERR_UNSUPPORTED.  For timing
 * against the pointwise kernel; it is not part of the layer. */
hstu_status hstu_softmax_attention_fwd(const hstu_config* cfg, const float* rab_pos,
                                       const float* rab_time, const void* g,
                                       const int64_t* seq_offsets, int32_t B, int64_t T,
                                       const int64_t* timestamps, const int32_t* num_targets,
                                       void* o_out, void* workspace, size_t ws_bytes,
                                       cudaStream_t stream);

/* Bytes of workspace the attention entry points need. Host only.
 * The work list of the tensor-core kernel is required.  For bf16 with
 * head_dim 32 the size also holds a copy of V|Q|K with every head
 * zero-padded to 64 columns (T * 3 * H * 64 * 2 bytes, after the work list
 * rounded up to 256 bytes): with it those heads run on the head_dim-64
 * tensor-core kernel; hstu_attention_fwd given a workspace that holds the
 * work list but not the copy runs them on the CUDA-core kernel instead.
 * hstu_attention_fwd_cached and hstu_softmax_attention_fwd never use the
 * copy. */
size_t hstu_attention_workspace_size(const hstu_config* cfg, int32_t B, int64_t T);

/* Equation (3), first half: Z = (LayerNorm(O) * gamma + beta) (.) U.
 * o [T][d] fp32, g [T][4d] (U = columns [0, d)), z_out [T][d];
 * mean_out, rstd_out fp32 [T] (either may be NULL). */
hstu_status hstu_ln_gate_fwd(const hstu_config* cfg, const void* ln_gamma, const void* ln_beta,
                             const void* o, const void* g, int64_t T, void* z_out,
                             float* mean_out, float* rstd_out, cudaStream_t stream);

/* Equation (3), second half: Y = Z W2 + b2 + X.  z [T][d] in cfg->dtype;
 * x (may be NULL: no residual) and y_out [T][d] in cfg->io_dtype. */
hstu_status hstu_proj_out_fwd(const hstu_config* cfg, const void* W2, const void* b2,
                              const void* z, const void* x, int64_t T, void* y_out,
                              cudaStream_t stream);

/* Backward of hstu_proj_out_fwd: dz_out = dY W2^T; dW2 += Z^T dY; db2 += sum dY.
 * dy, z, dz_out in cfg->dtype.  dW2/db2 may be NULL. */
hstu_status hstu_proj_out_bwd(const hstu_config* cfg, const void* W2, const void* z,
                              const void* dy, int64_t T, void* dz_out, float* dW2,
                              float* db2, cudaStream_t stream);

/* Backward of hstu_ln_gate_fwd (o fp32).  Writes dO [T][d] and, into the U columns of
 * dpre [T][4d], dPre_U = (dZ (.) LN(O)) (.) SiLU'(Pre_U).  Accumulates
 * dgamma, dbeta (may be NULL). */
hstu_status hstu_ln_gate_bwd(const hstu_config* cfg, const void* ln_gamma, const void* ln_beta,
                             const void* dz, const void* o, const void* g, const void* pre,
                             const float* mean, const float* rstd, int64_t T,
                             void* do_out, void* dpre, float* dgamma, float* dbeta,
                             cudaStream_t stream);

/* Backward of hstu_attention_fwd.  Writes dPre_V, dPre_Q, dPre_K (the V, Q, K
 * columns of dpre [T][4d]) = d{V,Q,K} (.) SiLU'(Pre), and accumulates
 * drab_pos, drab_time (may be NULL).  workspace: at least
 * hstu_attention_bwd_workspace_size(B, T) bytes. */
hstu_status hstu_attention_bwd(const hstu_config* cfg, const float* rab_pos,
                               const float* rab_time, const void* g, const void* pre,
                               const void* dout, const int64_t* seq_offsets, int32_t B,
                               int64_t T, const int64_t* timestamps,
                               const int32_t* num_targets, void* dpre, float* drab_pos,
                               float* drab_time, void* workspace, size_t ws_bytes,
                               cudaStream_t stream);

size_t hstu_attention_bwd_workspace_size(const hstu_config* cfg, int32_t B, int64_t T);

/* Backward of hstu_proj_in_fwd from the assembled dPre [T][4d]:
 * dx_out = dPre W1^T + dy_resid (dy_resid may be NULL); dW1 += X^T dPre;
 * db1 += sum dPre.  x, dpre in cfg->dtype; dy_resid, dx_out in
 * cfg->io_dtype.  dW1/db1 may be NULL. */
hstu_status hstu_proj_in_bwd(const hstu_config* cfg, const void* W1, const void* x,
                             const void* dpre, const void* dy_resid, int64_t T,
                             void* dx_out, float* dW1, float* db1, cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* Layer-level entry points (compose the steps above)                        */
/* ------------------------------------------------------------------------ */

/* One layer forward.  x, y [T][d] in cfg->io_dtype.  saved: NULL for
 * inference, else a block of
 * hstu_workspace_size(...).saved_bytes laid out by hstu_saved_layout.
 * kv_out: NULL, or [T][2d] receiving each token's V|K (the M-FALCON history
 * cache of this layer). */
hstu_status hstu_fwd(const hstu_config* cfg, const hstu_weights* w, const void* x,
                     const int64_t* seq_offsets, int32_t B, int64_t T,
                     const int64_t* timestamps, const int32_t* num_targets, void* y,
                     void* saved, void* kv_out, void* workspace, size_t ws_bytes,
                     cudaStream_t stream);

/* hstu_fwd for a layer inside a stack whose residual stream is fp32
 * (io_dtype HSTU_F32) and whose operands are bf16 (dtype HSTU_BF16): the
 * bf16 copy of each layer's input, which the W1 projection reads, comes from
 * the previous layer's output epilogue instead of a separate conversion.
 *   x_low: NULL, or [T][d] bf16 already holding x rounded to bf16 (the
 *          previous layer's y_low).  With `saved`, the backward needs that
 *          copy inside the saved block: pass the block's HSTU_SAVED_XLOW part
 *          (hstu_saved_layout) to avoid a copy, else it is copied there.
 *   y_low: NULL, or [T][d] bf16 receiving y rounded to bf16 by the W2
 *          projection's epilogue (e.g. the next layer's saved XLOW part).  It
 *          must not overlap x, x_low, y or this layer's saved block.
 * Both are ignored when io_dtype equals dtype.  The results are those of
 * hstu_fwd bit for bit (the same rounding of the same fp32 values). */
hstu_status hstu_fwd_chain(const hstu_config* cfg, const hstu_weights* w, const void* x,
                           const void* x_low, const int64_t* seq_offsets, int32_t B, int64_t T,
                           const int64_t* timestamps, const int32_t* num_targets, void* y,
                           void* y_low, void* saved, void* kv_out, void* workspace,
                           size_t ws_bytes, cudaStream_t stream);

/* One layer forward of M-FALCON candidates against a cached history (see
 * hstu_attention_fwd_cached for the layouts).  cand_x, y [Tc][d] in
 * cfg->io_dtype; hist_kv in cfg->dtype. */
hstu_status hstu_fwd_cached(const hstu_config* cfg, const hstu_weights* w, const void* cand_x,
                            const int64_t* cand_offsets, int32_t B, int64_t Tc,
                            const int64_t* cand_timestamps, const void* hist_kv,
                            const int64_t* hist_offsets, int64_t T_hist,
                            const int64_t* hist_timestamps, void* y, void* workspace,
                            size_t ws_bytes, cudaStream_t stream);

/* One layer backward.  x is the layer input of the forward, saved the block
 * the forward filled; dy [T][d] upstream; dx [T][d] output (may alias dy);
 * x, dy, dx in cfg->io_dtype.
 * Gradients accumulate into *grads (members may be NULL). */
hstu_status hstu_bwd(const hstu_config* cfg, const hstu_weights* w, const void* x,
                     const void* dy, const void* saved, const int64_t* seq_offsets,
                     int32_t B, int64_t T, const int64_t* timestamps,
                     const int32_t* num_targets, void* dx, const hstu_grads* grads,
                     void* workspace, size_t ws_bytes, cudaStream_t stream);

/* hstu_bwd inside a stack (fp32 io, bf16 operands, as hstu_fwd_chain):
 *   dy_low: NULL, or [T][d] bf16 already holding dy rounded to bf16 (the
 *           layer above's dx_low); used as the dY operand of the W2
 *           gradients instead of converting dy.
 *   dx_low: NULL, or [T][d] bf16 receiving dx rounded to bf16 by the dX
 *           epilogue, for the layer below.  It may alias dy_low (which is
 *           read before dx is formed) but no other argument.
 * Both are ignored when io_dtype equals dtype; results equal hstu_bwd's bit
 * for bit. */
hstu_status hstu_bwd_chain(const hstu_config* cfg, const hstu_weights* w, const void* x,
                           const void* dy, const void* dy_low, const void* saved,
                           const int64_t* seq_offsets, int32_t B, int64_t T,
                           const int64_t* timestamps, const int32_t* num_targets, void* dx,
                           void* dx_low, const hstu_grads* grads, void* workspace,
                           size_t ws_bytes, cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* Stochastic Length (training-input subsampling)                            */
/* ------------------------------------------------------------------------ */
/* HSTU walkthrough, "Three more scaling components / Stochastic Length":
 * training usually replaces a long history by a shorter subsequence of it and
 * now and then keeps it whole; alpha = 1.6 maps a length of 4,096 to 776.
 * Readings taken: the subsequence length is L = floor(N^(alpha/2)) for the
 * maximum sequence length N; only the history (the first n - num_targets
 * positions) is sampled and targets are always kept, after it; a history with
 * h <= L is kept whole, a longer one is kept whole with probability L^2/h^2
 * and is otherwise reduced to the L positions with the smallest
 * (key, position) pairs, in their original order. */

/* L = floor(N^(alpha/2)) computed on the host; -1 for N < 0, alpha < 0,
 * alpha > 64 or NaN. */
int64_t hstu_sl_subsequence_length(int64_t max_len, double alpha);

/* Samples a jagged batch.  Inputs (device): seq_offsets int64 [B+1];
 * num_targets int32 [B] or NULL; keep_draw uint32 [B] (sequence b is kept
 * whole iff keep_draw[b] < (L*L / (h*h)) * 2^32, the quotient in fp64);
 * keys uint32 [T] (one ranking key per input row; i.i.d. uniform keys give a
 * uniform random subset).  sub_len = L >= 0.
 * Outputs (device): new_offsets int64 [B+1] (new_offsets[B] = T', the sampled
 * row count, T' <= T); gather_index int64 [capacity T]: output row r is input
 * row gather_index[r], r < T'.  Build the sampled rows (embeddings,
 * timestamps, ...) with hstu_gather_rows; num_targets is unchanged.
 * Requires T < 2^31; int64 arrays 8-byte and uint32/int32 arrays 4-byte
 * aligned.  Two launches, no synchronisation.
 * Malformed offsets (check them with hstu_validate_inputs) give a wrong
 * sample but no out-of-range access: each sequence's rows are clamped into
 * [0, T] and no write lands past the T entries of gather_index. */
hstu_status hstu_stochastic_length(const int64_t* seq_offsets, const int32_t* num_targets,
                                   int32_t B, int64_t T, int64_t sub_len,
                                   const uint32_t* keep_draw, const uint32_t* keys,
                                   int64_t* new_offsets, int64_t* gather_index,
                                   cudaStream_t stream);

/* dst row r = src row gather_index[r] for r < min(*d_num_rows, max_rows)
 * (d_num_rows is a DEVICE int64, e.g. new_offsets + B, so no host sync is
 * needed); row_bytes bytes per row, strides in bytes.  Rows whose index is
 * outside [0, src_rows) are skipped (left unwritten).  dst must hold
 * max_rows rows and must not overlap src.  Copies in the widest of
 * 16/8/4/2/1-byte vectors that the pointers, strides and row size allow. */
hstu_status hstu_gather_rows(const void* src, int64_t src_stride_bytes, int64_t src_rows,
                             const int64_t* gather_index, const int64_t* d_num_rows,
                             int64_t max_rows, int64_t row_bytes, void* dst,
                             int64_t dst_stride_bytes, cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* Support                                                                    */
/* ------------------------------------------------------------------------ */

/* Input-data validation flags (bits of *d_flags, a device uint32). */
#define HSTU_FLAG_OFFSETS_START    0x1u  /* seq_offsets[0] != 0                 */
#define HSTU_FLAG_OFFSETS_ORDER    0x2u  /* seq_offsets decreasing              */
#define HSTU_FLAG_OFFSETS_END      0x4u  /* seq_offsets[B] != T                 */
#define HSTU_FLAG_SEQ_TOO_LONG     0x8u  /* a length > max_seq_len              */
#define HSTU_FLAG_TARGETS_RANGE    0x10u /* num_targets[b] < 0 or > length      */
#define HSTU_FLAG_TIME_ORDER       0x20u /* timestamps decrease in a sequence   */

/* Checks the jagged metadata on the device and ORs HSTU_FLAG_* bits into
 * *d_flags (device uint32, not cleared).  Never traps. */
hstu_status hstu_validate_inputs(const int64_t* seq_offsets, int32_t B, int64_t T,
                                 const int64_t* timestamps, const int32_t* num_targets,
                                 int32_t max_seq_len, uint32_t* d_flags, cudaStream_t stream);

/* Kernel-level profiler: while enabled, each kernel launch of this library is
 * bracketed by CUDA events on its own stream. */
typedef enum {
  HSTU_K_PROJ_IN = 0, HSTU_K_ATTN_FWD = 1, HSTU_K_LN_FWD = 2, HSTU_K_PROJ_OUT = 3,
  HSTU_K_PROJ_OUT_BWD = 4, HSTU_K_LN_BWD = 5, HSTU_K_ATTN_BWD = 6, HSTU_K_PROJ_IN_BWD = 7,
  HSTU_K_ATTN_CACHED = 8, HSTU_K_MISC = 9, HSTU_K_SOFTMAX = 10, HSTU_K_COUNT = 11
} hstu_kernel_id;

void hstu_profiler_enable(int32_t on);
/* NVTX ranges: while on, each of those regions is also an NVTX push/pop
 * range on the calling host thread, named after its kernel class
 * ("proj_in", "attn_fwd", "ln_fwd", "proj_out", "proj_out_bwd", "ln_bwd",
 * "attn_bwd", "proj_in_bwd", "attn_cached", "misc", "softmax_fwd"), so that an
 * NVTX-aware tracer or `ncu --nvtx` can select the library's steps.  Off by
 * default; the environment variable HSTU_NVTX=1 turns it on when the library
 * loads.  A switch flipped between a region's begin and end leaves that one
 * range unbalanced: flip it between calls. */
void hstu_nvtx_enable(int32_t on);
/* Waits for the recorded events, then returns launches and total milliseconds
 * of kernel class `id` since the last reset. */
hstu_status hstu_profiler_collect(int32_t id, int64_t* launches, double* total_ms);
void hstu_profiler_reset(void);
/* Number of kernel launches issued by this library since the last reset
 * (counted on the host whether or not the profiler is enabled). */
int64_t hstu_launch_count(void);

/* Device status word of this library on the current device: bit
 * HSTU_DEVICE_TIMEOUT is set when a kernel's bounded wait ran out (the kernel
 * then abandoned its work and exited cleanly; its outputs are not valid);
 * bit HSTU_DEVICE_SMEM_ALIGN when a kernel that packs its whole shared-memory
 * budget found its dynamic shared memory not 1024-byte aligned (it exits at
 * once; outputs not valid); bit HSTU_DEVICE_BOUNDS, in the debug build only
 * (libhstu_debug.so, compiled with -DHSTU_DEBUG), when an index check on a
 * direct global access of an attention kernel failed (the access was skipped;
 * outputs not valid).  Copies the word to *host_out, synchronising `stream`;
 * clears it when `clear` is non-zero. */
#define HSTU_DEVICE_TIMEOUT 0x100u
#define HSTU_DEVICE_SMEM_ALIGN 0x200u
#define HSTU_DEVICE_BOUNDS 0x400u
hstu_status hstu_device_status(uint32_t* host_out, int32_t clear, cudaStream_t stream);

/* Diagnostic of the bounded-wait path (the pages have no counterpart: this
 * is this library's failure detection).  Launches one small kernel on
 * `stream` that waits on an mbarrier nothing ever arrives on, with a limit of
 * limit_ns nanoseconds (1 .. 100,000,000); the wait runs out, sets
 * HSTU_DEVICE_TIMEOUT in the device status word and the kernel returns.  It
 * issues no copy or tensor-core instruction.  d_result (device int32,
 * nullable) receives 0 when the wait ran out, 1 if it had completed.
 * Returns HSTU_ERR_INVALID for a limit outside the range, without launching. */
hstu_status hstu_selftest_wait_timeout(uint64_t limit_ns, int32_t* d_result, cudaStream_t stream);

const char* hstu_status_string(hstu_status s);
const char* hstu_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HSTU_H_ */
