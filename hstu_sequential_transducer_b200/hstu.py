"""Thin Python binding of libhstu.so (include/hstu.h).

Argument marshalling only: every step of the layer runs in the library's
CUDA kernels.  PyTorch provides device memory and the current stream.  If
the library is missing this module raises on first use; there is no
fallback.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, Structure, c_char_p, c_double, c_float, c_int32, c_int64, c_size_t, c_uint32, c_void_p
from dataclasses import dataclass
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# HSTU_DEBUG_BUILD=1 loads the debug build (-DHSTU_DEBUG: index checks on the
# attention kernels' direct global accesses, reported as HSTU_DEVICE_BOUNDS)
DEBUG_BUILD = os.environ.get("HSTU_DEBUG_BUILD") == "1"
LIB_PATH = os.path.join(_HERE, "libhstu_debug.so" if DEBUG_BUILD else "libhstu.so")

HSTU_F32, HSTU_BF16 = 0, 1
SAVED_PRE, SAVED_G, SAVED_O, SAVED_Z, SAVED_MEAN, SAVED_RSTD, SAVED_XLOW, SAVED_COUNT = range(8)
K_PROJ_IN, K_ATTN_FWD, K_LN_FWD, K_PROJ_OUT, K_PROJ_OUT_BWD, K_LN_BWD, K_ATTN_BWD, \
    K_PROJ_IN_BWD, K_ATTN_CACHED, K_MISC, K_SOFTMAX, K_COUNT = range(12)
KERNEL_NAMES = ["proj_in", "attn_fwd", "ln_fwd", "proj_out", "proj_out_bwd", "ln_bwd",
                "attn_bwd", "proj_in_bwd", "attn_cached", "misc", "softmax_fwd"]

FLAG_OFFSETS_START, FLAG_OFFSETS_ORDER, FLAG_OFFSETS_END = 0x1, 0x2, 0x4
FLAG_SEQ_TOO_LONG, FLAG_TARGETS_RANGE, FLAG_TIME_ORDER = 0x8, 0x10, 0x20


class Config(Structure):
    _fields_ = [("d_model", c_int32), ("num_heads", c_int32), ("head_dim", c_int32),
                ("num_pos_buckets", c_int32), ("num_time_buckets", c_int32),
                ("max_seq_len", c_int32), ("norm_N", c_float), ("ln_eps", c_float),
                ("dtype", c_int32), ("io_dtype", c_int32)]


class Weights(Structure):
    _fields_ = [("W1", c_void_p), ("b1", c_void_p), ("W2", c_void_p), ("b2", c_void_p),
                ("ln_gamma", c_void_p), ("ln_beta", c_void_p), ("rab_pos", c_void_p),
                ("rab_time", c_void_p)]


class Grads(Structure):
    _fields_ = [("dW1", c_void_p), ("db1", c_void_p), ("dW2", c_void_p), ("db2", c_void_p),
                ("dgamma", c_void_p), ("dbeta", c_void_p), ("drab_pos", c_void_p),
                ("drab_time", c_void_p)]


class HSTUError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_string(status)} (status {status})")
        self.status = status


_lib = None
V, S, I32, I64, P = c_void_p, c_size_t, c_int32, c_int64, c_void_p
_CP = POINTER(Config)
_WP = POINTER(Weights)
_GP = POINTER(Grads)

_SIGS = {
    "hstu_workspace_size": (I32, [_CP, I32, I64, POINTER(c_size_t), POINTER(c_size_t)]),
    "hstu_saved_layout": (I32, [_CP, I64, POINTER(c_size_t)]),
    "hstu_proj_in_fwd": (I32, [_CP, _WP, P, I64, P, P, P]),
    "hstu_attention_fwd": (I32, [_CP, P, P, P, P, I32, I64, P, P, P, P, S, P]),
    "hstu_attention_fwd_cached": (I32, [_CP, P, P, P, P, I32, I64, P, P, P, I64, P, P, P, S, P]),
    "hstu_attention_workspace_size": (S, [_CP, I32, I64]),
    "hstu_softmax_attention_fwd": (I32, [_CP, P, P, P, P, I32, I64, P, P, P, P, S, P]),
    "hstu_attention_fwd_noalloc": (I32, [_CP, P, P, P, P, I32, I64, P, P, P, P]),
    "hstu_ln_gate_fwd": (I32, [_CP, P, P, P, P, I64, P, P, P, P]),
    "hstu_proj_out_fwd": (I32, [_CP, P, P, P, P, I64, P, P]),
    "hstu_proj_out_bwd": (I32, [_CP, P, P, P, I64, P, P, P, P]),
    "hstu_ln_gate_bwd": (I32, [_CP, P, P, P, P, P, P, P, P, I64, P, P, P, P, P]),
    "hstu_attention_bwd": (I32, [_CP, P, P, P, P, P, P, I32, I64, P, P, P, P, P, P, S, P]),
    "hstu_attention_bwd_workspace_size": (S, [_CP, I32, I64]),
    "hstu_proj_in_bwd": (I32, [_CP, P, P, P, P, I64, P, P, P, P]),
    "hstu_fwd": (I32, [_CP, _WP, P, P, I32, I64, P, P, P, P, P, P, S, P]),
    "hstu_fwd_cached": (I32, [_CP, _WP, P, P, I32, I64, P, P, P, I64, P, P, P, S, P]),
    "hstu_bwd": (I32, [_CP, _WP, P, P, P, P, I32, I64, P, P, P, _GP, P, S, P]),
    "hstu_fwd_chain": (I32, [_CP, _WP, P, P, P, I32, I64, P, P, P, P, P, P, P, S, P]),
    "hstu_bwd_chain": (I32, [_CP, _WP, P, P, P, P, P, I32, I64, P, P, P, P, _GP, P, S, P]),
    "hstu_validate_inputs": (I32, [P, I32, I64, P, P, I32, P, P]),
    "hstu_sl_subsequence_length": (I64, [I64, c_double]),
    "hstu_stochastic_length": (I32, [P, P, I32, I64, I64, P, P, P, P, P]),
    "hstu_gather_rows": (I32, [P, I64, I64, P, P, I64, I64, P, I64, P]),
    "hstu_profiler_enable": (None, [I32]),
    "hstu_nvtx_enable": (None, [I32]),
    "hstu_profiler_collect": (I32, [I32, POINTER(c_int64), POINTER(c_double)]),
    "hstu_profiler_reset": (None, []),
    "hstu_launch_count": (I64, []),
    "hstu_device_status": (I32, [POINTER(c_uint32), I32, P]),
    "hstu_selftest_wait_timeout": (I32, [ctypes.c_uint64, P, P]),
    "hstu_status_string": (c_char_p, [I32]),
    "hstu_version": (c_char_p, []),
}


def lib():
    """Loads libhstu.so (built by hstu_sequential_transducer_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run `python -m "
                               "hstu_sequential_transducer_b200.build"
                               f"{' --debug' if DEBUG_BUILD else ''}` first")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def exported_symbols() -> Sequence[str]:
    return list(_SIGS)


def status_string(s: int) -> str:
    return lib().hstu_status_string(int(s)).decode()


def _check(s: int, where: str):
    if s != 0:
        raise HSTUError(s, where)


def ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    return t.data_ptr()


def stream_ptr(stream: Optional[torch.cuda.Stream] = None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def torch_dtype(dtype: int):
    return torch.bfloat16 if dtype == HSTU_BF16 else torch.float32


def make_config(d_model: int, num_heads: int, norm_N: float, dtype: int = HSTU_BF16,
                num_pos_buckets: int = 32, num_time_buckets: int = 32, max_seq_len: int = 8192,
                ln_eps: float = 1e-5, io_dtype: Optional[int] = None) -> Config:
    """io_dtype (x, y, dy, dx) defaults to fp32: a bf16 layer then keeps its
    residual stream in fp32 and only the contraction operands are bf16."""
    io = HSTU_F32 if io_dtype is None else io_dtype
    return Config(d_model, num_heads, d_model // num_heads, num_pos_buckets, num_time_buckets,
                  max_seq_len, float(norm_N), float(ln_eps), dtype, io)


@dataclass
class LayerWeights:
    """Device tensors of one layer (dtype of the config; rab tables fp32)."""
    W1: torch.Tensor
    W2: torch.Tensor
    rab_pos: Optional[torch.Tensor] = None
    rab_time: Optional[torch.Tensor] = None
    b1: Optional[torch.Tensor] = None
    b2: Optional[torch.Tensor] = None
    ln_gamma: Optional[torch.Tensor] = None
    ln_beta: Optional[torch.Tensor] = None

    def c(self) -> Weights:
        return Weights(ptr(self.W1), ptr(self.b1), ptr(self.W2), ptr(self.b2), ptr(self.ln_gamma),
                       ptr(self.ln_beta), ptr(self.rab_pos), ptr(self.rab_time))


@dataclass
class LayerGradBufs:
    dW1: Optional[torch.Tensor] = None
    dW2: Optional[torch.Tensor] = None
    db1: Optional[torch.Tensor] = None
    db2: Optional[torch.Tensor] = None
    dgamma: Optional[torch.Tensor] = None
    dbeta: Optional[torch.Tensor] = None
    drab_pos: Optional[torch.Tensor] = None
    drab_time: Optional[torch.Tensor] = None

    @staticmethod
    def zeros_like(w: LayerWeights, device) -> "LayerGradBufs":
        z = lambda t: None if t is None else torch.zeros(t.shape, dtype=torch.float32, device=device)
        return LayerGradBufs(z(w.W1), z(w.W2), z(w.b1), z(w.b2), z(w.ln_gamma), z(w.ln_beta),
                             z(w.rab_pos), z(w.rab_time))

    def c(self) -> Grads:
        return Grads(ptr(self.dW1), ptr(self.db1), ptr(self.dW2), ptr(self.db2), ptr(self.dgamma),
                     ptr(self.dbeta), ptr(self.drab_pos), ptr(self.drab_time))


# ----------------------------------------------------------------------------
# Sizes
# ----------------------------------------------------------------------------

def workspace_size(cfg: Config, B: int, T: int):
    ws, sv = c_size_t(0), c_size_t(0)
    _check(lib().hstu_workspace_size(ctypes.byref(cfg), B, T, ctypes.byref(ws), ctypes.byref(sv)),
           "hstu_workspace_size")
    return ws.value, sv.value


def attention_workspace_size(cfg: Config, B: int, T: int) -> int:
    return int(lib().hstu_attention_workspace_size(ctypes.byref(cfg), B, T))


def saved_layout(cfg: Config, T: int):
    off = (c_size_t * (SAVED_COUNT + 1))()
    _check(lib().hstu_saved_layout(ctypes.byref(cfg), T, off), "hstu_saved_layout")
    return list(off)


def saved_views(cfg: Config, saved: torch.Tensor, T: int):
    """Typed views of one layer's saved block: pre, g, o, z, mean, rstd."""
    off = saved_layout(cfg, T)
    d = cfg.d_model
    dt = torch_dtype(cfg.dtype)
    es = 2 if cfg.dtype == HSTU_BF16 else 4

    def view(i, n, dtype, shape):
        nbytes = n * (4 if dtype == torch.float32 else es)
        return saved[off[i]:off[i] + nbytes].view(dtype).view(*shape)
    out = {"pre": view(SAVED_PRE, T * 4 * d, dt, (T, 4 * d)),
            "g": view(SAVED_G, T * 4 * d, dt, (T, 4 * d)),
            "o": view(SAVED_O, T * d, torch.float32, (T, d)),
            "z": view(SAVED_Z, T * d, dt, (T, d)),
            "mean": view(SAVED_MEAN, T, torch.float32, (T,)),
            "rstd": view(SAVED_RSTD, T, torch.float32, (T,))}
    if cfg.io_dtype != cfg.dtype:
        out["xlow"] = view(SAVED_XLOW, T * d, dt, (T, d))
    return out


_ws_cache = {}


def workspace(nbytes: int, device, key="default") -> torch.Tensor:
    """A cached uint8 device buffer of at least nbytes (allocated by torch)."""
    k = (str(device), key)
    t = _ws_cache.get(k)
    if t is None or t.numel() < nbytes:
        t = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
        _ws_cache[k] = t
    return t


# ----------------------------------------------------------------------------
# Step-level calls
# ----------------------------------------------------------------------------

def proj_in_fwd(cfg, w: LayerWeights, x, pre_out, g_out, stream=None):
    _check(lib().hstu_proj_in_fwd(ctypes.byref(cfg), ctypes.byref(w.c()), ptr(x), x.shape[0],
                                  ptr(pre_out), ptr(g_out), stream_ptr(stream)), "hstu_proj_in_fwd")


def attention_fwd(cfg, rab_pos, rab_time, g, offsets, timestamps, num_targets, o_out, stream=None,
                  ws_bytes=None):
    """ws_bytes: workspace bytes passed to the call (default: the full
    hstu_attention_workspace_size)."""
    B, T = offsets.numel() - 1, g.shape[0]
    n = lib().hstu_attention_workspace_size(ctypes.byref(cfg), B, T)
    ws = workspace(n, g.device, "attn")
    nb = ws.numel() if ws_bytes is None else min(int(ws_bytes), ws.numel())
    _check(lib().hstu_attention_fwd(ctypes.byref(cfg), ptr(rab_pos), ptr(rab_time), ptr(g),
                                    ptr(offsets), B, T, ptr(timestamps), ptr(num_targets),
                                    ptr(o_out), ptr(ws), nb, stream_ptr(stream)),
           "hstu_attention_fwd")


def softmax_attention_fwd(cfg, rab_pos, rab_time, g, offsets, timestamps, num_targets, o_out,
                          stream=None):
    """The softmax comparison attention (same score and mask, softmax weights)."""
    B, T = offsets.numel() - 1, g.shape[0]
    n = lib().hstu_attention_workspace_size(ctypes.byref(cfg), B, T)
    ws = workspace(n, g.device, "attn")
    _check(lib().hstu_softmax_attention_fwd(ctypes.byref(cfg), ptr(rab_pos), ptr(rab_time), ptr(g),
                                            ptr(offsets), B, T, ptr(timestamps), ptr(num_targets),
                                            ptr(o_out), ptr(ws), ws.numel(), stream_ptr(stream)),
           "hstu_softmax_attention_fwd")


def attention_fwd_noalloc(cfg, rab_pos, rab_time, g, offsets, timestamps, num_targets, o_out,
                          stream=None):
    """hstu_attention_fwd without a workspace (static device scratch)."""
    B, T = offsets.numel() - 1, g.shape[0]
    _check(lib().hstu_attention_fwd_noalloc(ctypes.byref(cfg), ptr(rab_pos), ptr(rab_time), ptr(g),
                                            ptr(offsets), B, T, ptr(timestamps), ptr(num_targets),
                                            ptr(o_out), stream_ptr(stream)),
           "hstu_attention_fwd_noalloc")


def attention_fwd_cached(cfg, rab_pos, rab_time, cand_g, cand_offsets, cand_ts, hist_kv,
                         hist_offsets, hist_ts, o_out, stream=None):
    B, Tc, Th = cand_offsets.numel() - 1, cand_g.shape[0], hist_kv.shape[0]
    n = lib().hstu_attention_workspace_size(ctypes.byref(cfg), B, Tc)
    ws = workspace(n, cand_g.device, "attn")
    _check(lib().hstu_attention_fwd_cached(ctypes.byref(cfg), ptr(rab_pos), ptr(rab_time),
                                           ptr(cand_g), ptr(cand_offsets), B, Tc, ptr(cand_ts),
                                           ptr(hist_kv), ptr(hist_offsets), Th, ptr(hist_ts),
                                           ptr(o_out), ptr(ws), ws.numel(), stream_ptr(stream)),
           "hstu_attention_fwd_cached")


def ln_gate_fwd(cfg, gamma, beta, o, g, z_out, mean_out=None, rstd_out=None, stream=None):
    _check(lib().hstu_ln_gate_fwd(ctypes.byref(cfg), ptr(gamma), ptr(beta), ptr(o), ptr(g),
                                  o.shape[0], ptr(z_out), ptr(mean_out), ptr(rstd_out),
                                  stream_ptr(stream)), "hstu_ln_gate_fwd")


def proj_out_fwd(cfg, W2, b2, z, x, y_out, stream=None):
    _check(lib().hstu_proj_out_fwd(ctypes.byref(cfg), ptr(W2), ptr(b2), ptr(z), ptr(x), z.shape[0],
                                   ptr(y_out), stream_ptr(stream)), "hstu_proj_out_fwd")


def proj_out_bwd(cfg, W2, z, dy, dz_out, dW2=None, db2=None, stream=None):
    _check(lib().hstu_proj_out_bwd(ctypes.byref(cfg), ptr(W2), ptr(z), ptr(dy), dy.shape[0],
                                   ptr(dz_out), ptr(dW2), ptr(db2), stream_ptr(stream)),
           "hstu_proj_out_bwd")


def ln_gate_bwd(cfg, gamma, beta, dz, o, g, pre, mean, rstd, do_out, dpre, dgamma=None,
                dbeta=None, stream=None):
    _check(lib().hstu_ln_gate_bwd(ctypes.byref(cfg), ptr(gamma), ptr(beta), ptr(dz), ptr(o), ptr(g),
                                  ptr(pre), ptr(mean), ptr(rstd), dz.shape[0], ptr(do_out),
                                  ptr(dpre), ptr(dgamma), ptr(dbeta), stream_ptr(stream)),
           "hstu_ln_gate_bwd")


def attention_bwd(cfg, rab_pos, rab_time, g, pre, dout, offsets, timestamps, num_targets, dpre,
                  drab_pos=None, drab_time=None, stream=None):
    B, T = offsets.numel() - 1, g.shape[0]
    n = lib().hstu_attention_bwd_workspace_size(ctypes.byref(cfg), B, T)
    ws = workspace(n, g.device, "attn_bwd")
    _check(lib().hstu_attention_bwd(ctypes.byref(cfg), ptr(rab_pos), ptr(rab_time), ptr(g), ptr(pre),
                                    ptr(dout), ptr(offsets), B, T, ptr(timestamps),
                                    ptr(num_targets), ptr(dpre), ptr(drab_pos), ptr(drab_time),
                                    ptr(ws), ws.numel(), stream_ptr(stream)), "hstu_attention_bwd")


def proj_in_bwd(cfg, W1, x, dpre, dy_resid, dx_out, dW1=None, db1=None, stream=None):
    _check(lib().hstu_proj_in_bwd(ctypes.byref(cfg), ptr(W1), ptr(x), ptr(dpre), ptr(dy_resid),
                                  dpre.shape[0], ptr(dx_out), ptr(dW1), ptr(db1),
                                  stream_ptr(stream)), "hstu_proj_in_bwd")


def validate_inputs(offsets, timestamps, num_targets, max_seq_len, stream=None) -> int:
    """Runs the device validator and returns its flag word (synchronises)."""
    B = offsets.numel() - 1
    T = timestamps.numel()
    flags = torch.zeros(1, dtype=torch.int32, device=offsets.device)
    _check(lib().hstu_validate_inputs(ptr(offsets), B, T, ptr(timestamps), ptr(num_targets),
                                      max_seq_len, ptr(flags), stream_ptr(stream)),
           "hstu_validate_inputs")
    return int(flags.item())


# ----------------------------------------------------------------------------
# Stochastic Length sampler
# ----------------------------------------------------------------------------

def sl_subsequence_length(max_len: int, alpha: float) -> int:
    """L = floor(N^(alpha/2)), computed by the library on the host."""
    v = int(lib().hstu_sl_subsequence_length(int(max_len), float(alpha)))
    if v < 0:
        raise HSTUError(1, "hstu_sl_subsequence_length")
    return v


def stochastic_length(offsets, num_targets, sub_len, keep_draw, keys, new_offsets=None,
                      gather_index=None, stream=None):
    """Samples the jagged batch; returns (new_offsets [B+1], gather_index [T])
    on the device.  new_offsets[B] is the sampled row count; entries of
    gather_index past it are not written."""
    B, T = offsets.numel() - 1, keys.numel()
    for name, t, sizes in (("offsets", offsets, (8,)), ("keep_draw", keep_draw, (4,)),
                           ("keys", keys, (4,)), ("num_targets", num_targets, (4,))):
        if t is not None and (t.element_size() not in sizes or not t.is_contiguous()):
            raise ValueError(f"stochastic_length: {name} must be contiguous with "
                             f"{sizes[0]}-byte elements")
    if keep_draw.numel() != B:
        raise ValueError("stochastic_length: keep_draw needs one entry per sequence")
    if new_offsets is None:
        new_offsets = torch.empty(B + 1, dtype=torch.int64, device=offsets.device)
    if gather_index is None:
        gather_index = torch.empty(max(T, 1), dtype=torch.int64, device=offsets.device)
    _check(lib().hstu_stochastic_length(ptr(offsets), ptr(num_targets), B, T, int(sub_len),
                                        ptr(keep_draw), ptr(keys), ptr(new_offsets),
                                        ptr(gather_index), stream_ptr(stream)),
           "hstu_stochastic_length")
    return new_offsets, gather_index


def gather_rows(src, gather_index, d_num_rows, out, stream=None):
    """out[r] = src[gather_index[r]] for r < d_num_rows (a device int64
    scalar view) and r < out.shape[0]; src and out are 1-D or 2-D tensors with
    contiguous rows of the same width and dtype."""
    src2 = src.reshape(src.shape[0], -1)
    out2 = out.reshape(out.shape[0], -1)
    if src2.dtype != out2.dtype or src2.shape[1] != out2.shape[1] or \
            src2.stride(1) != 1 or out2.stride(1) != 1:
        raise ValueError("gather_rows: src and out need the same dtype, width and unit inner stride")
    es = src2.element_size()
    _check(lib().hstu_gather_rows(ptr(src2), src2.stride(0) * es, src2.shape[0],
                                  ptr(gather_index), ptr(d_num_rows), out2.shape[0],
                                  src2.shape[1] * es, ptr(out2), out2.stride(0) * es,
                                  stream_ptr(stream)),
           "hstu_gather_rows")
    return out


# ----------------------------------------------------------------------------
# Layer-level calls
# ----------------------------------------------------------------------------

def fwd(cfg, w: LayerWeights, x, offsets, timestamps, num_targets=None, y=None, saved=None,
        kv_out=None, stream=None, x_low=None, y_low=None):
    """One layer forward; returns y.  `saved` (uint8, saved_bytes) is filled
    for a later bwd() when given.  x_low / y_low (bf16 [T][d] buffers, fp32
    io only): the bf16 copy of x from the previous layer, and where to write
    the bf16 copy of y for the next one (hstu_fwd_chain)."""
    B, T = offsets.numel() - 1, x.shape[0]
    ws_n, _ = workspace_size(cfg, B, T)
    ws = workspace(ws_n, x.device)
    if y is None:
        y = torch.empty_like(x)
    if x_low is None and y_low is None:
        _check(lib().hstu_fwd(ctypes.byref(cfg), ctypes.byref(w.c()), ptr(x), ptr(offsets), B, T,
                              ptr(timestamps), ptr(num_targets), ptr(y), ptr(saved), ptr(kv_out),
                              ptr(ws), ws.numel(), stream_ptr(stream)), "hstu_fwd")
    else:
        _check(lib().hstu_fwd_chain(ctypes.byref(cfg), ctypes.byref(w.c()), ptr(x), ptr(x_low),
                                    ptr(offsets), B, T, ptr(timestamps), ptr(num_targets), ptr(y),
                                    ptr(y_low), ptr(saved), ptr(kv_out), ptr(ws), ws.numel(),
                                    stream_ptr(stream)), "hstu_fwd_chain")
    return y


def fwd_cached(cfg, w: LayerWeights, cand_x, cand_offsets, cand_ts, hist_kv, hist_offsets, hist_ts,
               y=None, stream=None):
    B, Tc = cand_offsets.numel() - 1, cand_x.shape[0]
    ws_n, _ = workspace_size(cfg, B, Tc)
    ws = workspace(ws_n, cand_x.device)
    if y is None:
        y = torch.empty_like(cand_x)
    _check(lib().hstu_fwd_cached(ctypes.byref(cfg), ctypes.byref(w.c()), ptr(cand_x),
                                 ptr(cand_offsets), B, Tc, ptr(cand_ts), ptr(hist_kv),
                                 ptr(hist_offsets), hist_kv.shape[0], ptr(hist_ts), ptr(y), ptr(ws),
                                 ws.numel(), stream_ptr(stream)), "hstu_fwd_cached")
    return y


def bwd(cfg, w: LayerWeights, x, dy, saved, offsets, timestamps, num_targets=None, dx=None,
        grads: Optional[LayerGradBufs] = None, stream=None, dy_low=None, dx_low=None):
    """One layer backward; returns dx.  dy_low / dx_low (bf16 [T][d], fp32 io
    only): the bf16 copy of dy from the layer above, and where to write the
    bf16 copy of dx for the layer below (hstu_bwd_chain)."""
    B, T = offsets.numel() - 1, x.shape[0]
    ws_n, _ = workspace_size(cfg, B, T)
    ws = workspace(ws_n, x.device)
    if dx is None:
        dx = torch.empty_like(x)
    g = grads.c() if grads is not None else Grads()
    if dy_low is None and dx_low is None:
        _check(lib().hstu_bwd(ctypes.byref(cfg), ctypes.byref(w.c()), ptr(x), ptr(dy), ptr(saved),
                              ptr(offsets), B, T, ptr(timestamps), ptr(num_targets), ptr(dx),
                              ctypes.byref(g), ptr(ws), ws.numel(), stream_ptr(stream)), "hstu_bwd")
    else:
        _check(lib().hstu_bwd_chain(ctypes.byref(cfg), ctypes.byref(w.c()), ptr(x), ptr(dy),
                                    ptr(dy_low), ptr(saved), ptr(offsets), B, T, ptr(timestamps),
                                    ptr(num_targets), ptr(dx), ptr(dx_low), ctypes.byref(g),
                                    ptr(ws), ws.numel(), stream_ptr(stream)), "hstu_bwd_chain")
    return dx


# ----------------------------------------------------------------------------
# Profiler
# ----------------------------------------------------------------------------

def profiler_enable(on: bool = True):
    lib().hstu_profiler_enable(1 if on else 0)


def nvtx_enable(on: bool = True):
    """NVTX ranges named after the kernel classes around the library's steps."""
    lib().hstu_nvtx_enable(1 if on else 0)


def profiler_reset():
    lib().hstu_profiler_reset()


def profiler_collect(kernel_id: int):
    n, ms = c_int64(0), c_double(0.0)
    _check(lib().hstu_profiler_collect(kernel_id, ctypes.byref(n), ctypes.byref(ms)),
           "hstu_profiler_collect")
    return n.value, ms.value


def launch_count() -> int:
    return int(lib().hstu_launch_count())


def device_status(clear: bool = True, stream=None) -> int:
    """The library's device status word (synchronises the stream)."""
    v = c_uint32(0)
    _check(lib().hstu_device_status(ctypes.byref(v), 1 if clear else 0, stream_ptr(stream)),
           "hstu_device_status")
    return v.value


def selftest_wait_timeout(limit_ns: int, result=None, stream=None):
    """Launches the library's bounded-wait diagnostic (a wait nothing ends
    but its limit); the device status word then carries HSTU_DEVICE_TIMEOUT."""
    _check(lib().hstu_selftest_wait_timeout(int(limit_ns), ptr(result), stream_ptr(stream)),
           "hstu_selftest_wait_timeout")


DEVICE_TIMEOUT, DEVICE_SMEM_ALIGN, DEVICE_BOUNDS = 0x100, 0x200, 0x400


def version() -> str:
    return lib().hstu_version().decode()
