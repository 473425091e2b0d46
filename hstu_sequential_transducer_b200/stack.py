"""Device-side drivers for stacks of HSTU layers (plumbing only).

Moves a seeded workload to the GPU and runs it through the C ABI: a forward
stack, a forward+backward training step, M-FALCON scoring (history pass
with K/V caching, then candidate microbatches against the cache), and
Stochastic Length sampling of a training batch.  Every layer step runs in
libhstu.so.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional

import numpy as np
import torch

from . import hstu as H
from .workloads import Workload


def _t(a, dtype, device):
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(device=device, dtype=dtype)


@dataclass
class DeviceWorkload:
    cfg: H.Config
    x: torch.Tensor
    offsets: torch.Tensor
    timestamps: torch.Tensor
    num_targets: Optional[torch.Tensor]
    layers: List[H.LayerWeights]
    dy: Optional[torch.Tensor]
    w: Workload

    @staticmethod
    def from_workload(w: Workload, device="cuda", with_targets=True,
                      io_dtype: int = H.HSTU_F32) -> "DeviceWorkload":
        """io_dtype: dtype of the residual stream (x, y, dy, dx)."""
        dtype_id = H.HSTU_BF16 if w.dtype == "bf16" else H.HSTU_F32
        dt = H.torch_dtype(dtype_id)
        io_dt = H.torch_dtype(io_dtype)
        cfg = H.make_config(w.d_model, w.num_heads, w.norm_N, dtype_id, w.num_pos_buckets,
                            w.num_time_buckets, max(int(w.lengths.max(initial=1)), 1), w.ln_eps,
                            io_dtype=io_dtype)
        layers = []
        for p in w.params:
            layers.append(H.LayerWeights(
                W1=_t(p.W1, dt, device), W2=_t(p.W2, dt, device),
                rab_pos=_t(p.rab_pos, torch.float32, device),
                rab_time=_t(p.rab_time, torch.float32, device),
                b1=_t(p.b1, dt, device), b2=_t(p.b2, dt, device),
                ln_gamma=_t(p.gamma, dt, device), ln_beta=_t(p.beta, dt, device)))
        nt = _t(w.num_targets, torch.int32, device) if (with_targets and w.num_targets is not None) \
            else None
        return DeviceWorkload(cfg, _t(w.x, io_dt, device), _t(w.seq_offsets, torch.int64, device),
                              _t(w.timestamps, torch.int64, device), nt, layers,
                              _t(w.dy, io_dt, device), w)

    @property
    def B(self):
        return self.offsets.numel() - 1

    @property
    def T(self):
        return self.x.shape[0]


def forward_stack(dw: DeviceWorkload, num_layers: Optional[int] = None, stream=None,
                  chain: bool = True):
    """Inference forward through the stack; returns the last layer's output.
    With an fp32 residual stream and bf16 operands, each layer's output
    epilogue also writes the bf16 copy the next layer reads (two alternating
    buffers) unless chain is False."""
    y = dw.x
    layers = dw.layers[:num_layers]
    n = len(layers)
    ch = chain and dw.cfg.io_dtype != dw.cfg.dtype and n > 1
    lo = []
    if ch:
        lt = H.torch_dtype(dw.cfg.dtype)
        lo = [torch.empty(dw.T, dw.cfg.d_model, dtype=lt, device=dw.x.device) for _ in range(2)]
    for i, w in enumerate(layers):
        y = H.fwd(dw.cfg, w, y, dw.offsets, dw.timestamps, dw.num_targets, stream=stream,
                  x_low=lo[i % 2] if ch and i > 0 else None,
                  y_low=lo[(i + 1) % 2] if ch and i + 1 < n else None)
    return y


class TrainStep:
    """Buffers for a forward+backward step over the whole stack, allocated once."""

    def __init__(self, dw: DeviceWorkload, chain: bool = True):
        self.dw = dw
        T = dw.T
        _, saved_n = H.workspace_size(dw.cfg, dw.B, T)
        dev = dw.x.device
        self.saved = [torch.empty(saved_n, dtype=torch.uint8, device=dev) for _ in dw.layers]
        self.acts = [dw.x] + [torch.empty_like(dw.x) for _ in dw.layers]
        self.gbuf = [torch.empty_like(dw.x), torch.empty_like(dw.x)]
        # fp32 residual stream with bf16 operands: each layer's output epilogue
        # also writes the bf16 copy the next layer reads (forward: straight
        # into that layer's saved block; backward: two alternating buffers)
        self.chain = chain and dw.cfg.io_dtype != dw.cfg.dtype
        self.xlow = []
        self.dlow = []
        if self.chain:
            self.xlow = [H.saved_views(dw.cfg, sv, T)["xlow"] for sv in self.saved]
            lt = H.torch_dtype(dw.cfg.dtype)
            self.dlow = [torch.empty(T, dw.cfg.d_model, dtype=lt, device=dev) for _ in range(2)]
        # every layer's fp32 gradients are views of one flat buffer (one
        # all-reduce in data-parallel training)
        names = ("W1", "W2", "b1", "b2", "ln_gamma", "ln_beta", "rab_pos", "rab_time")
        gnames = ("dW1", "dW2", "db1", "db2", "dgamma", "dbeta", "drab_pos", "drab_time")
        total = 0
        for w in dw.layers:
            for n in names:
                t = getattr(w, n)
                if t is not None:
                    total += (t.numel() + 63) // 64 * 64
        self.flat_grads = torch.zeros(max(total, 1), dtype=torch.float32, device=dev)
        self.grads = []
        # layer i's gradients occupy elements [sum(sizes[:i]), sum(sizes[:i+1]))
        # of the flat buffer: one bucket per layer for an overlapped all-reduce
        self.layer_grad_sizes = []
        o = 0
        for w in dw.layers:
            gb = H.LayerGradBufs()
            o0 = o
            for n, gn in zip(names, gnames):
                t = getattr(w, n)
                if t is not None:
                    setattr(gb, gn, self.flat_grads[o:o + t.numel()].view(t.shape))
                    o += (t.numel() + 63) // 64 * 64
            self.grads.append(gb)
            self.layer_grad_sizes.append(o - o0)

    def zero_grads(self):
        self.flat_grads.zero_()

    def run(self, dy=None, stream=None, on_layer_grads=None):
        """Forward (keeping activations) then backward from dy; returns dX.
        on_layer_grads(i), when given, is called right after layer i's
        backward has been issued (layers in reverse order), e.g. to start the
        all-reduce of that layer's gradients."""
        dw = self.dw
        L = len(dw.layers)
        ch = self.chain
        for i, w in enumerate(dw.layers):
            H.fwd(dw.cfg, w, self.acts[i], dw.offsets, dw.timestamps, dw.num_targets,
                  y=self.acts[i + 1], saved=self.saved[i], stream=stream,
                  x_low=self.xlow[i] if ch and i > 0 else None,
                  y_low=self.xlow[i + 1] if ch and i + 1 < L else None)
        g = dw.dy if dy is None else dy
        for i in range(L - 1, -1, -1):
            out = self.gbuf[i % 2]
            H.bwd(dw.cfg, dw.layers[i], self.acts[i], g, self.saved[i], dw.offsets, dw.timestamps,
                  dw.num_targets, dx=out, grads=self.grads[i], stream=stream,
                  dy_low=self.dlow[(i + 1) % 2] if ch and i < L - 1 else None,
                  dx_low=self.dlow[i % 2] if ch and i > 0 else None)
            if on_layer_grads is not None:
                on_layer_grads(i)
            g = out
        return g

    @property
    def y(self):
        return self.acts[-1]


def _gather(src, rows: np.ndarray, out=None):
    """out[r] = src[rows[r]] through the library's row gather (the index and
    the row count are uploaded once per call; no PyTorch indexing)."""
    dev = src.device
    idx = torch.from_numpy(np.ascontiguousarray(rows, dtype=np.int64)).to(dev)
    count = torch.tensor([len(rows)], dtype=torch.int64, device=dev)
    if out is None:
        out = torch.empty((len(rows),) + tuple(src.shape[1:]), dtype=src.dtype, device=dev)
    return H.gather_rows(src, idx, count, out)


def mfalcon_score(dw: DeviceWorkload, history: int, candidates: int, microbatch: int, stream=None):
    """M-FALCON scoring of a workload whose users are `history` tokens followed
    by `candidates` tokens: one history pass caching each layer's V|K, then the
    candidates in microbatches against the cache.  Returns (y_hist, y_cand)
    with candidate rows in input order.  Row selection and reordering run in
    the library's gather kernel."""
    w = dw.w
    B = w.B
    dev = dw.x.device
    d = w.d_model
    n = history + candidates
    assert np.all(w.lengths == n)
    base = np.arange(B) * n
    hist_rows = (base[:, None] + np.arange(history)[None, :]).reshape(-1)
    x_hist = _gather(dw.x, hist_rows)
    ts_hist = _gather(dw.timestamps, hist_rows)
    hist_off = torch.arange(B + 1, dtype=torch.int64, device=dev) * history
    caches = []
    y = x_hist
    for lw in dw.layers:
        kv = torch.empty(y.shape[0], 2 * d, dtype=H.torch_dtype(dw.cfg.dtype), device=dev)
        y = H.fwd(dw.cfg, lw, y, hist_off, ts_hist, None, kv_out=kv, stream=stream)
        caches.append(kv)
    y_hist = y
    # microbatch k writes its B * mb_k rows (user-major) into its own slice of
    # ybuf; one gather then puts every candidate back in input order
    ybuf = torch.empty(B * candidates, d, dtype=dw.x.dtype, device=dev)
    src_rows = np.empty((B, candidates), dtype=np.int64)
    done = 0
    for k0 in range(0, candidates, microbatch):
        mb = min(microbatch, candidates - k0)
        rows = (base[:, None] + history + k0 + np.arange(mb)[None, :]).reshape(-1)
        xc = _gather(dw.x, rows)
        tc = _gather(dw.timestamps, rows)
        coff = torch.arange(B + 1, dtype=torch.int64, device=dev) * mb
        out = ybuf[done:done + B * mb]
        for li, lw in enumerate(dw.layers):
            last = li == len(dw.layers) - 1
            xc = H.fwd_cached(dw.cfg, lw, xc, coff, tc, caches[li], hist_off, ts_hist,
                              y=out if last else None, stream=stream)
        src_rows[:, k0:k0 + mb] = done + np.arange(B)[:, None] * mb + np.arange(mb)[None, :]
        done += B * mb
    y_cand = _gather(ybuf, src_rows.reshape(-1))
    return y_hist, y_cand


class StochasticLength:
    """Stochastic Length sampling of a jagged batch on the device, with
    buffers of the input's capacity allocated once.  `run` launches the
    sampler and the row gathers without synchronising; `batch` reads the
    sampled row count (one 8-byte device-to-host copy) and returns a
    DeviceWorkload of the sampled batch (weights and config shared)."""

    def __init__(self, dw: DeviceWorkload, alpha: float, max_len: Optional[int] = None):
        self.dw = dw
        self.sub_len = H.sl_subsequence_length(int(max_len or dw.cfg.max_seq_len), alpha)
        dev = dw.x.device
        self.new_offsets = torch.empty(dw.B + 1, dtype=torch.int64, device=dev)
        self.gather_index = torch.empty(max(dw.T, 1), dtype=torch.int64, device=dev)
        self.x = torch.empty_like(dw.x)
        self.timestamps = torch.empty_like(dw.timestamps)

    def run(self, keep_draw: torch.Tensor, keys: torch.Tensor, stream=None):
        dw = self.dw
        H.stochastic_length(dw.offsets, dw.num_targets, self.sub_len, keep_draw, keys,
                            self.new_offsets, self.gather_index, stream=stream)
        count = self.new_offsets[dw.B:]
        H.gather_rows(dw.x, self.gather_index, count, self.x, stream=stream)
        H.gather_rows(dw.timestamps, self.gather_index, count, self.timestamps, stream=stream)

    def batch(self) -> DeviceWorkload:
        dw = self.dw
        t = int(self.new_offsets[dw.B].item())
        return DeviceWorkload(dw.cfg, self.x[:t], self.new_offsets, self.timestamps[:t],
                              dw.num_targets, dw.layers, None, dw.w)
