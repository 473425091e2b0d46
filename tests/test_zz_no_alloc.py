"""The attention forward entry point that allocates nothing.

Callers held to a device-memory budget fixed at start-up (no allocation on the
serving path) or plain C hosts owning only their buffers cannot provide the
workspace hstu_attention_fwd asks for; hstu_attention_fwd_noalloc keeps that
scratch in a static device array instead.  This file is collected last so that
a run stopping at its first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

from hstu_sequential_transducer_b200 import build
from hstu_sequential_transducer_b200 import hstu as H
from hstu_sequential_transducer_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL = 2e-2  # the bf16 step tolerance of the parity tests: |err_i| / (rms + |ref_i|)


def _inputs(seed):
    d, Hh = 256, 2
    w = W.custom([300, 1, 0, 129, 64, 65, 257], d=d, H=Hh, dtype="bf16", N=300.0,
                 num_targets=[40, 1, 0, 129, 0, 7, 100], mean_gap=3000.0, seed=seed)
    rng = np.random.default_rng(seed)
    g = W.round_to_bf16(rng.normal(0.0, 0.5, size=(w.T, 4 * d)).astype(np.float32))
    dev = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).to("cuda", dt)
    cfg = H.make_config(d, Hh, 300.0, H.HSTU_BF16, max_seq_len=300)
    p = w.params[0]
    return (cfg, dev(p.rab_pos, torch.float32), dev(p.rab_time, torch.float32),
            dev(g, torch.bfloat16), dev(w.seq_offsets, torch.int64), dev(w.timestamps, torch.int64),
            dev(w.num_targets, torch.int32), w.T, d)


def test_noalloc_matches_attention_fwd_twice():
    build.build()
    for seed in (21, 22):   # two calls in a row reuse (and must clear) the shared scratch
        cfg, rp, rt, g, offs, ts, nt, T, d = _inputs(seed)
        ref = torch.empty(T, d, dtype=torch.float32, device="cuda")
        H.attention_fwd(cfg, rp, rt, g, offs, ts, nt, ref)
        got = torch.full((T, d), float("nan"), dtype=torch.float32, device="cuda")
        H.attention_fwd_noalloc(cfg, rp, rt, g, offs, ts, nt, got)
        torch.cuda.synchronize()
        assert H.device_status() == 0
        r = ref.cpu().double().numpy()
        o = got.cpu().double().numpy()
        assert np.isfinite(o).all()
        rms = np.sqrt(np.mean(r ** 2))
        err = float(np.max(np.abs(o - r) / (rms + np.abs(r))))
        assert err <= TOL, f"seed {seed}: {err:.3e}"


def test_noalloc_rejects_sizes_beyond_its_scratch():
    build.build()
    cfg = H.make_config(1024, 8, 8192.0, H.HSTU_BF16)
    B, T = 4, 40_000_000          # a work list far larger than the 2 MiB scratch
    offs = torch.zeros(B + 1, dtype=torch.int64, device="cuda")
    ts = torch.zeros(16, dtype=torch.int64, device="cuda")
    g = torch.zeros(16, 16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(H.HSTUError) as ei:
        H.lib()  # loaded
        st = H.lib().hstu_attention_fwd_noalloc(
            __import__("ctypes").byref(cfg), None, None, H.ptr(g), H.ptr(offs), B, T, H.ptr(ts),
            None, H.ptr(g), H.stream_ptr())
        H._check(st, "hstu_attention_fwd_noalloc")
    assert ei.value.status == 4
