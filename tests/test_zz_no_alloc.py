"""The attention forward entry point that allocates nothing.

Callers held to a device-memory budget fixed at start-up (no allocation on the
serving path) or plain C hosts owning only their buffers cannot provide the
workspace hstu_attention_fwd asks for; hstu_attention_fwd_noalloc keeps that
scratch in a static device array instead.  Both entry points run the same
kernel on the same work list, so their outputs must agree bit for bit.  This
file is collected last so that a run stopping at its first failure has
already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from hstu_sequential_transducer_b200 import build
from hstu_sequential_transducer_b200 import hstu as H
from hstu_sequential_transducer_b200 import workloads as W

pytestmark = pytest.mark.gpu

# (floor(T / 128) + B + 1) * H items fit in the 2 MiB scratch up to this many
CAPACITY_ITEMS = 261_344


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    H.lib()


def _dev(a, dt):
    return torch.from_numpy(np.ascontiguousarray(a)).to("cuda", dt)


def _inputs(seed, dtype, dh):
    Hh = 2
    d = Hh * dh
    w = W.custom([300, 1, 0, 129, 64, 65, 257], d=d, H=Hh, dtype=dtype, N=300.0,
                 num_targets=[40, 1, 0, 129, 0, 7, 100], mean_gap=3000.0, seed=seed)
    rng = np.random.default_rng(seed)
    g = rng.normal(0.0, 0.5, size=(w.T, 4 * d)).astype(np.float32)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    if dtype == "bf16":
        g = W.round_to_bf16(g)
    cfg = H.make_config(d, Hh, 300.0, H.HSTU_BF16 if dtype == "bf16" else H.HSTU_F32,
                        max_seq_len=300)
    p = w.params[0]
    return (cfg, _dev(p.rab_pos, torch.float32), _dev(p.rab_time, torch.float32), _dev(g, tdt),
            _dev(w.seq_offsets, torch.int64), _dev(w.timestamps, torch.int64),
            _dev(w.num_targets, torch.int32), w.T, d)


def _noalloc(cfg, rp, rt, g, offs, ts, nt, out, B=None, T=None):
    B = offs.numel() - 1 if B is None else B
    T = g.shape[0] if T is None else T
    return H.lib().hstu_attention_fwd_noalloc(ctypes.byref(cfg), H.ptr(rp), H.ptr(rt), H.ptr(g),
                                              H.ptr(offs), B, T, H.ptr(ts), H.ptr(nt), H.ptr(out),
                                              H.stream_ptr())


@pytest.mark.parametrize("dtype,dh", [("bf16", 128), ("bf16", 32), ("f32", 32)])
def test_noalloc_matches_attention_fwd_twice(dtype, dh):
    """Two calls in a row (different inputs: the second must not see the first
    one's work list) equal hstu_attention_fwd bit for bit; bf16 dh 128 runs the
    tensor-core kernel, bf16 dh 32 the same kernel on heads zero-padded to 64
    columns (the padded copy also fits in the scratch), fp32 dh 32 the
    CUDA-core one."""
    for i, seed in enumerate((21, 22)):
        cfg, rp, rt, g, offs, ts, nt, T, d = _inputs(seed, dtype, dh)
        ref = torch.full((T, d), float("nan"), dtype=torch.float32, device="cuda")
        H.attention_fwd(cfg, rp, rt, g, offs, ts, nt, ref)
        got = torch.full((T, d), float("nan"), dtype=torch.float32, device="cuda")
        torch.cuda.synchronize()
        free0, _ = torch.cuda.mem_get_info()
        n_alloc0 = torch.cuda.memory_stats().get("allocation.all.allocated", 0)
        assert _noalloc(cfg, rp, rt, g, offs, ts, nt, got) == 0
        torch.cuda.synchronize()
        free1, _ = torch.cuda.mem_get_info()
        n_alloc1 = torch.cuda.memory_stats().get("allocation.all.allocated", 0)
        assert H.device_status() == 0
        assert torch.isfinite(got).all()
        assert torch.equal(got, ref), f"seed {seed}: max diff {(got - ref).abs().max().item()}"
        assert n_alloc1 == n_alloc0
        if i > 0:   # the first call on a device may load the module's code
            assert free1 == free0, f"device memory changed by {free0 - free1} bytes"


def test_noalloc_capacity_boundary():
    """A work list of exactly the capacity runs and matches; one more item
    (one more sequence) is refused with HSTU_ERR_WORKSPACE before any launch."""
    Hh, dh = 8, 128
    d = Hh * dh
    T = 128
    B = CAPACITY_ITEMS // Hh - 1 - T // 128     # 32,666 sequences, all but the first empty
    assert (T // 128 + B + 1) * Hh == CAPACITY_ITEMS
    rng = np.random.default_rng(5)
    cfg = H.make_config(d, Hh, 128.0, H.HSTU_BF16, max_seq_len=128)
    offs = np.full(B + 2, T, np.int64)
    offs[0] = 0
    g = _dev(W.round_to_bf16(rng.normal(0, 0.5, size=(T, 4 * d)).astype(np.float32)), torch.bfloat16)
    ts = _dev(np.cumsum(rng.integers(1, 100, size=T)).astype(np.int64), torch.int64)
    rp = _dev(rng.normal(0, 0.1, size=(Hh, 32)).astype(np.float32), torch.float32)
    rt = _dev(rng.normal(0, 0.1, size=(Hh, 32)).astype(np.float32), torch.float32)
    offs_fit = _dev(offs[:B + 1], torch.int64)
    ref = torch.full((T, d), float("nan"), dtype=torch.float32, device="cuda")
    H.attention_fwd(cfg, rp, rt, g, offs_fit, ts, None, ref)
    got = torch.full((T, d), float("nan"), dtype=torch.float32, device="cuda")
    assert _noalloc(cfg, rp, rt, g, offs_fit, ts, None, got) == 0
    torch.cuda.synchronize()
    assert H.device_status() == 0
    assert torch.equal(got, ref)
    over = torch.full((T, d), float("nan"), dtype=torch.float32, device="cuda")
    assert _noalloc(cfg, rp, rt, g, _dev(offs, torch.int64), ts, None, over) == 4
    torch.cuda.synchronize()
    assert torch.isnan(over).all()          # nothing was launched


def test_noalloc_rejects_sizes_beyond_its_scratch():
    cfg = H.make_config(1024, 8, 8192.0, H.HSTU_BF16)
    B, T = 4, 40_000_000          # a work list far larger than the 2 MiB scratch
    offs = torch.zeros(B + 1, dtype=torch.int64, device="cuda")
    ts = torch.zeros(16, dtype=torch.int64, device="cuda")
    g = torch.zeros(16, 16, dtype=torch.bfloat16, device="cuda")
    assert _noalloc(cfg, None, None, g, offs, ts, None, g, B=B, T=T) == 4


def test_noalloc_empty_input_is_ok():
    cfg = H.make_config(256, 2, 64.0, H.HSTU_BF16)
    offs = torch.zeros(3, dtype=torch.int64, device="cuda")
    ts = torch.zeros(1, dtype=torch.int64, device="cuda")
    g = torch.zeros(1, 1024, dtype=torch.bfloat16, device="cuda")
    o = torch.zeros(1, 256, dtype=torch.float32, device="cuda")
    assert _noalloc(cfg, None, None, g, offs, ts, None, o, B=2, T=0) == 0
    assert _noalloc(cfg, None, None, g, offs[:1], ts, None, o, B=0, T=0) == 0
