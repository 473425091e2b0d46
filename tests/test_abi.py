"""The C-ABI library loads, exports every declared entry point, and rejects
host-checkable errors before touching the GPU (CPU only; no compute calls)."""
import ctypes
import os
import re

import pytest

from hstu_sequential_transducer_b200 import build
from hstu_sequential_transducer_b200 import hstu as H

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return H.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "hstu.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(hstu_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 20
    for n in names:
        assert hasattr(L, n), n
    # and the binding covers every one of them
    assert set(names) <= set(H.exported_symbols())


def test_status_strings(L):
    assert H.status_string(0) == "ok"
    assert "workspace" in H.status_string(4)
    assert H.version().startswith("hstu-b200")


def cfg(**kw):
    c = H.make_config(kw.pop("d", 64), kw.pop("H", 2), kw.pop("N", 64.0), kw.pop("dtype", H.HSTU_BF16))
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def test_config_validation(L):
    ws, sv = ctypes.c_size_t(0), ctypes.c_size_t(0)
    call = lambda c: L.hstu_workspace_size(ctypes.byref(c) if c is not None else None, 4, 100,
                                           ctypes.byref(ws), ctypes.byref(sv))
    assert call(None) == 1
    assert call(cfg()) == 0 and ws.value > 0 and sv.value > 0
    assert call(cfg(head_dim=48, d_model=96)) == 2           # dh not built
    assert call(cfg(d_model=65, head_dim=65, num_heads=1)) == 2      # dh not built
    assert call(cfg(num_heads=3)) == 1                         # d != H * dh
    assert call(cfg(norm_N=0.0)) == 1
    assert call(cfg(num_pos_buckets=33)) == 2
    assert call(cfg(dtype=7)) == 1
    assert L.hstu_workspace_size(ctypes.byref(cfg()), -1, 10, None, None) == 1


def test_saved_layout_sizes(L):
    c = cfg(d=1024, H=8)
    off = H.saved_layout(c, 1000)
    d, es = 1024, 2
    assert off[1] - off[0] >= 1000 * 4 * d * es
    assert off[3] - off[2] >= 1000 * d * es
    assert off[6] >= off[5] + 1000 * 4
    assert all(o % 256 == 0 for o in off)


def test_host_argument_errors_return_before_launch(L):
    c = cfg()
    w = H.Weights(None, None, None, None, None, None, None, None)
    # null x with T > 0
    assert L.hstu_proj_in_fwd(ctypes.byref(c), ctypes.byref(w), None, 10, None, None, None) == 1
    # misaligned pointer -> unsupported
    w.W1 = 0x1000
    assert L.hstu_proj_in_fwd(ctypes.byref(c), ctypes.byref(w), 0x2001, 10, None, 0x3000, None) == 2
    # workspace too small for the layer forward
    off = (ctypes.c_int64 * 3)()
    w.W2 = 0x1000
    st = L.hstu_fwd(ctypes.byref(c), ctypes.byref(w), 0x2000, ctypes.addressof(off), 2, 10,
                    0x4000, None, 0x5000, None, None, 0x6000, 16, None)
    assert st == 4
    # empty input is a no-op success (no launch)
    st = L.hstu_fwd(ctypes.byref(c), ctypes.byref(w), None, ctypes.addressof(off), 0, 0, None, None,
                    None, None, None, None, 1 << 30, None)
    assert st == 0
    # negative sizes
    assert L.hstu_ln_gate_fwd(ctypes.byref(c), None, None, None, None, -1, None, None, None,
                              None) == 1
    # the chained layer calls: a misaligned bf16 copy is refused, a short
    # workspace too, before any launch
    st = L.hstu_fwd_chain(ctypes.byref(c), ctypes.byref(w), 0x2000, 0x7001, ctypes.addressof(off),
                          2, 10, 0x4000, None, 0x5000, None, None, None, 0x6000, 1 << 30, None)
    assert st == 2
    st = L.hstu_fwd_chain(ctypes.byref(c), ctypes.byref(w), 0x2000, 0x7000, ctypes.addressof(off),
                          2, 10, 0x4000, None, 0x5000, 0x8000, None, None, 0x6000, 16, None)
    assert st == 4
    st = L.hstu_bwd_chain(ctypes.byref(c), ctypes.byref(w), 0x2000, 0x3000, 0x7000, 0x9000,
                          ctypes.addressof(off), 2, 10, 0x4000, None, 0x5000, 0x8001, None,
                          0x6000, 1 << 30, None)
    assert st == 2


def test_sl_subsequence_length_host(L):
    """The library's host computation of L = floor(N^(alpha/2)) matches the
    walkthrough's printed pair (alpha = 1.6: 4,096 -> 776) and the closed forms
    in tests/golden/stochastic_length.txt."""
    rows = [l.split() for l in open(os.path.join(ROOT, "tests", "golden", "stochastic_length.txt"))
            if l.strip() and not l.startswith("#")]
    assert rows
    for n, a, want in rows:
        assert L.hstu_sl_subsequence_length(int(n), float(a)) == int(want), (n, a)
    assert L.hstu_sl_subsequence_length(0, 1.6) == 0
    assert L.hstu_sl_subsequence_length(-1, 1.6) == -1
    assert L.hstu_sl_subsequence_length(4096, -0.5) == -1
    assert L.hstu_sl_subsequence_length(4096, float("nan")) == -1


def test_sl_host_argument_errors(L):
    off = (ctypes.c_int64 * 3)()
    a = ctypes.addressof(off)
    # negative sizes / sub_len
    assert L.hstu_stochastic_length(a, None, -1, 0, 5, None, None, a, None, None) == 1
    assert L.hstu_stochastic_length(a, None, 2, 10, -1, 0x1000, 0x1000, a, 0x1000, None) == 1
    # missing draws or outputs
    assert L.hstu_stochastic_length(a, None, 2, 10, 5, None, 0x1000, a, 0x1000, None) == 1
    assert L.hstu_stochastic_length(a, None, 2, 10, 5, 0x1000, 0x1000, a, None, None) == 1
    # misaligned int64 arrays, too many rows
    assert L.hstu_stochastic_length(a + 4, None, 2, 10, 5, 0x1000, 0x1000, a, 0x1000, None) == 2
    assert L.hstu_stochastic_length(a, None, 2, 1 << 31, 5, 0x1000, 0x1000, a, 0x1000, None) == 2
    # gather: empty is a no-op, bad strides and nulls are rejected
    assert L.hstu_gather_rows(None, 0, 0, None, None, 0, 16, None, 0, None) == 0
    assert L.hstu_gather_rows(0x1000, 8, 4, 0x2000, 0x3000, 4, 16, 0x4000, 16, None) == 1
    assert L.hstu_gather_rows(0x1000, 16, 4, None, 0x3000, 4, 16, 0x4000, 16, None) == 1
    assert L.hstu_gather_rows(0x1000, 16, 4, 0x2004, 0x3000, 4, 16, 0x4000, 16, None) == 2


def test_sl_binding_rejects_wrong_dtypes(L):
    import torch
    offs = torch.zeros(3, dtype=torch.int64)
    keep = torch.zeros(2, dtype=torch.int32)
    with pytest.raises(ValueError):
        H.stochastic_length(offs, None, 5, keep, torch.zeros(4, dtype=torch.int64))
    with pytest.raises(ValueError):
        H.stochastic_length(offs.to(torch.int32), None, 5, keep, torch.zeros(4, dtype=torch.int32))
    with pytest.raises(ValueError):
        H.stochastic_length(offs, None, 5, torch.zeros(3, dtype=torch.int32),
                            torch.zeros(4, dtype=torch.int32))


@pytest.mark.parametrize("d,nh", [(512, 4), (1024, 8)])
def test_saved_activation_budget_within_14d(L, d, nh):
    """The HSTU walkthrough ("Gating instead of a separate FFN") puts an HSTU
    layer's saved activation state at 14d bf16 values per token (against 33d
    for a Transformer layer).  The layer's saved block (Pre and G = SiLU(Pre)
    in bf16, O in fp32, Z, the bf16 copy of the residual input, the LayerNorm
    statistics) stays within that: 24d + 8 bytes = 12d + 4 bf16 values."""
    T = 1_000_000
    c = H.make_config(d, nh, 8192.0, H.HSTU_BF16)
    off = H.saved_layout(c, T)
    per_token = off[-1] / T
    assert per_token <= 24 * d + 8 + 1e-3 * d
    assert per_token <= 2 * 14 * d


def test_attention_workspace_holds_the_padded_head32_copy(L):
    """bf16 heads of 32 get a zero-padded copy of V|Q|K (forward) and of
    V|Q|K and dO (backward) in the attention workspace, after the work list
    rounded up to 256 bytes; fp32 heads of 32 and heads of 64 get none."""
    B, T, nh = 7, 1000, 2
    al = lambda v: (v + 255) // 256 * 256
    f = lambda c: L.hstu_attention_workspace_size(ctypes.byref(c), B, T)
    b = lambda c: L.hstu_attention_bwd_workspace_size(ctypes.byref(c), B, T)
    c32, c64 = cfg(d=64, H=nh), cfg(d=128, H=nh)
    c32f = cfg(d=64, H=nh, dtype=H.HSTU_F32)
    assert c32.head_dim == 32 and c64.head_dim == 64
    sched = f(c64)                                   # the work list alone (same B, T, H)
    assert f(c32f) == sched
    assert f(c32) == al(sched) + T * 3 * nh * 64 * 2
    # backward: work list (+ padding) rounded to 256, then the fp32 dQ [T][d]
    dq32 = al(T * 64 * 4)
    assert b(c32f) < b(c32)
    assert b(c32) - dq32 >= T * 4 * nh * 64 * 2
