"""The softmax comparison attention (hstu_softmax_attention_fwd) against its
fp64 oracle (oracle/softmax_ref.py), through the C ABI.

Tolerance: as the pointwise attention's single-step outputs, every element
within 2e-2 (rms(ref) + |ref_i|): P is rounded to bf16 once (relative 2^-9)
before the P V contraction, and the running sums are fp32.
"""
import numpy as np
import pytest
import torch

from oracle import hstu_ref as R
from oracle import softmax_ref as SR
from hstu_sequential_transducer_b200 import build
from hstu_sequential_transducer_b200 import hstu as H
from hstu_sequential_transducer_b200 import stack as S
from hstu_sequential_transducer_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL = 2e-2


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    H.lib()


def _check_el(got, ref, what):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    rms = np.sqrt(np.mean(ref ** 2))
    e = float(np.max(np.abs(got - ref) / (rms + np.abs(ref) + 1e-30)))
    assert e <= TOL, f"{what}: max|err|/(rms+|ref|) = {e:.3e} > {TOL:.1e}"
    return e


def _run(w, g):
    dw = S.DeviceWorkload.from_workload(w)
    lw = dw.layers[0]
    gd = torch.from_numpy(np.ascontiguousarray(g, dtype=np.float32)).to("cuda", torch.bfloat16)
    o = torch.full((w.T, w.d_model), float("nan"), dtype=torch.float32, device="cuda")
    H.softmax_attention_fwd(dw.cfg, lw.rab_pos, lw.rab_time, gd, dw.offsets, dw.timestamps,
                            dw.num_targets, o)
    torch.cuda.synchronize()
    assert H.device_status() == 0
    return o.cpu().numpy().astype(np.float64)


def _oracle(w, g):
    p = w.params[0]
    cfg = R.LayerConfig(w.num_heads, w.norm_N, w.num_pos_buckets, w.num_time_buckets, w.ln_eps)
    return SR.softmax_attention_forward(g, w.seq_offsets, w.timestamps, w.num_targets, p.rab_pos,
                                        p.rab_time, cfg)


def _g(w, seed, scale=0.5):
    rng = np.random.default_rng(seed)
    return W.round_to_bf16(rng.normal(0.0, scale, size=(w.T, 4 * w.d_model)).astype(np.float32))


@pytest.mark.parametrize("dh", [64, 128])
@pytest.mark.parametrize("targets", [False, True])
def test_softmax_attention_parity(dh, targets):
    lengths = [300, 1, 0, 129, 64, 65, 257]
    nt = [40, 1, 0, 129, 0, 7, 100] if targets else None
    w = W.custom(lengths, d=2 * dh, H=2, dtype="bf16", N=300.0, num_targets=nt, mean_gap=3000.0,
                 seed=41)
    g = _g(w, 42)
    _check_el(_run(w, g), _oracle(w, g), f"O dh={dh} targets={targets}")


def test_softmax_attention_large_scores():
    """Scores of tens of units: the running maximum moves several times along
    a row (the lazy rescale of O and l in TMEM)."""
    w = W.custom([700, 333], d=256, H=2, dtype="bf16", N=300.0, seed=43)
    g = _g(w, 44, scale=1.5)
    _check_el(_run(w, g), _oracle(w, g), "O large scores")


def test_softmax_attention_full_length():
    """One causal sequence of exactly 8,192 tokens and one 8,192-token sequence
    with 1,024 M-FALCON candidates (H = 2, dh = 128)."""
    w = W.custom([8192, 8192], d=256, H=2, dtype="bf16", N=8192.0, num_targets=[0, 1024],
                 seed=45)
    g = _g(w, 46)
    _check_el(_run(w, g), _oracle(w, g), "O 8,192")


def test_softmax_attention_unsupported_dtype():
    w = W.custom([10], d=64, H=2, dtype="f32", N=10.0)
    dw = S.DeviceWorkload.from_workload(w)
    g = torch.zeros(w.T, 4 * 64, dtype=torch.float32, device="cuda")
    o = torch.zeros(w.T, 64, dtype=torch.float32, device="cuda")
    with pytest.raises(H.HSTUError) as ei:
        H.softmax_attention_fwd(dw.cfg, None, None, g, dw.offsets, dw.timestamps, None, o)
    assert ei.value.status == 2
