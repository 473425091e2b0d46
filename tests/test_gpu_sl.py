"""Parity of the Stochastic Length sampler (CUDA, through the C ABI) with the
oracle in ``oracle/stochastic_length.py``.  Integer and byte work: every
comparison is bit-exact (new offsets, gather index, gathered rows)."""
import zlib

import numpy as np
import pytest
import torch

from oracle import stochastic_length as SL
from hstu_sequential_transducer_b200 import build
from hstu_sequential_transducer_b200 import hstu as H
from hstu_sequential_transducer_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    H.lib()


def run_gpu(offs, nt, L, keep, keys):
    o = torch.from_numpy(np.asarray(offs, np.int64)).to(DEV)
    n = None if nt is None else torch.from_numpy(np.asarray(nt, np.int32)).to(DEV)
    kd = torch.from_numpy(np.asarray(keep, np.uint32).view(np.int32)).to(DEV)
    ky = torch.from_numpy(np.asarray(keys, np.uint32).view(np.int32)).to(DEV)
    new_offs, gi = H.stochastic_length(o, n, L, kd, ky)
    torch.cuda.synchronize()
    assert H.device_status() == 0
    no = new_offs.cpu().numpy()
    return no, gi.cpu().numpy()[:int(no[-1])]


def check(offs, nt, L, keep, keys):
    want_offs, want_gi = SL.sample(offs, nt, L, keep, keys)
    got_offs, got_gi = run_gpu(offs, nt, L, keep, keys)
    np.testing.assert_array_equal(got_offs, want_offs)
    np.testing.assert_array_equal(got_gi, want_gi)
    return want_offs, want_gi


def test_sl_training_lengths():
    """64 sequences with lengths U{1024..8192}, N = 8192, alpha = 1.6."""
    rng = np.random.default_rng(5)
    lengths = rng.integers(1024, 8193, size=64)
    offs = W.offsets_from_lengths(lengths)
    L = SL.subsequence_length(8192, 1.6)
    assert L == H.sl_subsequence_length(8192, 1.6) == 1351
    keep, keys = W.sl_draws(21, 64, int(offs[-1]))
    new_offs, gi = check(offs, None, L, keep, keys)
    assert new_offs[-1] < offs[-1]


@pytest.mark.parametrize("case", [
    "empty_batch", "all_empty_seqs", "all_short", "ties", "targets", "targets_whole_seq",
    "L_zero", "h_L_plus_one", "keep_all", "keep_none", "many_seqs", "one_long"])
def test_sl_edge_cases(case):
    rng = np.random.default_rng(zlib.crc32(case.encode()))
    nt = None
    key_range = None
    L = 100
    keep_fix = None
    if case == "empty_batch":
        lengths = np.zeros(0, np.int64)
    elif case == "all_empty_seqs":
        lengths = np.zeros(5, np.int64)
    elif case == "all_short":
        lengths = rng.integers(0, 101, size=40)
    elif case == "ties":
        lengths = rng.integers(1, 3000, size=24)
        key_range = 4
    elif case == "targets":
        lengths = rng.integers(1, 2000, size=30)
        nt = np.array([int(rng.integers(0, n + 1)) for n in lengths], np.int32)
    elif case == "targets_whole_seq":
        lengths = rng.integers(150, 400, size=8)
        nt = lengths.astype(np.int32)
    elif case == "L_zero":
        lengths = rng.integers(0, 700, size=12)
        nt = np.array([int(rng.integers(0, min(n, 5) + 1)) for n in lengths], np.int32)
        L = 0
    elif case == "h_L_plus_one":
        lengths = np.full(16, 101, np.int64)
        keep_fix = 0xFFFFFFFF
    elif case == "keep_all":
        lengths = rng.integers(500, 3000, size=16)
        keep_fix = 0
    elif case == "keep_none":
        lengths = rng.integers(500, 3000, size=16)
        keep_fix = 0xFFFFFFFF
    elif case == "many_seqs":
        lengths = rng.integers(0, 300, size=3000)
    elif case == "one_long":
        lengths = np.array([100_000], np.int64)
        L = 50_000
        keep_fix = 0xFFFFFFFF
        key_range = 1 << 20
    offs = W.offsets_from_lengths(lengths)
    keep, keys = W.sl_draws(7, len(lengths), int(offs[-1]), key_range=key_range)
    if keep_fix is not None:
        keep[:] = keep_fix
    check(offs, nt, L, keep, keys)


@pytest.mark.parametrize("kind", ["bf16_d1024", "f32_d1024", "f32_d1000", "i64_ts", "f32_d50",
                                  "u8_3"])
def test_sl_gather_rows(kind):
    rng = np.random.default_rng(9)
    lengths = rng.integers(200, 2500, size=20)
    offs = W.offsets_from_lengths(lengths)
    T = int(offs[-1])
    L = 300
    keep, keys = W.sl_draws(3, len(lengths), T)
    new_offs, gi = SL.sample(offs, None, L, keep, keys)
    Tn = int(new_offs[-1])
    if kind == "bf16_d1024":
        x = W.round_to_bf16(rng.standard_normal((T, 1024)).astype(np.float32))
        xt = torch.from_numpy(x).to(DEV).to(torch.bfloat16)
    elif kind == "f32_d1024":
        x = rng.standard_normal((T, 1024)).astype(np.float32)
        xt = torch.from_numpy(x).to(DEV)
    elif kind == "f32_d1000":  # 250 16-byte vectors: a ragged last segment
        x = rng.standard_normal((T, 1000)).astype(np.float32)
        xt = torch.from_numpy(x).to(DEV)
    elif kind == "i64_ts":
        x = W.draw_timestamps(rng, lengths)
        xt = torch.from_numpy(x).to(DEV)
    elif kind == "f32_d50":
        x = rng.standard_normal((T, 50)).astype(np.float32)
        xt = torch.from_numpy(x).to(DEV)
    else:
        x = rng.integers(0, 256, size=(T, 3)).astype(np.uint8)
        xt = torch.from_numpy(x).to(DEV)
    o = torch.from_numpy(offs).to(DEV)
    kd = torch.from_numpy(keep.view(np.int32)).to(DEV)
    ky = torch.from_numpy(keys.view(np.int32)).to(DEV)
    new_o, gidx = H.stochastic_length(o, None, L, kd, ky)
    # capacity T rows; only the first new_offsets[B] are written
    out = torch.zeros((T,) + tuple(xt.shape[1:]), dtype=xt.dtype, device=DEV)
    H.gather_rows(xt, gidx, new_o[-1:], out)
    torch.cuda.synchronize()
    got = out[:Tn]
    if kind == "bf16_d1024":
        got = got.float()
    got = got.cpu().numpy()
    want = SL.gather(x, gi)
    np.testing.assert_array_equal(got, want)
    assert not out[Tn:].any().item()


def test_sl_then_layer_forward():
    """The product path (sampler, row gathers, one layer forward on the sampled
    batch) against the oracle path (oracle sampler, then the fp64 layer) on a
    fp32 workload with targets: max |err| <= 1e-4 rms."""
    from oracle import hstu_ref as R
    from hstu_sequential_transducer_b200 import stack as S
    rng = np.random.default_rng(17)
    lengths = rng.integers(50, 400, size=12)
    nt = np.array([int(rng.integers(0, 9)) for _ in lengths], np.int32)
    w = W.custom(lengths, d=64, H=2, N=400.0, dtype="f32", layers=1, seed=23, num_targets=nt)
    dw = S.DeviceWorkload.from_workload(w)
    sl = S.StochasticLength(dw, alpha=1.6, max_len=400)
    L = SL.subsequence_length(400, 1.6)
    assert sl.sub_len == L == 120
    keep, keys = W.sl_draws(29, w.B, w.T)
    sl.run(torch.from_numpy(keep.view(np.int32)).to(DEV),
           torch.from_numpy(keys.view(np.int32)).to(DEV))
    sb = sl.batch()
    y = H.fwd(sb.cfg, sb.layers[0], sb.x, sb.offsets, sb.timestamps, sb.num_targets)
    torch.cuda.synchronize()

    new_offs, gi = SL.sample(w.seq_offsets, nt, L, keep, keys)
    np.testing.assert_array_equal(sb.offsets.cpu().numpy(), new_offs)
    p = w.params[0]
    lp = R.LayerParams(p.W1, p.W2, p.rab_pos, p.rab_time, p.b1, p.b2, p.gamma, p.beta)
    cfg = R.LayerConfig(w.num_heads, w.norm_N, w.num_pos_buckets, w.num_time_buckets, w.ln_eps)
    want, _ = R.layer_forward(SL.gather(w.x, gi), new_offs, SL.gather(w.timestamps, gi), nt,
                              lp, cfg)
    got = y.double().cpu().numpy()
    rms = np.sqrt(np.mean(want ** 2))
    assert np.max(np.abs(got - want)) <= 1e-4 * rms


def test_sl_then_train_step():
    """A training step (fwd + bwd, 2 fp32 layers) on a sampled batch against
    the oracle's forward and backward on the oracle-sampled batch: Y, dX and
    dW1 within 3e-4 rms, max-abs (three times the fp32 layer bound, for
    values that went through the backward of two layers)."""
    from oracle import hstu_ref as R
    from hstu_sequential_transducer_b200 import stack as S
    rng = np.random.default_rng(31)
    lengths = rng.integers(60, 300, size=6)
    w = W.custom(lengths, d=64, H=2, N=300.0, dtype="f32", layers=2, seed=37, backward=True)
    dw = S.DeviceWorkload.from_workload(w)
    sl = S.StochasticLength(dw, alpha=1.6, max_len=300)
    keep, keys = W.sl_draws(41, w.B, w.T)
    sl.run(torch.from_numpy(keep.view(np.int32)).to(DEV),
           torch.from_numpy(keys.view(np.int32)).to(DEV))
    batch = sl.batch()
    new_offs, gi = SL.sample(w.seq_offsets, None, sl.sub_len, keep, keys)
    dy = w.dy[gi]
    step = S.TrainStep(batch)
    step.zero_grads()
    dx = step.run(torch.from_numpy(dy).to(DEV))
    torch.cuda.synchronize()
    plist = [R.LayerParams(p.W1, p.W2, p.rab_pos, p.rab_time, p.b1, p.b2, p.gamma, p.beta)
             for p in w.params]
    cfg = R.LayerConfig(w.num_heads, w.norm_N, w.num_pos_buckets, w.num_time_buckets, w.ln_eps)
    y, rdx, rgr = R.stack_forward_backward(SL.gather(w.x, gi), new_offs, SL.gather(w.timestamps, gi),
                                           None, plist, cfg, dy)
    for got, ref in ((step.y, y), (dx, rdx), (step.grads[0].dW1, rgr[0].dW1)):
        got = got.double().cpu().numpy()
        assert np.max(np.abs(got - ref)) <= 1e-4 * np.sqrt(np.mean(ref ** 2)) * 3


def test_gather_rows_skips_out_of_range_indices():
    """Indices outside [0, src_rows) leave their output rows unwritten (the
    documented behaviour of hstu_gather_rows); the row count comes from the
    device and caps at max_rows."""
    src = torch.arange(40 * 12, dtype=torch.float32, device=DEV).reshape(40, 12)
    idx = torch.tensor([3, -1, 39, 40, 7, 1 << 40, 0, 5], dtype=torch.int64, device=DEV)
    count = torch.tensor([7], dtype=torch.int64, device=DEV)      # the last index is not used
    out = torch.full((8, 12), -5.0, dtype=torch.float32, device=DEV)
    H.gather_rows(src, idx, count, out)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    s = src.cpu().numpy()
    for r, i in enumerate([3, -1, 39, 40, 7, 1 << 40, 0]):
        if 0 <= i < 40:
            np.testing.assert_array_equal(got[r], s[i])
        else:
            assert (got[r] == -5.0).all()
    assert (got[7] == -5.0).all()
