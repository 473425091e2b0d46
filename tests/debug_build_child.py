"""Run by tests/test_gpu_debug_build.py in a process of its own with
HSTU_DEBUG_BUILD=1, so that the index-checking debug build of the library
(libhstu_debug.so) is the one loaded.  Prints "debug build ok" on success.

1. Valid inputs: the attention forward and backward (tensor-core kernels, head
   widths 64 and 128, M-FALCON targets) match the fp64 oracle and no check
   fires.
2. Query rows past the declared row count: the call declares T_small rows of
   the query tensors while the offsets reach T; every buffer holds T rows, so
   nothing is read or written outside an allocation, but the kernels' checks
   see row indices past T_small and report HSTU_DEVICE_BOUNDS.
"""
import ctypes
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from hstu_sequential_transducer_b200 import build  # noqa: E402
from hstu_sequential_transducer_b200 import hstu as H  # noqa: E402
from hstu_sequential_transducer_b200 import stack as S  # noqa: E402
from hstu_sequential_transducer_b200 import workloads as W  # noqa: E402
from oracle import hstu_ref as R  # noqa: E402

TOL = 2e-2


def check(got, ref, what):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape and np.isfinite(got).all(), what
    rms = np.sqrt(np.mean(ref ** 2))
    e = float(np.max(np.abs(got - ref) / (rms + np.abs(ref) + 1e-30)))
    assert e <= TOL, f"{what}: {e:.3e}"


def dev(a, dt):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to("cuda", dt)


def valid_inputs(dh):
    nh = 2
    d = nh * dh
    w = W.custom([300, 1, 0, 129, 64, 257], d=d, H=nh, dtype="bf16", N=300.0,
                 num_targets=[40, 1, 0, 129, 0, 100], mean_gap=3000.0, seed=5 + dh)
    rng = np.random.default_rng(dh)
    pre = W.round_to_bf16(rng.normal(0, 1, size=(w.T, 4 * d)).astype(np.float32))
    g = W.round_to_bf16(R.silu(pre.astype(np.float64)).astype(np.float32))
    dout = W.round_to_bf16(rng.normal(0, 1, size=(w.T, d)).astype(np.float32))
    dw = S.DeviceWorkload.from_workload(w)
    lw = dw.layers[0]
    p = w.params[0]
    cfg = R.LayerConfig(nh, w.norm_N, w.num_pos_buckets, w.num_time_buckets, w.ln_eps)
    o = torch.full((w.T, d), float("nan"), dtype=torch.float32, device="cuda")
    H.attention_fwd(dw.cfg, lw.rab_pos, lw.rab_time, dev(g, torch.bfloat16), dw.offsets,
                    dw.timestamps, dw.num_targets, o)
    dpre = torch.full((w.T, 4 * d), float("nan"), dtype=torch.bfloat16, device="cuda")
    drp, drt = torch.zeros_like(lw.rab_pos), torch.zeros_like(lw.rab_time)
    H.attention_bwd(dw.cfg, lw.rab_pos, lw.rab_time, dev(g, torch.bfloat16),
                    dev(pre, torch.bfloat16), dev(dout, torch.bfloat16), dw.offsets,
                    dw.timestamps, dw.num_targets, dpre, drp, drt)
    torch.cuda.synchronize()
    assert H.device_status() == 0, "a check fired on valid inputs"
    ref = R.attention_forward(g, w.seq_offsets, w.timestamps, w.num_targets, p.rab_pos,
                              p.rab_time, cfg)
    check(o.cpu().numpy(), ref, f"O dh={dh}")
    dg, _, _ = R.attention_backward(g, dout, w.seq_offsets, w.timestamps, w.num_targets,
                                    p.rab_pos, p.rab_time, cfg)
    sg = R.silu_grad(pre.astype(np.float64))
    got = dpre.float().cpu().numpy()
    for name, sl in (("dPre_V", slice(d, 2 * d)), ("dPre_Q", slice(2 * d, 3 * d)),
                     ("dPre_K", slice(3 * d, 4 * d))):
        check(got[:, sl], dg[:, sl] * sg[:, sl], f"{name} dh={dh}")


def rows_past_declared_count():
    nh, dh = 2, 128
    d = nh * dh
    w = W.custom([300, 129, 257], d=d, H=nh, dtype="bf16", N=300.0, seed=9)
    dw = S.DeviceWorkload.from_workload(w)
    lw = dw.layers[0]
    rng = np.random.default_rng(9)
    g = dev(W.round_to_bf16(rng.normal(0, 0.5, size=(w.T, 4 * d)).astype(np.float32)),
            torch.bfloat16)
    o = torch.zeros(w.T, d, dtype=torch.float32, device="cuda")
    T_small = 300 + 129                   # the last sequence's rows lie past it
    ws = torch.zeros(H.attention_workspace_size(dw.cfg, w.B, w.T), dtype=torch.uint8,
                     device="cuda")      # sized for the rows the offsets reach
    st = H.lib().hstu_attention_fwd(ctypes.byref(dw.cfg), H.ptr(lw.rab_pos),
                                    H.ptr(lw.rab_time), H.ptr(g), H.ptr(dw.offsets), w.B,
                                    T_small, H.ptr(dw.timestamps), None, H.ptr(o), H.ptr(ws),
                                    ws.numel(), H.stream_ptr())
    assert st == 0, st
    torch.cuda.synchronize()
    word = H.device_status()
    assert word & H.DEVICE_BOUNDS, f"status {word:#x}: no bounds report"
    assert H.device_status() == 0          # the read above cleared it


def main():
    assert H.DEBUG_BUILD and H.LIB_PATH.endswith("libhstu_debug.so")
    build.build(debug=True)
    H.lib()
    H.device_status()
    for dh in (64, 128):
        valid_inputs(dh)
    rows_past_declared_count()
    print("debug build ok")


if __name__ == "__main__":
    main()
