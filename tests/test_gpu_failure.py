"""Failure detection on the GPU, in forms that neither trap nor hang it.

Every mbarrier wait in the library's kernels is bounded in time; when one
runs out the kernel sets HSTU_DEVICE_TIMEOUT in the device status word and
returns.  The diagnostic entry point waits on a barrier that nothing arrives
on, with a limit of microseconds, so its wait can only end by running out:
the call returns, the status word reports the timeout, and the library's next
ordinary call is unaffected.
"""
import numpy as np
import pytest
import torch

from oracle import hstu_ref as R
from hstu_sequential_transducer_b200 import build
from hstu_sequential_transducer_b200 import hstu as H
from hstu_sequential_transducer_b200 import stack as S
from hstu_sequential_transducer_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    H.lib()


def test_bounded_wait_runs_out_and_reports():
    H.device_status(clear=True)
    res = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    H.selftest_wait_timeout(5_000, res)          # 5 microseconds
    torch.cuda.synchronize()
    assert int(res.item()) == 0                  # the wait gave up ...
    st = H.device_status(clear=True)
    assert st & H.DEVICE_TIMEOUT                 # ... and said so
    assert H.device_status(clear=True) == 0      # cleared


def test_limit_outside_range_is_refused_without_launch():
    n0 = H.launch_count()
    for bad in (0, 100_000_001):
        with pytest.raises(H.HSTUError) as ei:
            H.selftest_wait_timeout(bad)
        assert ei.value.status == 1
    assert H.launch_count() == n0


def test_next_call_after_a_timeout_still_matches_the_oracle():
    H.selftest_wait_timeout(5_000)
    torch.cuda.synchronize()
    assert H.device_status(clear=True) & H.DEVICE_TIMEOUT
    w = W.custom([200, 7, 130], d=256, H=2, dtype="bf16", N=200.0, num_targets=[20, 0, 0],
                 seed=17)
    dw = S.DeviceWorkload.from_workload(w)
    y = S.forward_stack(dw)
    torch.cuda.synchronize()
    assert H.device_status() == 0
    ref = R.stack_forward(w.x, w.seq_offsets, w.timestamps, w.num_targets,
                          [R.LayerParams(p.W1, p.W2, p.rab_pos, p.rab_time, p.b1, p.b2, p.gamma,
                                         p.beta) for p in w.params],
                          R.LayerConfig(w.num_heads, w.norm_N, w.num_pos_buckets,
                                        w.num_time_buckets, w.ln_eps))
    got = y.detach().float().cpu().numpy().astype(np.float64)
    rms = np.sqrt(np.mean(ref ** 2))
    assert np.max(np.abs(got - ref)) <= 2e-2 * rms
