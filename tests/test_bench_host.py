"""Host-side pieces of bench.py on CPU: its algorithmic work counts against
the oracle's, and the JSON lines of the CPU-only reference arms of its extra
measurement modes (no GPU is touched)."""
import json
import os
import subprocess
import sys

import numpy as np

from oracle import hstu_ref as R
from hstu_sequential_transducer_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

KEYS = {"metric", "value", "unit", "impl", "n_gpus", "steps", "warmup", "higher_is_better",
        "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"}


def test_work_counts_match_the_oracle():
    rng = np.random.default_rng(3)
    for nt in (None, [3, 0, 7, 1]):
        lengths = rng.integers(1, 300, size=4)
        if nt is not None:
            nt = [min(m, int(n)) for m, n in zip(nt, lengths)]
        w = W.custom(lengths, d=64, H=2, layers=3, num_targets=nt)
        f, pairs = bench.workload_flops(w, backward=False)
        assert f == 3 * R.layer_flops_fwd(lengths, nt, 64)
        fb, _ = bench.workload_flops(w, backward=True)
        assert fb == 3 * f
        # the pair count is the number of allowed (i, j) of the mask
        assert pairs == sum(int(R.allowed_mask(int(n), 0 if nt is None else int(m)).sum())
                            for n, m in zip(lengths, nt or [0] * 4))


def run_line(args):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args,
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    return json.loads(lines[0])


def test_sampler_reference_line():
    d = run_line(["--sampler", "--impl", "reference", "--batch", "2", "--steps", "1",
                  "--warmup", "0"])
    assert KEYS <= set(d) and d["impl"] == "reference" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"


def test_attention_8k_reference_line():
    d = run_line(["--attention-8k", "--impl", "reference", "--cpu-budget", "0.1"])
    assert KEYS <= set(d) and d["impl"] == "reference" and d["unit"] == "TFLOP/s"
    assert d["value"] > 0


def test_softmax_8k_reference_line():
    d = run_line(["--softmax-8k", "--impl", "reference", "--cpu-budget", "0.1"])
    assert KEYS <= set(d) and d["impl"] == "reference" and d["unit"] == "TFLOP/s"
    assert d["value"] > 0 and "softmax" in d["metric"]


def test_split_shards_partition_one_batch():
    """--split: every rank draws the same batch and keeps its LPT share; the
    shares partition the batch's sequences and tokens."""
    w = W.custom([9, 3, 12, 5, 7, 2, 30], d=16, H=2, layers=1, seed=4)
    for world in (1, 2, 3):
        parts = [bench.split_shard(w, r, world) for r in range(world)]
        assert sum(p.T for p in parts) == w.T
        assert sum(p.B for p in parts) == w.B
        rows = np.concatenate([p.x for p in parts])
        assert sorted(map(tuple, rows.round(6))) == sorted(map(tuple, w.x.round(6)))


def test_training_reference_line():
    """The default reference arm (the oracle on a bounded sample) prints one
    JSON line with the base contract's keys."""
    d = run_line(["--impl", "reference", "--batch", "2", "--layers", "1", "--steps", "1",
                  "--warmup", "0"])
    assert KEYS <= set(d) and d["impl"] == "reference" and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0
