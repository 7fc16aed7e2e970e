"""bench.py's host logic on the CPU: the algorithmic bytes behind `value` and
`roofline.achieved` are the bytes of the arrays the oracle's encoders
produce for the format (codes, scales / palettes / zero points, the outlier
column list), plus the activations in fp16 and the outputs in fp32 -- for
every format, a ragged row count and two batch sizes."""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
import oracle  # noqa: E402

N, K = 70, 576  # 70 rows: three int8km groups, the last one ragged; K - 64 outlier columns = 512


def _weights():
    rng = np.random.default_rng(3)
    return (rng.standard_normal((N, K)) * 0.02).astype(np.float32)


def _encoded_bytes(fmt):
    W = _weights()
    if fmt == "fp4":
        arrays = oracle.encode_fp4(W)[:2]
    elif fmt == "int4":
        arrays = oracle.encode_int4(W)[:2]
    elif fmt == "int8":
        arrays = oracle.encode_int8(W)[:2]
    elif fmt == "int4aff":
        arrays = oracle.encode_int4aff(W)[:2]
    elif fmt == "int4km":
        arrays = oracle.kmeans_int4km(W, iters=1)[:2]
    elif fmt == "int8km":
        arrays = oracle.kmeans_int8km(W, iters=1)[:2]
    else:
        arrays = oracle.encode_int4km_o8(W, bench.O8_COLS, iters=1)[:5]
    return sum(a.nbytes for a in arrays)


@pytest.mark.parametrize("fmt", ["fp4", "int4", "int8", "int4aff", "int4km", "int8km", "int4km_o8"])
@pytest.mark.parametrize("B", [1, 4])
def test_algorithmic_bytes_are_the_encoded_bytes(fmt, B):
    want = _encoded_bytes(fmt) + B * K * 2 + B * N * 4
    assert bench.algorithmic_bytes(fmt, N, K, B) == want


def test_whole_job_rate_counts_every_rank():
    # 2 ranks x 1 GB in 0.5 ms (the slowest rank's time) = 4000 GB/s
    assert bench.whole_job_gbs(1_000_000_000, 2, 0.5) == pytest.approx(4000.0)


def test_spread_percentiles():
    # 1..25: median 13, nearest-rank p10 / p90 at positions 2.4 -> 2 and 21.6 -> 22 (0-based)
    st = bench.spread([float(v) for v in range(25, 0, -1)])
    assert st["median"] == 13.0 and st["p10"] == 3.0 and st["p90"] == 23.0
    assert st["mean"] == 13.0 and st["reps"] == 25


def test_cpu_baseline_reports_oracle_encode_and_thread_counts():
    """The CPU leg times the oracle's encoders and its matvec on all cores
    and on one thread, on a bounded row sample, and says so."""
    import torch
    from weight_only_quantized_qmv_b200 import synth
    g = synth.generator(0, "cpu")
    W, _ = synth.weights(64, bench.K_HEAD, g)
    x = synth.activations(1, bench.K_HEAD, g)
    r = bench.cpu_baseline(W, x, seconds=0.2, rows=64)
    assert r["kind"] == "oracle" and r["unit"] == "GB/s"
    assert r["value"] > 0 and r["single_thread_gbs"] > 0
    assert r["cores"] == oracle.num_threads() >= 1
    assert set(r["encode_ms"]) == {"fp4", "int4", "int8"} and all(v > 0 for v in r["encode_ms"].values())
    assert "64 of 248320 rows" in r["sample"] and "on one" in r["sample"]
    assert isinstance(W, torch.Tensor)
