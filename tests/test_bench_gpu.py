"""bench.py's end-to-end leg on the GPU at a small size: the activations go
in from pinned host memory, the matvecs run, each output comes back to
pinned host memory on a copy stream ordered after its matvec by an event,
and the host copies equal the device results of the same step bit for bit
(the leg raises otherwise)."""
import os
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from weight_only_quantized_qmv_b200 import synth  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from weight_only_quantized_qmv_b200 import _build
    _build.build()
    import weight_only_quantized_qmv_b200 as q
    q.lib()
    return q


def test_e2e_leg_orders_copies_and_checks_outputs(q, monkeypatch):
    N = 4096 + 48
    monkeypatch.setattr(bench, "N_HEAD", N)
    dev = torch.device("cuda", 0)
    g = synth.generator(5, dev)
    W, _ = synth.weights(N, bench.K_HEAD, g, n_outlier_cols=2)
    x = synth.activations(1, bench.K_HEAD, g)
    ops = {"fp4": q.encode_fp4(W), "int8": q.encode_int8(W)}
    fmt_id = {"fp4": q.FMT_FP4, "int8": q.FMT_INT8}
    ref = {f: q.matvec(fmt_id[f], *ops[f], x).cpu() for f in ops}
    stream = torch.cuda.Stream(device=dev)
    r = bench.measure_e2e(q, ops, fmt_id, x, dev, stream, tuple(ops), ref, steps=20)
    assert r["checked"] is True
    assert r["h2d_bytes_per_step"] == bench.K_HEAD * 2
    assert r["d2h_bytes_per_step"] == 2 * N * 4
    assert r["ms_per_step_wall"] >= r["ms_per_step_device"] > 0
    # a wrong reference is caught
    bad = {f: v.clone() for f, v in ref.items()}
    bad["int8"][0, 7] += 1.0
    with pytest.raises(RuntimeError):
        bench.measure_e2e(q, ops, fmt_id, x, dev, stream, tuple(ops), bad, steps=20)
    assert q.status_fetch() == 0
