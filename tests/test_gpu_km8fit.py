"""GPU int8km palette fit (qmv_encode_int8km) against the oracle's k-means:
the 256-entry fp16 palettes (bits) and the 8-bit indices bit-exact."""
import numpy as np
import pytest
import torch

import oracle as orc
from weight_only_quantized_qmv_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from weight_only_quantized_qmv_b200 import _build
    _build.build()
    import weight_only_quantized_qmv_b200 as q
    q.lib()
    assert q.status_fetch() == 0
    return q


def fit_both(q, Wn, iters):
    idx, lut = q.encode_int8km(torch.from_numpy(Wn).cuda(), iters=iters)
    flags = q.status_fetch()
    lut_o, idx_o, fl_o = orc.kmeans_int8km(Wn, iters=iters)
    return (lut.cpu().numpy().view(np.uint16), idx.cpu().numpy(), flags), (lut_o.view(np.uint16), idx_o, fl_o)


@pytest.mark.parametrize("N,K,iters", [(64, 512, 0), (64, 512, 1), (64, 512, 3), (70, 96, 3), (33, 544, 2),
                                       (32, 2048, 2), (5, 2080, 3), (1, 96, 3), (33, 32, 2), (32, 16384, 1)])
def test_encode_int8km_bit_exact(q, N, K, iters):
    """Shapes: groups whose keys fit one shared-memory sort chunk and ones that
    take the global strides (up to 32 x 16384 = 2^19 keys, the largest
    group), a single row, K = 32 with a one-row last group."""
    g = synth.generator(N * 13 + K + iters, "cpu")
    W, _ = synth.weights(N, K, g, n_outlier_cols=2)
    (lut, idx, fl), (lut_o, idx_o, fl_o) = fit_both(q, W.numpy(), iters)
    assert fl == 0 and fl_o == 0
    assert np.array_equal(lut, lut_o)
    assert np.array_equal(idx, idx_o)


def test_encode_int8km_duplicates_zeros_and_ranges(q):
    """Groups with few distinct values (duplicate centres keep their value and
    lose every tie), both signed zeros, and values spanning many binades."""
    rng = np.random.default_rng(3)
    N, K = 96, 256
    W = np.empty((N, K), np.float32)
    W[:32] = rng.choice(np.array([-0.5, -0.0, 0.0, 0.25, 0.25, 1.0], np.float32), size=(32, K))
    W[32:64] = (rng.standard_normal((32, K)) * np.exp2(rng.integers(-30, 4, size=(32, K)))).astype(np.float32)
    W[64:] = np.float32(0.125)
    W[64:, ::7] = -0.0
    (lut, idx, fl), (lut_o, idx_o, fl_o) = fit_both(q, W, 4)
    assert np.array_equal(lut, lut_o)
    assert np.array_equal(idx, idx_o)


def test_encode_int8km_nonfinite_group(q):
    g = synth.generator(8, "cpu")
    W, _ = synth.weights(96, 128, g)
    Wn = W.numpy().copy()
    Wn[40, 17] = np.inf
    (lut, idx, fl), (lut_o, idx_o, fl_o) = fit_both(q, Wn, 2)
    assert fl == q.FLAG_NONFINITE and fl_o == q.FLAG_NONFINITE
    assert np.array_equal(lut, lut_o) and np.all(lut[1] == 0)
    assert np.array_equal(idx, idx_o) and np.all(idx[32:64] == 0)


def test_encode_int8km_then_matvec(q):
    """The GPU fit feeds the int8km matvec; the result matches the oracle's
    matvec on the oracle's fit of the same weights (same tables)."""
    N, K, B = 256, 1024, 3
    g = synth.generator(21, "cpu")
    W, _ = synth.weights(N, K, g)
    x = synth.activations(B, K, g)
    idx, lut = q.encode_int8km(W.cuda(), iters=3)
    y = q.matvec_int8km(idx, lut, x.cuda()).cpu().numpy()
    lut_o, idx_o, _ = orc.kmeans_int8km(W.numpy(), iters=3)
    assert np.array_equal(lut.cpu().numpy().view(np.uint16), lut_o.view(np.uint16))
    r = orc.matvec(orc.FMT_INT8KM, idx_o, lut_o, x.numpy(), N, K)
    err = np.abs(y - r).max(axis=1) / np.abs(r).max(axis=1)
    assert err.max() < 1e-3
    assert q.status_fetch() == 0


def test_encode_int8km_head_groups_sampled(q):
    """The 130560 x 2048 int8 head shape fitted on the GPU (20 Lloyd steps,
    4080 groups); sampled groups compared with the oracle bit for bit."""
    N, K = 130560, 2048
    g = synth.generator(5, "cuda")
    W, _ = synth.weights(N, K, g)
    idx, lut = q.encode_int8km(W, iters=20)
    assert q.status_fetch() == 0
    for grp in (0, 1777, 4079):
        Wg = W[grp * 32:(grp + 1) * 32].cpu().numpy()
        lut_o, idx_o, _ = orc.kmeans_int8km(Wg, iters=20)
        assert np.array_equal(lut[grp].cpu().numpy().view(np.uint16), lut_o[0].view(np.uint16)), grp
        assert np.array_equal(idx[grp * 32:(grp + 1) * 32].cpu().numpy(), idx_o), grp
