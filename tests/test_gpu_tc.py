"""GPU parity of the fp4 tensor-core (tcgen05) matvec against the CPU oracle.

The kernel is switched on with set_fp4_tensor_cores(True) and serves dense
fp4 matvecs at 2..16 activation columns with K a multiple of 512 up to 4608.  Bar as in
test_gpu_parity: max relative error 1e-3 per activation row against the fp64
oracle; one-hot columns bit-exact (every scaled E2M1 value of a row within
2^36 of its largest block is exact in the kernel's fp16 operands).
"""
import numpy as np
import pytest
import torch

import oracle as orc
from weight_only_quantized_qmv_b200 import synth

pytestmark = pytest.mark.gpu

TOL = 1e-3


@pytest.fixture(scope="module")
def q():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from weight_only_quantized_qmv_b200 import _build
    _build.build()
    import weight_only_quantized_qmv_b200 as q
    q.lib()
    assert q.status_fetch() == 0
    q.set_fp4_tensor_cores(True)
    yield q
    q.set_fp4_tensor_cores(False)


def rel_err(y, r):
    y = np.asarray(y, np.float64).reshape(r.shape)
    num = np.abs(y - r).max(axis=-1)
    den = np.abs(r).max(axis=-1)
    den = np.where(den == 0, 1.0, den)
    return float((num / den).max())


def fp4_inputs(N, K, B, seed):
    g = synth.generator(seed, "cpu")
    W, _ = synth.weights(N, K, g, n_outlier_cols=2)
    x = synth.activations(B, K, g)
    c, s, _ = orc.encode_fp4(W.numpy())
    return c, s, x.numpy()


def run(q, c, s, x):
    return q.matvec_fp4(torch.from_numpy(c).cuda(), torch.from_numpy(s).cuda(), torch.from_numpy(x).cuda())


@pytest.mark.parametrize("N,K", [(1, 512), (1000, 512), (600, 2048), (130, 4096), (257, 4608), (129, 1024)])
@pytest.mark.parametrize("B", [2, 4, 9, 16])
def test_tc_matvec_parity(q, N, K, B):
    c, s, x = fp4_inputs(N, K, B, seed=N + K + B)
    y = run(q, c, s, x).cpu().numpy()
    r = orc.matvec(orc.FMT_FP4, c, s, x, N, K)
    e = rel_err(y, r)
    assert e < TOL, e
    assert q.status_fetch() == 0


def test_tc_many_tiles_per_cta(q):
    """Three and more 128-row tiles per CTA on a full grid (the scale, A and
    accumulator buffers change parity across tiles), a ragged last tile."""
    N, K, B = 148 * 128 * 3 + 77, 512, 4
    c, s, x = fp4_inputs(N, K, B, seed=3)
    y = run(q, c, s, x).cpu().numpy()
    r = orc.matvec(orc.FMT_FP4, c, s, x, N, K)
    assert rel_err(y, r) < TOL
    assert q.status_fetch() == 0


def test_tc_head_sampled_rows(q):
    """The 248320 x 2048 head at batch 16 (the verify-batch launch the bench
    times), checked on sampled rows: the first and last tiles and random rows."""
    N, K, B = 248320, 2048, 16
    g = synth.generator(41, "cuda")
    W, _ = synth.weights(N, K, g)
    c, s = q.encode_fp4(W)
    del W
    x = synth.activations(B, K, g)
    y = q.matvec_fp4(c, s, x).cpu().numpy()
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([np.arange(130), np.arange(N - 130, N), rng.integers(0, N, 512)]))
    ri = torch.from_numpy(rows).cuda()
    c_r, s_r = c[ri].cpu().numpy(), s[ri].cpu().numpy()
    r = orc.matvec(orc.FMT_FP4, c_r, s_r, x.cpu().numpy(), len(rows), K)
    assert rel_err(y[:, rows], r) < TOL
    assert q.status_fetch() == 0


def test_tc_one_hot_columns_bit_exact(q):
    """x = e_k (16 columns) returns column k of the dequantized W exactly:
    pins the nibble order, the swizzled code reads, the block-scale indexing
    and the A / B operand layouts."""
    N, K = 300, 2048
    c, s, _ = fp4_inputs(N, K, 1, seed=5)
    D = orc.dequant(orc.FMT_FP4, c, s, N, K)
    ks = [0, 1, 2, 7, 8, 15, 16, 31, 32, 63, 64, 127, 128, 255, 256, K - 1]
    for start in (0, 600, 1500):
        kk = [min(K - 1, k + start) for k in ks]
        x = np.zeros((16, K), np.float16)
        x[np.arange(16), kk] = 1.0
        y = run(q, c, s, x).cpu().numpy()
        for i, k in enumerate(kk):
            assert np.array_equal(y[i], D[:, k]), k


def test_tc_wide_scale_range_rows(q):
    """Rows whose block scales span more than 2^36: blocks further below the
    row's largest are dropped; the error stays below fp32 resolution of the
    row's result.  Random codes, scales 60..200."""
    N, K, B = 384, 2048, 8
    g = synth.generator(17, "cpu")
    c = synth.int_codes(N, K, 4, g).numpy()
    s = torch.randint(60, 201, (N, K // 32), generator=g, dtype=torch.int32).to(torch.uint8).numpy()
    x = synth.activations(B, K, g).numpy()
    y = run(q, c, s, x).cpu().numpy()
    r = orc.matvec(orc.FMT_FP4, c, s, x, N, K)
    assert rel_err(y, r) < 1e-5
    # one-hot: columns of blocks within 2^36 of the row's largest are exact
    D = orc.dequant(orc.FMT_FP4, c, s, N, K)
    kk = np.arange(0, K, K // 16)
    xo = np.zeros((16, K), np.float16)
    xo[np.arange(16), kk] = 1.0
    yo = run(q, c, s, xo).cpu().numpy()
    emax = s.astype(np.int32).max(axis=1)
    for i, k in enumerate(kk):
        keep = s[:, k // 32].astype(np.int32) >= emax - 36
        assert np.array_equal(yo[i][keep], D[keep, k]), k
        assert np.all(yo[i][~keep] == 0.0), k


def test_tc_refused_shapes_use_mma_sync(q):
    """K not a multiple of 512 or above 4608, and batch 1, keep the mma.sync
    kernel; results still match the oracle."""
    for N, K, B in ((200, 544, 16), (100, 2080, 4), (300, 2048, 1), (64, 7680, 16)):
        c, s, x = fp4_inputs(N, K, B, seed=B + K)
        y = run(q, c, s, x).cpu().numpy()
        r = orc.matvec(orc.FMT_FP4, c, s, x, N, K)
        assert rel_err(y, r) < TOL


def test_tc_deterministic_and_matches_mma_sync(q):
    N, K, B = 5000, 2048, 16
    c, s, x = fp4_inputs(N, K, B, seed=9)
    y1 = run(q, c, s, x).cpu().numpy()
    y2 = run(q, c, s, x).cpu().numpy()
    assert np.array_equal(y1, y2)
    q.set_fp4_tensor_cores(False)
    try:
        y3 = run(q, c, s, x).cpu().numpy()
    finally:
        q.set_fp4_tensor_cores(True)
    r = orc.matvec(orc.FMT_FP4, c, s, x, N, K)
    assert rel_err(y1, r) < TOL and rel_err(y3, r) < TOL
    assert q.status_fetch() == 0


def test_tc_output_guard_bands(q):
    """Writes stay inside y: canaries around the output survive."""
    N, K, B = 333, 1024, 5
    c, s, x = fp4_inputs(N, K, B, seed=13)
    buf = torch.full((B * N + 2048,), 7.25, dtype=torch.float32, device="cuda")
    out = buf[1024:1024 + B * N].view(B, N)
    q.matvec_fp4(torch.from_numpy(c).cuda(), torch.from_numpy(s).cuda(), torch.from_numpy(x).cuda(), out=out)
    b = buf.cpu().numpy()
    assert np.all(b[:1024] == 7.25) and np.all(b[1024 + B * N:] == 7.25)
    r = orc.matvec(orc.FMT_FP4, c, s, x, N, K)
    assert rel_err(out.cpu().numpy(), r) < TOL
