"""GPU parity of libqmv (through its C ABI binding) against the CPU oracle.

Bar: packed codes, scales and dequantized weights bit-exact; matvec outputs
within max relative error 1e-3 of the fp64 oracle, read per activation row as
||y_b - r_b||_inf / ||r_b||_inf (a per-element ratio is ill-conditioned where
r is near zero).  The expected fp32-accumulation error is ~1e-6, so the
tests also report the observed figure in their assertion messages.
"""
import numpy as np
import pytest
import torch

import oracle as orc
from weight_only_quantized_qmv_b200 import synth

pytestmark = pytest.mark.gpu

TOL = 1e-3
FMTS = ("fp4", "int4", "int4km", "int8", "int4aff", "int8km")
KM8_ITERS = 3  # Lloyd steps of the int8km test fits (256 centres per 32 rows: the fit dominates test time)


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


def rel_err(y, r):
    """max over activation rows of ||y_b - r_b||_inf / ||r_b||_inf."""
    y = np.asarray(y, np.float64).reshape(r.shape)
    num = np.abs(y - r).max(axis=-1)
    den = np.abs(r).max(axis=-1)
    den = np.where(den == 0, 1.0, den)
    return float((num / den).max())


def gen_w(N, K, seed=0, n_out=0, device="cuda"):
    g = synth.generator(seed, device)
    W, _ = synth.weights(N, K, g, n_outlier_cols=n_out)
    return W, g


def encode_gpu(q, fmt, W, W_np=None):
    """GPU encode (fp4/int4/int8) or oracle fit (int4km: no GPU encoder)."""
    if fmt == "fp4":
        return q.encode_fp4(W)
    if fmt == "int4":
        return q.encode_int4(W)
    if fmt == "int8":
        return q.encode_int8(W)
    if fmt == "int4aff":
        return q.encode_int4aff(W)
    lut, idx, _ = orc.kmeans_int4km(W.cpu().numpy() if W_np is None else W_np)
    return torch.from_numpy(idx).cuda(), torch.from_numpy(lut).cuda()


def encode_orc(fmt, Wn):
    if fmt == "fp4":
        c, s, f = orc.encode_fp4(Wn)
    elif fmt == "int4":
        c, s, f = orc.encode_int4(Wn)
    elif fmt == "int8":
        c, s, f = orc.encode_int8(Wn)
    elif fmt == "int4aff":
        c, s, f = orc.encode_int4aff(Wn)
    elif fmt == "int8km":
        s, c, f = orc.kmeans_int8km(Wn, iters=KM8_ITERS)
    else:
        s, c, f = orc.kmeans_int4km(Wn)
    return c, s, f


FID = {"fp4": orc.FMT_FP4, "int4": orc.FMT_INT4, "int4km": orc.FMT_INT4KM, "int8": orc.FMT_INT8,
       "int4aff": orc.FMT_INT4AFF, "int8km": orc.FMT_INT8KM}


def np_bits(t):
    a = t.cpu().numpy()
    return a.view(np.uint8) if a.dtype in (np.int8, np.uint8) else a.view(np.uint16)


# ---------------------------------------------------------------------------
# encoders
# ---------------------------------------------------------------------------

def test_e2m1_hardware_conversion_matches_oracle_table(q):
    """Blocks whose max is 4 or 7.99 have scale 2^0, so each code is the
    hardware E2M1 conversion of the weight itself: it must equal the
    oracle's nearest-even table at every tie and threshold."""
    grid = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    pts = [(a + b) / 2 for a, b in zip(grid, grid[1:])] + grid + [7.0]
    vals = []
    for c in pts:
        v = np.float32(c)
        vals.append(v)
        lo = hi = v
        for _ in range(3):
            lo = np.nextafter(lo, np.float32(-1), dtype=np.float32)
            hi = np.nextafter(hi, np.float32(9), dtype=np.float32)
            vals += [lo, hi]
    vals = np.array([v for v in vals if 0 <= v < 7.99], np.float32)
    vals = np.concatenate([vals, -vals, np.array([-0.0, 1e-30, -1e-30], np.float32)])
    n = (len(vals) + 30) // 31
    W = np.zeros((n, 32), np.float32)
    W[:, 0] = np.where(np.arange(n) % 2 == 0, 4.0, 7.99)
    W[:, 1:].flat[:len(vals)] = vals
    c_gpu, s_gpu = q.encode_fp4(torch.from_numpy(W).cuda())
    c_orc, s_orc, _ = orc.encode_fp4(W)
    assert np.array_equal(s_gpu.cpu().numpy(), s_orc)
    assert (s_orc == 127).all()
    assert np.array_equal(c_gpu.cpu().numpy(), c_orc)
    assert q.status_fetch() == 0


@pytest.mark.parametrize("fmt", ["fp4", "int4", "int8", "int4aff"])
@pytest.mark.parametrize("N,K", [(1, 32), (40, 96), (300, 544), (64, 2080), (33, 4096)])
def test_encoder_bit_exact(q, fmt, N, K):
    W, _ = gen_w(N, K, seed=N + K, n_out=max(1, K // 1000))
    W[0, :32] = 0.0  # all-zero block
    if N > 2:
        W[1, 32 % K:32 % K + 32] = 1e-30  # tiny block: scale underflow paths
        W[2, :] *= 1e4  # large row
    Wn = W.cpu().numpy()
    c_g, s_g = encode_gpu(q, fmt, W)
    c_o, s_o, f = encode_orc(fmt, Wn)
    assert f == 0
    assert np.array_equal(np_bits(c_g), c_o.view(np.uint8))
    assert np.array_equal(np_bits(s_g), s_o.view(np.uint8) if fmt in ("fp4", "int4aff") else s_o.view(np.uint16))
    assert q.status_fetch() == 0


def test_encode_int4aff_special_blocks(q):
    """Blocks of one sign (zero point at an end of the range), a constant
    block, a block whose range gives an fp16-subnormal scale, halfway cases
    of w / s, and a last odd block (its zero-point byte's high nibble stays 0)."""
    K = 96
    W = np.zeros((6, K), np.float32)
    rng = np.random.default_rng(5)
    W[0] = np.abs(rng.standard_normal(K)).astype(np.float32) * 0.02  # all >= 0: z = 0
    W[1] = -np.abs(rng.standard_normal(K)).astype(np.float32) * 0.02  # all <= 0: z = 15
    W[2] = 0.375  # constant block
    W[3] = rng.standard_normal(K).astype(np.float32) * 1e-7  # scale in the fp16 subnormal range
    W[4] = (np.arange(K) % 31 - 15).astype(np.float32) * 0.5 / 15.0  # w / s on halfway points
    W[5] = rng.standard_normal(K).astype(np.float32)
    c_g, a_g = q.encode_int4aff(torch.from_numpy(W).cuda())
    c_o, a_o, f = orc.encode_int4aff(W)
    assert f == 0 and q.status_fetch() == 0
    assert np.array_equal(c_g.cpu().numpy(), c_o)
    assert np.array_equal(a_g.cpu().numpy(), a_o)
    assert (a_o[:, -1] >> 4 == 0).all()  # K / 32 = 3 blocks: the last byte holds one zero point


def test_int4aff_unaligned_aux(q):
    """An aux plane starting at an odd byte (and one at 4 mod 8) takes the
    bytewise staging path on a shape that is otherwise copied asynchronously."""
    N, K = 70, 2048
    for B in (1, 3):
        c_o, a_o, xn = _inputs("int4aff", N, K, B, seed=19 + B)
        r = orc.matvec(orc.FMT_INT4AFF, c_o, a_o, xn, N, K)
        c, x = torch.from_numpy(c_o).cuda(), torch.from_numpy(xn).cuda()
        y0 = q.matvec_int4aff(c, torch.from_numpy(a_o).cuda(), x)
        for off in (1, 4):
            ab = torch.zeros(a_o.size + off, dtype=torch.uint8, device="cuda")
            ab[off:] = torch.from_numpy(a_o.reshape(-1)).cuda()
            y = q.matvec_int4aff(c, ab[off:].view(N, -1), x)
            assert rel_err(y.cpu().numpy(), r) < TOL
            if B == 1:
                # batch 1 leaves the block-column form for the general one: same tolerance
                assert rel_err(y.cpu().numpy(), y0.cpu().numpy().astype(np.float64)) < TOL
            else:
                assert torch.equal(y, y0)  # same form, same summation order
    assert q.status_fetch() == 0


@pytest.mark.parametrize("K", [32768, 65536])
def test_int8km_batch1_long_rows(q, K):
    """Batch 1 with long rows: at K = 32768 the batch-1 kernel's fp32
    activation row leaves room for one CTA per SM; at K = 65536 it does not
    fit at all and the general kernel (fp16 rows) takes the call.  Both match
    the oracle on stand-in tables."""
    N = 40
    c_o, s_o, xn = _inputs("int8km", N, K, 1, seed=K + 3)
    y = q.matvec_int8km(torch.from_numpy(c_o).cuda(), torch.from_numpy(s_o).cuda(),
                        torch.from_numpy(xn).cuda()).cpu().numpy()
    r = orc.matvec(FID["int8km"], c_o, s_o, xn, N, K)
    e = rel_err(y, r)
    assert e < TOL, e
    assert q.status_fetch() == 0


def test_int8km_lut_checks_and_unaligned_lut(q):
    """The binding rejects a LUT of the wrong group count; a LUT plane that
    starts 2 bytes past a 16-byte boundary gives the same outputs."""
    N, K, B = 70, 2080, 3
    c_o, s_o, xn = _inputs("int8km", N, K, B, seed=41)
    c, x = torch.from_numpy(c_o).cuda(), torch.from_numpy(xn).cuda()
    y0 = q.matvec_int8km(c, torch.from_numpy(s_o).cuda(), x)
    with pytest.raises(ValueError):
        q.matvec_int8km(c, torch.from_numpy(s_o[:2].copy()).cuda(), x)
    lb = torch.zeros(s_o.size + 1, dtype=torch.float16, device="cuda")
    lb[1:] = torch.from_numpy(s_o.reshape(-1)).cuda()
    y = q.matvec_int8km(c, lb[1:].view(s_o.shape), x)
    assert torch.equal(y, y0)
    assert rel_err(y.cpu().numpy(), orc.matvec(orc.FMT_INT8KM, c_o, s_o, xn, N, K)) < TOL
    assert q.status_fetch() == 0


def test_c1_tiny_fp4_round_trip_and_matvec(q):
    """512x1024 fp4, 8 outlier columns x20, x ~N(0,1) fp16, seed 0."""
    g = synth.generator(0, "cpu")
    W, _ = synth.weights(512, 1024, g, n_outlier_cols=8)
    x = synth.activations(1, 1024, g)
    Wn, xn = W.numpy(), x.numpy()
    codes, scales = q.encode_fp4(W.cuda())
    c_o, s_o, _ = orc.encode_fp4(Wn)
    assert np.array_equal(codes.cpu().numpy(), c_o) and np.array_equal(scales.cpu().numpy(), s_o)
    D = q.dequant(q.FMT_FP4, codes, scales).cpu().numpy()
    D_o = orc.dequant(orc.FMT_FP4, c_o, s_o, 512, 1024)
    assert np.array_equal(D.view(np.uint32), D_o.view(np.uint32))
    y = q.matvec_fp4(codes, scales, x.cuda())
    r = orc.matvec(orc.FMT_FP4, c_o, s_o, xn, 512, 1024)
    assert rel_err(y.cpu().numpy(), r) < TOL
    assert q.status_fetch() == 0


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("N,K", [(17, 96), (200, 544), (130, 2048), (64, 2080), (48, 4096)])
def test_dequant_bit_exact(q, fmt, N, K):
    W, _ = gen_w(N, K, seed=3 * N + K, n_out=2)
    Wn = W.cpu().numpy()
    c_o, s_o, _ = encode_orc(fmt, Wn)
    c = torch.from_numpy(c_o).cuda()
    s = torch.from_numpy(s_o).cuda()
    D = q.dequant(q.__dict__["FMT_" + fmt.upper()], c, s).cpu().numpy()
    D_o = orc.dequant(FID[fmt], c_o, s_o, N, K)
    assert np.array_equal(D.view(np.uint32), D_o.view(np.uint32))


# ---------------------------------------------------------------------------
# fused dequant + matvec
# ---------------------------------------------------------------------------

def _inputs(fmt, N, K, B, seed):
    g = synth.generator(seed, "cpu")
    W, _ = synth.weights(N, K, g, n_outlier_cols=2)
    x = synth.activations(B, K, g)
    Wn = W.numpy()
    big = (fmt == "int4km" and N * K > 2_000_000) or (fmt == "int8km" and N * K > 600_000)
    c_o, s_o, _ = encode_orc(fmt, Wn) if not big else (None, None, 0)
    if c_o is None:  # stand-in tables where the CPU fit is too slow
        lut, idx = (synth.palette_tables8 if fmt == "int8km" else synth.palette_tables)(N, K, g)
        c_o, s_o = idx.numpy(), lut.numpy()
    return c_o, s_o, x.numpy()


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("N,K", [(1, 32), (17, 96), (1000, 544), (600, 2048), (70, 2080), (130, 4096),
                                 (40, 6144)])
@pytest.mark.parametrize("B", [1, 3, 8, 9, 16])
def test_matvec_parity(q, fmt, N, K, B):
    c_o, s_o, xn = _inputs(fmt, N, K, B, seed=N * 7 + K + B)
    c, s, x = torch.from_numpy(c_o).cuda(), torch.from_numpy(s_o).cuda(), torch.from_numpy(xn).cuda()
    if B * K * 2 > 160 * 1024 and fmt == "int8km":
        # int8km's kernel stages all of K: activations beyond the on-chip
        # staging are rejected on the host (the other formats stage them in
        # K-phases)
        with pytest.raises(q.QmvError) as ei:
            q.matvec(q.__dict__["FMT_" + fmt.upper()], c, s, x)
        assert ei.value.status == q.ERR_UNSUPPORTED
        return
    y = q.matvec(q.__dict__["FMT_" + fmt.upper()], c, s, x).cpu().numpy()
    r = orc.matvec(FID[fmt], c_o, s_o, xn, N, K)
    e = rel_err(y, r)
    assert e < TOL, e
    assert q.status_fetch() == 0


@pytest.mark.parametrize("B", [7, 8])
def test_int4km_palette_copy_fallback_parity(q, B):
    """int4km at up to 8 columns looks rows g+8 up in lane palette copies in
    shared memory where they fit beside the staged activations: at K = 8704
    they just fit with 7 columns (one 8-warp CTA per SM), and with 8 columns
    they do not, so the byte-permute lookups serve that launch (no refusal)."""
    N, K = 300, 8704
    c_o, s_o, xn = _inputs("int4km", N, K, B, seed=91 + B)
    y = q.matvec_int4km(torch.from_numpy(c_o).cuda(), torch.from_numpy(s_o).cuda(), torch.from_numpy(xn).cuda())
    r = orc.matvec(FID["int4km"], c_o, s_o, xn, N, K)
    assert rel_err(y.cpu().numpy(), r) < TOL
    assert q.status_fetch() == 0


def test_int4km_palette_copy_equals_register_lookup(q):
    """The shared-memory palette lookups (8 columns) and the byte-permute
    lookups (9 columns) return the same fp16 weights: on a shape where every
    output is one lane's sum over all of K, the first 8 outputs of the 9-column
    launch equal the 8-column launch bit for bit."""
    N, K = 37905, 2048
    g = synth.generator(17, "cuda")
    lut, idx = synth.palette_tables(N, K, g)
    x9 = synth.activations(9, K, g)
    y8 = q.matvec_int4km(idx, lut, x9[:8].contiguous())
    y9 = q.matvec_int4km(idx, lut, x9)
    assert torch.equal(y8, y9[:8])
    assert q.status_fetch() == 0


PHASED_FMTS = ("fp4", "int4", "int4km", "int8", "int4aff")


@pytest.mark.parametrize("fmt", PHASED_FMTS)
@pytest.mark.parametrize("N,K,B", [(100, 16384, 16), (40, 6144, 9), (300, 8192, 12), (33, 32768, 3)])
def test_matvec_phased_staging_parity(q, fmt, N, K, B):
    """Activations larger than the on-chip staging (B * K * 2 bytes beyond
    ~160 KB) are staged one K-phase at a time: the result still matches the
    oracle (several phases, ragged row tiles, 3..16 columns)."""
    c_o, s_o, xn = _inputs(fmt, N, K, B, seed=N + K + B)
    y = q.matvec(q.__dict__["FMT_" + fmt.upper()], torch.from_numpy(c_o).cuda(), torch.from_numpy(s_o).cuda(),
                 torch.from_numpy(xn).cuda()).cpu().numpy()
    r = orc.matvec(FID[fmt], c_o, s_o, xn, N, K)
    assert rel_err(y, r) < TOL
    assert q.status_fetch() == 0


@pytest.mark.parametrize("fmt", ("fp4", "int4km"))
def test_gather_phased_staging_parity(q, fmt):
    """Per-slot activations of 64 (token, slot) pairs at K = 4096 (512 KB)
    are staged in K-phases: every slot still equals the oracle's matvec with
    its expert."""
    E, N, K, B, topk = 16, 64, 4096, 8, 8
    g = synth.generator(77, "cpu")
    W, _ = synth.weights(E * N, K, g)
    Wn = W.numpy()
    c_o, s_o, _ = encode_orc(fmt, Wn)
    ids = synth.routing(B, topk, E, g)
    x = synth.activations(B, K, g, extra_shape=(topk,))
    c = torch.from_numpy(c_o).cuda().view(E, N, -1)
    a = torch.from_numpy(s_o).cuda().view(E, N, -1)
    y = q.gather_matvec(q.__dict__["FMT_" + fmt.upper()], c, a, ids.cuda(), x.cuda(), x_per_slot=True).cpu().numpy()
    xn, ids_n = x.numpy(), ids.numpy()
    for b in range(B):
        for j in range(topk):
            e = ids_n[b, j]
            r = orc.matvec(FID[fmt], c_o[e * N:(e + 1) * N], s_o[e * N:(e + 1) * N], xn[b, j][None], N, K)
            assert rel_err(y[b, j][None], r) < TOL, (b, j)
    assert q.status_fetch() == 0


def test_argmax_phased_staging(q):
    """The fused argmax over a launch with phased activation staging equals
    torch.argmax of the unfused outputs (16 columns, K = 12288)."""
    N, K, B = 3000, 12288, 16
    g = synth.generator(78, "cuda")
    W, _ = synth.weights(N, K, g)
    codes, scales = q.encode_fp4(W)
    x = synth.activations(B, K, g)
    y = q.matvec_fp4(codes, scales, x)
    idx, val = q.matvec_argmax(q.FMT_FP4, codes, scales, x, q.argmax_workspace())
    assert torch.equal(idx.long(), torch.argmax(y, dim=1))
    assert torch.equal(val, y.max(dim=1).values)
    assert q.status_fetch() == 0


@pytest.mark.parametrize("fmt", FMTS)
def test_matvec_one_hot_columns_bit_exact(q, fmt):
    """x = e_k picks column k of Wdq: the kernel must return it exactly
    (pins layout, nibble order, scale indexing and the k-permutation)."""
    N, K = 100, 544
    c_o, s_o, _ = _inputs(fmt, N, K, 1, seed=5)
    ks = [0, 1, 7, 8, 31, 32, 100, 257, K - 1, K - 2, 300, 511, 64, 65, 200, 450]
    x = np.zeros((len(ks), K), np.float16)
    x[np.arange(len(ks)), ks] = 1.0
    y = q.matvec(q.__dict__["FMT_" + fmt.upper()], torch.from_numpy(c_o).cuda(), torch.from_numpy(s_o).cuda(),
                 torch.from_numpy(x).cuda()).cpu().numpy()
    D = orc.dequant(FID[fmt], c_o, s_o, N, K)
    for i, k in enumerate(ks):
        assert np.array_equal(y[i], D[:, k]), (fmt, k)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("N,K", [(100, 512), (37, 2048), (40, 1056)])
def test_matvec_batch1_one_hot_bit_exact(q, fmt, N, K):
    """Batch 1 with K a multiple of 256 takes the form whose MMA columns carry
    blocks: x = e_k, one launch per k, must return column k of Wdq exactly
    (pins the block-to-column and in-block k mapping of that form; int8km's
    batch-1 kernel: its 512-wide chunks, ragged at K = 1056)."""
    c_o, s_o, _ = _inputs(fmt, N, K, 1, seed=23 + K)
    c, s = torch.from_numpy(c_o).cuda(), torch.from_numpy(s_o).cuda()
    D = orc.dequant(FID[fmt], c_o, s_o, N, K)
    for k in [0, 1, 2, 3, 4, 7, 8, 9, 15, 16, 31, 32, 33, 63, 64, 100, 255, 256, 300, K - 33, K - 1]:
        x = torch.zeros((1, K), dtype=torch.float16, device="cuda")
        x[0, k] = 1.0
        y = q.matvec(q.__dict__["FMT_" + fmt.upper()], c, s, x).cpu().numpy()
        assert np.array_equal(y[0], D[:, k]), (fmt, k)


@pytest.mark.parametrize("fmt", FMTS)
def test_matvec_batch1_whole_units(q, fmt):
    """Enough 16-row tiles that every warp takes whole tiles (no K split), a
    ragged last tile, batch 1."""
    N, K = 37905, 2048  # 2370 tiles: at least one whole tile per warp of a full grid
    c_o, s_o, xn = _inputs(fmt, N, K, 1, seed=29)
    y = q.matvec(q.__dict__["FMT_" + fmt.upper()], torch.from_numpy(c_o).cuda(), torch.from_numpy(s_o).cuda(),
                 torch.from_numpy(xn).cuda()).cpu().numpy()
    r = orc.matvec(FID[fmt], c_o, s_o, xn, N, K)
    assert rel_err(y, r) < TOL
    y2 = q.matvec(q.__dict__["FMT_" + fmt.upper()], torch.from_numpy(c_o).cuda(), torch.from_numpy(s_o).cuda(),
                  torch.from_numpy(xn).cuda()).cpu().numpy()
    assert np.array_equal(y, y2)


@pytest.mark.parametrize("fmt", FMTS)
def test_weight_prefetch_same_results_and_ordering(q, fmt):
    """With early weight reads on, results are bit-identical, and each launch
    still sees activations (and weights) written by the work just before it
    on the same stream."""
    N, K = 3000, 2048
    f = q.__dict__["FMT_" + fmt.upper()]
    c_o, s_o, xn = _inputs(fmt, N, K, 1, seed=31)
    c, s = torch.from_numpy(c_o).cuda(), torch.from_numpy(s_o).cuda()
    xs = [torch.from_numpy(synth.activations(1, K, synth.generator(40 + i, "cpu")).numpy()).cuda() for i in range(4)]
    ref = [q.matvec(f, c, s, x) for x in xs]
    torch.cuda.synchronize()
    st = torch.cuda.Stream()
    xbuf = torch.empty_like(xs[0])
    outs = [torch.empty((1, N), dtype=torch.float32, device="cuda") for _ in xs]
    try:
        q.set_weight_prefetch(True)
        with torch.cuda.stream(st):
            for _ in range(3):
                for i, x in enumerate(xs):
                    xbuf.copy_(x)  # a kernel on the same stream writes the activations
                    q.matvec(f, c, s, xbuf, out=outs[i], stream=st)
        st.synchronize()
    finally:
        q.set_weight_prefetch(False)
    for r, o in zip(ref, outs):
        assert torch.equal(r, o)
    # weights rewritten right before the call (prefetch off, the default)
    c2 = torch.zeros_like(c) if fmt != "int4km" else c.clone()
    s2 = s.clone()
    with torch.cuda.stream(st):
        c2.copy_(c)
        s2.copy_(s)
        y = q.matvec(f, c2, s2, xs[0], stream=st)
    st.synchronize()
    assert torch.equal(y, ref[0])
    assert q.status_fetch() == 0


def test_matvec_output_guard_bands(q):
    """Sentinels around the output rows stay untouched (no out-of-bounds
    writes on a ragged last tile)."""
    N, K, B = 37, 2048, 3
    c_o, s_o, xn = _inputs("fp4", N, K, B, seed=11)
    buf = torch.full((B * N + 64,), 12345.0, device="cuda")
    out = buf[32:32 + B * N].view(B, N)
    q.matvec_fp4(torch.from_numpy(c_o).cuda(), torch.from_numpy(s_o).cuda(), torch.from_numpy(xn).cuda(), out=out)
    b = buf.cpu().numpy()
    assert (b[:32] == 12345.0).all() and (b[32 + B * N:] == 12345.0).all()
    assert rel_err(out.cpu().numpy(), orc.matvec(orc.FMT_FP4, c_o, s_o, xn, N, K)) < TOL


def test_unaligned_fp4_scale_plane(q):
    """A scale plane starting at an odd byte takes the staged-block path."""
    N, K, B = 50, 2048, 2
    c_o, s_o, xn = _inputs("fp4", N, K, B, seed=13)
    sb = torch.zeros(s_o.size + 1, dtype=torch.uint8, device="cuda")
    sb[1:] = torch.from_numpy(s_o.reshape(-1)).cuda()
    s_view = sb[1:].view(N, K // 32)
    y = q.matvec_fp4(torch.from_numpy(c_o).cuda(), s_view, torch.from_numpy(xn).cuda())
    assert rel_err(y.cpu().numpy(), orc.matvec(orc.FMT_FP4, c_o, s_o, xn, N, K)) < TOL


def test_matvec_is_deterministic(q):
    N, K, B = 3000, 2048, 4
    c_o, s_o, xn = _inputs("int4", N, K, B, seed=17)
    args = (torch.from_numpy(c_o).cuda(), torch.from_numpy(s_o).cuda(), torch.from_numpy(xn).cuda())
    y1 = q.matvec_int4(*args)
    y2 = q.matvec_int4(*args)
    assert torch.equal(y1, y2)


# ---------------------------------------------------------------------------
# int4km encoder (GPU palette fit) against the oracle's k-means
# ---------------------------------------------------------------------------

def _km_rows(K, seed):
    """Rows that stress the fit: synthetic weights with outliers, few distinct
    values, signed zeros, constant, two values, duplicated quantile values."""
    g = synth.generator(seed, "cpu")
    W, _ = synth.weights(40, K, g, n_outlier_cols=2)
    W = W.numpy().copy()
    rng = np.random.default_rng(seed)
    W[1] = rng.choice(np.array([-0.03, -0.01, 0.0, 0.02, 0.05], np.float32), K)
    W[2] = np.where(rng.random(K) < 0.5, -0.0, 0.0).astype(np.float32)
    W[3] = 0.0125
    W[4] = np.where(rng.random(K) < 0.3, -0.02, 0.04).astype(np.float32)
    W[5, : K // 2] = 0.01
    W[6] = np.round(W[6] * 64) / 64  # coarse grid: many ties
    W[7] = rng.standard_normal(K).astype(np.float32) * 1e-6
    W[8] = (rng.standard_normal(K) * 30.0).astype(np.float32)
    return W


@pytest.mark.parametrize("K", [32, 96, 544, 2048, 4096])
@pytest.mark.parametrize("iters", [0, 1, 20])
def test_encode_int4km_bit_exact(q, K, iters):
    W = _km_rows(K, seed=K + iters)
    lut_o, idx_o, fl_o = orc.kmeans_int4km(W, iters=iters)
    idx, lut = q.encode_int4km(torch.from_numpy(W).cuda(), iters=iters)
    assert np.array_equal(lut.cpu().numpy().view(np.uint16), lut_o.view(np.uint16))
    assert np.array_equal(idx.cpu().numpy(), idx_o)
    assert q.status_fetch() == fl_o == 0


def test_encode_int4km_nonfinite_rows(q):
    W = _km_rows(256, seed=5)
    W[3, 7] = np.inf
    W[9, 100] = np.nan
    lut_o, idx_o, fl_o = orc.kmeans_int4km(W)
    idx, lut = q.encode_int4km(torch.from_numpy(W).cuda())
    assert np.array_equal(lut.cpu().numpy().view(np.uint16), lut_o.view(np.uint16))
    assert np.array_equal(idx.cpu().numpy(), idx_o)
    assert fl_o == q.FLAG_NONFINITE
    assert q.status_fetch() == q.FLAG_NONFINITE


def test_encode_int4km_then_matvec(q):
    """GPU palette fit -> GPU matvec against the oracle's fit -> fp64 matvec."""
    N, K, B = 1000, 2048, 2
    g = synth.generator(13, "cpu")
    W, _ = synth.weights(N, K, g, n_outlier_cols=2)
    x = synth.activations(B, K, g).numpy()
    idx, lut = q.encode_int4km(W.cuda())
    y = q.matvec_int4km(idx, lut, torch.from_numpy(x).cuda()).cpu().numpy()
    lut_o, idx_o, _ = orc.kmeans_int4km(W.numpy())
    assert rel_err(y, orc.matvec(orc.FMT_INT4KM, idx_o, lut_o, x, N, K)) < TOL


def test_encode_int4km_argument_checks(q):
    W = torch.zeros((4, 64), dtype=torch.float32, device="cuda")
    with pytest.raises(q.QmvError) as ei:
        q.encode_int4km(W, iters=-1)
    assert ei.value.status == q.ERR_ARG
    with pytest.raises(q.QmvError) as ei:
        q.encode_int4km(torch.zeros((4, 32768), dtype=torch.float32, device="cuda"))
    assert ei.value.status == q.ERR_UNSUPPORTED


# ---------------------------------------------------------------------------
# fused matvec + argmax
# ---------------------------------------------------------------------------

def _first_argmax(y):
    """Lowest index of the maximum per row (values compared with -0 == +0)."""
    y = np.asarray(y, np.float64) + 0.0
    m = y.max(axis=1, keepdims=True)
    return (y == m).argmax(axis=1), m[:, 0]


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("N,K,B", [(17, 96, 1), (1000, 2048, 1), (1000, 2048, 3), (300, 544, 16), (37905, 2048, 1),
                                   (37905, 2048, 9)])
def test_matvec_argmax_matches_unfused(q, fmt, N, K, B):
    """The fused argmax equals the argmax of the same kernel's materialised y
    (bit-identical outputs, lowest index on ties) and is within tolerance of
    the fp64 oracle's maximum."""
    f = q.__dict__["FMT_" + fmt.upper()]
    c_o, s_o, xn = _inputs(fmt, N, K, B, seed=N + K + B)
    c, s, x = torch.from_numpy(c_o).cuda(), torch.from_numpy(s_o).cuda(), torch.from_numpy(xn).cuda()
    ws = q.argmax_workspace()
    idx, val = q.matvec_argmax(f, c, s, x, ws)
    y = q.matvec(f, c, s, x).cpu().numpy()
    want_i, want_v = _first_argmax(y)
    assert np.array_equal(idx.cpu().numpy(), want_i)
    assert np.array_equal(val.cpu().numpy(), want_v.astype(np.float32))
    r = orc.matvec(FID[fmt], c_o, s_o, xn, N, K)
    got = r[np.arange(B), idx.cpu().numpy()]
    assert np.all(got >= r.max(axis=1) - TOL * np.abs(r).max(axis=1))
    assert int(ws.count_nonzero()) == 0  # left zero-filled for the next call
    assert q.status_fetch() == 0


@pytest.mark.parametrize("fmt", FMTS)
def test_matvec_argmax_planted_and_ties(q, fmt):
    """A planted maximum is found exactly; two identical rows holding the
    maximum resolve to the lower index; repeated calls reuse the workspace."""
    N, K, B = 3000, 1024, 2
    f = q.__dict__["FMT_" + fmt.upper()]
    g = synth.generator(77, "cpu")
    W, _ = synth.weights(N, K, g, n_outlier_cols=0)
    x = synth.activations(B, K, g).numpy()
    Wn = W.numpy()
    # row 2321 aligned with x[0]; rows 777 and 2900 identical and aligned with
    # x[1] (int8km: 777 and 778, one LUT group, so their weights stay equal)
    tw = 778 if fmt == "int8km" else 2900
    Wn[2321] = np.sign(x[0].astype(np.float32)) * 0.05
    Wn[777] = np.sign(x[1].astype(np.float32)) * 0.05
    Wn[tw] = Wn[777]
    c_o, s_o, _ = encode_orc(fmt, Wn)
    c, s, xg = torch.from_numpy(c_o).cuda(), torch.from_numpy(s_o).cuda(), torch.from_numpy(x).cuda()
    ws = q.argmax_workspace()
    r = orc.matvec(FID[fmt], c_o, s_o, x, N, K)
    for _ in range(3):
        idx, val = q.matvec_argmax(f, c, s, xg, ws)
        got = idx.cpu().numpy()
        assert got[0] == 2321 and r[0].argmax() == 2321
        assert got[1] == 777 and r[1, 777] == r[1, tw] and r[1].argmax() == 777


def test_matvec_argmax_rejects_short_workspace(q):
    N, K = 64, 256
    c = torch.zeros((N, K // 2), dtype=torch.uint8, device="cuda")
    s = torch.zeros((N, K // 32), dtype=torch.uint8, device="cuda")
    x = torch.zeros((1, K), dtype=torch.float16, device="cuda")
    ws = torch.zeros(q.argmax_workspace_bytes() - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(q.QmvError) as ei:
        q.matvec_argmax(q.FMT_FP4, c, s, x, ws)
    assert ei.value.status == q.ERR_ARG


# ---------------------------------------------------------------------------
# gather over routed experts
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("B,topk,x_per_slot", [(1, 8, 0), (3, 2, 1), (8, 8, 0), (8, 8, 1), (16, 4, 0)])
def test_gather_parity(q, fmt, B, topk, x_per_slot):
    E, N, K = 12, 80, 544
    g = synth.generator(B * 100 + topk, "cpu")
    Ws = [synth.weights(N, K, g)[0].numpy() for _ in range(E)]
    enc = [encode_orc(fmt, W) for W in Ws]
    cs = np.stack([e[0] for e in enc])
    aus = np.stack([e[1] for e in enc])
    ids = synth.routing(B, topk, E, g).numpy()
    if B >= 3:
        ids[1, 0] = ids[0, 0]  # two tokens share an expert
    x = synth.activations(B, K, g, extra_shape=(topk,) if x_per_slot else ()).numpy()
    F = q.__dict__["FMT_" + fmt.upper()]
    y = q.gather_matvec(F, torch.from_numpy(cs).cuda(), torch.from_numpy(aus).cuda(), torch.from_numpy(ids).cuda(),
                        torch.from_numpy(x).cuda(), x_per_slot=bool(x_per_slot)).cpu().numpy()
    r, fl = orc.gather_matvec(FID[fmt], cs, aus, E, N, K, ids, x, x_per_slot)
    assert fl == 0
    assert rel_err(y.reshape(-1, N), r.reshape(-1, N)) < TOL
    # identical, bit for bit, to the dense kernel on the chosen expert's
    # weights taking the same tensor-core path: a batch of two (dense batch 1
    # may take a batch-1 form with another summation order)
    for b in range(B):
        for j in range(topk):
            e = ids[b, j]
            xb = x[b, j] if x_per_slot else x[b]
            yd = q.matvec(F, torch.from_numpy(cs[e]).cuda(), torch.from_numpy(aus[e]).cuda(),
                          torch.from_numpy(np.stack([xb, xb])).cuda()).cpu().numpy()[0]
            assert np.array_equal(yd, y[b, j]), (b, j)
    assert q.status_fetch() == 0


def test_gather_bad_expert_id_flags_and_zeroes(q):
    E, N, K, B, topk = 4, 64, 256, 2, 3
    g = synth.generator(1, "cpu")
    W = synth.weights(E * N, K, g)[0].numpy()
    c, s, _ = orc.encode_fp4(W)
    cs, ss = c.reshape(E, N, -1), s.reshape(E, N, -1)
    ids = np.array([[0, 9, 2], [-1, 3, 3]], np.int32)
    x = synth.activations(B, K, g).numpy()
    y = torch.full((B, topk, N), 7.0, device="cuda")
    q.gather_matvec(q.FMT_FP4, torch.from_numpy(cs).cuda(), torch.from_numpy(ss).cuda(), torch.from_numpy(ids).cuda(),
                    torch.from_numpy(x).cuda(), out=y)
    flags = q.status_fetch()
    assert flags & q.FLAG_BAD_EXPERT
    yn = y.cpu().numpy()
    assert not yn[0, 1].any() and not yn[1, 0].any()
    r, fl = orc.gather_matvec(orc.FMT_FP4, cs, ss, E, N, K, ids, x, 0)
    assert fl & orc.FLAG_BAD_EXPERT
    assert rel_err(yn.reshape(-1, N), r.reshape(-1, N)) < TOL


# ---------------------------------------------------------------------------
# data faults and argument errors
# ---------------------------------------------------------------------------

def test_nonfinite_weights_flag_and_zero_blocks(q):
    W, _ = gen_w(8, 128, seed=2)
    W[3, 40] = float("nan")
    W[5, 100] = float("inf")
    Wn = W.cpu().numpy()
    for fmt in ("fp4", "int4", "int8", "int4aff"):
        c, s = encode_gpu(q, fmt, W)
        flags = q.status_fetch()
        assert flags & q.FLAG_NONFINITE, fmt
        c_o, s_o, f = encode_orc(fmt, Wn)
        assert f & orc.FLAG_NONFINITE
        assert np.array_equal(np_bits(c), c_o.view(np.uint8))


def test_scale_overflow_flag(q):
    W = torch.zeros(2, 32, device="cuda")
    W[1, 0] = 1e6  # 1e6 / 7 > 65504: no finite fp16 scale for clip 1.0
    c, s = q.encode_int4(W, clips=[1.0])
    assert q.status_fetch() & q.FLAG_SCALE_OVERFLOW
    c_o, s_o, f = orc.encode_int4(W.cpu().numpy(), np.array([1.0], np.float32))
    assert f & orc.FLAG_SCALE_OVERFLOW
    assert np.array_equal(c.cpu().numpy(), c_o) and np.array_equal(np_bits(s), s_o.view(np.uint16))
    # affine int4: (1e6 - 0) / 15 > 65504
    c, a = q.encode_int4aff(W)
    assert q.status_fetch() & q.FLAG_SCALE_OVERFLOW
    c_o, a_o, f = orc.encode_int4aff(W.cpu().numpy())
    assert f & orc.FLAG_SCALE_OVERFLOW
    assert np.array_equal(c.cpu().numpy(), c_o) and np.array_equal(a.cpu().numpy(), a_o)


def test_argument_errors_raise(q):
    codes = torch.zeros(16, 64, dtype=torch.uint8, device="cuda")
    scales = torch.zeros(16, 4, dtype=torch.uint8, device="cuda")
    xb = torch.zeros(2 * 128 + 1, dtype=torch.float16, device="cuda")
    with pytest.raises(q.QmvError) as ei:
        q.matvec_fp4(codes, scales, xb[1:129])  # x misaligned by 2 bytes
    assert ei.value.status == q.ERR_ARG
    with pytest.raises(q.QmvError) as ei:
        q.matvec_fp4(codes, scales, torch.zeros(17, 128, dtype=torch.float16, device="cuda"))
    assert ei.value.status == q.ERR_UNSUPPORTED
    assert q.status_fetch() == 0


# ---------------------------------------------------------------------------
# the workloads at full size (sampled rows against the oracle)
# ---------------------------------------------------------------------------

def sample_rows(N, n_rand=384, seed=0):
    rng = np.random.default_rng(seed)
    rows = np.concatenate([np.arange(min(N, 48)), np.arange(max(0, N - 48), N), rng.integers(0, N, n_rand)])
    return np.unique(rows)


def _full_encode_check(q, fmt, W, rows):
    c, s = encode_gpu(q, fmt, W)
    c_o, s_o, f = encode_orc(fmt, W[torch.from_numpy(rows).cuda()].cpu().numpy())
    assert f == 0
    assert np.array_equal(np_bits(c)[rows], c_o.view(np.uint8))
    assert np.array_equal(np_bits(s)[rows], s_o.view(np.uint8) if fmt in ("fp4", "int4aff") else s_o.view(np.uint16))
    return c, s, c_o, s_o


def _sampled_matvec(q, fmt, c, s, c_o, s_o, xn, rows, K):
    y = q.matvec(q.__dict__["FMT_" + fmt.upper()], c, s, torch.from_numpy(xn).cuda())
    r = orc.matvec(FID[fmt], c_o, s_o, xn, len(rows), K)
    e = rel_err(y.cpu().numpy()[:, rows], r)
    assert e < TOL, (fmt, e)
    return e


@pytest.mark.slow
def test_full_int8_head_130560x2048(q):
    N, K = 130560, 2048
    g = synth.generator(0, "cuda")
    W, _ = synth.weights(N, K, g)
    x = synth.activations(1, K, g).cpu().numpy()
    rows = sample_rows(N)
    c, s, c_o, s_o = _full_encode_check(q, "int8", W, rows)
    _sampled_matvec(q, "int8", c, s, c_o, s_o, x, rows, K)
    assert q.status_fetch() == 0


@pytest.mark.slow
def test_full_int4_and_fp4_head_248320x2048(q):
    """int4 (11 clips), affine int4 and fp4 on the same outlier-bearing head;
    affine int4 at batch 1 and 16, fp4 at batch 1, 4 and 16."""
    N, K = 248320, 2048
    g = synth.generator(0, "cuda")
    W, _ = synth.weights(N, K, g, n_outlier_cols=2)
    x16 = synth.activations(16, K, g).cpu().numpy()
    rows = sample_rows(N)
    c, s, c_o, s_o = _full_encode_check(q, "int4", W, rows)
    _sampled_matvec(q, "int4", c, s, c_o, s_o, x16[:1], rows, K)
    del c, s
    c, s, c_o, s_o = _full_encode_check(q, "int4aff", W, rows)
    for B in (1, 16):
        _sampled_matvec(q, "int4aff", c, s, c_o, s_o, x16[:B], rows, K)
    del c, s
    c, s, c_o, s_o = _full_encode_check(q, "fp4", W, rows)
    for B in (1, 4, 16):
        _sampled_matvec(q, "fp4", c, s, c_o, s_o, x16[:B], rows, K)
    assert q.status_fetch() == 0


@pytest.mark.slow
def test_full_int4km_head_248320x2048(q):
    """int4km at full size with per-row palettes of the workload's shape
    (random tables: the CPU fit of 248320 rows is covered at smaller sizes)."""
    N, K = 248320, 2048
    g = synth.generator(0, "cuda")
    lut, idx = synth.palette_tables(N, K, g)
    x = synth.activations(1, K, g).cpu().numpy()
    rows = sample_rows(N)
    y = q.matvec_int4km(idx, lut, torch.from_numpy(x).cuda())
    r = orc.matvec(orc.FMT_INT4KM, idx.cpu().numpy()[rows], lut.cpu().numpy()[rows], x, len(rows), K)
    assert rel_err(y.cpu().numpy()[:, rows], r) < TOL


@pytest.mark.slow
@pytest.mark.parametrize("B", [1, 8])
def test_full_decode_step_int4km(q, B):
    """lm_head + 10 x (q_proj 2048->4096, o_proj 4096->2048) + routed experts
    256 x (gate/up 2048->512, down 512->2048), top-8 routing; gate and up as
    one [256, 1024, 2048] stack (one gather launch serves both)."""
    g = synth.generator(1000 + B, "cuda")
    dense = [(248320, 2048)] + [(4096, 2048), (2048, 4096)] * 10
    for i, (N, K) in enumerate(dense):
        lut, idx = synth.palette_tables(N, K, g)
        x = synth.activations(B, K, g).cpu().numpy()
        rows = sample_rows(N, n_rand=64, seed=i)
        y = q.matvec_int4km(idx, lut, torch.from_numpy(x).cuda())
        r = orc.matvec(orc.FMT_INT4KM, idx.cpu().numpy()[rows], lut.cpu().numpy()[rows], x, len(rows), K)
        assert rel_err(y.cpu().numpy()[:, rows], r) < TOL, (i, N, K)
    E, topk = 256, 8
    ids = synth.routing(B, topk, E, g)
    for name, N, K, per_slot in (("gate_up", 1024, 2048, 0), ("down", 2048, 512, 1)):
        lut, idx = synth.palette_tables(E * N, K, g)
        lut, idx = lut.view(E, N, 16), idx.view(E, N, K // 2)
        x = synth.activations(B, K, g, extra_shape=(topk,) if per_slot else ())
        y = q.gather_matvec(q.FMT_INT4KM, idx, lut, ids, x, x_per_slot=bool(per_slot)).cpu().numpy()
        ids_n, xn = ids.cpu().numpy(), x.cpu().numpy()
        for b in range(B):
            for j in range(topk):
                e = ids_n[b, j]
                rows = sample_rows(N, n_rand=32, seed=b * topk + j)
                xb = xn[b, j] if per_slot else xn[b]
                r = orc.matvec(orc.FMT_INT4KM, idx[e].cpu().numpy()[rows], lut[e].cpu().numpy()[rows], xb[None],
                               len(rows), K)
                assert rel_err(y[b, j][rows][None], r) < TOL, (name, b, j)
    assert q.status_fetch() == 0


# ---------------------------------------------------------------------------
# mixed int4km + int8 outlier columns
# ---------------------------------------------------------------------------

def _outlier_w(N, K, C, seed):
    g = np.random.default_rng(seed)
    W = (g.standard_normal((N, K)) * 0.02).astype(np.float32)
    cols = np.sort(g.choice(K, C, replace=False))
    W[:, cols] *= 20.0
    return W


@pytest.mark.parametrize("N,K,C", [(3000, 256, 32), (40, 4096, 64), (7, 1088, 96), (300, 2048, 0)])
def test_outlier_columns_exact(q, N, K, C):
    """The GPU column choice equals the oracle's, with ties, a NaN column and
    several blocks of the rank kernel."""
    W = _outlier_w(N, K, max(C, 32), seed=N + K)
    W[:, 5] = W[:, K - 3]  # equal maxima: the lower column first
    W[N // 2, 9] = np.nan
    got = q.outlier_columns(torch.from_numpy(W).cuda(), C).cpu().numpy()
    assert np.array_equal(got, orc.outlier_columns(W, C))
    assert q.status_fetch() == 0


@pytest.mark.parametrize("N,K,C", [(200, 1088, 64), (33, 544, 32), (64, 2048, 0)])
def test_encode_int4km_o8_bit_exact(q, N, K, C):
    W = _outlier_w(N, K, max(C, 32), seed=3 * N + K)
    cols, lut, idx, oc, osc = q.encode_int4km_o8(torch.from_numpy(W).cuda(), C)
    c_o, lut_o, idx_o, oc_o, osc_o, f = orc.encode_int4km_o8(W, C)
    assert f == 0 and q.status_fetch() == 0
    assert np.array_equal(cols.cpu().numpy(), c_o)
    assert np.array_equal(lut.cpu().numpy().view(np.uint16), lut_o.view(np.uint16))
    assert np.array_equal(idx.cpu().numpy(), idx_o)
    assert np.array_equal(oc.cpu().numpy(), oc_o)
    assert np.array_equal(osc.cpu().numpy().view(np.uint16), osc_o.view(np.uint16))


@pytest.mark.parametrize("N,K,C", [(70, 544, 32), (600, 2048, 64), (130, 4096, 128), (17, 96, 64)])
@pytest.mark.parametrize("B", [1, 3, 9, 16])
def test_matvec_int4km_o8_parity(q, N, K, C, B):
    W = _outlier_w(N, K, C, seed=7 * N + K + B)
    c_o, lut_o, idx_o, oc_o, osc_o, _ = orc.encode_int4km_o8(W, C)
    x = synth.activations(B, K, synth.generator(N + B, "cpu")).numpy()
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    y = q.matvec_int4km_o8(t(c_o), t(lut_o), t(idx_o), t(oc_o), t(osc_o), t(x)).cpu().numpy()
    r = orc.matvec_int4km_o8(c_o, lut_o, idx_o, oc_o, osc_o, x, N, K)
    assert rel_err(y, r) < TOL
    assert q.status_fetch() == 0


def test_matvec_int4km_o8_main_part_staging(q):
    """With the outlier codes zeroed, the mixed matvec is the int4km kernel
    on the main columns of x, bit for bit (the kernel's column map)."""
    N, K, C, B = 300, 2048, 96, 3
    W = _outlier_w(N, K, C, seed=61)
    c_o, lut_o, idx_o, oc_o, osc_o, _ = orc.encode_int4km_o8(W, C)
    x = synth.activations(B, K, synth.generator(62, "cpu")).numpy()
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    y = q.matvec_int4km_o8(t(c_o), t(lut_o), t(idx_o), t(np.zeros_like(oc_o)), t(osc_o), t(x))
    main = np.setdiff1d(np.arange(K), c_o)
    y_main = q.matvec_int4km(t(idx_o), t(lut_o), t(x[:, main]))
    assert torch.equal(y, y_main)


def test_matvec_int4km_o8_no_outliers_is_int4km(q):
    N, K, B = 300, 2048, 2
    W = _outlier_w(N, K, 32, seed=51)
    c_o, lut_o, idx_o, oc_o, osc_o, _ = orc.encode_int4km_o8(W, 0)
    x = torch.from_numpy(synth.activations(B, K, synth.generator(52, "cpu")).numpy()).cuda()
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    y = q.matvec_int4km_o8(t(c_o), t(lut_o), t(idx_o), t(oc_o), t(osc_o), x)
    assert torch.equal(y, q.matvec_int4km(t(idx_o), t(lut_o), x))


@pytest.mark.slow
def test_matvec_int4km_o8_full_head_sampled(q):
    """The 248320 x 2048 head with 64 outlier columns, GPU-encoded (bit-exact
    with the oracle per row, checked on sampled rows) at batch 1 and 16."""
    N, K, C = 248320, 2048, 64
    g = synth.generator(0, "cuda")
    W, _ = synth.weights(N, K, g, n_outlier_cols=2)
    cols, lut, idx, oc, osc = q.encode_int4km_o8(W, C)
    rows = sample_rows(N, n_rand=256)
    Wr = W[torch.from_numpy(rows).cuda()].cpu().numpy()
    c_o = orc.outlier_columns(W.cpu().numpy(), C)
    assert np.array_equal(cols.cpu().numpy(), c_o)
    _, lut_o, idx_o, oc_o, osc_o, _ = orc.encode_int4km_o8(Wr, C, cols=c_o)
    assert np.array_equal(lut.cpu().numpy()[rows].view(np.uint16), lut_o.view(np.uint16))
    assert np.array_equal(idx.cpu().numpy()[rows], idx_o) and np.array_equal(oc.cpu().numpy()[rows], oc_o)
    x16 = synth.activations(16, K, g)
    for B in (1, 16):
        y = q.matvec_int4km_o8(cols, lut, idx, oc, osc, x16[:B]).cpu().numpy()[:, rows]
        r = orc.matvec_int4km_o8(c_o, lut_o, idx_o, oc_o, osc_o, x16[:B].cpu().numpy(), len(rows), K)
        assert rel_err(y, r) < TOL
    assert q.status_fetch() == 0


def test_int4km_o8_argument_errors(q):
    W = torch.zeros(64, 256, device="cuda")
    with pytest.raises(q.QmvError) as ei:
        q.outlier_columns(W, 48)  # C % 32 != 0
    assert ei.value.status == q.ERR_SHAPE
    with pytest.raises(q.QmvError) as ei:
        q.outlier_columns(W, 256)  # C == K
    assert ei.value.status == q.ERR_SHAPE
    cols, lut, idx, oc, osc = q.encode_int4km_o8(W, 32)
    x = torch.zeros(1, 256, dtype=torch.float16, device="cuda")
    with pytest.raises(ValueError):
        q.matvec_int4km_o8(cols, lut, idx, oc[:, :16].contiguous(), osc, x)  # outlier codes of the wrong width
    with pytest.raises(q.QmvError) as ei:
        q.matvec_int4km_o8(cols, lut, idx, oc, osc, torch.zeros(17, 256, dtype=torch.float16, device="cuda"))
    assert ei.value.status == q.ERR_UNSUPPORTED  # B > 16
    assert q.status_fetch() == 0
