"""The no-allocation argmax entry point (qmv_matvec_argmax_static) against
the workspace entry point (qmv_matvec_argmax): same results on two calls in
a row (the static scratch is left zeroed by each call), per format."""
import pytest
import torch

from weight_only_quantized_qmv_b200 import synth

pytestmark = pytest.mark.gpu

FMTS = ("fp4", "int4", "int4km", "int8")


@pytest.fixture(scope="module")
def q():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from weight_only_quantized_qmv_b200 import _build
    _build.build()
    import weight_only_quantized_qmv_b200 as q
    q.lib()
    return q


def _codes(q, fmt, N, K, g):
    if fmt == "int8":
        c = synth.int_codes(N, K, 8, g).view(torch.int8)
    else:
        c = torch.randint(0, 256, (N, K // 2), generator=g, dtype=torch.int32).to(torch.uint8)
    if fmt == "fp4":
        a = torch.randint(118, 125, (N, K // 32), generator=g, dtype=torch.int32).to(torch.uint8)
    elif fmt == "int4km":
        a = synth.palette_tables(N, K, g)[0]
    else:
        a = (torch.rand((N, K // 32), generator=g) * 0.01 + 0.001).to(torch.float16)
    return c.cuda(), a.cuda()


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("N,K,B", [(4096, 2048, 1), (37905, 2048, 3), (300, 544, 16)])
def test_static_scratch_matches_workspace_entry(q, fmt, N, K, B):
    f = q.__dict__["FMT_" + fmt.upper()]
    g = synth.generator(101 + N + B, "cpu")
    c, a = _codes(q, fmt, N, K, g)
    x = synth.activations(B, K, g).cuda()
    ws = q.argmax_workspace()
    want_i, want_v = q.matvec_argmax(f, c, a, x, ws)
    for _ in range(2):
        got_i, got_v = q.matvec_argmax_static(f, c, a, x)
        assert torch.equal(got_i, want_i)
        assert torch.equal(got_v, want_v)
    assert q.status_fetch() == 0
