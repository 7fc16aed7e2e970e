"""The no-allocation argmax entry point (qmv_matvec_argmax_static) against
the workspace entry point (qmv_matvec_argmax): same results on two calls in
a row (the static scratch is left zeroed by each call), per format.  int8km
at batch 1 takes its own kernel (the batch-1 row-loop form) with its own
argmax epilogue and grid, so it is covered beside the general form."""
import pytest
import torch

from weight_only_quantized_qmv_b200 import synth

pytestmark = pytest.mark.gpu

FMTS = ("fp4", "int4", "int4km", "int8", "int4aff", "int8km")


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
    if fmt == "int8km":
        lut, idx = synth.palette_tables8(N, K, g)
        return idx.cuda(), lut.cuda()
    if fmt == "int8":
        c = synth.int_codes(N, K, 8, g).view(torch.int8)
    else:
        c = torch.randint(0, 256, (N, K // 2), generator=g, dtype=torch.int32).to(torch.uint8)
    if fmt == "fp4":
        a = torch.randint(118, 125, (N, K // 32), generator=g, dtype=torch.int32).to(torch.uint8)
    elif fmt == "int4km":
        a = synth.palette_tables(N, K, g)[0]
    elif fmt == "int4aff":
        # fp16 scales, then the zero points two per byte
        nb = K // 32
        s = (torch.rand((N, nb), generator=g) * 0.01 + 0.001).to(torch.float16).view(torch.uint8)
        z = torch.randint(0, 256, (N, q.int4aff_aux_row_bytes(K) - 2 * nb), generator=g,
                          dtype=torch.int32).to(torch.uint8)
        a = torch.cat([s, z], dim=1).contiguous()
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
