"""The byte-mix reference passes (cf_diag_stream_mix, and
cf_diag_stream_mix_tma through the encode's row pipeline) compute what they
state, so the times bench.py reports for them are the times of that work:
a = x - r and r = x + r elementwise in fp32, over ragged sizes."""
import pytest
import torch

from activation_residual_compression_cf_b200 import cf

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n", [8, 1000, 3 * 148 * 128 * 8 * 4 + 40])
def test_stream_mix_computes_difference_and_sum(n):
    g = torch.Generator(device="cuda").manual_seed(n)
    x = torch.randn(n, device="cuda", generator=g).to(torch.bfloat16)
    r = torch.randn(n, device="cuda", generator=g)
    a = torch.empty(n, device="cuda")
    r0 = r.clone()
    cf.cf_diag_stream_mix(x.view(torch.int16), r, a)
    torch.cuda.synchronize()
    xf = x.float()
    assert torch.equal(a, xf - r0) and torch.equal(r, xf + r0)


def test_stream_mix_rejects_ragged_groups():
    x = torch.zeros(12, dtype=torch.int16, device="cuda")
    r = torch.zeros(12, device="cuda")
    with pytest.raises(cf.CFError) as ei:
        cf.cf_diag_stream_mix(x, r, r.clone())
    assert ei.value.status == 1


# bulk stores need two ring slots and two output rows in one CTA's shared
# memory (C <= 8296); the longest row runs with per-thread stores only
_MIX_CASES = [(rows, C, bulk) for rows, C in ((1, 8), (37, 1920), (3 * 148 * 4 + 5, 1920), (300, 3072))
              for bulk in (False, True)] + [(5, 15360, False)]


@pytest.mark.parametrize("rows,C,bulk", _MIX_CASES)
def test_stream_mix_tma_computes_difference_and_sum(rows, C, bulk):
    g = torch.Generator(device="cuda").manual_seed(rows * C)
    x = torch.randn(rows, C, device="cuda", generator=g).to(torch.bfloat16)
    r = torch.randn(rows, C, device="cuda", generator=g)
    a = torch.full((rows, C), float("nan"), device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    r0 = r.clone()
    cf.cf_diag_stream_mix_tma(x.view(torch.int16), r, a, rows, C, st, bulk=bulk)
    torch.cuda.synchronize()
    xf = x.float()
    assert st.item() == 0
    assert torch.equal(a, xf - r0) and torch.equal(r, xf + r0)


def test_stream_mix_tma_rejects_bad_shapes():
    x = torch.zeros(4, 24, dtype=torch.int16, device="cuda")
    r = torch.zeros(4, 24, device="cuda")
    for rows, C, code in ((4, 12, 1), (-1, 24, 1), (1, 16392, 1)):
        with pytest.raises(cf.CFError) as ei:
            cf.cf_diag_stream_mix_tma(x, r, r.clone(), rows, C)
        assert ei.value.status == code
    with pytest.raises(cf.CFError) as ei:     # bulk: 2 slots + 2 output rows beyond a CTA's shared memory
        cf.cf_diag_stream_mix_tma(torch.zeros(1, 8304, dtype=torch.int16, device="cuda"),
                                  torch.zeros(1, 8304, device="cuda"), torch.zeros(1, 8304, device="cuda"),
                                  1, 8304, bulk=True)
    assert ei.value.status == 3
    big = torch.zeros(1, 15368, device="cuda")
    with pytest.raises(cf.CFError) as ei:
        cf.cf_diag_stream_mix_tma(torch.zeros(1, 15368, dtype=torch.int16, device="cuda"), big, big.clone(),
                                  1, 15368)
    assert ei.value.status == 3
    # nothing to do
    cf.cf_diag_stream_mix_tma(x, r, r.clone(), 0, 24)
