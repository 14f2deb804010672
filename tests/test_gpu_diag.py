"""The byte-mix ceiling pass (cf_diag_stream_mix) computes what it states,
so the time bench.py reports for it is the time of that work: a = x - r and
r = x + r elementwise in fp32, over a ragged number of elements."""
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
