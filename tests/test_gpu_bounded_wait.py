"""The bounded wait every TMA and tensor-core pipeline of the library uses
ends on the device: a wait on an mbarrier that nothing signals gives up after
its poll limit and reports CF_ERR_TIMEOUT, and the context stays usable.
The failure is made by construction (a barrier that nothing arrives on), not
by a fault, a trap or an endless loop."""
import pytest
import torch

from activation_residual_compression_cf_b200 import cf
from activation_residual_compression_cf_b200 import workloads as W

pytestmark = pytest.mark.gpu

CF_ERR_TIMEOUT = 7


@pytest.mark.parametrize("polls", [1, 256, 65536])
def test_unsignalled_wait_gives_up_and_context_stays_usable(polls):
    out = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    cf.cf_diag_bounded_wait(polls, out)
    torch.cuda.synchronize()
    assert out.tolist() == [1, CF_ERR_TIMEOUT]
    # the next launch on the same context works
    wl = W.WORKLOADS["tiny"]
    x = W.trajectory(wl, 0, steps=1, device="cuda")[0]
    d = cf.desc(wl.tokens, wl.channels, wl.bits)
    recon = torch.empty(wl.tokens, wl.channels, dtype=torch.float32, device="cuda")
    err = torch.empty_like(recon)
    cf.cf_state_init(d, x.view(torch.int16), recon, err)
    torch.cuda.synchronize()
    assert torch.equal(recon, x.float())
    assert not torch.any(err)
