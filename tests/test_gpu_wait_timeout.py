"""The kernels' failure path on a GPU: a bounded mbarrier wait that nothing completes gives up
after its limit, records MORE_DEVERR_WAIT_TIMEOUT in the library's device error word and returns,
and the context stays usable for routing afterwards.  No fault, trap or endless loop is involved:
the wait is the same bounded wait the persistent kernels use, on a barrier nothing arrives at."""
import numpy as np
import pytest
import torch

import synthetic as syn
from tests import parity

pytestmark = pytest.mark.gpu

MORE_DEVERR_WAIT_TIMEOUT = 0x1


def test_bounded_wait_gives_up_and_the_context_stays_usable():
    import mixture_experts_rank_b200 as m
    assert m.device_status() == 0
    out = m.selftest_wait_timeout()
    assert m.device_status() & MORE_DEVERR_WAIT_TIMEOUT
    assert int(out.item()) == 2, "the wait should have given up, not completed"
    assert m.device_status() == 0, "reading the error word clears it"
    # routing still works on the same context
    N, h, r, M, k = 1000, 256, 32, 1024, 8
    X, R1, R2 = syn.router_inputs(N, h, r, M, seed=4)
    dev = lambda b: torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16).cuda()
    idx, gate, cnt, logits = m.route(dev(X), dev(R1), dev(R2), k, variant="fused_tc")
    torch.cuda.synchronize()
    assert m.device_status() == 0
    parity.compare(X, R1, R2, N, h, r, M, k, idx.cpu().numpy(), gate.cpu().numpy(), cnt.cpu().numpy(),
                   logits.cpu().numpy())
