"""The bounded wait of the pipelined kernels gives up and reports instead of
hanging: an mbarrier that nothing completes, MOE_ERR_TIMEOUT in the status
word after about a second, and the context still usable afterwards."""
import time

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    from combine_moe_topk_gate_b200 import api
    dev = torch.device("cuda", 0)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    t0 = time.monotonic()
    api.moe_selftest_bounded_wait(st)
    torch.cuda.synchronize(dev)
    waited = time.monotonic() - t0
    assert int(st.item()) == api.MOE_ERR_TIMEOUT
    assert 0.9 < waited < 30.0
    # the context is still usable: a small combine runs and is exact
    y = torch.ones((8, 64), dtype=torch.bfloat16, device=dev)
    slots = torch.arange(8, dtype=torch.int32, device=dev).reshape(4, 2)
    w = torch.full((4, 2), 0.5, dtype=torch.float32, device=dev)
    out = api.moe_combine(y, slots, w)
    torch.cuda.synchronize(dev)
    assert np.array_equal(out.float().cpu().numpy(), np.ones((4, 64), np.float32))
