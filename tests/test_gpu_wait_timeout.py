"""Failure detection without a GPU fault: a bounded in-kernel wait on an
mbarrier that nothing arrives on gives up, sets DF_DEVERR_TIMEOUT in the
call's error word and returns; the context stays usable afterwards."""

import pytest
import torch

from dual_flow_transformer_b200 import _lib as L
from dual_flow_transformer_b200 import api

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_the_context_survives(cuda_device):
    lib = L.load()
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    st = lib.dualflow_selftest_wait_timeout(err.data_ptr(), None)
    assert st == L.DF_OK
    torch.cuda.synchronize()
    assert int(err.item()) == L.DF_DEVERR_TIMEOUT
    # the same process and context go on to run a normal call correctly
    x = torch.randn(4, 256, device=cuda_device).to(torch.bfloat16)
    y = api.rmsnorm(x)
    torch.cuda.synchronize()
    ref = (x.float() / torch.sqrt((x.float() ** 2).mean(dim=1, keepdim=True) + 1e-5))
    assert torch.allclose(y.float(), ref, atol=2e-2, rtol=1e-2)

