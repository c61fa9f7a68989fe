"""Failure detection on the GPU without a GPU fault: a device wait that nothing
completes runs out after a short limit, the kernel records
GSA_ERR_DEVICE_TIMEOUT in the context's error word and returns, the host reads
the code through gsa_get_status, and the context keeps working."""
import pytest
import torch

import sparse_global_attention_b200 as gsa
from gsa_inputs import GSAConfig, make_inputs

pytestmark = pytest.mark.gpu

CFG = GSAConfig("expire_small", 2, 8, 8, 8, 8, 1, 2, 64, 4, 3, "bf16")


def test_expired_wait_is_reported_and_the_context_stays_usable():
    x = {k: v.cuda() for k, v in make_inputs(CFG, seed=3).items()}
    layer = gsa.GSALayer.from_workload(CFG)
    try:
        ref = layer.forward(x)
        torch.cuda.synchronize()
        assert gsa.gsa_get_status(layer.ctx) == gsa.GSA_OK

        gsa.gsa_debug_expire_wait(layer.ctx, 20000)          # 20 ms, nothing ever arrives
        assert gsa.gsa_get_status(layer.ctx) == 6            # GSA_ERR_DEVICE_TIMEOUT, read and cleared
        assert gsa.gsa_get_status(layer.ctx) == gsa.GSA_OK

        again = layer.forward(x)                               # the context still computes the same layer
        torch.cuda.synchronize()
        assert gsa.gsa_get_status(layer.ctx) == gsa.GSA_OK
        for k in ref:
            assert torch.equal(ref[k], again[k]), k
    finally:
        layer.close()


def test_expire_wait_rejects_limits_out_of_range():
    layer = gsa.GSALayer.from_workload(CFG)
    try:
        for bad in (0, 1000001):
            with pytest.raises(gsa.GSAError):
                gsa.gsa_debug_expire_wait(layer.ctx, bad)
    finally:
        layer.close()
