"""Failure detection on the GPU without a GPU fault: a bounded wait that
nothing satisfies (an mbarrier no thread arrives on) gives up after its
limit, records its bit in the device error word and returns; the host reads
the status and the same process and CUDA context then run a normal layer step
that matches the oracle."""
import numpy as np
import pytest
import torch

import oracle
import orthogonal_equivalence_b200 as px
import poetx_inputs as pi
from orthogonal_equivalence_b200 import build as pbuild

from gpu_util import check, dev, host64, make_layer

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_the_context_stays_usable():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    pbuild.build()
    px.lib()
    px.poetx_device_error()                      # clear
    out = torch.full((2,), -1, dtype=torch.int64, device="cuda")
    limit_us = 50_000
    px.poetx_selftest_wait_timeout(limit_us, out)
    torch.cuda.synchronize()
    arrived, waited_ns = out.tolist()
    assert arrived == 0
    assert limit_us * 1000 <= waited_ns < 5_000_000_000
    assert px.poetx_device_error() == 1          # bit 1: a bounded wait timed out
    assert px.poetx_device_error() == 0          # read and cleared
    # the context is still usable: one layer step against the oracle
    inp = pi.layer_inputs(pi.CONFIGS["attn3b"], 0, T=300, m=512, n=512, b=256)
    L = make_layer(inp)
    x, dz = dev(inp.x, "bf16"), dev(inp.dz, "bf16")
    z, y = L.forward(x)
    dx, dqR, dqP = L.backward(x, y, dz)
    torch.cuda.synchronize()
    GR, GP = oracle.cnp_blocks(inp.qR, inp.b), oracle.cnp_blocks(inp.qP, inp.b)
    W0 = inp.W0lin64.T
    check(host64(z), oracle.forward(inp.x64, W0, inp.permR, GR, inp.permP, GP), "bf16", "z after the timeout")
    dxo, dqRo, dqPo = oracle.layer_backward(inp.x64, W0, inp.permR, inp.qR, inp.permP, inp.qP, inp.b, inp.dz64)
    check(host64(dx), dxo, "bf16", "dx after the timeout")
    check(host64(dqR), dqRo, "bf16", "dqR after the timeout")
    assert px.poetx_device_error() == 0


def test_selftest_rejects_bad_arguments():
    pbuild.build()
    out = torch.zeros(2, dtype=torch.int64, device="cuda")
    for bad in (0, 1_000_001):
        with pytest.raises(px.PoetxError) as e:
            px.poetx_selftest_wait_timeout(bad, out)
        assert e.value.status == 1
