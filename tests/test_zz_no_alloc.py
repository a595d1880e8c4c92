"""poetx_cnp_build_fixed: the CNP build for callers that cannot allocate
device memory (its scratch is a fixed array inside the library).  On the same
inputs it runs the same kernels as poetx_cnp_build with a caller workspace, so
its G must carry the same bits, call after call (the calls share the array),
and match the oracle; requests larger than its fixed scratch are refused.
This file is collected last so a failure here never hides the results of the
other GPU tests."""
import numpy as np
import pytest
import torch

import oracle
import orthogonal_equivalence_b200 as px
from orthogonal_equivalence_b200 import build as pbuild

from gpu_util import bits, check, host64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def library():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    pbuild.build()
    px.lib()


# (dtype, b, nblk): the b = 256 bf16 pair kernel (191 is the largest batch its
# 24 MiB scratch holds: 128 KiB of bf16 Q per block), the tf32 GEMM chain at
# b = 512 (7 is the largest), the fp32 chain
CASES = [("bf16", 256, 24), ("bf16", 256, 191), ("fp32", 64, 12), ("bf16", 512, 7)]


@pytest.mark.parametrize("dtype,b,nblk", CASES)
def test_fixed_scratch_build_matches_workspace_build(dtype, b, nblk):
    pd = px.POETX_BF16 if dtype == "bf16" else px.POETX_FP32
    td = torch.bfloat16 if dtype == "bf16" else torch.float32
    nb = px.poetx_cnp_workspace_bytes(nblk, b, pd)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    for call in range(2):  # two calls in a row share the fixed scratch
        g = np.random.Generator(np.random.PCG64(7000 + 10 * b + nblk + call))
        q_host = (g.standard_normal((nblk, b * (b - 1) // 2)) * 0.02).astype(np.float32)
        q = torch.from_numpy(q_host).cuda()
        G_ref = torch.empty((nblk, b, b), dtype=td, device="cuda")
        G_fix = torch.full((nblk, b, b), float("nan"), dtype=td, device="cuda")
        px.poetx_cnp_build(nblk, b, q, pd, G_ref, ws, nb)
        px.poetx_cnp_build_fixed(nblk, b, q, pd, G_fix)
        torch.cuda.synchronize()
        assert np.array_equal(bits(G_fix), bits(G_ref)), f"fixed-scratch G differs from the workspace build, call {call}"
        for t in sorted({0, nblk // 2, nblk - 1}):
            check(host64(G_fix[t]), oracle.cnp_blocks(q_host[t:t + 1], b)[0], dtype, f"G[{t}], call {call}")


@pytest.mark.parametrize("dtype,b,nblk", [("bf16", 256, 192), ("bf16", 512, 8)])
def test_fixed_scratch_refuses_oversized_requests(dtype, b, nblk):
    pd = px.POETX_BF16 if dtype == "bf16" else px.POETX_FP32
    q = torch.zeros((nblk, b * (b - 1) // 2), dtype=torch.float32, device="cuda")
    G = torch.full((nblk, b, b), 7.0, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(px.PoetxError) as e:
        px.poetx_cnp_build_fixed(nblk, b, q, pd, G)
    assert e.value.status == 5
    torch.cuda.synchronize()
    assert bool(torch.all(G == 7.0)), "a refused call must queue nothing"
