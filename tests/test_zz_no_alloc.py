"""poetx_cnp_build_fixed: the CNP build for callers that cannot allocate
device memory (its scratch is a fixed array inside the library).  It must
give the same G as poetx_cnp_build with a caller workspace, call after call,
and refuse requests larger than its fixed scratch.  This file is collected
last so a failure here never hides the results of the other GPU tests."""
import numpy as np
import pytest
import torch

import orthogonal_equivalence_b200 as px
from orthogonal_equivalence_b200 import build as pbuild

from gpu_util import check, host64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,b,nblk", [("bf16", 256, 24), ("fp32", 64, 12), ("bf16", 512, 7)])
def test_fixed_scratch_build_matches_workspace_build(dtype, b, nblk):
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    pbuild.build()
    pd = px.POETX_BF16 if dtype == "bf16" else px.POETX_FP32
    td = torch.bfloat16 if dtype == "bf16" else torch.float32
    nb = px.poetx_cnp_workspace_bytes(nblk, b, pd)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    for call in range(2):  # two calls in a row share the fixed scratch
        g = np.random.Generator(np.random.PCG64(7000 + 10 * b + call))
        q = torch.from_numpy((g.standard_normal((nblk, b * (b - 1) // 2)) * 0.01).astype(np.float32)).cuda()
        G_ref = torch.empty((nblk, b, b), dtype=td, device="cuda")
        G_fix = torch.full((nblk, b, b), float("nan"), dtype=td, device="cuda")
        px.poetx_cnp_build(nblk, b, q, pd, G_ref, ws, nb)
        px.poetx_cnp_build_fixed(nblk, b, q, pd, G_fix)
        torch.cuda.synchronize()
        check(host64(G_fix), host64(G_ref), dtype, f"fixed-scratch G, call {call}")


def test_fixed_scratch_refuses_oversized_requests():
    pbuild.build()
    q = torch.zeros((32, 256 * 255 // 2), dtype=torch.float32, device="cuda")
    G = torch.empty((32, 256, 256), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(px.PoetxError) as e:
        px.poetx_cnp_build_fixed(32, 256, q, px.POETX_BF16, G)
    assert e.value.status == 5
