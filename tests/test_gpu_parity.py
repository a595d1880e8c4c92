"""GPU parity of libpoetx.so against the float64 oracle on the same seeded
inputs (POET-X write-up, sections 1-3 and the merge step).

Bars: permutation / frame / index work bit-exact; fp32 layers normwise max
error <= 1e-5; bf16 layers relative Frobenius error <= 1e-2 on z, dx, dqR, dqP
and the merged weight.  Reduced shapes keep every recipe of the workloads but
span several tiles with ragged token tails; the full-size workloads are
checked on sampled token rows and sampled blocks, in the launch configuration
the benchmark uses."""
import numpy as np
import pytest
import torch

import oracle
import orthogonal_equivalence_b200 as px
import poetx_inputs as pi
from orthogonal_equivalence_b200 import build as pbuild

from gpu_util import bits, check, dev, host64, make_layer, poetx_dtype

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def library():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    pbuild.build()
    px.lib()
    px.poetx_device_error()  # clear
    yield
    torch.cuda.synchronize()
    assert px.poetx_device_error() == 0, "a kernel recorded a device error (timeout or bad index)"


# (workload recipe, m, n, b, T[, fold]); None = the workload's own size.
# Without a fold entry the layer is evaluated input-centrically (fold 0), also
# where T > m, n; the cases with FOLD also take the weight-fold paths.
FOLD = px.POETX_FOLD_ALL
SMALL = [
    ("tiny", None, None, None, None),
    ("tiny", 192, 320, 64, 77),
    ("attn3b", 512, 512, 256, 300),
    ("up8b", 512, 1792, 256, 200),
    ("down13b", 1536, 1024, 512, 130),
    ("block8b", 1024, 256, 256, 257),
    ("block8b", 256, 768, 256, 1),
    ("block8b", 512, 1024, 256, 1000),   # >= 4 token tiles: block-resident G path
    ("down13b", 1024, 1536, 512, 777),
    ("down13b", 1024, 512, 512, 2000),   # T > m, n, input-centric at b = 512
    ("attn3b", 256, 384, 128, 1000),     # T > m, n, input-centric at b = 128
    ("block8b", 512, 256, 256, 2000),    # T > m, n, input-centric at b = 256 (fused bdg on both sides)
    ("down13b", 1024, 512, 512, 2000, FOLD),   # T > m, n: both weight folds at b = 512
    ("attn3b", 256, 384, 128, 1000, FOLD),     # T > m, n: both weight folds at b = 128
    ("block8b", 512, 256, 256, 2000, FOLD),    # T > m, n: both weight folds at b = 256
]

# One layer case per b at the triangle scale where leaving out the Q^4 or the
# 2Q^3 term of G misses the bf16 bar by >= 3x (tests/test_parity_sigma.py
# proves it on the oracle for these shapes).
SIGMA_LAYERS = [("block8b", 192, 320, 64, 300), ("attn3b", 256, 384, 128, 1000), ("attn3b", 512, 512, 256, 300),
                ("down13b", 1024, 1536, 512, 130), ("block8b", 512, 256, 256, 2000, FOLD)]


def _inputs(name, m, n, b, T, *fold, layer=0, **kw):
    return pi.layer_inputs(pi.CONFIGS[name], layer=layer, T=T, m=m, n=n, b=b, **kw)


def _fold(case):
    return case[5] if len(case) > 5 else 0


def _oracle_all(inp):
    W0 = inp.W0lin64.T
    GR = oracle.cnp_blocks(inp.qR, inp.b)
    GP = oracle.cnp_blocks(inp.qP, inp.b)
    z = oracle.forward(inp.x64, W0, inp.permR, GR, inp.permP, GP)
    dX, dGR, dGP = oracle.backward(inp.x64, W0, inp.permR, GR, inp.permP, GP, inp.dz64)
    return z, dX, oracle.cnp_backward(inp.qR, inp.b, dGR), oracle.cnp_backward(inp.qP, inp.b, dGP), GR, GP


def _run(L, inp):
    x = dev(inp.x, inp.dtype)
    dz = dev(inp.dz, inp.dtype)
    z, y = L.forward(x)
    dx, dqR, dqP = L.backward(x, y, dz)
    torch.cuda.synchronize()
    return z, y, dx, dqR, dqP


@pytest.mark.parametrize("case", SMALL, ids=lambda c: "-".join(str(v) for v in c))
def test_layer_forward_backward_parity(case):
    inp = _inputs(*case)
    L = make_layer(inp, _fold(case))
    z, _, dx, dqR, dqP = _run(L, inp)
    zo, dxo, dqRo, dqPo, _, _ = _oracle_all(inp)
    check(host64(z), zo, inp.dtype, "z")
    check(host64(dx), dxo, inp.dtype, "dx")
    check(host64(dqR), dqRo, inp.dtype, "dqR")
    check(host64(dqP), dqPo, inp.dtype, "dqP")


def _skew_from_packed(p, b):
    # packed upper triangles [nblk][b(b-1)/2] (row-major over i < j) -> [nblk][b][b], lower part zero
    out = np.zeros((p.shape[0], b, b))
    iu = np.triu_indices(b, 1)
    out[:, iu[0], iu[1]] = p
    return out


def _tilewise(a, o, what, tile=32, bar=3e-2):
    # relative Frobenius error of every 32 x 32 tile of every block (tiles whose
    # reference is all zero, i.e. the empty lower tiles of a packed triangle,
    # must be zero too), so that one wrong tile cannot hide in the whole-block norm
    nblk, b, _ = o.shape
    t = min(tile, b)
    for k in range(nblk):
        for I in range(0, b, t):
            for J in range(0, b, t):
                at, ot = a[k, I:I + t, J:J + t], o[k, I:I + t, J:J + t]
                no = np.linalg.norm(ot)
                if no == 0:
                    assert np.all(at == 0), f"{what}: block {k} tile ({I}, {J}) should be empty"
                    continue
                e = np.linalg.norm(at - ot) / no
                assert e <= bar, f"{what}: block {k} tile ({I}, {J}) relative error {e:.3e} > {bar}"


@pytest.mark.parametrize("case", SIGMA_LAYERS, ids=lambda c: "-".join(str(v) for v in c))
def test_layer_parity_at_discriminating_sigma(case):
    inp = _inputs(*case, sigma_q=pi.PARITY_SIGMA[case[3]])
    L = make_layer(inp, _fold(case))
    z, _, dx, dqR, dqP = _run(L, inp)
    zo, dxo, dqRo, dqPo, _, _ = _oracle_all(inp)
    check(host64(z), zo, inp.dtype, "z")
    check(host64(dx), dxo, inp.dtype, "dx")
    check(host64(dqR), dqRo, inp.dtype, "dqR")
    check(host64(dqP), dqPo, inp.dtype, "dqP")


# sigma None: the workloads' scale 0.01; "parity": pi.PARITY_SIGMA[b], where
# every term of G shows through the bar
@pytest.mark.parametrize("dtype,b,nblk,sigma", [("fp32", 64, 8, None), ("bf16", 256, 5, None),
                                                ("bf16", 512, 3, None), ("bf16", 64, 9, None), ("fp32", 6, 4, None),
                                                ("bf16", 256, 5, "parity"), ("bf16", 512, 3, "parity"),
                                                ("bf16", 128, 4, "parity"), ("bf16", 64, 9, "parity"),
                                                ("fp32", 64, 8, "parity")])
def test_cnp_build_and_backward_parity(dtype, b, nblk, sigma):
    g = np.random.Generator(np.random.PCG64(1000 + b + nblk))
    scale = pi.PARITY_SIGMA[b] if sigma == "parity" else 0.01
    q = (g.standard_normal((nblk, b * (b - 1) // 2)) * scale).astype(np.float32)
    dG = g.standard_normal((nblk, b, b)).astype(np.float32)
    pd = poetx_dtype(dtype)
    td = torch.bfloat16 if dtype == "bf16" else torch.float32
    qd = torch.from_numpy(q).cuda()
    G = torch.empty((nblk, b, b), dtype=td, device="cuda")
    nb = px.poetx_cnp_workspace_bytes(nblk, b, pd)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    px.poetx_cnp_build(nblk, b, qd, pd, G, ws, nb)
    dq = torch.empty_like(qd)
    px.poetx_cnp_backward(nblk, b, qd, torch.from_numpy(dG).cuda(), dq, 0, pd, ws, nb)
    torch.cuda.synchronize()
    Go = oracle.cnp_blocks(q, b)
    dqo = oracle.cnp_backward(q, b, dG.astype(np.float64))
    check(host64(G), Go, dtype, "G")
    check(host64(dq), dqo, dtype, "dq")
    if dtype == "bf16":
        # G rounded to bf16 alone leaves up to ~1.2% per tile of G - I at sigma 0.01
        _tilewise(host64(G) - np.eye(b), Go - np.eye(b), "G - I", bar=5e-2)
        _tilewise(_skew_from_packed(host64(dq), b), _skew_from_packed(dqo, b), "dq")
    # accumulate adds onto what is there
    px.poetx_cnp_backward(nblk, b, qd, torch.from_numpy(dG).cuda(), dq, 1, pd, ws, nb)
    torch.cuda.synchronize()
    check(host64(dq), 2 * dqo, dtype, "dq accumulated")


@pytest.mark.parametrize("sigma", [0.01, pi.PARITY_SIGMA[256]])
def test_cnp_full_batch_of_the_8b_block(sigma):
    """The 8B block's batched CNP size (320 blocks of b = 256: several blocks
    per pair of SMs): build and backward on sampled blocks against the oracle,
    a sub-batch gives the same bits as the full batch, and accumulating adds
    exactly the plain result."""
    nblk, b = 320, 256
    g = np.random.Generator(np.random.PCG64(4242))
    q = (g.standard_normal((nblk, b * (b - 1) // 2)) * sigma).astype(np.float32)
    dG = g.standard_normal((nblk, b, b)).astype(np.float32)
    qd, dGd = torch.from_numpy(q).cuda(), torch.from_numpy(dG).cuda()
    G = torch.empty((nblk, b, b), dtype=torch.bfloat16, device="cuda")
    nb = px.poetx_cnp_workspace_bytes(nblk, b, px.POETX_BF16)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    px.poetx_cnp_build(nblk, b, qd, px.POETX_BF16, G, ws, nb)
    dq = torch.full_like(qd, float("nan"))
    px.poetx_cnp_backward(nblk, b, qd, dGd, dq, 0, px.POETX_BF16, ws, nb)
    # blocks 147..149 alone (one block per pair)
    sub_q, sub_dG = qd[147:150].contiguous(), dGd[147:150].contiguous()
    sub_G = torch.empty((3, b, b), dtype=torch.bfloat16, device="cuda")
    sub_dq = torch.empty_like(sub_q)
    px.poetx_cnp_build(3, b, sub_q, px.POETX_BF16, sub_G, ws, nb)
    px.poetx_cnp_backward(3, b, sub_q, sub_dG, sub_dq, 0, px.POETX_BF16, ws, nb)
    acc = dq.clone()
    px.poetx_cnp_backward(nblk, b, qd, dGd, acc, 1, px.POETX_BF16, ws, nb)
    torch.cuda.synchronize()
    assert np.array_equal(bits(sub_G), bits(G[147:150])) and np.array_equal(bits(sub_dq), bits(dq[147:150]))
    assert np.array_equal(bits(acc), bits(2 * dq))
    for t in [0, 1, 73, 74, 147, 148, 221, 295, 319]:
        Go = oracle.cnp_blocks(q[t:t + 1], b)
        dqo = oracle.cnp_backward(q[t:t + 1], b, dG[t:t + 1].astype(np.float64))
        check(host64(G[t]), Go[0], "bf16", f"G[{t}]")
        check(host64(dq[t]), dqo[0], "bf16", f"dq[{t}]")
        _tilewise(host64(G[t:t + 1]) - np.eye(b), Go - np.eye(b), f"G[{t}] - I", bar=5e-2)
        _tilewise(_skew_from_packed(host64(dq[t:t + 1]), b), _skew_from_packed(dqo, b), f"dq[{t}]")


@pytest.mark.parametrize("name", ["block8b", "tiny"])
def test_batched_build_of_several_layers(name):
    # one CNP build for the R and P blocks of several layers equals the
    # per-layer builds and the oracle
    cfg = pi.CONFIGS[name]
    shapes = [(512, 256), (256, 768), (1024, 512)] if name == "block8b" else [(128, 192), (256, 64)]
    inps = [_inputs(name, m, n, None, 8, layer=k) for k, (m, n) in enumerate(shapes)]
    Ls = [make_layer(i) for i in inps]
    ref = [(L.GR.clone(), L.GP.clone()) for L in Ls]
    for L in Ls:
        L.GR.zero_()
        L.GP.zero_()
    px.LayerGroup(Ls).build()
    torch.cuda.synchronize()
    for L, inp, (gr, gp) in zip(Ls, inps, ref):
        assert np.array_equal(bits(L.GR), bits(gr)) and np.array_equal(bits(L.GP), bits(gp))
        check(host64(L.GR), oracle.cnp_blocks(inp.qR, inp.b), inp.dtype, "GR")
        check(host64(L.GP), oracle.cnp_blocks(inp.qP, inp.b), inp.dtype, "GP")


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_zero_q_gives_identity_and_plain_linear(dtype):
    name = "tiny" if dtype == "fp32" else "attn3b"
    b = 64 if dtype == "fp32" else 256
    inp = _inputs(name, 512, 768, b, 150, zero_q=True)
    L = make_layer(inp)
    eye = np.broadcast_to(np.eye(b), (512 // b, b, b))
    assert np.array_equal(host64(L.GR), eye)
    assert np.array_equal(host64(L.GP), np.broadcast_to(np.eye(b), (768 // b, b, b)))
    z, _ = L.forward(dev(inp.x, dtype))
    torch.cuda.synchronize()
    check(host64(z), inp.x64 @ inp.W0lin64.T, dtype, "z with Q = 0")


@pytest.mark.parametrize("dtype,m,n", [("fp32", 192, 320), ("bf16", 1024, 768), ("bf16", 14336, 256)])
def test_frame_import_export_bit_exact(dtype, m, n):
    name = "tiny" if dtype == "fp32" else "block8b"
    inp = _inputs(name, m, n, 64, 4)
    L = make_layer(inp)
    torch.cuda.synchronize()
    want = oracle.to_frame(inp.W0lin, inp.permR, inp.permP)
    assert np.array_equal(bits(L.W), want.view(np.uint16 if dtype == "bf16" else np.uint32))
    back = L.export_weight()
    torch.cuda.synchronize()
    assert np.array_equal(bits(back), inp.W0lin.view(np.uint16 if dtype == "bf16" else np.uint32))


def _merge_check(inp, merge_index=1, cfg=None, layer=0):
    L = make_layer(inp)
    x = dev(inp.x, inp.dtype)
    z_before, _ = L.forward(x, save=False)
    if cfg is None:
        cfg = pi.CONFIGS["tiny"] if inp.dtype == "fp32" else pi.CONFIGS["down13b"]
    newR, newP = pi.merge_perms(cfg, layer, merge_index, inp.m, inp.n)
    L.merge(torch.from_numpy(newR).cuda(), torch.from_numpy(newP).cuda())
    W_nat = L.export_weight()
    torch.cuda.synchronize()
    GR = oracle.cnp_blocks(inp.qR, inp.b)
    GP = oracle.cnp_blocks(inp.qP, inp.b)
    W_o = oracle.merge(inp.W0lin64.T, inp.permR, GR, inp.permP, GP)   # natural m x n
    check(host64(W_nat), W_o.T, inp.dtype, "merged weight")
    assert not np.any(host64(L.qR)) and not np.any(host64(L.qP))
    assert np.array_equal(host64(L.GR), np.broadcast_to(np.eye(inp.b), L.GR.shape))
    assert np.array_equal(bits(L.permR), newR.view(np.uint32))
    # function preservation: same z before and after the merge
    z_after, _ = L.forward(x, save=False)
    torch.cuda.synchronize()
    check(host64(z_after), host64(z_before), inp.dtype, "z after merge")
    return L


@pytest.mark.parametrize("case", [("tiny", None, None, None, 64), ("down13b", 1536, 1024, 512, 64),
                                  ("attn3b", 768, 512, 256, 33)], ids=lambda c: c[0])
def test_merge_parity(case):
    _merge_check(_inputs(*case))


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_merge_with_zero_q_is_exact_reframing(dtype):
    name = "tiny" if dtype == "fp32" else "attn3b"
    b = 64 if dtype == "fp32" else 256
    inp = _inputs(name, 512, 768, b, 8, zero_q=True)
    L = make_layer(inp)
    newR, newP = pi.merge_perms(pi.CONFIGS[name], 0, 1, 512, 768)
    L.merge(torch.from_numpy(newR).cuda(), torch.from_numpy(newP).cuda())
    torch.cuda.synchronize()
    want = oracle.to_frame(inp.W0lin, newR, newP)
    assert np.array_equal(bits(L.W), want.view(np.uint16 if dtype == "bf16" else np.uint32))


@pytest.mark.parametrize("m,n", [(36864, 256), (256, 40960)], ids=["wide-m", "wide-n"])
def test_wide_rows_take_the_one_row_permutation(m, n):
    # bf16 rows wider than the double-buffered permutation holds with its index
    # table (about 34K columns) go through the kernels that stage one row at a
    # time: frame bit-exact, layer and merge against the oracle
    inp = _inputs("up8b", m, n, 256, 72)
    L = make_layer(inp)
    torch.cuda.synchronize()
    want = oracle.to_frame(inp.W0lin, inp.permR, inp.permP)
    assert np.array_equal(bits(L.W), want.view(np.uint16))
    z, _, dx, dqR, dqP = _run(L, inp)
    zo, dxo, dqRo, dqPo, _, _ = _oracle_all(inp)
    check(host64(z), zo, "bf16", "z (wide)")
    check(host64(dx), dxo, "bf16", "dx (wide)")
    check(host64(dqR), dqRo, "bf16", "dqR (wide)")
    check(host64(dqP), dqPo, "bf16", "dqP (wide)")
    _merge_check(inp)


def test_empty_and_single_token():
    inp = _inputs("attn3b", 512, 512, 256, 1)
    L = make_layer(inp)
    x = dev(inp.x, "bf16")
    z = torch.empty((0, 512), dtype=torch.bfloat16, device="cuda")
    L.forward(x[:0], z=z)          # T = 0: no-op
    dqR = torch.full_like(L.qR, 7.0)
    dqP = torch.full_like(L.qP, 7.0)
    L.backward(x[:0], z, z, need_dx=True, dx=torch.empty((0, 512), dtype=torch.bfloat16, device="cuda"),
               dqR=dqR, dqP=dqP)
    torch.cuda.synchronize()
    assert not torch.any(dqR) and not torch.any(dqP)
    z1, _, dx1, dqR1, dqP1 = _run(L, inp)
    zo, dxo, dqRo, dqPo, _, _ = _oracle_all(inp)
    check(host64(z1), zo, "bf16", "z T=1")
    check(host64(dx1), dxo, "bf16", "dx T=1")
    check(host64(dqR1), dqRo, "bf16", "dqR T=1")


@pytest.mark.parametrize("case", [("up8b", 512, 1024, 256, 700), ("tiny", 192, 320, 64, 77)], ids=lambda c: c[0])
def test_saved_xg_backward_matches_regather(case):
    # the forward's optional Xg = x[:, permR] gives the backward the same result
    # (bit for bit) as gathering x again
    inp = _inputs(*case)
    L = make_layer(inp)
    x, dz = dev(inp.x, inp.dtype), dev(inp.dz, inp.dtype)
    z1, s1 = L.forward(x)
    z2, s2 = L.forward(x, save_xg=True)
    dx1, r1, p1 = L.backward(x, s1, dz)
    dx2, r2, p2 = L.backward(None, s2, dz)
    torch.cuda.synchronize()
    assert np.array_equal(bits(z1), bits(z2))
    assert np.array_equal(bits(s2.xg), bits(x)[:, inp.permR])
    for a, b in ((dx1, dx2), (r1, r2), (p1, p2)):
        assert np.array_equal(bits(a), bits(b))


@pytest.mark.parametrize("case", [("block8b", 512, 256, 256, 2000), ("up8b", 256, 768, 256, 1500),
                                  ("attn3b", 512, 512, 256, 300), ("block8b", 512, 256, 256, 2000, FOLD),
                                  ("up8b", 256, 768, 256, 1500, FOLD)], ids=lambda c: f"{c[0]}-{c[4]}-{_fold(c)}")
def test_forward_without_saving(case):
    """A forward that saves nothing (inference, or the recomputing backward's
    forward): input-centric by default; with POETX_FOLD_WEIGHT_CENTRIC and
    T above 6nm/(2m+4n) the whole layer is one GEMM with the weight folded
    into the natural frames; z against the oracle and against the forward that
    saves Y (which takes the token-row path)."""
    inp = _inputs(*case)
    L = make_layer(inp, _fold(case))
    x = dev(inp.x, inp.dtype)
    z_nosave, _ = L.forward(x, save=False)
    z_save, _ = L.forward(x)
    torch.cuda.synchronize()
    zo, _, _, _, _, _ = _oracle_all(inp)
    check(host64(z_nosave), zo, inp.dtype, "z (nothing saved)")
    check(host64(z_nosave), host64(z_save), inp.dtype, "z (nothing saved vs saved)")


@pytest.mark.parametrize("case", [("up8b", 512, 1024, 256, 700), ("tiny", 192, 320, 64, 77),
                                  ("block8b", 512, 256, 256, 600),
                                  ("block8b", 512, 256, 256, 600, FOLD)],   # T > m, n: both weight folds
                         ids=lambda c: f"{c[0]}-{c[4]}-{_fold(c)}")
def test_recomputing_backward_mem_variant(case):
    # the "mem" variant keeps nothing from the forward: the backward recomputes
    # Y from x and must match the saved-Y backward bit for bit
    inp = _inputs(*case)
    L = make_layer(inp, _fold(case))
    x, dz = dev(inp.x, inp.dtype), dev(inp.dz, inp.dtype)
    _, saved = L.forward(x)
    dx1, r1, p1 = L.backward(x, saved, dz)
    dx2, r2, p2 = L.backward(x, None, dz)
    torch.cuda.synchronize()
    for a, b in ((dx1, dx2), (r1, r2), (p1, p2)):
        assert np.array_equal(bits(a), bits(b))
    _, dxo, dqRo, dqPo, _, _ = _oracle_all(inp)
    check(host64(dx2), dxo, inp.dtype, "dx (mem variant)")
    check(host64(r2), dqRo, inp.dtype, "dqR (mem variant)")
    check(host64(p2), dqPo, inp.dtype, "dqP (mem variant)")


@pytest.mark.parametrize("name,m,n,b,T", [("up8b", 512, 768, 256, 300), ("tiny", 192, 320, 64, 77)],
                         ids=["bf16", "fp32"])
def test_xq_weight_quantization_and_layer_parity(name, m, n, b, T):
    # POET-XQ: codes and scales bit-exact against the oracle (both decide them
    # in float32), the dequantized weight bit-exact, and the layer run on the
    # dequantized weight against the oracle run on the same weight
    inp = _inputs(name, m, n, b, T)
    L = make_layer(inp)
    stored = host64(L.W)                      # exact stored (frame) weight values
    L.quantize_weight()
    z, saved = L.forward(dev(inp.x, inp.dtype))
    dx, dqR, dqP = L.backward(dev(inp.x, inp.dtype), saved, dev(inp.dz, inp.dtype))
    torch.cuda.synchronize()
    codes, scale = oracle.quantize_rows(stored)
    assert np.array_equal(L.Wq.cpu().numpy(), codes)
    assert np.array_equal(L.Wscale.cpu().numpy().view(np.uint32), scale.view(np.uint32))
    deq = oracle.dequantize_rows(codes, scale)
    want = oracle.round_to_bf16(deq) if inp.dtype == "bf16" else deq.astype(np.float64)
    assert np.array_equal(host64(L.W), want)
    W0 = oracle.from_frame(want, inp.permR, inp.permP).T
    GR, GP = oracle.cnp_blocks(inp.qR, inp.b), oracle.cnp_blocks(inp.qP, inp.b)
    check(host64(z), oracle.forward(inp.x64, W0, inp.permR, GR, inp.permP, GP), inp.dtype, "z (XQ)")
    dxo, dqRo, dqPo = oracle.layer_backward(inp.x64, W0, inp.permR, inp.qR, inp.permP, inp.qP, inp.b, inp.dz64)
    check(host64(dx), dxo, inp.dtype, "dx (XQ)")
    check(host64(dqR), dqRo, inp.dtype, "dqR (XQ)")
    check(host64(dqP), dqPo, inp.dtype, "dqP (XQ)")


def test_adamw_step_parity():
    g = np.random.Generator(np.random.PCG64(77))
    n = 10007                                  # not a multiple of 4: vector body + scalar tail
    q = (g.standard_normal(n) * 0.01).astype(np.float32)
    qd, md, vd = torch.from_numpy(q.copy()).cuda(), torch.zeros(n, device="cuda"), torch.zeros(n, device="cuda")
    qo, mo, vo = q.astype(np.float64), np.zeros(n), np.zeros(n)
    for step in range(1, 4):
        grad = g.standard_normal(n).astype(np.float32)
        px.poetx_adamw_step(n, qd, torch.from_numpy(grad).cuda(), md, vd, 1e-3, 0.9, 0.95, 1e-8, 0.1, step)
        qo, mo, vo = oracle.adamw_step(qo, grad, mo, vo, 1e-3, 0.9, 0.95, 1e-8, 0.1, step)
    torch.cuda.synchronize()
    check(host64(qd), qo, "fp32", "q after 3 AdamW steps")
    check(host64(md), mo, "fp32", "first moment")
    check(host64(vd), vo, "fp32", "second moment")


def test_fused_optimizer_step_and_rebuild():
    # AdamW on the flattened packed triangles of two layers, then the batched
    # CNP rebuild: q and G of each layer against the oracle
    inps = [_inputs("block8b", 512, 256, 256, 8, layer=0), _inputs("block8b", 256, 768, 256, 8, layer=1)]
    Ls = [make_layer(i) for i in inps]
    grp = px.LayerGroup(Ls)
    flat_q = grp.flatten_params()
    g = np.random.Generator(np.random.PCG64(5))
    grads = (g.standard_normal(flat_q.numel()) * 1e-2).astype(np.float32)
    grp.optimizer_step(torch.from_numpy(grads).cuda(), 1e-3, weight_decay=0.01)
    torch.cuda.synchronize()
    off = 0
    for L, inp in zip(Ls, inps):
        for name, q0 in (("qR", inp.qR), ("qP", inp.qP)):
            k = q0.size
            qo, _, _ = oracle.adamw_step(q0.ravel(), grads[off:off + k], np.zeros(k), np.zeros(k), 1e-3, 0.9, 0.95,
                                         1e-8, 0.01, 1)
            off += k
            q_gpu = getattr(L, name)
            check(host64(q_gpu).ravel(), qo, "fp32", f"{name} after the step")
            G = L.GR if name == "qR" else L.GP
            check(host64(G), oracle.cnp_blocks(host64(q_gpu), inp.b), "bf16", f"G rebuilt from {name}")


def test_backward_is_deterministic_and_accumulates():
    inp = _inputs("up8b", 512, 1024, 256, 700)
    L = make_layer(inp)
    x, dz = dev(inp.x, "bf16"), dev(inp.dz, "bf16")
    _, y = L.forward(x)
    _, a_R, a_P = L.backward(x, y, dz)
    _, b_R, b_P = L.backward(x, y, dz)
    torch.cuda.synchronize()
    assert np.array_equal(bits(a_R), bits(b_R)) and np.array_equal(bits(a_P), bits(b_P))
    acc_R, acc_P = a_R.clone(), a_P.clone()
    L.backward(x, y, dz, need_dx=False, dqR=acc_R, dqP=acc_P, accumulate=True)
    torch.cuda.synchronize()
    np.testing.assert_allclose(host64(acc_R), 2 * host64(a_R), rtol=1e-6, atol=0)


@pytest.mark.parametrize("case", [("up8b", 512, 1024, 256, 700), ("tiny", 192, 320, 64, 77),
                                  ("down13b", 1024, 1536, 512, 300)], ids=lambda c: c[0])
def test_dG_backward_and_batched_cnp_backward(case):
    """poetx_backward_dG: the token sums dG of both sides against the oracle's
    chain rule, and one poetx_cnp_backward over [dGR | dGP] gives the dq of
    poetx_backward bit for bit (same sums, same per-block arithmetic)."""
    inp = _inputs(*case)
    L = make_layer(inp)
    x, dz = dev(inp.x, inp.dtype), dev(inp.dz, inp.dtype)
    _, y = L.forward(x)
    b, nR, nP = inp.b, inp.m // inp.b, inp.n // inp.b
    dG = torch.full((nR + nP, b, b), float("nan"), dtype=torch.float32, device="cuda")
    dx_g = L.backward_dG(x, y, dz, dG[:nR], dG[nR:])
    dx, dqR, dqP = L.backward(x, y, dz)
    q = torch.cat([L.qR, L.qP])
    dq = torch.full_like(q, float("nan"))
    ws = torch.empty(px.poetx_cnp_workspace_bytes(nR + nP, b, L.dtype), dtype=torch.uint8, device="cuda")
    px.poetx_cnp_backward(nR + nP, b, q, dG, dq, 0, L.dtype, ws, ws.numel())
    torch.cuda.synchronize()
    assert np.array_equal(bits(dx_g), bits(dx))
    assert np.array_equal(bits(dq[:nR]), bits(dqR)) and np.array_equal(bits(dq[nR:]), bits(dqP))
    GR, GP = oracle.cnp_blocks(inp.qR, b), oracle.cnp_blocks(inp.qP, b)
    _, dGRo, dGPo = oracle.backward(inp.x64, inp.W0lin64.T, inp.permR, GR, inp.permP, GP, inp.dz64)
    check(host64(dG[:nR]), dGRo, inp.dtype, "dGR")
    check(host64(dG[nR:]), dGPo, inp.dtype, "dGP")
    # accumulate adds the same sums once more: exactly 2 dG
    acc = dG.clone()
    L.backward_dG(x, y, dz, acc[:nR], acc[nR:], need_dx=False, accumulate=True)
    torch.cuda.synchronize()
    assert np.array_equal(bits(acc), bits(2 * dG))


def test_batched_build_of_the_most_layers_one_call_takes():
    # 16 linears = 32 segments, the most one batched call takes: every
    # segment's G (its own output buffer) equals the per-layer build, and the
    # oracle on a few of them; one more linear is refused before any launch
    shapes = [(256, 256), (512, 256), (256, 512), (512, 512)] * 4
    inps = [_inputs("block8b", m, n, None, 8, layer=k) for k, (m, n) in enumerate(shapes)]
    Ls = [make_layer(i) for i in inps]
    ref = [(L.GR.clone(), L.GP.clone()) for L in Ls]
    for L in Ls:
        L.GR.fill_(float("nan"))
        L.GP.fill_(float("nan"))
    px.LayerGroup(Ls).build()
    torch.cuda.synchronize()
    for k, (L, inp, (gr, gp)) in enumerate(zip(Ls, inps, ref)):
        assert np.array_equal(bits(L.GR), bits(gr)) and np.array_equal(bits(L.GP), bits(gp)), f"layer {k}"
        if k in (0, 7, 15):
            check(host64(L.GR), oracle.cnp_blocks(inp.qR, inp.b), inp.dtype, f"GR of layer {k}")
            check(host64(L.GP), oracle.cnp_blocks(inp.qP, inp.b), inp.dtype, f"GP of layer {k}")
    extra = make_layer(_inputs("block8b", 256, 256, None, 8, layer=16))
    with pytest.raises(px.PoetxError):
        px.LayerGroup(Ls + [extra]).build()


def test_layer_group_batched_cnp_backward():
    """Several linears: backward_dG of each into one flat dG buffer, then one
    batched CNP backward into the flat dq, equals each layer's own dq."""
    shapes = [(512, 256), (256, 768), (1024, 512)]
    inps = [_inputs("block8b", m, n, 256, 300, layer=i) for i, (m, n) in enumerate(shapes)]
    layers = [make_layer(inp) for inp in inps]
    group = px.LayerGroup(layers)
    q = group.flatten_params()
    dG = group.dG_buffer()
    dq = torch.full_like(q, float("nan"))
    want = []
    for L, inp, (dGR, dGP) in zip(layers, inps, group.dG_views(dG)):
        x, dz = dev(inp.x, "bf16"), dev(inp.dz, "bf16")
        _, y = L.forward(x)
        L.backward_dG(x, y, dz, dGR, dGP, need_dx=False)
        _, dqR, dqP = L.backward(x, y, dz, need_dx=False)
        want += [dqR.flatten(), dqP.flatten()]
    group.cnp_backward(dG, dq)
    torch.cuda.synchronize()
    assert np.array_equal(bits(dq), bits(torch.cat(want)))
    for L, inp, (dqR, dqP) in zip(layers, inps, [(want[2 * i], want[2 * i + 1]) for i in range(len(layers))]):
        _, dqRo, dqPo = oracle.layer_backward(inp.x64, inp.W0lin64.T, inp.permR, inp.qR, inp.permP, inp.qP, inp.b,
                                              inp.dz64)
        check(host64(dqR).reshape(dqRo.shape), dqRo, "bf16", "dqR")
        check(host64(dqP).reshape(dqPo.shape), dqPo, "bf16", "dqP")


def test_check_perm_and_errors():
    n = 1000
    perm = torch.from_numpy(pi.permutation(5, n)).cuda()
    ok = torch.zeros(1, dtype=torch.int32, device="cuda")
    nb = px.poetx_check_perm_workspace_bytes(n)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    px.poetx_check_perm(perm, n, ok, ws, nb)
    torch.cuda.synchronize()
    assert ok.item() == 1
    bad = perm.clone()
    bad[3] = bad[4]
    px.poetx_check_perm(bad, n, ok, ws, nb)
    torch.cuda.synchronize()
    assert ok.item() == 0
    bad[3] = n + 5
    px.poetx_check_perm(bad, n, ok, ws, nb)
    torch.cuda.synchronize()
    assert ok.item() == 0
    # a workspace that is too small is refused before anything is queued
    inp = _inputs("attn3b", 512, 512, 256, 16)
    L = make_layer(inp)
    with pytest.raises(px.PoetxError) as e:
        px.poetx_forward(L.abi(), 16, dev(inp.x, "bf16"), torch.empty((16, 512), dtype=torch.bfloat16,
                                                                       device="cuda"), None, None, ws, 64)
    assert e.value.status == 5


# ------------------------------------------------------------------ full-size workloads
FULL = ["attn3b", "up8b", "down13b", "block8b"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled_parity(name):
    cfg = pi.CONFIGS[name]
    for layer in range(len(cfg.layers)):
        inp = pi.layer_inputs(cfg, layer)
        L = make_layer(inp)
        z, _, dx, dqR, dqP = _run(L, inp)
        rows = pi.random_token_rows(7 + layer, inp.T, 48)
        W0 = inp.W0lin64.T
        GR = oracle.cnp_blocks(inp.qR, inp.b)
        GP = oracle.cnp_blocks(inp.qP, inp.b)
        zo = oracle.forward(inp.x64[rows], W0, inp.permR, GR, inp.permP, GP)
        dxo, _, _ = oracle.backward(inp.x64[rows], W0, inp.permR, GR, inp.permP, GP, inp.dz64[rows])
        rows_t = torch.from_numpy(rows).cuda()
        check(host64(z[rows_t]), zo, "bf16", f"{name}[{layer}] z rows")
        check(host64(dx[rows_t]), dxo, "bf16", f"{name}[{layer}] dx rows")
        nR, nP = inp.m // inp.b, inp.n // inp.b
        for side, nblk, q, dq in (("R", nR, inp.qR, dqR), ("P", nP, inp.qP, dqP)):
            blocks = sorted({0, nblk // 2, nblk - 1})
            dGs = oracle.grad_G_blocks(inp.x64, W0, inp.permR, GR, inp.permP, GP, inp.dz64, side, blocks)
            dqo = np.stack([oracle.cnp_backward_block(q[j], inp.b, g) for j, g in zip(blocks, dGs)])
            check(host64(dq)[blocks], dqo, "bf16", f"{name}[{layer}] dq{side} blocks {blocks}")
        del L, z, dx, dqR, dqP
        torch.cuda.empty_cache()


def test_full_size_merge_down13b():
    inp = pi.layer_inputs(pi.CONFIGS["down13b"], 0, T=256)
    _merge_check(inp)


def test_full_size_merge_of_all_block8b_linears():
    """The merge step of the 8B block: each of its seven linears at full size
    (q, k, v, o, gate, up, down) merged with its own new permutations; merged
    weight against the oracle's R W0 P, q = 0, G = I, and z unchanged."""
    cfg = pi.CONFIGS["block8b"]
    for layer in range(len(cfg.layers)):
        inp = pi.layer_inputs(cfg, layer, T=64)
        L = _merge_check(inp, cfg=cfg, layer=layer)
        del L
        torch.cuda.empty_cache()
