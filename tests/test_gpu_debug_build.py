"""The debug build (-DPOETX_DEBUG: every TMA and bulk copy checked before it
is issued) on a layer step that reaches every kernel family of the b = 256
bf16 path: no copy fails a check, and the results are bit-identical to the
release build's (the checks never touch the arithmetic).  Each build runs in
its own process, since the package loads one library per process."""
import os
import subprocess
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r"""
import os, sys
import numpy as np
import torch
sys.path.insert(0, os.environ["POETX_ROOT"])
sys.path.insert(0, os.path.join(os.environ["POETX_ROOT"], "tests"))
from orthogonal_equivalence_b200 import build as pbuild
pbuild.build(debug=os.environ.get("POETX_DEBUG") == "1")
import orthogonal_equivalence_b200 as px
import poetx_inputs as pi
from gpu_util import dev, make_layer

px.poetx_device_error()
out = {}
# a: P side with G_P folded, R side fused; b: both folds; c: P side fused
# (T <= m); d: input-centric with T > m, n (both sides fused)
F = px.POETX_FOLD_ALL
for tag, (m, n, T, fold) in {"a": (512, 1024, 1000, F), "b": (1024, 512, 2000, F), "c": (1024, 512, 700, F),
                             "d": (1024, 512, 2000, 0)}.items():
    inp = pi.layer_inputs(pi.CONFIGS["block8b"], layer=0, T=T, m=m, n=n, b=256)
    L = make_layer(inp, fold)
    x, dz = dev(inp.x, "bf16"), dev(inp.dz, "bf16")
    z, saved = L.forward(x, save_xg=True)
    dx, dqR, dqP = L.backward(x, saved, dz)
    z2, _ = L.forward(x, save=False)
    dx2, dqR2, dqP2 = L.backward(x, None, dz)
    newR, newP = pi.merge_perms(pi.CONFIGS["block8b"], 0, 1, m, n)
    L.merge(torch.from_numpy(newR).cuda(), torch.from_numpy(newP).cuda())
    torch.cuda.synchronize()
    for k, t in {"z": z, "dx": dx, "dqR": dqR, "dqP": dqP, "z2": z2, "dx2": dx2, "dqR2": dqR2, "dqP2": dqP2,
                 "W": L.W}.items():
        out[tag + k] = t.detach().cpu().contiguous().view(torch.int16 if t.dtype == torch.bfloat16 else torch.int32).numpy()
out["error"] = np.array([px.poetx_device_error()])
np.savez(sys.argv[1], **out)
"""


def _run(tmp_path, debug: bool):
    path = str(tmp_path / ("debug.npz" if debug else "release.npz"))
    env = dict(os.environ, POETX_ROOT=ROOT, POETX_DEBUG="1" if debug else "0")
    r = subprocess.run([sys.executable, "-c", SCRIPT, path], env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    return dict(np.load(path))


def test_debug_build_checks_pass_and_match_release(tmp_path):
    rel = _run(tmp_path, False)
    dbg = _run(tmp_path, True)
    assert int(dbg["error"][0]) == 0, f"device error word {int(dbg['error'][0])} in the debug build"
    assert int(rel["error"][0]) == 0
    for k in rel:
        if k != "error":
            assert np.array_equal(rel[k], dbg[k]), k
