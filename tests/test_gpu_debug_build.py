"""The HA_DEBUG build on valid inputs: no bounds report, and the same results as the regular build.

The HA_DEBUG build (libhyper_attn_debug.so) checks every row index its tensor-core kernels read from a
permutation or a sample list; an index out of range would set a status bit (reported by hyper_attn_status) and
be replaced by row 0 instead of being read out of bounds. On valid inputs it must report nothing and compute
exactly what the regular build computes. Each build runs in a process of its own (HA_LIBRARY selects it).
"""
import os
import subprocess
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r"""
import sys, numpy as np, torch
sys.path.insert(0, sys.argv[1])
from approximate_long_context_b200 import binding, workload as wl
out = sys.argv[2]
res = {}
for name, n, d, bh, block, m, r, causal, base in [("level_d64", 4096, 64, 2, 256, 256, 8, False, 4096),
                                                 ("level_d128", 2048, 128, 2, 128, 200, 7, False, 4096),
                                                 ("causal_d128", 4096, 128, 2, 256, 128, 7, True, 1024)]:
    Qh, Kh, Vh = wl.make_inputs(n, d, bh, data_seed=21, dtype="bf16", sinks=causal)
    t = lambda a: torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    Q, K, V = t(Qh), t(Kh), t(Vh)
    O = torch.empty((bh, n, d), dtype=torch.float32, device="cuda")
    ha = binding.HyperAttention(0)
    ha.set_options(dtype="bf16", out_dtype="fp32", causal_base=base, kernel="tc",
                   stream=torch.cuda.current_stream().cuda_stream)
    ha.forward(Q, K, V, O, n=n, d=d, heads=bh, block=block, m=m, r=r, causal=causal, seed=77)
    torch.cuda.synchronize()
    assert ha.status() == 0, ha.last_error()
    res[name] = O.cpu().numpy()
    ha.close()
np.savez(out, **res)
"""


def run(lib, tmp_path):
    out = str(tmp_path / f"{lib}.npz")
    env = dict(os.environ)
    if lib == "debug":
        env["HA_LIBRARY"] = "debug"
    else:
        env.pop("HA_LIBRARY", None)
    subprocess.run([sys.executable, "-c", SCRIPT, ROOT, out], env=env, check=True, timeout=600)
    return np.load(out)


def test_debug_build_matches_regular_build(tmp_path):
    from approximate_long_context_b200 import build
    build.build(debug=True)
    reg = run("regular", tmp_path)
    dbg = run("debug", tmp_path)
    for name in reg.files:
        assert np.array_equal(reg[name], dbg[name]), name
