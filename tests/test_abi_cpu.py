"""Host-side checks of the C-ABI library (no GPU needed): it loads, exports every symbol the header
declares, its host-side draws equal the oracle's bit for bit, and handle creation fails cleanly without
a device."""
import ctypes
import os
import re

import numpy as np
import pytest

from approximate_long_context_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    import __graft_entry__  # noqa: F401  (build helper)
    from approximate_long_context_b200 import build
    build.build()
    return binding.lib()


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"^\s*(?:HA_API\s+)?(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(hyper_attn_[a-z_0-9]+)\s*\(", text, re.M)
    return sorted(set(names))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) >= 13
    for name in names:
        assert hasattr(lib, name), name
    assert sorted(binding.EXPORTS) == sorted(n for n in names if n in binding.EXPORTS)
    assert set(names) <= set(binding.EXPORTS)


def test_debug_build_exports_every_declared_symbol(lib):
    """The HA_DEBUG build (bounds-checked index reads in the tensor-core kernels) is the same library."""
    from approximate_long_context_b200 import build
    path = build.build(debug=True)
    dbg = ctypes.CDLL(path)
    for name in declared_functions():
        assert hasattr(dbg, name), name


def test_version(lib):
    assert lib.hyper_attn_version() >= 100


def test_create_without_device_fails_cleanly(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    h = ctypes.c_void_p()
    rc = lib.hyper_attn_create(ctypes.byref(h), 0)
    assert rc in (binding.HA_ERR_CUDA, binding.HA_ERR_UNSUPPORTED)
    assert not h.value


@pytest.mark.parametrize("seed,d,r,bh,n,m,causal,base", [
    (1234, 64, 6, 1, 1024, 64, False, 0),
    (1237, 64, 8, 3, 131072, 256, False, 0),
    (1236, 128, 7, 2, 32768, 256, True, 4096),
    (99, 128, 16, 1, 4096, 0, False, 0),
    (7, 64, 0, 2, 2048, 17, True, 256),
])
def test_draws_match_oracle(lib, ora, seed, d, r, bh, n, m, causal, base):
    P, S = binding.draw(seed, d, r, bh, n, m, causal=causal, base=base)
    assert np.array_equal(P.view(np.uint32), ora.draw_projection(seed, d, r).view(np.uint32))
    L, nodes = binding.levels(n, causal, base) if causal else (0, 1)
    for b in range(bh):
        for k in range(nodes):
            node = k + 1
            depth = node.bit_length() - 1
            N = n >> (depth + 1) if causal else n
            assert np.array_equal(S[b, k], ora.draw_samples(seed, b, node, N, m))


def test_levels(lib):
    assert binding.levels(32768, True, 4096) == (3, 7)
    assert binding.levels(524288, True, 8192) == (6, 63)
    assert binding.levels(4096, True, 8192) == (0, 0)
    with pytest.raises(binding.HAError):
        binding.levels(3 * 4096, True, 4096)
    with pytest.raises(binding.HAError):
        binding.draw(1, 64, 4, 1, 100, 101, causal=False)


def test_options_struct_mirrors_the_header(tmp_path):
    """The binding's ctypes Options has the C struct's size and field offsets (compiled here with gcc)."""
    fields = [f for f, _ in binding.Options._fields_]
    src = tmp_path / "layout.c"
    body = "".join(f'    printf("{f} %zu\\n", offsetof(ha_options, {f}));\n' for f in fields)
    src.write_text('#include <stddef.h>\n#include <stdio.h>\n#include "hyper_attn.h"\nint main(void) {\n'
                   '    printf("size %zu\\n", sizeof(ha_options));\n' + body + "    return 0;\n}\n")
    exe = tmp_path / "layout"
    import subprocess
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    out = dict(line.split() for line in subprocess.run([str(exe)], capture_output=True, text=True,
                                                       check=True).stdout.splitlines())
    assert int(out["size"]) == ctypes.sizeof(binding.Options)
    for f in fields:
        assert int(out[f]) == getattr(binding.Options, f).offset, f


def test_default_options_match_the_binding_defaults(lib):
    o = binding.Options()
    lib.hyper_attn_default_options(ctypes.byref(o))
    assert (o.dtype, o.out_dtype, o.batch, o.causal_base, o.kernel, o.debug_captures, o.bh_offset,
            o.test_stall_ms, o.sampling) == (0, -1, 1, 4096, 0, 0, 0, 0, 0)


def test_binding_selects_the_debug_build():
    """HA_LIBRARY=debug makes the binding load the HA_DEBUG build (in a fresh process); unset, the regular one."""
    import subprocess
    import sys
    code = "from approximate_long_context_b200 import binding; print(binding.LIB_PATH)"
    env = dict(os.environ, HA_LIBRARY="debug")
    out = subprocess.run([sys.executable, "-c", code], env=env, cwd=ROOT, capture_output=True, text=True,
                         check=True).stdout.strip()
    assert out.endswith("libhyper_attn_debug.so")
    env.pop("HA_LIBRARY")
    out = subprocess.run([sys.executable, "-c", code], env=env, cwd=ROOT, capture_output=True, text=True,
                         check=True).stdout.strip()
    assert out.endswith("libhyper_attn.so")
