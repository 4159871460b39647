"""The problems of a call split over several calls (as over ranks) with the bh_offset option give the same
output, bit for bit, as one call over all of them; a call keyed at offset 0 for the same problems does not.

"HyperAttention: Long-context Attention in Near-Linear Time" (research-map summary, "Approach"): every
(batch, head) problem is hashed, sorted and attended on its own, so a split needs no data exchange.
"""
import numpy as np
import pytest

from approximate_long_context_b200 import binding
from approximate_long_context_b200 import shard
from approximate_long_context_b200 import workload as wl

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

G = 5

CASES = [
    # name, n, d, block, m, r, causal, base, dtype, kernel
    ("tc_level", 2048, 64, 256, 256, 8, False, 0, "bf16", "auto"),
    ("simt_level", 1024, 64, 128, 64, 6, False, 0, "fp32", "auto"),
    ("tc_causal", 2048, 128, 256, 128, 7, True, 512, "bf16", "auto"),
]


def dev_tensor(a):
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(a).cuda()


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_split_calls_equal_one_call(case):
    _, n, d, block, m, r, causal, base, dtype, kernel = case
    Qh, Kh, Vh = wl.make_inputs(n, d, G, data_seed=0x5EED, dtype=dtype)
    Q, K, V = dev_tensor(Qh), dev_tensor(Kh), dev_tensor(Vh)
    kw = dict(n=n, d=d, block=block, m=m, r=r, causal=causal, seed=99)
    ha = binding.HyperAttention(0)
    try:
        def run(lo, hi, offset):
            O = torch.empty((hi - lo, n, d), dtype=torch.float32, device="cuda")
            ha.set_options(dtype=dtype, out_dtype="fp32", causal_base=base or 4096, kernel=kernel,
                           stream=torch.cuda.current_stream().cuda_stream, bh_offset=offset)
            ha.forward(Q[lo:hi].contiguous(), K[lo:hi].contiguous(), V[lo:hi].contiguous(), O, heads=hi - lo, **kw)
            torch.cuda.synchronize()
            assert ha.status() == 0, ha.last_error()
            return O.cpu()

        whole = run(0, G, 0)
        parts = []
        for rank in range(2):
            s = shard.shard_problems(G, 2, rank)
            parts.append(run(s.offset, s.offset + s.count, s.offset))
        assert torch.equal(torch.cat(parts), whole)
        # keyed at offset 0, problems 2.. draw other samples: the offset is what makes the split exact
        wrong = run(2, G, 0)
        assert not torch.equal(wrong, whole[2:])
    finally:
        ha.close()
