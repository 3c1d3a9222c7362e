"""GPU parity of gq_quant_error (expected / realised quantization error) with the oracle.

The per-element terms are bit-identical on both sides (same fit, same draws, same binary64
operations); only the order of the binary64 summation differs, hence the 1e-12 relative
bound."""
import numpy as np
import pytest
import torch

import gradient_quantization_communication_b200.gq as G
import oracle as O
from gpu_harness import configs

pytestmark = pytest.mark.gpu


def _gpu_err(cg, worker, step, g, r=None):
    with G.Plan(cg) as plan:
        out = torch.zeros(3, dtype=torch.float64, device="cuda")
        gd = torch.from_numpy(g).cuda()
        rd = torch.from_numpy(r).cuda() if r is not None else None
        G.gq_quant_error(plan.handle, worker, step, gd, rd, out)
        assert G.gq_plan_status(plan.handle) == G.GQ_OK
        if rd is not None:   # the residual is only read
            assert np.array_equal(rd.cpu().numpy(), r)
        return out.cpu().numpy()


@pytest.mark.parametrize("scheme,levels", [("orq", 5), ("orq", 3), ("orq", 9), ("qsgd", 5), ("terngrad", 3),
                                           ("bingrad_b", 2), ("bingrad_pb", 2)])
@pytest.mark.parametrize("d", [128, 512, 2048, 8192])
def test_quant_error_matches_oracle(scheme, levels, d):
    rng = np.random.default_rng(d + levels)
    nbk = 6 if d <= 2048 else 2
    n = nbk * d - 13
    g = (rng.laplace(0, 1e-3, n)).astype(np.float32)
    r = (rng.standard_normal(n) * 1e-4).astype(np.float32)
    for ef, clip in [(True, 0.0), (False, 0.0), (True, 2.5)]:
        cg, co = configs(scheme, levels, d, 1, ef, clip, 42, n)
        mine = _gpu_err(cg, 3, 7, g, r if ef else None)
        ref = O.quant_error(co, 3, 7, g, r if ef else None)
        assert np.all(np.abs(mine - ref) <= 1e-12 * np.abs(ref) + 1e-300), (ef, clip, mine, ref)


def test_quant_error_is_deterministic_and_launch_independent():
    rng = np.random.default_rng(1)
    n = 333 * 512 + 77
    g = (rng.standard_normal(n) * 1e-3).astype(np.float32)
    cg, _ = configs("orq", 5, 512, 1, False, 0.0, 42, n)
    a = _gpu_err(cg, 0, 0, g)
    b = _gpu_err(cg, 0, 0, g)
    assert np.array_equal(a, b)
    # a different stream (and an unrelated kernel running before) changes nothing
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        torch.randn(1 << 20, device="cuda").sum()
        c = _gpu_err(cg, 0, 0, g)
    assert np.array_equal(a, c)


def test_quant_error_empty():
    cg, _ = configs("orq", 5, 512, 1, False, 0.0, 1, 0)
    with G.Plan(cg) as plan:
        out = torch.full((3,), 7.0, dtype=torch.float64, device="cuda")
        G.gq_quant_error(plan.handle, 0, 0, None, None, out)
        torch.cuda.synchronize()
        assert out.cpu().tolist() == [0.0, 0.0, 0.0]
