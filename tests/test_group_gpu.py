"""GPU parity of the group kernels: buckets of 1024 .. 32768 values spread over d / 512 warps
(one CTA, or a cluster of 2 .. 8 CTAs from d = 8192), for ORQ, QSGD (2 .. 255 levels) and
TernGrad, fused and unfused, with and without error feedback and messages.  The cases hold
several groups per CTA, more buckets than resident groups (grid-stride), a ragged last bucket
(taken by the CTA kernel) and none.  Everything must equal the oracle bit for bit."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu

from gpu_harness import compare_steps, configs, run_gpu_fused, run_oracle_fused


def _grads(n, W, steps, seed, dist="t3"):
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(steps):
        row = []
        for _ in range(W):
            x = rng.standard_t(3, n) * 1e-3 if dist == "t3" else rng.laplace(0, 1e-3, n)
            row.append(x.astype(np.float32))
        out.append(row)
    return out


CASES = [("orq", 5), ("orq", 2), ("orq", 16), ("qsgd", 5), ("qsgd", 255), ("terngrad", 3)]
SIZES = [1024, 2048, 4096, 8192, 16384, 32768]


@pytest.mark.parametrize("scheme,levels", CASES)
@pytest.mark.parametrize("d", SIZES)
def test_group_fused(scheme, levels, d):
    nbk = max(2, 49152 // d)
    n = nbk * d + (d // 3 if d < 32768 else 0)
    W, steps = 3, 2
    cg, co = configs(scheme, levels, d, W, True, 0.0, 31, n)
    g = _grads(n, W, steps, seed=d + levels)
    compare_steps(run_gpu_fused(cg, steps, g), run_oracle_fused(co, steps, g), co, "%s-%d d=%d" % (scheme, levels, d))


@pytest.mark.parametrize("scheme,levels", [("orq", 5), ("qsgd", 5), ("terngrad", 3)])
@pytest.mark.parametrize("d", [2048, 8192, 32768])
def test_group_unfused(scheme, levels, d):
    n = 3 * d + 100
    cg, co = configs(scheme, levels, d, 2, True, 0.0, 8, n)
    g = _grads(n, 2, 2, seed=5 * d + levels, dist="laplace")
    compare_steps(run_gpu_fused(cg, 2, g, unfused=True), run_oracle_fused(co, 2, g), co, "unfused d=%d" % d)


@pytest.mark.parametrize("scheme,levels", [("orq", 5), ("qsgd", 5)])
@pytest.mark.parametrize("d", [4096, 16384])
def test_group_without_error_feedback(scheme, levels, d):
    n, W = 3 * d, 8
    cg, co = configs(scheme, levels, d, W, False, 0.0, 4, n)
    g = _grads(n, W, 1, seed=d, dist="laplace")
    o = run_oracle_fused(co, 1, g)
    compare_steps(run_gpu_fused(cg, 1, g), o, co, "no-ef d=%d" % d)
    a = run_gpu_fused(cg, 1, g, with_msgs=False)
    assert np.array_equal(a[0][0].view(np.uint32), o[0][0].view(np.uint32))


@pytest.mark.parametrize("d,nbk", [(1024, 3000), (8192, 400)])
def test_group_more_buckets_than_resident_groups(d, nbk):
    n = nbk * d + 5
    cg, co = configs("orq", 5, d, 2, True, 0.0, 77, n)
    g = _grads(n, 2, 1, seed=nbk)
    compare_steps(run_gpu_fused(cg, 1, g), run_oracle_fused(co, 1, g), co, "d=%d x %d" % (d, nbk))
