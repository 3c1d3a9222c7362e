"""GPU parity of the biased baselines (QSGD with rounding to the nearest level, and the scaled
sign) and of QSGD with l2 scaling with the oracle: codes, level tables, residuals and averages bit for bit, through the fused
and the unfused calls, with and without error feedback and clipping, on special and short
buckets; the quantization error within the 1e-12 bound of its binary64 summation order."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

import gradient_quantization_communication_b200.gq as G
import oracle as O
from gpu_harness import compare_steps, configs, run_gpu_fused, run_oracle_fused
from gradient_quantization_communication_b200 import synth

BIASED = [("qsgd_nearest", 2), ("qsgd_nearest", 3), ("qsgd_nearest", 5), ("qsgd_nearest", 15),
          ("qsgd_nearest", 16), ("signsgd", 2), ("qsgd_l2", 3), ("qsgd_l2", 5), ("qsgd_l2", 16)]


def _grads(n, W, steps, seed):
    rng = np.random.default_rng(seed)
    return [[(rng.laplace(0, 1e-3, n)).astype(np.float32) for _ in range(W)] for _ in range(steps)]


@pytest.mark.parametrize("scheme,levels", BIASED)
@pytest.mark.parametrize("d", [128, 256, 512])
def test_fused(scheme, levels, d):
    n, W, steps = 9 * d + 37, 3, 3
    cg, co = configs(scheme, levels, d, W, True, 0.0, 42, n)
    g = _grads(n, W, steps, seed=d + levels)
    compare_steps(run_gpu_fused(cg, steps, g), run_oracle_fused(co, steps, g), co, "%s-%d d=%d" % (scheme, levels, d))


@pytest.mark.parametrize("scheme,levels", [("qsgd_nearest", 3), ("qsgd_nearest", 15), ("signsgd", 2), ("qsgd_l2", 3)])
@pytest.mark.parametrize("ef,clip", [(True, 0.0), (False, 0.0), (True, 2.5), (False, 2.5)])
def test_unfused_clip_and_no_error_feedback(scheme, levels, ef, clip):
    d = 512
    n, W, steps = 5 * d + 100, 2, 2
    cg, co = configs(scheme, levels, d, W, ef, clip, 1, n)
    g = _grads(n, W, steps, seed=levels + int(ef) + int(clip))
    compare_steps(run_gpu_fused(cg, steps, g, unfused=True), run_oracle_fused(co, steps, g), co, "unfused")
    compare_steps(run_gpu_fused(cg, steps, g), run_oracle_fused(co, steps, g), co, "fused")


@pytest.mark.parametrize("kind", ["zero", "constant", "negconst", "grid", "twovalue", "tiny", "spike", "subnormal"])
@pytest.mark.parametrize("scheme,levels", [("qsgd_nearest", 5), ("signsgd", 2), ("qsgd_l2", 3)])
def test_special_buckets(kind, scheme, levels):
    d, W = 512, 2
    parts = [synth.special_bucket(kind, d, seed=w).numpy() for w in range(W)]
    rng = np.random.default_rng(0)
    g = [[np.concatenate([parts[w], (rng.standard_normal(d + 40) * 1e-3).astype(np.float32)]) for w in range(W)]]
    n = g[0][0].size
    cg, co = configs(scheme, levels, d, W, True, 0.0, 3, n)
    compare_steps(run_gpu_fused(cg, 1, g), run_oracle_fused(co, 1, g), co, kind)


@pytest.mark.parametrize("n", [1, 3, 127, 129, 500])
@pytest.mark.parametrize("scheme,levels", [("qsgd_nearest", 5), ("signsgd", 2), ("qsgd_l2", 5)])
def test_short_vectors(n, scheme, levels):
    for d in (128, 512):
        cg, co = configs(scheme, levels, d, 2, True, 0.0, 9, n)
        g = _grads(n, 2, 2, seed=n)
        compare_steps(run_gpu_fused(cg, 2, g), run_oracle_fused(co, 2, g), co, "n=%d d=%d" % (n, d))


@pytest.mark.parametrize("scheme,levels", [("qsgd_nearest", 5), ("qsgd_nearest", 3), ("signsgd", 2), ("qsgd_l2", 3)])
@pytest.mark.parametrize("d", [128, 512])
def test_quant_error(scheme, levels, d):
    rng = np.random.default_rng(d + levels)
    n = 6 * d - 13
    g = (rng.laplace(0, 1e-3, n)).astype(np.float32)
    r = (rng.standard_normal(n) * 1e-4).astype(np.float32)
    for ef, clip in [(True, 0.0), (False, 0.0), (True, 2.5)]:
        cg, co = configs(scheme, levels, d, 1, ef, clip, 42, n)
        with G.Plan(cg) as plan:
            out = torch.zeros(3, dtype=torch.float64, device="cuda")
            G.gq_quant_error(plan.handle, 3, 7, torch.from_numpy(g).cuda(),
                             torch.from_numpy(r).cuda() if ef else None, out)
            assert G.gq_plan_status(plan.handle) == G.GQ_OK
            mine = out.cpu().numpy()
        ref = O.quant_error(co, 3, 7, g, r if ef else None)
        assert np.all(np.abs(mine - ref) <= 1e-12 * np.abs(ref) + 1e-300), (ef, clip, mine, ref)
        if scheme != "qsgd_l2":  # deterministic rounding: the expected error is the realised one
            assert abs(mine[0] - mine[2]) <= 1e-12 * abs(mine[2]) + 1e-300


def test_no_randomness():
    """The seed and the step do not change the codes (only the residual history does)."""
    d, n = 512, 4 * 512
    g = _grads(n, 1, 1, seed=5)
    outs = []
    for seed in (0, 12345):
        cg, _ = configs("qsgd_nearest", 5, d, 1, False, 0.0, seed, n)
        outs.append(run_gpu_fused(cg, 1, g)[0][2][0])
    assert np.array_equal(outs[0], outs[1])


# INT8: the QSGD family with 129 .. 256 levels and 8-bit codes (255 levels with nearest
# rounding: the symmetric integers -127 .. 127 times m / 127)
INT8 = [("qsgd_nearest", 255), ("qsgd", 255), ("qsgd_nearest", 256), ("qsgd", 129), ("qsgd_l2", 255)]


@pytest.mark.parametrize("scheme,levels", INT8)
@pytest.mark.parametrize("d", [128, 512, 2048])
def test_int8_fused_and_unfused(scheme, levels, d):
    if d > 512 and scheme != "qsgd":
        pytest.skip("nearest rounding and l2 scaling run on the register path only (d <= 512)")
    n, W, steps = 5 * d + 37, 3, 2
    cg, co = configs(scheme, levels, d, W, True, 0.0, 42, n)
    g = _grads(n, W, steps, seed=d + levels)
    o = run_oracle_fused(co, steps, g)
    compare_steps(run_gpu_fused(cg, steps, g), o, co, "%s-%d d=%d" % (scheme, levels, d))
    compare_steps(run_gpu_fused(cg, steps, g, unfused=True), o, co, "unfused %s-%d d=%d" % (scheme, levels, d))


@pytest.mark.parametrize("kind", ["zero", "constant", "spike", "subnormal"])
def test_int8_special_buckets(kind):
    d, W = 512, 2
    parts = [synth.special_bucket(kind, d, seed=w).numpy() for w in range(W)]
    rng = np.random.default_rng(1)
    g = [[np.concatenate([parts[w], (rng.standard_normal(d + 40) * 1e-3).astype(np.float32)]) for w in range(W)]]
    n = g[0][0].size
    cg, co = configs("qsgd_nearest", 255, d, W, True, 0.0, 3, n)
    compare_steps(run_gpu_fused(cg, 1, g), run_oracle_fused(co, 1, g), co, kind)


def test_int8_level_counts_between_17_and_128_are_rejected():
    for levels in (17, 64, 128, 257):
        assert G.gq_config_check(G.gq_config("qsgd_nearest", levels, 512, 1, True, 0.0, 0, 1024)) == G.GQ_ERR_INVALID
    assert G.gq_config_check(G.gq_config("orq", 255, 512, 1, True, 0.0, 0, 1024)) == G.GQ_ERR_INVALID
