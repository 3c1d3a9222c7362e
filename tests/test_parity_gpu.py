"""GPU parity: the CUDA library against the CPU oracle, element by element.

Expected agreement is bit-exact for codes, level tables, residuals and averages: every fit
decision is taken from exact integer data on both sides and every floating-point operation
is a single IEEE rounding.  (The acceptance bar is looser: codes bit-exact for QSGD, TernGrad
and BinGrad, >= 99.99 % for ORQ, average within 1e-5 relative L2, residuals within 1e-6.)
Sizes span several buckets and a ragged tail; edge cases cover constant, zero, grid-aligned,
tiny and subnormal buckets, n < d, a single element, clipping, no error feedback, and every
bucket size 128 .. 32768.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

from gpu_harness import compare_steps, configs, run_gpu_fused, run_oracle_fused
from gradient_quantization_communication_b200 import synth


def _grads(n, W, steps, seed, dist="laplace"):
    rng = np.random.default_rng(seed)
    out = []
    for t in range(steps):
        row = []
        for w in range(W):
            if dist == "laplace":
                x = rng.laplace(0, 1e-3, n)
            elif dist == "t3":
                x = rng.standard_t(3, n) * 1e-3
            else:
                x = rng.standard_normal(n) * 1e-3
            row.append(x.astype(np.float32))
        out.append(row)
    return out


SCHEMES = [("qsgd", 5), ("qsgd", 2), ("qsgd", 9), ("terngrad", 3), ("bingrad_b", 2), ("bingrad_pb", 2),
           ("orq", 2), ("orq", 3), ("orq", 4), ("orq", 5), ("orq", 9), ("orq", 16), ("qsgd", 16)]


@pytest.mark.parametrize("scheme,levels", SCHEMES)
@pytest.mark.parametrize("d", [128, 256, 512])
def test_fused_register_path(scheme, levels, d):
    n, W, steps = 9 * d + 37, 3, 2
    cg, co = configs(scheme, levels, d, W, True, 0.0, 42, n)
    g = _grads(n, W, steps, seed=d + levels)
    compare_steps(run_gpu_fused(cg, steps, g), run_oracle_fused(co, steps, g), co, "%s-%d d=%d" % (scheme, levels, d))


@pytest.mark.parametrize("scheme,levels", [("qsgd", 5), ("terngrad", 3), ("bingrad_b", 2), ("bingrad_pb", 2),
                                           ("orq", 3), ("orq", 5), ("orq", 9)])
@pytest.mark.parametrize("d", [128, 512])
def test_unfused_matches_oracle(scheme, levels, d):
    n, W, steps = 7 * d + 40, 2, 2
    cg, co = configs(scheme, levels, d, W, True, 0.0, 7, n)
    g = _grads(n, W, steps, seed=3 * d + levels, dist="t3")
    compare_steps(run_gpu_fused(cg, steps, g, unfused=True), run_oracle_fused(co, steps, g), co, "unfused")


@pytest.mark.parametrize("scheme,levels", [("qsgd", 5), ("orq", 5), ("orq", 3), ("bingrad_b", 2), ("bingrad_pb", 2),
                                           ("terngrad", 3)])
@pytest.mark.parametrize("d", [1024, 2048, 8192, 32768])
def test_large_buckets(scheme, levels, d):
    nbk = {1024: 5, 2048: 3, 8192: 2, 32768: 2}[d]
    if scheme == "bingrad_pb" and d >= 8192:
        nbk = 1          # the oracle's exhaustive pair search is slow on big buckets
    n, W, steps = nbk * d - 37 if nbk > 1 else d - 37, 2, 2
    cg, co = configs(scheme, levels, d, W, True, 0.0, 11, n)
    g = _grads(n, W, steps, seed=d + levels, dist="t3")
    compare_steps(run_gpu_fused(cg, steps, g), run_oracle_fused(co, steps, g), co, "%s-%d d=%d" % (scheme, levels, d))


@pytest.mark.parametrize("scheme,levels", [("qsgd", 5), ("orq", 3), ("orq", 5), ("bingrad_b", 2), ("bingrad_pb", 2)])
@pytest.mark.parametrize("d", [512, 2048])
def test_clip(scheme, levels, d):
    n, W, steps = 4 * d + 100, 2, 2
    cg, co = configs(scheme, levels, d, W, True, 2.5, 5, n)
    g = _grads(n, W, steps, seed=99, dist="t3")
    g[0][0][17] = 0.5   # an outlier the clip must catch
    compare_steps(run_gpu_fused(cg, steps, g), run_oracle_fused(co, steps, g), co, "clip")


@pytest.mark.parametrize("scheme,levels", [("qsgd", 5), ("orq", 5), ("bingrad_b", 2)])
@pytest.mark.parametrize("d", [128, 512, 2048])
def test_no_error_feedback(scheme, levels, d):
    n, W, steps = 6 * d + 3, 8, 1
    cg, co = configs(scheme, levels, d, W, False, 0.0, 1, n)
    g = _grads(n, W, steps, seed=5, dist="normal")
    compare_steps(run_gpu_fused(cg, steps, g), run_oracle_fused(co, steps, g), co, "no-ef")


@pytest.mark.parametrize("kind", ["zero", "constant", "negconst", "grid", "twovalue", "tiny", "spike", "subnormal"])
@pytest.mark.parametrize("scheme,levels", [("qsgd", 5), ("orq", 5), ("orq", 9), ("bingrad_b", 2), ("bingrad_pb", 2)])
@pytest.mark.parametrize("d", [512, 1024])
def test_special_buckets(kind, scheme, levels, d):
    W = 2
    parts = [synth.special_bucket(kind, d, seed=w).numpy() for w in range(W)]
    # a normal bucket after the special one, then a ragged tail
    rng = np.random.default_rng(0)
    g = [[np.concatenate([parts[w], (rng.standard_normal(d + 40) * 1e-3).astype(np.float32)]) for w in range(W)]]
    n = g[0][0].size
    cg, co = configs(scheme, levels, d, W, True, 0.0, 3, n)
    compare_steps(run_gpu_fused(cg, 1, g), run_oracle_fused(co, 1, g), co, kind)


@pytest.mark.parametrize("n", [1, 3, 4, 127, 129, 500])
@pytest.mark.parametrize("scheme,levels", [("orq", 5), ("qsgd", 3), ("bingrad_b", 2), ("bingrad_pb", 2)])
def test_short_vectors(n, scheme, levels):
    for d in (128, 512, 2048):
        cg, co = configs(scheme, levels, d, 2, True, 0.0, 9, n)
        g = _grads(n, 2, 2, seed=n)
        compare_steps(run_gpu_fused(cg, 2, g), run_oracle_fused(co, 2, g), co, "n=%d d=%d" % (n, d))


def test_fused_without_messages_matches():
    n, W = 20 * 512 + 5, 4
    cg, co = configs("orq", 5, 512, W, True, 0.0, 42, n)
    g = _grads(n, W, 2, seed=1)
    a = run_gpu_fused(cg, 2, g, with_msgs=False)
    o = run_oracle_fused(co, 2, g)
    for (ga, gr, _), (oa, orr, _) in zip(a, o):
        assert np.array_equal(ga.view(np.uint32), oa.view(np.uint32))
        assert all(np.array_equal(x, y) for x, y in zip(gr, orr))


@pytest.mark.parametrize("scheme,levels", [("orq", 5), ("qsgd", 5), ("bingrad_b", 2), ("bingrad_pb", 2)])
@pytest.mark.parametrize("d", [1024, 8192, 16384, 32768])
def test_large_buckets_fused_without_messages(scheme, levels, d):
    """One CTA walks the W workers of a bucket and keeps the running sum on chip: in shared
    memory up to d = 8192, in the average's own slice (L2) above; with and without messages
    the average and residuals equal the oracle's, including a ragged last bucket."""
    W = 5
    nbk = 1 if (scheme == "bingrad_pb" and d >= 8192) else 2
    n = nbk * d + (77 if d < 32768 else -300)
    cg, co = configs(scheme, levels, d, W, True, 0.0, 21, n)
    g = _grads(n, W, 2, seed=d + 7 * levels, dist="t3")
    o = run_oracle_fused(co, 2, g)
    for with_msgs in (False, True):
        a = run_gpu_fused(cg, 2, g, with_msgs=with_msgs)
        if with_msgs:
            compare_steps(a, o, co, "%s-%d d=%d" % (scheme, levels, d))
        for (ga, gr, _), (oa, orr, _) in zip(a, o):
            assert np.array_equal(ga.view(np.uint32), oa.view(np.uint32))
            assert all(np.array_equal(x, y) for x, y in zip(gr, orr))


def test_many_workers():
    n, W = 3 * 512 + 11, 64
    cg, co = configs("orq", 5, 512, W, True, 0.0, 2, n)
    g = _grads(n, W, 1, seed=64)
    compare_steps(run_gpu_fused(cg, 1, g), run_oracle_fused(co, 1, g), co, "W=64")


def test_empty_vector():
    import gradient_quantization_communication_b200.gq as G
    cg, _ = configs("orq", 5, 512, 2, True, 0.0, 1, 0)
    with G.Plan(cg) as plan:
        e = torch.empty(0, device="cuda")
        G.gq_fused_step(plan.handle, 0, [e, e], [e, e], None, e)
        assert G.gq_plan_status(plan.handle) == G.GQ_OK


def test_nonfinite_input_is_flagged():
    import gradient_quantization_communication_b200.gq as G
    for d in (512, 2048):
        n = 3 * d
        cg, _ = configs("orq", 5, d, 2, True, 0.0, 1, n)
        g = [torch.randn(n, device="cuda") * 1e-3 for _ in range(2)]
        g[1][d + 5] = float("nan")
        g[0][7] = float("inf")
        r = [torch.zeros(n, device="cuda") for _ in range(2)]
        with G.Plan(cg) as plan:
            msgs = [torch.zeros(plan.msg_bytes, dtype=torch.uint8, device="cuda") for _ in range(2)]
            avg = torch.zeros(n, device="cuda")
            G.gq_fused_step(plan.handle, 0, g, r, msgs, avg)
            assert G.gq_plan_status(plan.handle) == G.GQ_ERR_NONFINITE
            # the flag is cleared by reading it; clean input raises nothing
            g[1][d + 5] = 0.0
            g[0][7] = 0.0
            G.gq_fused_step(plan.handle, 1, g, [torch.zeros(n, device="cuda") for _ in range(2)], msgs, avg)
            assert G.gq_plan_status(plan.handle) == G.GQ_OK


def test_invalid_arguments_rejected():
    import gradient_quantization_communication_b200.gq as G
    cg, _ = configs("orq", 5, 512, 2, True, 0.0, 1, 1024)
    with G.Plan(cg) as plan:
        g = torch.zeros(1024, device="cuda")
        msg = torch.zeros(plan.msg_bytes, dtype=torch.uint8, device="cuda")
        with pytest.raises(G.GQError) as ei:   # residual required with error feedback on
            G.gq_encode(plan.handle, 0, 0, g, None, msg)
        assert ei.value.status == G.GQ_ERR_INVALID
        with pytest.raises(G.GQError):         # misaligned gradient
            G.gq_encode(plan.handle, 0, 0, g.data_ptr() + 4, g, msg)
        with pytest.raises(G.GQError):         # misaligned average
            G.gq_fused_step(plan.handle, 0, [g, g], [g.clone(), g.clone()], None, g.data_ptr() + 4)


def test_deterministic_repeat():
    """Two runs on the same inputs are bitwise identical (catches races in shared memory)."""
    n, W = 50 * 512 + 9, 4
    cg, _ = configs("orq", 5, 512, W, True, 0.0, 3, n)
    g = _grads(n, W, 2, seed=8)
    a = run_gpu_fused(cg, 2, g)
    b = run_gpu_fused(cg, 2, g)
    for (aa, ar, am), (ba, br, bm) in zip(a, b):
        assert np.array_equal(aa.view(np.uint32), ba.view(np.uint32))
        assert all(np.array_equal(x, y) for x, y in zip(am, bm))


def test_checkpoint_resume_is_bit_identical():
    """The only state is the residual and the step: 4 steps in one go equal 2 + save/restore + 2."""
    import gradient_quantization_communication_b200.gq as G
    n, W = 10 * 512 + 3, 2
    cg, _ = configs("orq", 3, 512, W, True, 0.0, 77, n)
    g = _grads(n, W, 4, seed=12)
    full = run_gpu_fused(cg, 4, g)
    with G.Plan(cg) as plan:
        r = [torch.zeros(n, device="cuda") for _ in range(W)]
        for t in range(2):
            G.gq_fused_step(plan.handle, t, [torch.from_numpy(x).cuda() for x in g[t]], r, None,
                            torch.empty(n, device="cuda"))
        saved = [x.cpu().clone() for x in r]
    with G.Plan(cg) as plan:
        r = [x.cuda() for x in saved]
        for t in range(2, 4):
            avg = torch.empty(n, device="cuda")
            G.gq_fused_step(plan.handle, t, [torch.from_numpy(x).cuda() for x in g[t]], r, None, avg)
            assert np.array_equal(avg.cpu().numpy().view(np.uint32), full[t][0].view(np.uint32))
        assert all(np.array_equal(x.cpu().numpy(), y) for x, y in zip(r, full[3][1]))


def _bingrad_buckets(kind, d, rng):
    """Buckets that stress BinGrad's split search: duplicates, gaps, heavy tails, huge dynamic
    range, narrow all-positive ranges (where the grid cannot separate the values) and
    distributions whose best split is far from the middle."""
    if kind == "integers":
        return rng.integers(-3, 4, d).astype(np.float32)
    if kind == "bimodal":
        x = np.concatenate([rng.normal(-1.0, 0.01, d // 2), rng.normal(2.0, 0.01, d - d // 2)])
        return (rng.permutation(x) * 1e-3).astype(np.float32)
    if kind == "cauchy":
        return (rng.standard_cauchy(d) * 1e-4).astype(np.float32)
    if kind == "dynamic":
        return (np.sign(rng.standard_normal(d)) * 10.0 ** rng.uniform(-30, 0, d)).astype(np.float32)
    if kind == "narrow":
        return (1.0 + rng.standard_normal(d) * 1e-6).astype(np.float32)
    if kind == "skewed":
        return (rng.exponential(1.0, d) ** 3 * 1e-3).astype(np.float32)
    if kind == "uniform":
        return rng.uniform(-1e-3, 1e-3, d).astype(np.float32)
    if kind == "fewvalues":
        return rng.choice(np.array([-2e-3, -1e-3, 5e-4, 3e-3], np.float32), d)
    raise KeyError(kind)


@pytest.mark.parametrize("kind", ["integers", "bimodal", "cauchy", "dynamic", "narrow", "skewed", "uniform",
                                  "fewvalues"])
@pytest.mark.parametrize("scheme", ["bingrad_b", "bingrad_pb"])
@pytest.mark.parametrize("d", [128, 512])
def test_bingrad_split_search_stress(kind, scheme, d):
    """The register path's split search sorts only the grid cells that can hold the best split
    (falling back to a full sort when they hold too many values); every choice must still be
    the exhaustive one, bit for bit."""
    rng = np.random.default_rng(sum(map(ord, kind)) + d)
    W, nbk = 2, 12
    g = [[np.concatenate([_bingrad_buckets(kind, d, rng) for _ in range(nbk)] + [_bingrad_buckets(kind, 77, rng)])
          for _ in range(W)]]
    n = g[0][0].size
    cg, co = configs(scheme, 2, d, W, True, 0.0, 13, n)
    compare_steps(run_gpu_fused(cg, 1, g), run_oracle_fused(co, 1, g), co, "%s %s d=%d" % (scheme, kind, d))


@pytest.mark.parametrize("d", [128, 512, 2048])
def test_bingrad_pb_interior_optima(d):
    """Buckets whose best admissible pair lies strictly inside the admissible range (A below the
    largest admissible lower index, or B above the smallest admissible upper one): integer values
    0 .. 63 on the exact grid, from the oracle pins' interior cases repeated to the bucket size.
    There the kernel's per-column search cannot stop at the range's corner: along a column it
    must find an interior minimum (the bisection), and the pair must still be the exhaustive
    scan's, bit for bit."""
    import oracle as O
    from test_oracle_pins import _PB_INNER, _grid32
    rng = np.random.default_rng(77 + d)
    buckets, inner = [], 0
    for lst in _PB_INNER:
        u = np.resize(np.array(lst, np.float32), d)
        rng.shuffle(u)
        buckets.append(u)
        A, B, _, _ = O.bingrad_pb_fit(u)
        a_b, b_b = O.bingrad_b_fit(u)[:2]
        grid = _grid32(u)
        amax = max([j for j in range(64) if grid[j] <= a_b], default=0)
        bmin = min([j for j in range(64) if grid[j] >= b_b], default=63)
        inner += A < amax or B > bmin
    assert inner >= 20, inner
    W = 2
    g = [[np.concatenate([buckets[(i + 5 * w) % len(buckets)] for i in range(len(buckets))]) for w in range(W)]]
    n = g[0][0].size
    cg, co = configs("bingrad_pb", 2, d, W, True, 0.0, 21, n)
    compare_steps(run_gpu_fused(cg, 1, g), run_oracle_fused(co, 1, g), co, "bingrad_pb interior d=%d" % d)


@pytest.mark.parametrize("W", [1, 4, 5, 8])
@pytest.mark.parametrize("scheme,levels,d", [("orq", 5, 512), ("qsgd", 3, 128), ("qsgd", 255, 256), ("orq", 9, 2048)])
def test_decode_worker_counts(W, scheme, levels, d):
    """gq_decode_accumulate for 1, 4 and 8 messages (the staged decode, the count a template
    argument) and for 5 (the generic one), 3-, 2-, 8- and 4-bit codes, against the oracle."""
    n = 6 * d + 71
    cg, co = configs(scheme, levels, d, W, True, 0.0, 91 + W, n)
    g = _grads(n, W, 1, seed=7 * W + d)
    compare_steps(run_gpu_fused(cg, 1, g, unfused=True), run_oracle_fused(co, 1, g), co,
                  "decode W=%d %s-%d d=%d" % (W, scheme, levels, d))
