"""The allocation-free quantization-error entry point (gq_quant_error_noalloc).

It serves callers that cannot call cudaMalloc (code inside a caching allocator or memory pool,
processes with device memory reserved up front, plugins given buffers but no allocator): it
takes a configuration instead of a plan and keeps its scratch in a static device array of the
library.  Its results must equal those of gq_quant_error bit for bit, call after call, even
though every call reuses the same scratch.  This file is collected last so that a failure here
cannot stop a run before the other tests.
"""
import numpy as np
import pytest
import torch

import gradient_quantization_communication_b200.gq as G

pytestmark = pytest.mark.gpu


def _inputs(n, seed):
    rng = np.random.default_rng(seed)
    g = torch.from_numpy((rng.laplace(0, 1e-3, n)).astype(np.float32)).cuda()
    r = torch.from_numpy((rng.standard_normal(n) * 1e-4).astype(np.float32)).cuda()
    return g, r


@pytest.mark.parametrize("scheme,levels,d", [("orq", 5, 512), ("qsgd", 5, 128), ("bingrad_pb", 2, 256),
                                             ("orq", 3, 2048)])
def test_noalloc_matches_planned_call_twice(scheme, levels, d):
    n = 37 * d + 19
    cfg = G.gq_config(scheme, levels, d, 1, True, 0.0, 42, n)
    out_plan = torch.zeros(3, dtype=torch.float64, device="cuda")
    out_free = torch.zeros(3, dtype=torch.float64, device="cuda")
    for call in range(2):  # two calls in a row: the static scratch keeps the previous contents
        g, r = _inputs(n, seed=100 * call + d)
        with G.Plan(cfg) as plan:
            G.gq_quant_error(plan.handle, call, call + 5, g, r, out_plan)
        out_free.fill_(-1.0)
        G.gq_quant_error_noalloc(cfg, call, call + 5, g, r, out_free)
        torch.cuda.synchronize()
        a, b = out_plan.cpu().numpy(), out_free.cpu().numpy()
        # same kernels, same fixed reduction order: the same bits
        assert np.array_equal(a.view(np.uint64), b.view(np.uint64)), (call, a, b)


@pytest.mark.parametrize("workers", [0, 1, 100])
def test_noalloc_ignores_the_worker_count(workers):
    d, n = 512, 9 * 512 + 3
    g, r = _inputs(n, seed=7)
    ref = torch.zeros(3, dtype=torch.float64, device="cuda")
    out = torch.zeros(3, dtype=torch.float64, device="cuda")
    G.gq_quant_error_noalloc(G.gq_config("orq", 5, d, 1, True, 0.0, 3, n), 2, 1, g, r, ref)
    G.gq_quant_error_noalloc(G.gq_config("orq", 5, d, workers, True, 0.0, 3, n), 2, 1, g, r, out)
    torch.cuda.synchronize()
    assert np.array_equal(ref.cpu().numpy().view(np.uint64), out.cpu().numpy().view(np.uint64))


def test_noalloc_reports_a_raised_status_as_nan_then_recovers():
    """A status bit raised by the call's kernels (here: a non-finite input) turns all three
    outputs into NaN; the next call clears the word and is exact again."""
    d, n = 256, 20 * 256
    cfg = G.gq_config("qsgd", 5, d, 1, False, 0.0, 11, n)
    g, _ = _inputs(n, seed=5)
    bad = g.clone()
    bad[3 * d + 17] = float("nan")
    out = torch.zeros(3, dtype=torch.float64, device="cuda")
    G.gq_quant_error_noalloc(cfg, 0, 0, bad, None, out)
    torch.cuda.synchronize()
    assert np.all(np.isnan(out.cpu().numpy()))
    ref = torch.zeros(3, dtype=torch.float64, device="cuda")
    with G.Plan(cfg) as plan:
        G.gq_quant_error(plan.handle, 0, 0, g, None, ref)
    G.gq_quant_error_noalloc(cfg, 0, 0, g, None, out)
    torch.cuda.synchronize()
    assert np.array_equal(ref.cpu().numpy().view(np.uint64), out.cpu().numpy().view(np.uint64))


def test_noalloc_rejects_inputs_beyond_its_scratch():
    d = 128
    n = 16384 * d + 1   # 16385 buckets: one more than the static scratch holds
    cfg = G.gq_config("orq", 5, d, 1, False, 0.0, 1, n)
    g = torch.zeros(n, device="cuda")
    out = torch.zeros(3, dtype=torch.float64, device="cuda")
    with pytest.raises(G.GQError) as ei:
        G.gq_quant_error_noalloc(cfg, 0, 0, g, None, out)
    assert ei.value.status == G.GQ_ERR_UNSUPPORTED
