"""Failure path of the kernels' bounded waits, exercised on the GPU without a fault.

Every wait of the kernels for a bulk copy gives up after a time limit and raises the plan's
timeout flag instead of hanging.  gq_selftest_bounded_wait runs that same wait on a barrier that
nothing completes; the flag must come back as GQ_ERR_TIMEOUT, be cleared by the report, and the
plan and the CUDA context must stay usable (a fused step afterwards still matches the oracle).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from gpu_harness import G, compare_steps, configs, run_gpu_fused, run_oracle_fused  # noqa: E402


@pytest.mark.gpu
def test_bounded_wait_times_out_and_context_stays_usable():
    n, W = 4 * 512 + 17, 2
    cg, co = configs("orq", 5, 512, W, True, 0.0, 5, n)
    with G.Plan(cg) as plan:
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        G.gq_selftest_bounded_wait(plan.handle, 5_000_000)  # 5 ms
        b.record()
        assert G.gq_plan_status(plan.handle) == G.GQ_ERR_TIMEOUT
        assert a.elapsed_time(b) >= 4.0  # the wait ran to its limit
        assert G.gq_plan_status(plan.handle) == G.GQ_OK  # the report cleared the flag
        assert "timed out" in G.gq_status_string(G.GQ_ERR_TIMEOUT)
    rng = np.random.default_rng(5)
    g = [[(rng.standard_normal(n) * 1e-3).astype(np.float32) for _ in range(W)]]
    compare_steps(run_gpu_fused(cg, 1, g), run_oracle_fused(co, 1, g), co, "after a timed-out wait")
