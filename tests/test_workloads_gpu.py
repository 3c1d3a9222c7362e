"""GPU parity on the workloads at their full sizes, in the launch configuration the benchmark
times (gq_fused_step with messages).  The whole 65,536-element workload goes through the
oracle; for the large ones the oracle recomputes a sample of buckets (the first, the last /
ragged one, and random ones) from the same generated gradients, following its own residual
chain across the steps."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

import gradient_quantization_communication_b200.gq as G
import oracle as O
from gpu_harness import assert_same_f32, compare_steps, configs, run_gpu_fused, run_oracle_fused
from gradient_quantization_communication_b200 import synth


def test_gauss64k_full():
    wl = synth.WORKLOADS["gauss64k"]
    g = [[synth.gradient("gauss64k", w, 0).numpy() for w in range(wl.workers)]]
    for scheme, levels, clip in wl.schemes:
        cg, co = configs(scheme, levels, wl.bucket, wl.workers, True, clip, wl.rounding_seed, wl.n)
        compare_steps(run_gpu_fused(cg, 1, g), run_oracle_fused(co, 1, g), co, "gauss64k " + scheme)


def sampled_parity(name, scheme, levels, clip, d, steps, nsample=40, seed=0):
    wl = synth.WORKLOADS[name]
    W, n, ef = wl.workers, wl.n, wl.error_feedback
    cg, co = configs(scheme, levels, d, W, ef, clip, wl.rounding_seed, n)
    nb = (n + d - 1) // d
    rng = np.random.default_rng(seed)
    sample = sorted(set([0, nb - 1] + rng.choice(nb, size=min(nsample, nb), replace=False).tolist()))
    words = d * O.bits(levels) // 32
    L = O.table_len(co.scheme, levels)
    dev = torch.device("cuda")
    plan = G.Plan(cg)
    _, coff, loff = O.message_layout(co)
    g = [torch.empty(n, dtype=torch.float32, device=dev) for _ in range(W)]
    r = [torch.zeros(n, dtype=torch.float32, device=dev) for _ in range(W)] if ef else None
    msgs = [torch.zeros(plan.msg_bytes, dtype=torch.uint8, device=dev) for _ in range(W)]
    avg = torch.empty(n, dtype=torch.float32, device=dev)
    r_or = {b: [np.zeros(min(d, n - b * d), np.float32) for _ in range(W)] for b in sample} if ef else None
    try:
        for t in range(steps):
            for w in range(W):
                synth.gradient(name, w, t, out=g[w])
            g_s = {b: [g[w][b * d:min(n, (b + 1) * d)].cpu().numpy() for w in range(W)] for b in sample}
            G.gq_fused_step(plan.handle, t, g, r, msgs, avg)
            assert G.gq_plan_status(plan.handle) == G.GQ_OK
            for b in sample:
                lo, hi = b * d, min(n, (b + 1) * d)
                o_avg, o_r, o_words, o_tab = O.fused_bucket(co, t, b, g_s[b], r_or[b] if ef else None)
                assert_same_f32(avg[lo:hi].cpu().numpy(), o_avg, "%s %s t%d bucket %d avg" % (name, scheme, t, b))
                for w in range(W):
                    cw = msgs[w][coff + b * words * 4: coff + (b + 1) * words * 4].cpu().numpy().view(np.uint32)
                    assert np.array_equal(cw, o_words[w]), "%s %s t%d bucket %d w%d codes" % (name, scheme, t, b, w)
                    tb = msgs[w][loff + b * L * 4: loff + (b + 1) * L * 4].cpu().numpy().view(np.float32)
                    assert_same_f32(tb, o_tab[w], "table")
                    if ef:
                        assert_same_f32(r[w][lo:hi].cpu().numpy(), o_r[w], "residual")
                if ef:
                    r_or[b] = o_r
    finally:
        plan.close()
        del g, r, msgs, avg
        torch.cuda.empty_cache()


@pytest.mark.parametrize("scheme,levels,clip", synth.WORKLOADS["resnet18"].schemes)
def test_resnet18(scheme, levels, clip):
    sampled_parity("resnet18", scheme, levels, clip, 512, steps=3)


@pytest.mark.parametrize("scheme,levels,clip", synth.WORKLOADS["resnet50"].schemes)
def test_resnet50(scheme, levels, clip):
    sampled_parity("resnet50", scheme, levels, clip, 512, steps=2, nsample=24)


@pytest.mark.parametrize("d", synth.WORKLOADS["mixture100m"].buckets_sweep)
@pytest.mark.parametrize("scheme,levels,clip", synth.WORKLOADS["mixture100m"].schemes)
def test_mixture100m(scheme, levels, clip, d):
    sampled_parity("mixture100m", scheme, levels, clip, d, steps=1, nsample=8 if d >= 8192 else 24)


@pytest.mark.parametrize("scheme,levels,clip", synth.WORKLOADS["blocks1b"].schemes)
def test_blocks1b(scheme, levels, clip):
    sampled_parity("blocks1b", scheme, levels, clip, 512, steps=2, nsample=24)
