"""Helpers for the GPU parity tests: run the CUDA library (through the C ABI binding) and the
CPU oracle on the same seeded inputs and compare element by element."""
import numpy as np
import torch

import gradient_quantization_communication_b200.gq as G
import oracle as O

SCHEME_ID = {"qsgd": 0, "terngrad": 1, "bingrad_b": 2, "bingrad_pb": 3, "orq": 4, "qsgd_nearest": 5, "signsgd": 6, "qsgd_l2": 7}


def configs(scheme, levels, d, W, ef, clip, seed, n):
    sid = SCHEME_ID[scheme]
    return (G.gq_config(sid, levels, d, W, ef, clip, seed, n),
            O.Config(sid, levels, d, W, int(ef), clip, seed, n))


def msg_views(buf, cfg_o):
    """(codes words, level tables) of one message (numpy uint8 buffer)."""
    nb = O.num_buckets(cfg_o)
    words = cfg_o.bucket * O.bits(cfg_o.levels) // 32
    L = O.table_len(cfg_o.scheme, cfg_o.levels)
    _, coff, loff = O.message_layout(cfg_o)
    codes = buf[coff:coff + nb * words * 4].view(np.uint32).reshape(nb, words)
    tables = buf[loff:loff + nb * L * 4].view(np.float32).reshape(nb, L)
    return codes, tables


def assert_same_f32(a, b, what):
    a = np.asarray(a, dtype=np.float32)
    b = np.asarray(b, dtype=np.float32)
    assert a.shape == b.shape, what
    bad = np.flatnonzero(a.view(np.uint32) != b.view(np.uint32))
    if bad.size:
        # +0 / -0 compare equal numerically; anything else is a mismatch
        num = np.flatnonzero(a[bad] != b[bad])
        assert num.size == 0, "%s: %d of %d values differ, first at %d: %r vs %r" % (
            what, num.size, a.size, bad[num[0]], a[bad[num[0]]], b[bad[num[0]]])


def assert_same_msg(gpu_buf, ora_buf, cfg_o, what):
    gc, gt = msg_views(gpu_buf, cfg_o)
    oc, ot = msg_views(ora_buf, cfg_o)
    badb = np.flatnonzero((gc != oc).any(axis=1))
    assert badb.size == 0, "%s: packed codes differ in %d of %d buckets (first %d)" % (
        what, badb.size, gc.shape[0], badb[0])
    assert_same_f32(gt, ot, what + " level tables")


def run_gpu_fused(cfg_g, steps, grads_np, with_msgs=True, unfused=False):
    """grads_np[t][w]: float32 arrays.  Returns per step (avg, residuals, msgs) as numpy."""
    W = cfg_g.workers
    n = cfg_g.n
    dev = torch.device("cuda")
    ef = bool(cfg_g.error_feedback)
    plan = G.Plan(cfg_g)
    r = [torch.zeros(n, dtype=torch.float32, device=dev) for _ in range(W)] if ef else None
    out = []
    try:
        for t in range(steps):
            g = [torch.from_numpy(np.ascontiguousarray(grads_np[t][w])).to(dev) for w in range(W)]
            avg = torch.full((n,), float("nan"), dtype=torch.float32, device=dev)
            msgs = [torch.zeros(plan.msg_bytes, dtype=torch.uint8, device=dev) for _ in range(W)] \
                if (with_msgs or unfused) else None
            if unfused:
                for w in range(W):
                    G.gq_encode(plan.handle, w, t, g[w], r[w] if ef else None, msgs[w])
                G.gq_decode_accumulate(plan.handle, msgs, avg)
            else:
                G.gq_fused_step(plan.handle, t, g, r, msgs, avg)
            st = G.gq_plan_status(plan.handle)
            assert st == G.GQ_OK, G.gq_status_string(st)
            out.append((avg.cpu().numpy(),
                        [x.cpu().numpy().copy() for x in r] if ef else None,
                        [m.cpu().numpy() for m in msgs] if msgs is not None else None))
    finally:
        plan.close()
    return out


def run_oracle_fused(cfg_o, steps, grads_np):
    W = cfg_o.workers
    ef = bool(cfg_o.error_feedback)
    r = [np.zeros(cfg_o.n, dtype=np.float32) for _ in range(W)] if ef else None
    out = []
    for t in range(steps):
        gs = [np.ascontiguousarray(grads_np[t][w], dtype=np.float32) for w in range(W)]
        avg, msgs = O.fused_step(cfg_o, t, gs, r, with_msgs=True)
        out.append((avg, [x.copy() for x in r] if ef else None, msgs))
    return out


def compare_steps(gpu, ora, cfg_o, label):
    for t, ((ga, gr, gm), (oa, orr, om)) in enumerate(zip(gpu, ora)):
        assert_same_f32(ga, oa, "%s step %d avg" % (label, t))
        if orr is not None:
            for w in range(len(orr)):
                assert_same_f32(gr[w], orr[w], "%s step %d residual w%d" % (label, t, w))
        if gm is not None:
            for w in range(len(om)):
                assert_same_msg(gm[w], om[w], cfg_o, "%s step %d msg w%d" % (label, t, w))
