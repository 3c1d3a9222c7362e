"""GPU parity of base-s messages written by the quantization kernel itself (gq_plan_set_format
with GQ_FORMAT_BASE_S) and read by gq_decode_accumulate: no dense message exists on the way.

For every base-s level count (3, 5, 9), ORQ and the QSGD family, d = 128 / 256 / 512, a ragged
last bucket and vectors shorter than a bucket: the messages must equal the oracle's dense
messages packed by the oracle's base-s packer byte for byte (codes and level tables), and the
average and residuals must equal the oracle's fused step bit for bit, fused and unfused."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

import gradient_quantization_communication_b200.gq as G
import oracle as O
from gpu_harness import assert_same_f32, configs


def _grads(n, W, steps, seed):
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(steps):
        row = []
        for _ in range(W):
            x = rng.laplace(0, 1e-3, n)
            if n > 7:
                x[::7] *= 20.0
            row.append(x.astype(np.float32))
        out.append(row)
    return out


def _regions(buf, co, nb):
    words = O.entropy_words(co)
    L = O.table_len(co.scheme, co.levels)
    _, coff, loff = O.entropy_layout(co)
    return (buf[coff:coff + nb * words * 4], buf[loff:loff + nb * L * 4])


def _run(scheme, levels, d, n, W=3, steps=2, ef=True, unfused=False, fill=0xA5, seed=5):
    cg, co = configs(scheme, levels, d, W, ef, 0.0, seed, n)
    g = _grads(n, W, steps, seed=d * 7 + levels + n)
    dev = torch.device("cuda")
    nb = (n + d - 1) // d
    rs = [np.zeros(n, np.float32) for _ in range(W)] if ef else None
    with G.Plan(cg, fmt=G.GQ_FORMAT_BASE_S) as plan:
        assert plan.msg_bytes == O.entropy_layout(co)[0]
        r = [torch.zeros(n, device=dev) for _ in range(W)] if ef else None
        for t in range(steps):
            gt = [torch.from_numpy(x).to(dev) for x in g[t]]
            msgs = [torch.full((plan.msg_bytes,), fill, dtype=torch.uint8, device=dev) for _ in range(W)]
            avg = torch.full((n,), float("nan"), device=dev)
            if unfused:
                for w in range(W):
                    G.gq_encode(plan.handle, w, t, gt[w], r[w] if ef else None, msgs[w])
                G.gq_decode_accumulate(plan.handle, msgs, avg)
            else:
                G.gq_fused_step(plan.handle, t, gt, r, msgs, avg)
            assert G.gq_plan_status(plan.handle) == G.GQ_OK
            oavg, omsgs = O.fused_step(co, t, g[t], rs)
            assert_same_f32(avg.cpu().numpy(), oavg, "avg step %d" % t)
            if ef:
                for w in range(W):
                    assert_same_f32(r[w].cpu().numpy(), rs[w], "residual w%d" % w)
            for w in range(W):
                want = _regions(O.entropy_pack(co, omsgs[w]), co, nb)
                got = _regions(msgs[w].cpu().numpy(), co, nb)
                assert np.array_equal(got[0], want[0]), "codes of w%d step %d" % (w, t)
                assert np.array_equal(got[1], want[1]), "level tables of w%d step %d" % (w, t)
            # the decode of the base-s messages gives the average again
            avg2 = torch.full((n,), float("nan"), device=dev)
            G.gq_decode_accumulate(plan.handle, msgs, avg2)
            assert_same_f32(avg2.cpu().numpy(), oavg, "decoded avg step %d" % t)


CASES = [("orq", 3), ("orq", 5), ("orq", 9), ("qsgd", 3), ("qsgd", 5), ("qsgd", 9), ("terngrad", 3),
         ("qsgd_nearest", 5), ("qsgd_l2", 3)]


@pytest.mark.parametrize("scheme,levels", CASES)
@pytest.mark.parametrize("d", [128, 256, 512])
def test_base_s_fused(scheme, levels, d):
    _run(scheme, levels, d, 7 * d + 37)


@pytest.mark.parametrize("scheme,levels", [("orq", 5), ("qsgd", 9), ("orq", 3)])
@pytest.mark.parametrize("d", [128, 512])
def test_base_s_unfused(scheme, levels, d):
    _run(scheme, levels, d, 5 * d + 100, W=2, unfused=True)


@pytest.mark.parametrize("n", [1, 5, 127, 300])
def test_base_s_short_vectors(n):
    _run("orq", 5, 512, n, W=2)


def test_base_s_without_error_feedback_and_many_buckets():
    _run("orq", 5, 512, 512 * 700 + 3, W=8, steps=1, ef=False)


def test_base_s_without_messages_matches_dense():
    """With no message buffers the base-s plan computes the same average and residuals."""
    n, W = 512 * 9 + 11, 3
    cg, co = configs("orq", 5, 512, W, True, 0.0, 2, n)
    g = _grads(n, W, 1, seed=4)
    rs = [np.zeros(n, np.float32) for _ in range(W)]
    oavg, _ = O.fused_step(co, 0, g[0], rs, with_msgs=False)
    with G.Plan(cg, fmt=G.GQ_FORMAT_BASE_S) as plan:
        r = [torch.zeros(n, device="cuda") for _ in range(W)]
        avg = torch.empty(n, device="cuda")
        G.gq_fused_step(plan.handle, 0, [torch.from_numpy(x).cuda() for x in g[0]], r, None, avg)
        assert_same_f32(avg.cpu().numpy(), oavg, "avg")
        for w in range(W):
            assert_same_f32(r[w].cpu().numpy(), rs[w], "residual")


def test_base_s_format_checks():
    for scheme, levels, d in [("orq", 4, 512), ("orq", 5, 1024), ("bingrad_b", 2, 512), ("signsgd", 2, 512),
                              ("qsgd", 7, 512)]:
        cg, _ = configs(scheme, levels, d, 1, True, 0.0, 1, 1000)
        with G.Plan(cg) as plan:
            with pytest.raises(G.GQError) as ei:
                G.gq_plan_set_format(plan.handle, G.GQ_FORMAT_BASE_S)
            assert ei.value.status == G.GQ_ERR_UNSUPPORTED
    cg, co = configs("orq", 5, 512, 1, True, 0.0, 1, 1000)
    with G.Plan(cg) as plan:
        with pytest.raises(G.GQError):
            G.gq_plan_set_format(plan.handle, 7)
        G.gq_plan_set_format(plan.handle, G.GQ_FORMAT_BASE_S)
        assert G.gq_plan_message_layout(plan.handle) == tuple(O.entropy_layout(co))
        G.gq_plan_set_format(plan.handle, G.GQ_FORMAT_DENSE)
        assert G.gq_plan_message_layout(plan.handle) == tuple(O.message_layout(co))
