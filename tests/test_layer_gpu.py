"""GPU parity of TernGrad with one scale per parameter tensor (GQ_TERNGRAD_LAYER) with the
oracle: codes, scales, residuals and averages bit for bit through gq_fused_step, gq_encode and
gq_decode_accumulate, for ResNet-shaped tensors (small ones included), ragged vectors, every
bucket layout, with and without error feedback."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

import gradient_quantization_communication_b200.gq as G
import oracle as O
from gradient_quantization_communication_b200 import synth


def _offsets(n, sizes):
    off = [0]
    for s in sizes:
        if off[-1] + s >= n:
            break
        off.append(off[-1] + s)
    off.append(n)
    return np.array(off, dtype=np.int64)


def _run(n, d, W, steps, off, ef, seed=5):
    rng = np.random.default_rng(seed)
    grads = [[(rng.laplace(0, 1, n) * 10.0 ** rng.uniform(-4, -2, n)).astype(np.float32) for _ in range(W)]
             for _ in range(steps)]
    cfg = G.gq_config("terngrad_layer", 3, d, W, ef, 0.0, 17, n)
    ocfg = O.Config(G.GQ_TERNGRAD_LAYER, 3, d, W, int(ef), 0.0, 17, n)
    dev = torch.device("cuda")
    with G.Plan(cfg, segments=off) as plan:
        assert plan.msg_bytes == O.tg_layer_layout(ocfg, len(off) - 1)[0]
        r = [torch.zeros(n, device=dev) for _ in range(W)] if ef else None
        ro = [np.zeros(n, np.float32) for _ in range(W)] if ef else None
        # stale bytes in the messages: every byte must be written
        msgs = [torch.full((plan.msg_bytes,), 0xA5, dtype=torch.uint8, device=dev) for _ in range(W)]
        avg = torch.empty(n, device=dev)
        for t in range(steps):
            g = [torch.from_numpy(x).to(dev) for x in grads[t]]
            G.gq_fused_step(plan.handle, t, g, r, msgs, avg)
            assert G.gq_plan_status(plan.handle) == G.GQ_OK
            om = [O.tg_layer_encode(ocfg, off, w, t, grads[t][w], ro[w] if ef else None) for w in range(W)]
            oavg = O.tg_layer_decode_accumulate(ocfg, off, om)
            for w in range(W):
                assert np.array_equal(msgs[w].cpu().numpy(), om[w]), (t, w)
                if ef:
                    assert np.array_equal(r[w].cpu().numpy(), ro[w]), (t, w)
            assert np.array_equal(avg.cpu().numpy().view(np.uint32), oavg.view(np.uint32)), t
            # the unfused calls give the same messages and average
            avg2 = torch.empty(n, device=dev)
            G.gq_decode_accumulate(plan.handle, msgs, avg2)
            assert np.array_equal(avg2.cpu().numpy().view(np.uint32), oavg.view(np.uint32))


@pytest.mark.parametrize("d", [128, 512, 2048])
def test_resnet18_tensors(d):
    sizes = synth.resnet_param_sizes(18)
    n = 200000 + 37
    _run(n, d, 3, 2, _offsets(n, sizes), True)


@pytest.mark.parametrize("ef", [True, False])
def test_tiny_and_empty_tensors(ef):
    n, d = 5 * 512 + 19, 512
    off = np.array([0, 0, 9, 9, 73, 600, 601, 1200, 2048, n], dtype=np.int64)
    _run(n, d, 2, 2, off, ef, seed=8)


def test_one_tensor_and_encode_per_worker():
    n, d = 4 * 512 + 3, 512
    off = np.array([0, n], dtype=np.int64)
    rng = np.random.default_rng(9)
    g = (rng.standard_normal(n) * 1e-3).astype(np.float32)
    cfg = G.gq_config("terngrad_layer", 3, d, 2, False, 0.0, 1, n)
    ocfg = O.Config(G.GQ_TERNGRAD_LAYER, 3, d, 2, 0, 0.0, 1, n)
    with G.Plan(cfg, segments=off) as plan:
        msg = torch.full((plan.msg_bytes,), 0xFF, dtype=torch.uint8, device="cuda")
        G.gq_encode(plan.handle, 1, 4, torch.from_numpy(g).cuda(), None, msg)
        assert np.array_equal(msg.cpu().numpy(), O.tg_layer_encode(ocfg, off, 1, 4, g))


def test_segments_required_and_checked():
    n = 1000
    cfg = G.gq_config("terngrad_layer", 3, 128, 1, False, 0.0, 1, n)
    with pytest.raises(G.GQError):
        G.gq_message_layout(cfg)
    with G.Plan(cfg) as plan:
        g = torch.zeros(n, device="cuda")
        msg = torch.zeros(1024, dtype=torch.uint8, device="cuda")
        with pytest.raises(G.GQError):      # no segments yet
            G.gq_encode(plan.handle, 0, 0, g, None, msg)
        for bad in ([1, n], [0, 500], [0, 600, 500, n]):
            with pytest.raises(G.GQError):
                G.gq_plan_set_segments(plan.handle, bad)
        G.gq_plan_set_segments(plan.handle, [0, 400, n])
        assert G.gq_plan_message_layout(plan.handle)[0] == O.tg_layer_layout(
            O.Config(G.GQ_TERNGRAD_LAYER, 3, 128, 1, 0, 0.0, 1, n), 2)[0]


@pytest.mark.parametrize("W,ef", [(2, True), (8, True), (1, False), (5, True)])
def test_long_vector_many_tensors(W, ef):
    """More chunks than the grid has warps, so that every warp walks a run of chunks and slices
    across many tensor boundaries (random sizes from 0 to 40000, so boundaries fall inside a
    lane's four elements, across chunk edges, and empty tensors follow each other); 1, 2 and 8
    workers take the staged encode, 5 the generic one; a ragged last chunk."""
    rng = np.random.default_rng(21)
    n = 3_000_000 + 13 if W <= 2 else 1_000_000 + 77
    sizes = rng.integers(0, 40000, 400)
    sizes[rng.integers(0, 400, 40)] = 0
    _run(n, 512, W, 1, _offsets(n, sizes.tolist()), ef, seed=22 + W)
