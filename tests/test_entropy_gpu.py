"""GPU parity of the base-s packing (gq_entropy_pack / gq_entropy_unpack) with the oracle.

Dense messages come from the oracle's encoder (or, at the full 1e9-element size, from the
library's encoder, whose messages the fused-step tests pin to the oracle); the base-s message
must equal the oracle's byte for byte, padding included, and unpacking must give the dense
message back exactly.  Sizes span several tiles of the kernel and a ragged last bucket; the
full-size case runs in the benchmark's launch configuration (one launch per 1e9-element
message) and checks a sample of buckets against the oracle and the whole round trip on the GPU."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

import gradient_quantization_communication_b200.gq as G
import oracle as O
from gradient_quantization_communication_b200 import synth

CANARY = 64  # bytes after each output buffer that must stay untouched


def _dev_buf(nbytes, fill):
    return torch.full((nbytes + CANARY,), fill, dtype=torch.uint8, device="cuda")


def _oracle_msg(scheme, levels, d, n, seed):
    rng = np.random.default_rng(seed)
    co = O.Config(scheme, levels, d, 1, 0, 0.0, seed, n)
    g = (rng.standard_normal(n) * 1e-3).astype(np.float32)
    if n > 7:
        g[::7] *= 50.0  # spread the codes over all levels
    return co, O.encode(co, 0, 3, g)


@pytest.mark.parametrize("scheme,levels", [(4, 3), (4, 5), (4, 9), (0, 5), (1, 3), (0, 9), (0, 3)])
@pytest.mark.parametrize("d,n", [(128, 1), (128, 128 * 1500 + 77), (512, 512 * 300 + 5), (2048, 2048 * 70 + 2047),
                                 (8192, 8192 * 9), (32768, 32768 * 4 + 100)])
def test_entropy_parity(scheme, levels, d, n):
    co, msg = _oracle_msg(scheme, levels, d, n, 11 * d + levels + scheme)
    cg = G.gq_config(scheme, levels, d, 1, False, 0.0, co.seed, n)
    ebytes = G.gq_entropy_layout(cg)[0]
    nbytes = G.gq_message_layout(cg)[0]
    assert msg.size == nbytes
    ref = O.entropy_pack(co, msg)
    d_msg = torch.from_numpy(msg).cuda()
    d_emsg = _dev_buf(ebytes, 0xAB)
    G.gq_entropy_pack(cg, d_msg, d_emsg)
    d_back = _dev_buf(nbytes, 0xCD)
    G.gq_entropy_unpack(cg, d_emsg, d_back)
    torch.cuda.synchronize()
    emsg = d_emsg.cpu().numpy()
    back = d_back.cpu().numpy()
    bad = np.flatnonzero(emsg[:ebytes] != ref)
    assert bad.size == 0, "base-s message differs in %d of %d bytes (first at %d)" % (bad.size, ebytes, bad[0])
    assert (emsg[ebytes:] == 0xAB).all() and (back[nbytes:] == 0xCD).all(), "write past the message"
    bad = np.flatnonzero(back[:nbytes] != msg)
    assert bad.size == 0, "unpacked message differs in %d of %d bytes (first at %d)" % (bad.size, nbytes, bad[0])
    assert np.array_equal(O.entropy_unpack(co, ref), msg)


def test_entropy_streams_and_sync():
    """Work is enqueued on the given stream only; consecutive calls on two streams agree."""
    co, msg = _oracle_msg(4, 5, 512, 512 * 2000 + 1, 5)
    cg = G.gq_config(4, 5, 512, 1, False, 0.0, co.seed, co.n)
    ebytes = G.gq_entropy_layout(cg)[0]
    d_msg = torch.from_numpy(msg).cuda()
    outs = []
    for _ in range(2):
        s = torch.cuda.Stream()
        e = torch.zeros(ebytes, dtype=torch.uint8, device="cuda")
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            G.gq_entropy_pack(cg, d_msg, e, stream=s)
        s.synchronize()
        outs.append(e.cpu().numpy())
    assert np.array_equal(outs[0], outs[1])
    assert np.array_equal(outs[0], O.entropy_pack(co, msg))


def test_entropy_full_size_orq5():
    """The 1e9-element ORQ-5 d=512 message of the blocks1b workload (worker 0, step 0): sampled
    buckets against the oracle, the whole round trip on the GPU."""
    n, d, levels = 1_000_000_000, 512, 5
    wl = synth.WORKLOADS["blocks1b"]
    cg = G.gq_config("orq", levels, d, 1, False, 0.0, wl.rounding_seed, n)
    co = O.Config(O.ORQ, levels, d, 1, 0, 0.0, wl.rounding_seed, n)
    nb = (n + d - 1) // d
    nbytes, _, loff = G.gq_message_layout(cg)
    ebytes, _, eloff = G.gq_entropy_layout(cg)
    dw, ew, L = d * 3 // 32, O.entropy_words(co), levels
    g = synth.gradient("blocks1b", 0, 0, device="cuda")
    msg = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    plan = G.Plan(cg)
    try:
        G.gq_encode(plan.handle, 0, 0, g, None, msg)
        assert G.gq_plan_status(plan.handle) == G.GQ_OK
    finally:
        plan.close()
    del g
    emsg = _dev_buf(ebytes, 0xAB)
    G.gq_entropy_pack(cg, msg, emsg)
    back = _dev_buf(nbytes, 0xCD)
    G.gq_entropy_unpack(cg, emsg, back)
    torch.cuda.synchronize()
    assert torch.equal(back[:nbytes], msg), "round trip differs"
    assert bool((emsg[ebytes:] == 0xAB).all()) and bool((back[nbytes:] == 0xCD).all())

    rng = np.random.default_rng(1)
    sample = sorted(set([0, 1, nb - 2, nb - 1] + rng.choice(nb, size=60, replace=False).tolist()))
    # the sampled buckets as one small message: their code words, then their level tables
    k = len(sample)
    sub = O.Config(O.ORQ, levels, d, 1, 0, 0.0, wl.rounding_seed, k * d)
    sbytes, _, sloff = O.message_layout(sub)
    words = msg[:nb * dw * 4].view(torch.int32).view(nb, dw)
    tables = msg[loff:loff + nb * L * 4].view(torch.float32).view(nb, L)
    idx = torch.tensor(sample, device="cuda")
    sub_msg = np.zeros(sbytes, dtype=np.uint8)
    sub_msg[:k * dw * 4] = words[idx].cpu().numpy().view(np.uint8).reshape(-1)
    sub_msg[sloff:sloff + k * L * 4] = tables[idx].cpu().numpy().view(np.uint8).reshape(-1)
    ref = O.entropy_pack(sub, sub_msg)
    ref_words = ref[:k * ew * 4].view(np.uint32).reshape(k, ew)
    got = emsg[:nb * ew * 4].view(torch.int32).view(nb, ew)[idx].cpu().numpy().view(np.uint32)
    assert np.array_equal(got, ref_words)
    got_t = emsg[eloff:eloff + nb * L * 4].view(torch.float32).view(nb, L)[idx].cpu().numpy()
    assert np.array_equal(got_t.view(np.uint32), tables[idx].cpu().numpy().view(np.uint32))
