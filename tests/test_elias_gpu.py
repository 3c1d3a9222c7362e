"""GPU parity of the Elias-gamma coding (gq_elias_pack / gq_elias_unpack) with the oracle.

Dense messages come from the oracle's encoder; the GPU's Elias message must equal the oracle's
byte for byte over its used length (header, offsets, tables, stream and padding), leave the
rest of the buffer untouched, and unpack to the dense message exactly.  Sizes span several
scan tiles (4096 buckets each) and ragged last buckets; the 1e9-element QSGD-l2 message is
checked on sampled buckets against the oracle and round-trips whole on the GPU."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

import gradient_quantization_communication_b200.gq as G
import oracle as O
from gpu_harness import configs
from gradient_quantization_communication_b200 import synth

FILL = 0xAB


def _oracle_msg(co, seed):
    rng = np.random.default_rng(seed)
    g = (rng.laplace(0, 1e-3, co.n)).astype(np.float32)
    return O.encode(co, 0, 2, g)


@pytest.mark.parametrize("scheme,levels", [("qsgd", 3), ("qsgd", 5), ("terngrad", 3), ("qsgd_nearest", 9),
                                           ("qsgd_l2", 3), ("qsgd_l2", 15)])
@pytest.mark.parametrize("d,n", [(128, 1), (128, 128 * 9000 + 77), (256, 256 * 700 + 255), (512, 512 * 300)])
def test_elias_parity(scheme, levels, d, n):
    cg, co = configs(scheme, levels, d, 1, False, 0.0, 4, n)
    msg = _oracle_msg(co, d + levels)
    ref, used = O.elias_pack(co, msg)
    cap = G.gq_elias_layout(cg)[0]
    assert ref.size == cap
    d_msg = torch.from_numpy(msg).cuda()
    d_e = torch.full((cap,), FILL, dtype=torch.uint8, device="cuda")
    G.gq_elias_pack(cg, d_msg, d_e)
    back = torch.full((msg.size + 64,), FILL, dtype=torch.uint8, device="cuda")
    G.gq_elias_unpack(cg, d_e, back)
    torch.cuda.synchronize()
    e = d_e.cpu().numpy()
    T = int(e[:8].view(np.uint64)[0])
    assert G.gq_elias_used_bytes(cg, T) == used
    bad = np.flatnonzero(e[:used] != ref[:used])
    assert bad.size == 0, "Elias message differs in %d of %d bytes (first at %d)" % (bad.size, used, bad[0])
    assert (e[used:] == FILL).all(), "pack wrote past the used length"
    b = back.cpu().numpy()
    assert np.array_equal(b[:msg.size], msg) and (b[msg.size:] == FILL).all()


def test_elias_repeat_and_stream_order():
    """Two packs of the same message give the same bytes; pack on a side stream."""
    cg, co = configs("qsgd_l2", 3, 512, 1, False, 0.0, 1, 512 * 5000 + 3)
    msg = torch.from_numpy(_oracle_msg(co, 9)).cuda()
    cap = G.gq_elias_layout(cg)[0]
    outs = []
    for _ in range(2):
        s = torch.cuda.Stream()
        e = torch.zeros(cap, dtype=torch.uint8, device="cuda")
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            G.gq_elias_pack(cg, msg, e, stream=s)
        s.synchronize()
        outs.append(e.cpu().numpy())
    assert np.array_equal(outs[0], outs[1])


def _bits(words, start, length):
    v = 0
    for k in range(length):
        bit = start + k
        v |= ((int(words[bit // 32]) >> (bit % 32)) & 1) << k
    return v


def test_elias_full_size_qsgd_l2():
    """QSGD-l2 with 3 levels on the 1e9-element blocks1b gradient (worker 0, step 0): sampled
    buckets' codewords against the oracle, the whole round trip on the GPU, and about one bit
    per element."""
    n, d = 1_000_000_000, 512
    wl = synth.WORKLOADS["blocks1b"]
    cg = G.gq_config("qsgd_l2", 3, d, 1, False, 0.0, wl.rounding_seed, n)
    nb = n // d
    nbytes, _, loff = G.gq_message_layout(cg)
    cap, ooff, toff, soff = G.gq_elias_layout(cg)
    g = synth.gradient("blocks1b", 0, 0, device="cuda")
    msg = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    with G.Plan(cg) as plan:
        G.gq_encode(plan.handle, 0, 0, g, None, msg)
        assert G.gq_plan_status(plan.handle) == G.GQ_OK
    del g
    e = torch.zeros(cap, dtype=torch.uint8, device="cuda")
    G.gq_elias_pack(cg, msg, e)
    back = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    G.gq_elias_unpack(cg, e, back)
    torch.cuda.synchronize()
    assert torch.equal(back, msg), "round trip differs"
    T = int(e[:8].cpu().numpy().view(np.uint64)[0])
    assert 1.0 <= T / n < 1.2
    offs = e[ooff:ooff + 8 * nb].view(torch.int64)
    dw = d * 2 // 32
    rng = np.random.default_rng(3)
    sample = sorted(set([0, 1, nb - 1] + rng.choice(nb, size=40, replace=False).tolist()))
    words = msg[:nb * dw * 4].view(torch.int32).view(nb, dw)
    tables = msg[loff:loff + nb * 4].view(torch.float32)
    sub = O.Config(O.QSGD_L2, 3, d, 1, 0, 0.0, wl.rounding_seed, d)
    for bk in sample:
        one = np.zeros(O.message_layout(sub)[0], dtype=np.uint8)
        one[:dw * 4] = words[bk].cpu().numpy().view(np.uint8)
        one[O.message_layout(sub)[2]:O.message_layout(sub)[2] + 4] = tables[bk:bk + 1].cpu().numpy().view(np.uint8)
        ref, _ = O.elias_pack(sub, one)
        rT = int(ref[:8].view(np.uint64)[0])
        rs = ref[O.elias_layout(sub)[3]:].view(np.uint32)
        start = int(offs[bk].item())
        end = int(offs[bk + 1].item()) if bk + 1 < nb else T
        assert end - start == rT, bk
        lo, hi = start // 32, (end + 31) // 32 + 1
        gw = e[soff + 4 * lo:soff + 4 * min(hi, (cap - soff) // 4)].view(torch.int32).cpu().numpy().view(np.uint32)
        assert _bits(gw, start - 32 * lo, rT) == _bits(rs, 0, rT), bk
        assert e[toff + 4 * bk:toff + 4 * bk + 4].cpu().numpy().view(np.float32)[0] == tables[bk].item()
