"""The message exchange between ranks (gradient_quantization_communication_b200.exchange) on the
CPU with gloo ranks: each rank quantizes its own worker's gradient, the ranks all-gather the
packed messages in rank order, and each rank decodes and averages them.  The encode and decode
here are the oracle's (the CUDA library needs a GPU); the collective, the buffers and the order
of the calls are the module's own.  Every rank's average and residual must equal, bit for bit,
a single-process fused step over all ranks' gradients.
"""
import datetime
import os
import socket
import sys

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _grads(n, world, steps):
    rng = np.random.default_rng(77)
    return [[(rng.laplace(0, 1e-3, n)).astype(np.float32) for _ in range(world)] for _ in range(steps)]


def _rank_main(rank, world, port, out, scheme, levels, d, n, steps):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle as O
    from gradient_quantization_communication_b200 import gq as G
    from gradient_quantization_communication_b200.exchange import Exchange
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        sid = G.SCHEMES[scheme]
        ocfg = O.Config(sid, levels, d, world, 1, 0.0, 42, n)
        msg_bytes = O.message_layout(ocfg)[0]
        res = np.zeros(n, dtype=np.float32)

        def encode(step, r, grad, residual, msg):
            m = O.encode(ocfg, r, step, grad, residual)
            msg.copy_(torch.from_numpy(m))

        def decode(messages, avg):
            avg[:] = O.decode_accumulate(ocfg, [m.numpy() for m in messages])

        ex = Exchange(G.gq_config(sid, levels, d, world, True, 0.0, 42, n), encode=encode, decode=decode,
                      msg_bytes=msg_bytes)
        grads = _grads(n, world, steps)
        avgs = []
        for t in range(steps):
            avg = np.zeros(n, dtype=np.float32)
            ex.step(t, grads[t][rank], res, avg)
            avgs.append(avg.copy())
        np.save(os.path.join(out, "rank%d_avg.npy" % rank), np.stack(avgs))
        np.save(os.path.join(out, "rank%d_res.npy" % rank), res)
        ex.close()
    finally:
        dist.destroy_process_group()


def _run(tmp_path, scheme, levels, d, n, steps=3, world=2):
    import oracle as O
    from gradient_quantization_communication_b200 import gq as G
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path), scheme, levels, d, n, steps), nprocs=world, join=True)
    ocfg = O.Config(G.SCHEMES[scheme], levels, d, world, 1, 0.0, 42, n)
    grads = _grads(n, world, steps)
    rs = [np.zeros(n, dtype=np.float32) for _ in range(world)]
    ref = [O.fused_step(ocfg, t, grads[t], rs, with_msgs=False)[0] for t in range(steps)]
    for r in range(world):
        got = np.load(tmp_path / ("rank%d_avg.npy" % r))
        for t in range(steps):
            assert np.array_equal(got[t].view(np.uint32), ref[t].view(np.uint32)), (r, t)
        assert np.array_equal(np.load(tmp_path / ("rank%d_res.npy" % r)), rs[r])


def test_exchange_orq5_matches_fused_step(tmp_path):
    _run(tmp_path, "orq", 5, 512, 3 * 512 + 40)


def test_exchange_qsgd_ragged_matches_fused_step(tmp_path):
    _run(tmp_path, "qsgd", 3, 128, 5 * 128 + 7)


def test_exchange_rejects_a_worker_count_other_than_the_world(tmp_path):
    mp.spawn(_mismatch_main, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True)
    assert (tmp_path / "rank0.ok").exists() and (tmp_path / "rank1.ok").exists()


def _mismatch_main(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from gradient_quantization_communication_b200 import gq as G
    from gradient_quantization_communication_b200.exchange import Exchange
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        try:
            Exchange(G.gq_config("orq", 5, 512, 3, True, 0.0, 1, 1024), encode=lambda *a: None,
                     decode=lambda *a: None, msg_bytes=16)
        except ValueError:
            open(os.path.join(out, "rank%d.ok" % rank), "w").close()
    finally:
        dist.destroy_process_group()
