"""The message exchange on the GPU through NCCL: gq_encode of this rank's worker, the
all-gather of the packed messages, gq_decode_accumulate.  One GPU gives one rank, so the
exchange gathers one message; its average and residual must equal gq_fused_step's for the same
worker bit for bit, and the gathered message must equal the encoded one."""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _main(rank, port, out):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from gradient_quantization_communication_b200 import gq as G
    from gradient_quantization_communication_b200.exchange import Exchange
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dev = torch.device("cuda:0")
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60), device_id=dev)
    try:
        n, d = 40 * 512 + 77, 512
        cfg = G.gq_config("orq", 5, d, 1, True, 0.0, 42, n)
        rng = np.random.default_rng(3)
        gs = [torch.from_numpy(rng.laplace(0, 1e-3, n).astype(np.float32)).to(dev) for _ in range(3)]
        ex = Exchange(cfg, device=dev)
        r1 = torch.zeros(n, device=dev)
        r2 = torch.zeros(n, device=dev)
        ok = True
        with G.Plan(cfg) as plan:
            msg = torch.zeros(plan.msg_bytes, dtype=torch.uint8, device=dev)
            for t, g in enumerate(gs):
                a1 = torch.empty(n, device=dev)
                a2 = torch.empty(n, device=dev)
                ex.step(t, g, r1, a1)
                G.gq_fused_step(plan.handle, t, [g], [r2], [msg], a2)
                torch.cuda.synchronize()
                ok &= torch.equal(a1.view(torch.int32), a2.view(torch.int32))
                ok &= torch.equal(r1, r2)
                ok &= torch.equal(ex.buf.gathered, msg)
        ex.close()
        with open(os.path.join(out, "result"), "w") as f:
            f.write("ok" if ok else "mismatch")
    finally:
        dist.destroy_process_group()


def test_exchange_one_rank_matches_fused_step(tmp_path):
    mp.spawn(_main, args=(_free_port(), str(tmp_path)), nprocs=1, join=True)
    assert (tmp_path / "result").read_text() == "ok"
