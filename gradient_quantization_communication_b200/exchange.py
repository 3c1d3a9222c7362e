"""Data-parallel exchange of quantized gradients: one worker per rank.

The glossary "gradient quantization for communication" (sections The Problem, How Gradient
Quantization Works, Frameworks) describes the step this module runs across processes: every
worker quantizes its own gradient, the quantized messages travel over the collective library
(NCCL on GPUs), and every worker dequantizes and averages what it received.  Here

  1. rank w encodes its gradient into its message with gq_encode (Philox worker index w, error
     feedback on its own residual);
  2. the W messages are all-gathered in rank order (torch.distributed.all_gather_into_tensor:
     NCCL over NVLink between GPUs; the packed codes and level tables are the only bytes that
     cross the link, 0.414 B per element for ORQ-5 at d = 512);
  3. every rank decodes and sums the W messages with gq_decode_accumulate into its average.

The average equals, bit for bit, that of gq_fused_step over the same W gradients on one GPU:
the encode of worker w is the same, and the decode sums the workers in the same order.

Only plumbing lives here (buffers, the collective, the order of the calls); every step of the
path runs in the library's kernels.  The encode and decode callables can be replaced, which is
how the exchange logic is tested on CPU ranks.
"""
from dataclasses import dataclass
from typing import Callable, Optional

import torch
import torch.distributed as dist

from . import gq as G


@dataclass
class ExchangeBuffers:
    msg: torch.Tensor        # this rank's message (uint8)
    gathered: torch.Tensor   # the W messages, rank order (uint8, W * msg_bytes)


class Exchange:
    """One quantized all-gather step per call, for one worker per rank.

    cfg      gq_config_t of the whole job: workers = world size, n = elements per worker.
    group    the process group (default: the world).
    encode   encode(step, rank, grad, residual, msg) -> None; default gq_encode.
    decode   decode(messages, avg) -> None (messages: list of W uint8 tensors); default
             gq_decode_accumulate.
    """

    def __init__(self, cfg, group=None, device=None, encode: Optional[Callable] = None,
                 decode: Optional[Callable] = None, msg_bytes: Optional[int] = None):
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        if cfg.workers != self.world:
            raise ValueError("the configuration has %d workers, the group %d ranks" % (cfg.workers, self.world))
        self.cfg = cfg
        self.device = device if device is not None else torch.device("cpu")
        self.plan = None
        if encode is None or decode is None:
            self.plan = G.Plan(cfg)
            msg_bytes = self.plan.msg_bytes
        if msg_bytes is None:
            raise ValueError("msg_bytes is required with custom encode/decode callables")
        self.msg_bytes = msg_bytes
        self._encode = encode or self._gq_encode
        self._decode = decode or self._gq_decode
        self.buf = ExchangeBuffers(
            msg=torch.zeros(msg_bytes, dtype=torch.uint8, device=self.device),
            gathered=torch.zeros(self.world * msg_bytes, dtype=torch.uint8, device=self.device))

    def _gq_encode(self, step, rank, grad, residual, msg):
        G.gq_encode(self.plan.handle, rank, step, grad, residual, msg)

    def _gq_decode(self, messages, avg):
        G.gq_decode_accumulate(self.plan.handle, messages, avg)

    def messages(self):
        """Views of the W gathered messages, rank order."""
        b = self.msg_bytes
        return [self.buf.gathered[w * b:(w + 1) * b] for w in range(self.world)]

    def step(self, step, grad, residual, avg, events=None):
        """Quantize this rank's gradient, exchange the messages, write the average to avg.
        events: optional four CUDA events, recorded on the current stream before the encode,
        after it, after the all-gather (whose completion the current stream waits for) and after
        the decode."""
        if events is not None:
            events[0].record()
        self._encode(step, self.rank, grad, residual, self.buf.msg)
        if events is not None:
            events[1].record()
        dist.all_gather_into_tensor(self.buf.gathered, self.buf.msg, group=self.group)
        if events is not None:
            events[2].record()
        self._decode(self.messages(), avg)
        if events is not None:
            events[3].record()

    def close(self):
        if self.plan is not None:
            self.plan.close()
            self.plan = None
