"""Seeded synthetic gradients shaped like the workloads the pages describe.

This module holds no quantization arithmetic: it only draws inputs.  The tests feed the same
arrays to the CUDA library and to the CPU oracle; the benchmark draws them directly in HBM.

Workloads (named by what they are):

* ``gauss64k``   -- 65,536 elements (128 buckets of 512) i.i.d. N(0, 1e-3), W = 2, one step.
* ``resnet18``   -- 11,689,512 elements concatenated from the ResNet-18 parameter tensors (62
  tensors, torchvision order); tensor k ~ Laplace(0, b_k), log10 b_k ~ U[-4, -2]; W = 4.
* ``resnet50``   -- 25,557,032 elements from the ResNet-50 tensors (161); 1e-3 * Student-t(3),
  0.1 % of the entries (fixed draw without replacement) multiplied by 100; W = 8.
* ``mixture100m``-- 1e8 elements, each a fair-coin choice of N(0, 1e-4) or Laplace(0, 1e-3);
  W = 8; bucket sweep 128 ... 32768.
* ``blocks1b``   -- 1e9 elements in 1000 blocks of 1e6, block k ~ N(0, s_k) with
  log10 s_k ~ U[-5, -2]; W = 8.

The real gradients of the pages' CIFAR / ImageNet CNNs are replaced by these draws: the
tensor sizes are those of the architectures, no dataset or weight is used.
"""
from dataclasses import dataclass, field
from typing import List, Tuple

import torch


# ---------------------------------------------------------------------------------------------
# Parameter-tensor sizes of ResNet-18 / ResNet-50 (torchvision layout, 1000 classes)
# ---------------------------------------------------------------------------------------------
def _bn(c):
    return [c, c]


def resnet_param_sizes(depth: int) -> List[int]:
    """Sizes of the parameter tensors of ResNet-18 or ResNet-50, in registration order."""
    sizes = [64 * 3 * 7 * 7] + _bn(64)
    if depth == 18:
        blocks, expansion = [2, 2, 2, 2], 1
    elif depth == 50:
        blocks, expansion = [3, 4, 6, 3], 4
    else:
        raise ValueError(depth)
    inplanes = 64
    for stage, nblk in enumerate(blocks):
        planes = 64 * 2 ** stage
        for b in range(nblk):
            stride = 2 if (stage > 0 and b == 0) else 1
            out = planes * expansion
            if expansion == 1:
                sizes += [planes * inplanes * 9] + _bn(planes)
                sizes += [planes * planes * 9] + _bn(planes)
            else:
                sizes += [planes * inplanes] + _bn(planes)
                sizes += [planes * planes * 9] + _bn(planes)
                sizes += [out * planes] + _bn(out)
            if stride != 1 or inplanes != out:
                sizes += [out * inplanes] + _bn(out)
            inplanes = out
    sizes += [1000 * inplanes, 1000]
    return sizes


# ---------------------------------------------------------------------------------------------
# Distributions (inverse-CDF / ratio forms, drawn with a seeded torch.Generator)
# ---------------------------------------------------------------------------------------------
def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & 0x7FFFFFFFFFFFFFFF)
    return g


def _laplace_(out: torch.Tensor, b, gen: torch.Generator) -> torch.Tensor:
    """Laplace(0, b) into ``out`` by inverse CDF; ``b`` a float or a broadcastable tensor."""
    u = torch.rand(out.shape, generator=gen, device=out.device, dtype=torch.float32) - 0.5
    # |2u| < 1 strictly (torch.rand can return 0, i.e. u = -0.5, where the inverse CDF is infinite)
    a = (2.0 * u.abs()).clamp_(max=1.0 - 2.0 ** -24)
    out.copy_(-torch.sign(u) * torch.log1p(-a))
    out.mul_(b)
    return out


def _student_t3(n: int, gen: torch.Generator, device) -> torch.Tensor:
    z = torch.randn(n, generator=gen, device=device)
    chi2 = torch.zeros(n, device=device)
    for _ in range(3):
        chi2.add_(torch.randn(n, generator=gen, device=device).square_())
    return z / torch.sqrt(chi2.clamp_(min=1e-30) / 3.0)


def mix_seed(*parts: int) -> int:
    """Deterministic 63-bit seed from small integers (splitmix64 finaliser)."""
    h = 0x9E3779B97F4A7C15
    for p in parts:
        h = (h ^ (int(p) & 0xFFFFFFFFFFFFFFFF)) & 0xFFFFFFFFFFFFFFFF
        h = (h * 0xBF58476D1CE4E5B9) & 0xFFFFFFFFFFFFFFFF
        h ^= h >> 31
    return h & 0x7FFFFFFFFFFFFFFF


# ---------------------------------------------------------------------------------------------
# Workloads
# ---------------------------------------------------------------------------------------------
@dataclass
class Workload:
    name: str
    n: int
    workers: int
    bucket: int
    steps: int
    error_feedback: bool
    schemes: List[Tuple[str, int, float]] = field(default_factory=list)  # (scheme, levels, clip)
    buckets_sweep: Tuple[int, ...] = ()
    seeds: Tuple[int, ...] = ()          # per-worker data seeds (gauss64k)
    rounding_seed: int = 42


WORKLOADS = {
    "gauss64k": Workload("gauss64k", 65536, 2, 512, 1, True,
                         [("qsgd", 5, 0.0), ("bingrad_b", 2, 0.0), ("orq", 5, 0.0)], seeds=(0, 1)),
    "resnet18": Workload("resnet18", sum(resnet_param_sizes(18)), 4, 512, 10, True,
                         [("orq", 3, 0.0), ("orq", 5, 0.0), ("orq", 9, 0.0), ("terngrad", 3, 0.0)]),
    "resnet50": Workload("resnet50", sum(resnet_param_sizes(50)), 8, 512, 10, True,
                         [("bingrad_b", 2, 0.0), ("bingrad_pb", 2, 0.0), ("orq", 3, 2.5)]),
    "mixture100m": Workload("mixture100m", 100_000_000, 8, 512, 1, False,
                            [("orq", 5, 0.0), ("qsgd", 5, 0.0)],
                            buckets_sweep=(128, 512, 2048, 8192, 32768)),
    "blocks1b": Workload("blocks1b", 1_000_000_000, 8, 512, 5, True,
                         [("orq", 5, 0.0), ("bingrad_b", 2, 0.0)]),
}


def tensor_offsets(workload: str, n: int = None) -> List[int]:
    """The parameter tensors of a workload with tensor structure, as offsets into its gradient
    (nseg + 1 values from 0 to n): resnet18 / resnet50, their parameter tensors in order;
    blocks1b, its 1e6-element blocks.  ``n`` truncates the vector (the last tensor is cut)."""
    wl = WORKLOADS[workload]
    n = wl.n if n is None else int(n)
    if workload in ("resnet18", "resnet50"):
        sizes = resnet_param_sizes(18 if workload == "resnet18" else 50)
    elif workload == "blocks1b":
        sizes = [1_000_000] * ((n + 999_999) // 1_000_000)
    else:
        raise KeyError("%s has no tensor structure" % workload)
    off = [0]
    for sz in sizes:
        if off[-1] >= n:
            break
        off.append(min(n, off[-1] + sz))
    return off


def gradient(workload: str, worker: int, step: int, n: int = None, device="cpu",
             out: torch.Tensor = None) -> torch.Tensor:
    """Worker ``worker``'s fp32 gradient at ``step`` for ``workload``.

    ``n`` truncates the workload to its first n elements (same distribution per element
    position as the full vector for the segment-shaped workloads).  ``out`` (float32, length n,
    on ``device``) is filled in place when given.
    """
    wl = WORKLOADS[workload]
    n = wl.n if n is None else int(n)
    if out is None:
        out = torch.empty(n, dtype=torch.float32, device=device)
    elif out.numel() != n:
        raise ValueError("out holds %d elements, the request is for %d" % (out.numel(), n))
    device = out.device
    if workload == "gauss64k":
        seed = wl.seeds[worker] if worker < len(wl.seeds) else mix_seed(1, worker, step)
        gen = _gen(mix_seed(seed, step), device)
        torch.randn(n, generator=gen, device=device, out=out)
        out.mul_(1e-3)
    elif workload in ("resnet18", "resnet50"):
        depth = 18 if workload == "resnet18" else 50
        sizes = resnet_param_sizes(depth)
        gen = _gen(mix_seed(depth, worker, step), device)
        if depth == 18:
            # per-tensor Laplace scale, fixed per tensor (drawn from a workload-wide seed)
            sgen = torch.Generator().manual_seed(18)
            logb = torch.rand(len(sizes), generator=sgen) * 2.0 - 4.0
            scale = torch.repeat_interleave(10.0 ** logb, torch.tensor(sizes))[:n].to(device)
            _laplace_(out, scale, gen)
        else:
            out.copy_(_student_t3(n, gen, device) * 1e-3)
            ogen = torch.Generator().manual_seed(50)
            k = max(1, wl.n // 1000)
            idx = torch.randperm(wl.n, generator=ogen)[:k]
            idx = idx[idx < n].to(device)
            out[idx] *= 100.0
    elif workload == "mixture100m":
        gen = _gen(mix_seed(100, worker, step), device)
        a = torch.randn(n, generator=gen, device=device).mul_(1e-4)
        b = _laplace_(torch.empty(n, device=device), 1e-3, gen)
        coin = torch.rand(n, generator=gen, device=device) < 0.5
        out.copy_(torch.where(coin, a, b))
    elif workload == "blocks1b":
        gen = _gen(mix_seed(1000, worker, step), device)
        blk = 1_000_000
        nblk = (n + blk - 1) // blk
        sgen = torch.Generator().manual_seed(1000)
        sig = 10.0 ** (torch.rand(max(nblk, 1000), generator=sgen) * 3.0 - 5.0)
        torch.randn(n, generator=gen, device=device, out=out)
        full = (n // blk) * blk
        if full:
            out[:full].view(-1, blk).mul_(sig[: n // blk].to(device)[:, None])
        if full < n:
            out[full:].mul_(float(sig[n // blk]))
    else:
        raise KeyError(workload)
    return out


def special_bucket(kind: str, d: int, seed: int = 0) -> torch.Tensor:
    """Edge-case buckets: constant, zero, grid-aligned, two-valued, tiny, spiky."""
    gen = torch.Generator().manual_seed(seed)
    if kind == "zero":
        return torch.zeros(d)
    if kind == "constant":
        return torch.full((d,), 0.0123)
    if kind == "negconst":
        return torch.full((d,), -3.5e-4)
    if kind == "grid":
        # values exactly on the 64-point grid of [-1, 1]
        j = torch.randint(0, 64, (d,), generator=gen)
        return (-1.0 + j.float() * (2.0 / 63.0)).float()
    if kind == "twovalue":
        c = torch.rand(d, generator=gen) < 0.3
        return torch.where(c, torch.tensor(2e-3), torch.tensor(-5e-4))
    if kind == "tiny":
        return torch.randn(d, generator=gen) * 1e-30
    if kind == "spike":
        x = torch.randn(d, generator=gen) * 1e-4
        x[d // 3] = 0.5
        return x
    if kind == "subnormal":
        return torch.randn(d, generator=gen) * 1e-40
    raise KeyError(kind)
