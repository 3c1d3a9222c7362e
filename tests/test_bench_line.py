"""The benchmark's JSON line and roofline object, built on the CPU from given timings (the
GPU run feeds the same functions): every contract field, the metric's name, and the stored
DRAM traffic applied only to its captured configuration, scaled by the element count."""
import sys

import pytest

import bench
from gradient_quantization_communication_b200 import synth


def _args(*argv):
    old = sys.argv
    sys.argv = ["bench.py", *argv]
    try:
        return bench.parse_args()
    finally:
        sys.argv = old


def test_default_line_fields():
    args = _args()
    wl = synth.WORKLOADS[args.workload]
    W, n = wl.workers, wl.n
    bpe = bench.bytes_per_worker_elem(4, 5, 512, W, True, True)
    assert abs(bpe - 12.914) < 1e-3
    ms = 26.0
    peak = 6541.1
    achieved = bpe * W * n / (ms / 1000) / 1e9
    roof = bench.fused_roofline(args, 512, W, n, True, True, bpe, achieved, peak, "measured")
    value = W * n / (ms / 1000)
    line = bench.default_line(args, wl, value, 1, W, n, ms, bpe, peak, roof, None, None, 5, {})
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "roofline", "cpu_baseline", "e2e", "gpu_launches", "clocks"):
        assert k in line, k
    assert line["metric"] == bench.METRIC and line["config"]["workload"].startswith("blocks1b")
    assert line["pct_hbm_peak"] == pytest.approx(100 * achieved / peak, abs=0.01)
    assert line["pct_hbm_spec"] == pytest.approx(100 * achieved / 8000.0, abs=0.01)
    assert line["elem_per_s_per_worker"] == pytest.approx(n / (ms / 1000))
    r = line["roofline"]
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["frac"] == pytest.approx(achieved / peak, abs=1e-4)
    assert r["algorithmic_bytes_per_launch"] == pytest.approx(bpe * W * n)
    rec = bench.traffic_record("fused_orq5_d512_w8")
    if rec is None:  # the kernel's sources changed since the capture: the line must say null
        assert r["traffic"] is None
    else:
        assert r["traffic"] == pytest.approx(rec["bytes_per_launch"])
        # DRAM traffic within 2 % of the algorithmic bytes: nothing is read twice
        assert abs(r["traffic"] / r["algorithmic_bytes_per_launch"] - 1) < 0.02


def test_traffic_scaled_and_matched():
    args = _args("--elements", "5120000")
    n, W = 5120000, 8
    bpe = bench.bytes_per_worker_elem(4, 5, 512, W, True, True)
    r = bench.fused_roofline(args, 512, W, n, True, True, bpe, 4000.0, 6541.1, "measured")
    rec = bench.traffic_record("fused_orq5_d512_w8")
    if rec is not None:
        assert r["traffic"] == pytest.approx(rec["bytes_per_launch"] * n / 1e9)
    # other configurations have no stored figure
    assert bench.fused_roofline(args, 512, W, n, False, True, bpe, 4000.0, 6541.1, "measured")["traffic"] is None
    assert bench.fused_roofline(args, 512, W, n, True, False, bpe, 4000.0, 6541.1, "measured")["traffic"] is None
    a2 = _args("--workload", "mixture100m")
    assert bench.fused_roofline(a2, 512, W, n, True, True, bpe, 4000.0, 6541.1, "measured")["traffic"] is None
    a3 = _args("--scheme", "qsgd")
    assert bench.fused_roofline(a3, 512, W, n, True, True, bpe, 4000.0, 6541.1, "measured")["traffic"] is None
    # no roofline object above d = 512 (two kernels per step)
    assert bench.fused_roofline(args, 2048, W, n, True, True, bpe, None, 6541.1, "measured") is None


def test_metric_name_follows_the_configuration():
    assert bench.metric_name(_args()) == bench.METRIC
    assert "signsgd-2 d=512" in bench.metric_name(_args("--scheme", "signsgd", "--levels", "2"))
    assert "orq-5 d=2048" in bench.metric_name(_args("--bucket", "2048"))


@pytest.mark.parametrize("scheme,levels", [(4, 3), (4, 5), (4, 9), (0, 5), (1, 3)])
@pytest.mark.parametrize("d", [128, 256, 512])
def test_message_bytes_match_the_oracle_layouts(scheme, levels, d):
    """The bench's message bytes per element, dense and base-s, times the elements of whole
    buckets equal the oracle's message sizes without their 16-byte padding."""
    import oracle as O
    nb = 1000
    co = O.Config(scheme, levels, d, 1, 1, 0.0, 0, nb * d)
    L = O.table_len(scheme, levels)
    dense = bench.message_bytes_per_elem(scheme, levels, d) * d * nb
    assert dense == nb * d * ((levels - 1).bit_length()) / 8 + 4 * L * nb
    assert O.message_layout(co)[0] - dense < 32
    bases = bench.message_bytes_per_elem(scheme, levels, d, base_s=True) * d * nb
    assert abs(bases - (nb * O.entropy_words(co) * 4 + 4 * L * nb)) < 1e-6
    assert 0 <= O.entropy_layout(co)[0] - bases < 32
    args = _args("--base-s", "--levels", str(levels))
    assert args.base_s


def test_tensor_offsets():
    """The per-tensor TernGrad bench's tensors: the parameter tensors of the resnet workloads and
    the 1e6-element blocks of blocks1b, as offsets from 0 to n, cut at a truncated n."""
    off = synth.tensor_offsets("resnet50")
    assert len(off) - 1 == 161 and off[0] == 0 and off[-1] == synth.WORKLOADS["resnet50"].n
    assert all(b > a for a, b in zip(off, off[1:]))
    assert [b - a for a, b in zip(off, off[1:])] == synth.resnet_param_sizes(50)
    assert synth.tensor_offsets("blocks1b", 2_500_000) == [0, 1_000_000, 2_000_000, 2_500_000]
    cut = synth.tensor_offsets("resnet18", 100_000)
    assert cut[-1] == 100_000 and all(b > a for a, b in zip(cut, cut[1:]))
    with pytest.raises(KeyError):
        synth.tensor_offsets("mixture100m")
