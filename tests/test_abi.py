"""The C-ABI library without a GPU: it loads, exports every symbol include/gq.h declares, and
its host-side logic (argument checks, message layout, status strings) is right.  The layout is
checked against the oracle's own, independently written, layout computation."""
import ctypes
import os
import re
import subprocess

import pytest

import gradient_quantization_communication_b200.gq as G
import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    with open(os.path.join(ROOT, "include", "gq.h")) as f:
        hdr = f.read()
    return re.findall(r"GQ_API\s+[\w\s\*]+?\b(gq_\w+)\s*\(", hdr)


def test_exports_every_declared_symbol():
    names = _declared()
    assert len(names) >= 10
    L = ctypes.CDLL(G.LIB_PATH)
    for n in names:
        assert hasattr(L, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", G.LIB_PATH], capture_output=True, text=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln and ln.split()[-1].startswith("gq_")}
    assert exported == set(names)


def test_library_has_sm100a_code():
    out = subprocess.run(["cuobjdump", "--list-elf", G.LIB_PATH], capture_output=True, text=True).stdout
    assert "sm_100a" in out


def test_version_and_status_strings():
    assert G.gq_version().count(".") == 2
    assert G.gq_status_string(G.GQ_OK) == "ok"
    assert G.gq_status_string(G.GQ_ERR_NONFINITE) == "non-finite input value"
    assert "unknown" in G.gq_status_string(99)


@pytest.mark.parametrize("kw,ok", [
    (dict(scheme="orq", levels=5), True),
    (dict(scheme="orq", levels=16), True),
    (dict(scheme="orq", levels=17), False),
    (dict(scheme="orq", levels=1), False),
    (dict(scheme="qsgd", levels=2), True),
    (dict(scheme="terngrad", levels=0), True),
    (dict(scheme="terngrad", levels=5), False),
    (dict(scheme="bingrad_b", levels=0), True),
    (dict(scheme="bingrad_pb", levels=3), False),
    (dict(scheme=9, levels=3), False),
    (dict(scheme="terngrad_layer", levels=3), True),
    (dict(scheme="terngrad_layer", levels=0), True),
    (dict(scheme="terngrad_layer", levels=5), False),
    (dict(scheme="orq", levels=5, bucket=64), False),
    (dict(scheme="orq", levels=5, bucket=384), False),
    (dict(scheme="orq", levels=5, bucket=65536), False),
    (dict(scheme="orq", levels=5, bucket=32768), True),
    (dict(scheme="orq", levels=5, workers=0), False),
    (dict(scheme="orq", levels=5, workers=65), False),
    (dict(scheme="orq", levels=5, clip_sigma=-1.0), False),
    (dict(scheme="orq", levels=5, clip_sigma=float("inf")), False),
    (dict(scheme="orq", levels=5, n=-1), False),
    (dict(scheme="orq", levels=5, n=1 << 40), False),
    (dict(scheme="orq", levels=5, n=0), True),
])
def test_config_check(kw, ok):
    base = dict(bucket=512, workers=2, error_feedback=True, clip_sigma=0.0, seed=1, n=1000)
    base.update(kw)
    st = G.gq_config_check(G.gq_config(**base))
    assert (st == G.GQ_OK) == ok
    if not ok:
        assert st == G.GQ_ERR_INVALID


@pytest.mark.parametrize("scheme,levels", [(0, 5), (1, 3), (2, 2), (3, 2), (4, 2), (4, 5), (4, 9), (0, 16), (4, 3)])
@pytest.mark.parametrize("d", [128, 512, 4096, 32768])
@pytest.mark.parametrize("n", [0, 1, 127, 1000, 11689512, 10 ** 9])
def test_message_layout_matches_oracle(scheme, levels, d, n):
    mine = G.gq_message_layout(G.gq_config(scheme, levels, d, 1, True, 0.0, 0, n))
    ref = O.message_layout(O.Config(scheme, levels, d, 1, 1, 0.0, 0, n))
    assert mine == ref
    assert mine[2] % 16 == 0 and mine[0] % 16 == 0


def test_compression_ratio_orq5_d512():
    # 3 bits per element plus a 5-float table per 512-element bucket
    n = 512 * 1000
    nbytes, _, _ = G.gq_message_layout(G.gq_config("orq", 5, 512, 1, True, 0.0, 0, n))
    assert abs(32 * n / (8 * nbytes) - 9.6603773) < 1e-6


def test_plan_create_without_device_fails_cleanly():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    with pytest.raises(G.GQError) as ei:
        G.gq_plan_create(G.gq_config("orq", 5, 512, 1, True, 0.0, 0, 100))
    assert ei.value.status == G.GQ_ERR_CUDA


@pytest.mark.parametrize("scheme,levels", [(0, 5), (1, 0), (1, 3), (4, 3), (4, 5), (4, 9), (0, 9), (0, 3)])
@pytest.mark.parametrize("d", [128, 512, 4096, 32768])
@pytest.mark.parametrize("n", [0, 1, 127, 1000, 11689512, 10 ** 9])
def test_entropy_layout_matches_oracle(scheme, levels, d, n):
    mine = G.gq_entropy_layout(G.gq_config(scheme, levels, d, 1, True, 0.0, 0, n))
    ref = O.entropy_layout(O.Config(scheme, levels or 3, d, 1, 1, 0.0, 0, n))
    assert mine == ref
    assert mine[2] % 16 == 0 and mine[0] % 16 == 0


@pytest.mark.parametrize("scheme,levels", [(0, 2), (0, 4), (4, 16), (2, 0), (3, 2), (4, 7)])
def test_entropy_unsupported_levels(scheme, levels):
    cfg = G.gq_config(scheme, levels, 512, 1, True, 0.0, 0, 1000)
    for call in (lambda: G.gq_entropy_layout(cfg), lambda: G.gq_entropy_pack(cfg, 0, 0, stream=0),
                 lambda: G.gq_entropy_unpack(cfg, 0, 0, stream=0)):
        with pytest.raises(G.GQError) as ei:
            call()
        assert ei.value.status == G.GQ_ERR_UNSUPPORTED


def test_entropy_argument_checks_without_device():
    """Argument errors are found on the host before anything touches a device."""
    cfg = G.gq_config("orq", 5, 512, 1, True, 0.0, 0, 5000)
    nbytes, _, _ = G.gq_message_layout(cfg)
    ebytes, _, _ = G.gq_entropy_layout(cfg)
    base = 1 << 40  # never dereferenced: every case below fails its checks first
    cases = [(0, base), (base, 0), (base + 4, base + (1 << 30)), (base, base + (1 << 30) + 8),
             (base, base + 16),                      # overlapping
             (base + ebytes - 16, base)]             # overlapping the other way
    for a, b in cases:
        for call in (G.gq_entropy_pack, G.gq_entropy_unpack):
            with pytest.raises(G.GQError) as ei:
                call(cfg, a, b, stream=0)
            assert ei.value.status == G.GQ_ERR_INVALID, (call.__name__, a, b)
    bad = G.gq_config("orq", 5, 384, 1, True, 0.0, 0, 5000)
    with pytest.raises(G.GQError) as ei:
        G.gq_entropy_pack(bad, base, base + (1 << 30), stream=0)
    assert ei.value.status == G.GQ_ERR_INVALID
    # n = 0: a no-op, NULL pointers allowed
    G.gq_entropy_pack(G.gq_config("orq", 5, 512, 1, True, 0.0, 0, 0), 0, 0, stream=0)
    G.gq_entropy_unpack(G.gq_config("orq", 5, 512, 1, True, 0.0, 0, 0), 0, 0, stream=0)
    assert ebytes < nbytes


@pytest.mark.parametrize("scheme,levels,ratio", [(1, 3, 32 * 512 / (26 * 32 + 32)),      # TernGrad
                                                 (4, 3, 32 * 512 / (26 * 32 + 3 * 32)),  # ORQ-3
                                                 (0, 9, 32 * 512 / (52 * 32 + 32)),      # QSGD-9
                                                 (4, 9, 32 * 512 / (52 * 32 + 9 * 32))])  # ORQ-9
def test_entropy_compression_ratio_d512(scheme, levels, ratio):
    """Base-s messages at d = 512: 26 words (s = 3) or 52 words (s = 9) of codes per bucket plus
    the level table; without the table the ratios are 32 * 512 / 832 = 19.7 and 9.85."""
    n = 512 * 1000
    nbytes, _, _ = G.gq_entropy_layout(G.gq_config(scheme, levels, 512, 1, True, 0.0, 0, n))
    assert abs(32 * n / (8 * nbytes) - ratio) < 1e-9



@pytest.mark.parametrize("scheme,levels", [(5, 2), (5, 3), (5, 15), (5, 16), (6, 2), (6, 0), (7, 3), (7, 16)])
@pytest.mark.parametrize("d", [128, 256, 512])
@pytest.mark.parametrize("n", [0, 1, 1000, 10 ** 9])
def test_biased_layout_matches_oracle(scheme, levels, d, n):
    mine = G.gq_message_layout(G.gq_config(scheme, levels, d, 1, True, 0.0, 0, n))
    ref = O.message_layout(O.Config(scheme, levels or 2, d, 1, 1, 0.0, 0, n))
    assert mine == ref


def test_terngrad_layer_host_checks():
    """Per-tensor TernGrad: no clipping; its message is sized by the tensors, so the
    configuration-only layouts (dense, base-s, Elias) refuse it."""
    cfg = G.gq_config("terngrad_layer", 3, 512, 2, True, 0.0, 0, 1000)
    assert G.gq_config_check(cfg) == G.GQ_OK
    assert G.gq_config_check(G.gq_config("terngrad_layer", 3, 512, 2, True, 2.5, 0, 1000)) == G.GQ_ERR_UNSUPPORTED
    for call in (lambda: G.gq_message_layout(cfg), lambda: G.gq_entropy_layout(cfg), lambda: G.gq_elias_layout(cfg)):
        with pytest.raises(G.GQError) as ei:
            call()
        assert ei.value.status == G.GQ_ERR_UNSUPPORTED


@pytest.mark.parametrize("kw,status", [
    (dict(scheme="qsgd_nearest", levels=5, bucket=1024), "GQ_ERR_UNSUPPORTED"),
    (dict(scheme="signsgd", levels=2, bucket=2048), "GQ_ERR_UNSUPPORTED"),
    (dict(scheme="qsgd_l2", levels=3, bucket=1024), "GQ_ERR_UNSUPPORTED"),
    (dict(scheme="qsgd_l2", levels=3, bucket=512), "GQ_OK"),
    (dict(scheme="signsgd", levels=3, bucket=512), "GQ_ERR_INVALID"),
    (dict(scheme="qsgd_nearest", levels=17, bucket=512), "GQ_ERR_INVALID"),
    (dict(scheme="qsgd_nearest", levels=1, bucket=512), "GQ_ERR_INVALID"),
    (dict(scheme="signsgd", levels=0, bucket=512), "GQ_OK"),
    (dict(scheme="qsgd_nearest", levels=16, bucket=128), "GQ_OK"),
])
def test_biased_config_check(kw, status):
    cfg = G.gq_config(kw["scheme"], kw["levels"], kw["bucket"], 1, True, 0.0, 0, 1000)
    assert G.gq_config_check(cfg) == getattr(G, status)


@pytest.mark.parametrize("scheme,levels", [(0, 3), (0, 5), (1, 0), (5, 9), (7, 3), (7, 15)])
@pytest.mark.parametrize("d", [128, 256, 512])
@pytest.mark.parametrize("n", [0, 1, 1000, 10 ** 9])
def test_elias_layout_matches_oracle(scheme, levels, d, n):
    cfg = G.gq_config(scheme, levels, d, 1, True, 0.0, 0, n)
    mine = G.gq_elias_layout(cfg)
    ref = O.elias_layout(O.Config(scheme, levels or 3, d, 1, 1, 0.0, 0, n))
    assert mine == ref
    assert all(x % 16 == 0 for x in mine)
    assert G.gq_elias_used_bytes(cfg, 0) == mine[3]
    if n > 0:
        assert G.gq_elias_used_bytes(cfg, 33) == mine[3] + 16


@pytest.mark.parametrize("scheme,levels,d", [(4, 5, 512), (0, 4, 512), (0, 5, 1024), (2, 0, 512), (6, 2, 512),
                                             (7, 2, 256)])
def test_elias_unsupported(scheme, levels, d):
    cfg = G.gq_config(scheme, levels, d, 1, True, 0.0, 0, 1000)
    for call in (lambda: G.gq_elias_layout(cfg), lambda: G.gq_elias_pack(cfg, 0, 0, stream=0),
                 lambda: G.gq_elias_unpack(cfg, 0, 0, stream=0)):
        with pytest.raises(G.GQError) as ei:
            call()
        assert ei.value.status == G.GQ_ERR_UNSUPPORTED


def test_elias_argument_checks_without_device():
    cfg = G.gq_config("qsgd_l2", 3, 512, 1, True, 0.0, 0, 5000)
    cap = G.gq_elias_layout(cfg)[0]
    base = 1 << 40  # never dereferenced: every case fails its checks first
    for a, b in [(0, base), (base, 0), (base + 8, base + (1 << 30)), (base, base + 16), (base + 16, base)]:
        for call in (G.gq_elias_pack, G.gq_elias_unpack):
            with pytest.raises(G.GQError) as ei:
                call(cfg, a, b, stream=0)
            assert ei.value.status == G.GQ_ERR_INVALID
    with pytest.raises(G.GQError):
        G.gq_elias_used_bytes(cfg, 8 * cap)
    G.gq_elias_pack(G.gq_config("qsgd_l2", 3, 512, 1, True, 0.0, 0, 0), 0, 0, stream=0)
