"""ctypes wrapper of the plain C oracle (``oracle/gq_oracle.c``).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import this package.  It shares no code with the CUDA library.
"""
import ctypes
import os
from dataclasses import dataclass

import numpy as np

from . import build as _build

QSGD, TERNGRAD, BINGRAD_B, BINGRAD_PB, ORQ, QSGD_NEAREST, SIGNSGD, QSGD_L2 = 0, 1, 2, 3, 4, 5, 6, 7
SCHEMES = {"qsgd": QSGD, "terngrad": TERNGRAD, "bingrad_b": BINGRAD_B, "bingrad_pb": BINGRAD_PB, "orq": ORQ,
           "qsgd_nearest": QSGD_NEAREST, "signsgd": SIGNSGD, "qsgd_l2": QSGD_L2}


class _Cfg(ctypes.Structure):
    _fields_ = [("scheme", ctypes.c_int32), ("levels", ctypes.c_int32),
                ("bucket", ctypes.c_int32), ("workers", ctypes.c_int32),
                ("error_feedback", ctypes.c_int32), ("clip_sigma", ctypes.c_float),
                ("seed", ctypes.c_uint64), ("n", ctypes.c_int64)]


@dataclass
class Config:
    scheme: int
    levels: int
    bucket: int = 512
    workers: int = 1
    error_feedback: int = 1
    clip_sigma: float = 0.0
    seed: int = 0
    n: int = 0

    def c(self) -> _Cfg:
        return _Cfg(self.scheme, self.levels, self.bucket, self.workers, self.error_feedback,
                    self.clip_sigma, self.seed, self.n)


_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.POINTER
        f32p, i32p, u8p, u32p = P(ctypes.c_float), P(ctypes.c_int), P(ctypes.c_uint8), P(ctypes.c_uint32)
        i64 = ctypes.c_int64
        L.or_philox4x32_10.argtypes = [u32p, u32p, u32p]
        L.or_uniform.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint32, i64]
        L.or_uniform.restype = ctypes.c_float
        L.or_fexpo.argtypes = [ctypes.c_float]
        L.or_clip_threshold.argtypes = [f32p, ctypes.c_int, ctypes.c_float]
        L.or_clip_threshold.restype = ctypes.c_float
        L.or_grid.argtypes = [f32p, ctypes.c_int, f32p]
        L.or_sign_scale.argtypes = [f32p, ctypes.c_int]
        L.or_sign_scale.restype = ctypes.c_float
        L.or_l2_scale.argtypes = [f32p, ctypes.c_int]
        L.or_l2_scale.restype = ctypes.c_float
        L.or_elias_layout.argtypes = [P(_Cfg), P(i64), P(i64), P(i64), P(i64)]
        L.or_elias_pack.argtypes = [P(_Cfg), u8p, u8p]
        L.or_elias_pack.restype = i64
        L.or_elias_unpack.argtypes = [P(_Cfg), u8p, u8p]
        L.or_elias_gamma_len.argtypes = [ctypes.c_uint32]
        L.or_orq_select.argtypes = [f32p, ctypes.c_int, ctypes.c_int, i32p]
        L.or_orq_select.restype = ctypes.c_double
        L.or_bingrad_b_fit.argtypes = [f32p, ctypes.c_int, f32p, f32p, f32p, i32p]
        L.or_bingrad_pb_fit.argtypes = [f32p, ctypes.c_int, i32p, i32p, f32p, f32p]
        L.or_bits.argtypes = [ctypes.c_int]
        L.or_table_len.argtypes = [ctypes.c_int, ctypes.c_int]
        L.or_num_buckets.argtypes = [P(_Cfg)]
        L.or_num_buckets.restype = i64
        L.or_message_layout.argtypes = [P(_Cfg), P(i64), P(i64), P(i64)]
        L.or_encode_bucket.argtypes = [P(_Cfg), ctypes.c_int, ctypes.c_uint64, i64, f32p, ctypes.c_int,
                                       u8p, f32p, f32p]
        L.or_pack_bucket.argtypes = [P(_Cfg), u8p, ctypes.c_int, u32p]
        L.or_unpack_bucket.argtypes = [P(_Cfg), u32p, ctypes.c_int, u8p]
        L.or_dequant.argtypes = [P(_Cfg), f32p, ctypes.c_int]
        L.or_dequant.restype = ctypes.c_float
        L.or_encode.argtypes = [P(_Cfg), ctypes.c_int, ctypes.c_uint64, i64, i64, f32p, f32p, u8p]
        L.or_decode_accumulate.argtypes = [P(_Cfg), P(u8p), ctypes.c_int, i64, i64, f32p]
        L.or_fused_step.argtypes = [P(_Cfg), ctypes.c_uint64, i64, i64, P(f32p), P(f32p), P(u8p), f32p]
        L.or_quant_error.argtypes = [P(_Cfg), ctypes.c_int, ctypes.c_uint64, i64, i64, f32p, f32p,
                                     P(ctypes.c_double)]
        L.or_entropy_groups.argtypes = [ctypes.c_int, i32p, i32p]
        L.or_entropy_words.argtypes = [P(_Cfg)]
        L.or_entropy_words.restype = i64
        L.or_entropy_layout.argtypes = [P(_Cfg), P(i64), P(i64), P(i64)]
        L.or_entropy_pack.argtypes = [P(_Cfg), u8p, u8p]
        L.or_entropy_unpack.argtypes = [P(_Cfg), u8p, u8p]
        L.or_fused_bucket.argtypes = [P(_Cfg), ctypes.c_uint64, i64, ctypes.c_int, P(f32p), P(f32p), P(f32p),
                                      P(u32p), P(f32p), f32p]
        i64p = P(i64)
        L.or_tg_layer_layout.argtypes = [P(_Cfg), ctypes.c_int, P(i64), P(i64), P(i64)]
        L.or_tg_layer_encode.argtypes = [P(_Cfg), i64p, ctypes.c_int, ctypes.c_int, ctypes.c_uint64, f32p, f32p, u8p]
        L.or_tg_layer_decode_accumulate.argtypes = [P(_Cfg), i64p, ctypes.c_int, P(u8p), ctypes.c_int, f32p]
        _lib = L
    return _lib


def _p(a, ct):
    return a.ctypes.data_as(ctypes.POINTER(ct))


def _f32(a):
    a = np.ascontiguousarray(a, dtype=np.float32)
    return a


def philox(ctr, key):
    c = np.asarray(ctr, dtype=np.uint32).copy()
    k = np.asarray(key, dtype=np.uint32).copy()
    out = np.zeros(4, dtype=np.uint32)
    lib().or_philox4x32_10(_p(c, ctypes.c_uint32), _p(k, ctypes.c_uint32), _p(out, ctypes.c_uint32))
    return out


def uniform(seed, step, worker, i):
    return lib().or_uniform(seed, step, worker, i)


def fexpo(m):
    return lib().or_fexpo(float(m))


def clip_threshold(v, c):
    v = _f32(v)
    return lib().or_clip_threshold(_p(v, ctypes.c_float), len(v), c)


def sign_scale(u):
    u = _f32(u)
    return lib().or_sign_scale(_p(u, ctypes.c_float), len(u))


def l2_scale(u):
    u = _f32(u)
    return lib().or_l2_scale(_p(u, ctypes.c_float), len(u))


def grid(u):
    u = _f32(u)
    g = np.zeros(64, dtype=np.float32)
    ok = lib().or_grid(_p(u, ctypes.c_float), len(u), _p(g, ctypes.c_float))
    return bool(ok), g


def orq_select(u, s):
    u = _f32(u)
    idx = np.zeros(s, dtype=np.int32)
    var = lib().or_orq_select(_p(u, ctypes.c_float), len(u), s, _p(idx, ctypes.c_int))
    return var, idx


def bingrad_b_fit(u):
    u = _f32(u)
    a, b, t = ctypes.c_float(), ctypes.c_float(), ctypes.c_float()
    k = ctypes.c_int()
    lib().or_bingrad_b_fit(_p(u, ctypes.c_float), len(u), ctypes.byref(a), ctypes.byref(b),
                           ctypes.byref(t), ctypes.byref(k))
    return a.value, b.value, t.value, k.value


def bingrad_pb_fit(u):
    u = _f32(u)
    A, B = ctypes.c_int(), ctypes.c_int()
    ga, gb = ctypes.c_float(), ctypes.c_float()
    lib().or_bingrad_pb_fit(_p(u, ctypes.c_float), len(u), ctypes.byref(A), ctypes.byref(B),
                            ctypes.byref(ga), ctypes.byref(gb))
    return A.value, B.value, ga.value, gb.value


def bits(levels):
    return lib().or_bits(levels)


def table_len(scheme, levels):
    return lib().or_table_len(scheme, levels)


def num_buckets(cfg: Config):
    return lib().or_num_buckets(ctypes.byref(cfg.c()))


def message_layout(cfg: Config):
    b, c, l = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
    lib().or_message_layout(ctypes.byref(cfg.c()), ctypes.byref(b), ctypes.byref(c), ctypes.byref(l))
    return b.value, c.value, l.value


def encode_bucket(cfg: Config, worker, step, bucket, v):
    v = _f32(v)
    n = len(v)
    code = np.zeros(max(n, 1), dtype=np.uint8)
    q = np.zeros(max(n, 1), dtype=np.float32)
    table = np.zeros(16, dtype=np.float32)
    rc = lib().or_encode_bucket(ctypes.byref(cfg.c()), worker, step, bucket, _p(v, ctypes.c_float), n,
                                _p(code, ctypes.c_uint8), _p(q, ctypes.c_float), _p(table, ctypes.c_float))
    assert rc == 0
    return code[:n], q[:n], table[:table_len(cfg.scheme, cfg.levels)]


def pack_bucket(cfg: Config, code):
    code = np.ascontiguousarray(code, dtype=np.uint8)
    words = np.zeros(cfg.bucket * bits(cfg.levels) // 32, dtype=np.uint32)
    lib().or_pack_bucket(ctypes.byref(cfg.c()), _p(code, ctypes.c_uint8), len(code), _p(words, ctypes.c_uint32))
    return words


def unpack_bucket(cfg: Config, words, n):
    words = np.ascontiguousarray(words, dtype=np.uint32)
    code = np.zeros(max(n, 1), dtype=np.uint8)
    lib().or_unpack_bucket(ctypes.byref(cfg.c()), _p(words, ctypes.c_uint32), n, _p(code, ctypes.c_uint8))
    return code[:n]


def dequant(cfg: Config, table, code):
    table = _f32(table)
    return lib().or_dequant(ctypes.byref(cfg.c()), _p(table, ctypes.c_float), code)


def encode(cfg: Config, worker, step, g, r=None, b0=0, b1=None):
    """Encode one worker's vector; r (float32, in/out) is updated in place.  Returns the message."""
    assert g.dtype == np.float32 and g.flags.c_contiguous
    nbytes, _, _ = message_layout(cfg)
    msg = np.zeros(nbytes, dtype=np.uint8)
    b1 = num_buckets(cfg) if b1 is None else b1
    rp = _p(r, ctypes.c_float) if r is not None else None
    rc = lib().or_encode(ctypes.byref(cfg.c()), worker, step, b0, b1, _p(g, ctypes.c_float), rp,
                         _p(msg, ctypes.c_uint8))
    assert rc == 0
    return msg


def decode_accumulate(cfg: Config, msgs, b0=0, b1=None):
    b1 = num_buckets(cfg) if b1 is None else b1
    arr = (ctypes.POINTER(ctypes.c_uint8) * len(msgs))(*[_p(m, ctypes.c_uint8) for m in msgs])
    avg = np.zeros(cfg.n, dtype=np.float32)
    lib().or_decode_accumulate(ctypes.byref(cfg.c()), arr, len(msgs), b0, b1, _p(avg, ctypes.c_float))
    return avg


def fused_step(cfg: Config, step, gs, rs=None, with_msgs=True, b0=0, b1=None):
    """The whole step for W = len(gs) workers.  rs (list of float32 arrays) are updated in place.
    Returns (avg, msgs or None)."""
    W = len(gs)
    assert W == cfg.workers
    b1 = num_buckets(cfg) if b1 is None else b1
    f32p = ctypes.POINTER(ctypes.c_float)
    garr = (f32p * W)(*[_p(g, ctypes.c_float) for g in gs])
    rarr = (f32p * W)(*[_p(r, ctypes.c_float) for r in rs]) if rs is not None else None
    msgs = None
    marr = None
    if with_msgs:
        nbytes, _, _ = message_layout(cfg)
        msgs = [np.zeros(nbytes, dtype=np.uint8) for _ in range(W)]
        marr = (ctypes.POINTER(ctypes.c_uint8) * W)(*[_p(m, ctypes.c_uint8) for m in msgs])
    avg = np.zeros(cfg.n, dtype=np.float32)
    rc = lib().or_fused_step(ctypes.byref(cfg.c()), step, b0, b1, garr, rarr, marr, _p(avg, ctypes.c_float))
    assert rc == 0
    return avg, msgs


def fused_bucket(cfg: Config, step, bucket, gs, rs=None):
    """One bucket of the whole step from per-bucket slices.

    gs / rs: W float32 arrays holding the bucket's n values of each worker (rs None when error
    feedback is off).  Returns (avg, new residuals or None, packed words per worker, level
    tables per worker)."""
    W = len(gs)
    assert W == cfg.workers
    n = len(gs[0])
    f32p = ctypes.POINTER(ctypes.c_float)
    u32p = ctypes.POINTER(ctypes.c_uint32)
    gs = [_f32(g) for g in gs]
    garr = (f32p * W)(*[_p(g, ctypes.c_float) for g in gs])
    rin = rout = None
    routs = None
    if rs is not None:
        rs = [_f32(r) for r in rs]
        routs = [np.zeros(n, dtype=np.float32) for _ in range(W)]
        rin = (f32p * W)(*[_p(r, ctypes.c_float) for r in rs])
        rout = (f32p * W)(*[_p(r, ctypes.c_float) for r in routs])
    words = [np.zeros(cfg.bucket * bits(cfg.levels) // 32, dtype=np.uint32) for _ in range(W)]
    tables = [np.zeros(table_len(cfg.scheme, cfg.levels), dtype=np.float32) for _ in range(W)]
    warr = (u32p * W)(*[_p(x, ctypes.c_uint32) for x in words])
    tarr = (f32p * W)(*[_p(x, ctypes.c_float) for x in tables])
    avg = np.zeros(max(n, 1), dtype=np.float32)
    rc = lib().or_fused_bucket(ctypes.byref(cfg.c()), step, bucket, n, garr, rin, rout, warr, tarr,
                               _p(avg, ctypes.c_float))
    assert rc == 0
    return avg[:n], routs, words, tables


def quant_error(cfg: Config, worker, step, g, r=None, b0=0, b1=None):
    """(sum of expected squared rounding error, sum of u^2, realised sum of (Q(u)-u)^2)."""
    g = _f32(g)
    b1 = num_buckets(cfg) if b1 is None else b1
    out = np.zeros(3, dtype=np.float64)
    rp = _p(_f32(r), ctypes.c_float) if r is not None else None
    rc = lib().or_quant_error(ctypes.byref(cfg.c()), worker, step, b0, b1, _p(g, ctypes.c_float), rp,
                              _p(out, ctypes.c_double))
    assert rc == 0
    return out


def entropy_groups(levels):
    """(g, B): g codes of `levels` levels per B-bit group, or None if base-s packing has no
    grouping for that level count."""
    g, B = ctypes.c_int(), ctypes.c_int()
    if not lib().or_entropy_groups(levels, ctypes.byref(g), ctypes.byref(B)):
        return None
    return g.value, B.value


def entropy_words(cfg: Config):
    return lib().or_entropy_words(ctypes.byref(cfg.c()))


def entropy_layout(cfg: Config):
    b, c, l = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
    lib().or_entropy_layout(ctypes.byref(cfg.c()), ctypes.byref(b), ctypes.byref(c), ctypes.byref(l))
    return b.value, c.value, l.value


def entropy_pack(cfg: Config, msg):
    """Dense message -> base-s message."""
    msg = np.ascontiguousarray(msg, dtype=np.uint8)
    out = np.zeros(entropy_layout(cfg)[0], dtype=np.uint8)
    lib().or_entropy_pack(ctypes.byref(cfg.c()), _p(msg, ctypes.c_uint8), _p(out, ctypes.c_uint8))
    return out


def entropy_unpack(cfg: Config, emsg):
    """Base-s message -> dense message."""
    emsg = np.ascontiguousarray(emsg, dtype=np.uint8)
    out = np.zeros(message_layout(cfg)[0], dtype=np.uint8)
    lib().or_entropy_unpack(ctypes.byref(cfg.c()), _p(emsg, ctypes.c_uint8), _p(out, ctypes.c_uint8))
    return out


def elias_layout(cfg: Config):
    """(capacity bytes, offsets_off, tables_off, stream_off), or None if unsupported."""
    v = [ctypes.c_int64() for _ in range(4)]
    if not lib().or_elias_layout(ctypes.byref(cfg.c()), *[ctypes.byref(x) for x in v]):
        return None
    return tuple(x.value for x in v)


def elias_pack(cfg: Config, msg):
    """Dense message -> (Elias message buffer of the capacity size, bytes used)."""
    msg = np.ascontiguousarray(msg, dtype=np.uint8)
    out = np.zeros(elias_layout(cfg)[0], dtype=np.uint8)
    used = lib().or_elias_pack(ctypes.byref(cfg.c()), _p(msg, ctypes.c_uint8), _p(out, ctypes.c_uint8))
    return out, used


def elias_unpack(cfg: Config, emsg):
    emsg = np.ascontiguousarray(emsg, dtype=np.uint8)
    out = np.zeros(message_layout(cfg)[0], dtype=np.uint8)
    assert lib().or_elias_unpack(ctypes.byref(cfg.c()), _p(emsg, ctypes.c_uint8), _p(out, ctypes.c_uint8))
    return out


def elias_gamma_len(x):
    return lib().or_elias_gamma_len(x)


# ---------------------------------------------------------------------------------------------
# TernGrad with one scale per parameter tensor (segments [off[t], off[t+1]))
# ---------------------------------------------------------------------------------------------
def _offsets(off):
    off = np.ascontiguousarray(np.asarray(off, dtype=np.int64))
    return off, len(off) - 1


def tg_layer_layout(cfg: Config, nseg):
    b, c, s = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
    lib().or_tg_layer_layout(ctypes.byref(cfg.c()), nseg, ctypes.byref(b), ctypes.byref(c), ctypes.byref(s))
    return b.value, c.value, s.value


def tg_layer_encode(cfg: Config, off, worker, step, g, r=None):
    """One worker's message; r (float32, in/out) is updated in place when error feedback is on."""
    off, nseg = _offsets(off)
    assert g.dtype == np.float32 and g.flags.c_contiguous
    nbytes, _, _ = tg_layer_layout(cfg, nseg)
    msg = np.zeros(nbytes, dtype=np.uint8)
    rp = _p(r, ctypes.c_float) if r is not None else None
    rc = lib().or_tg_layer_encode(ctypes.byref(cfg.c()), _p(off, ctypes.c_int64), nseg, worker, step,
                                  _p(g, ctypes.c_float), rp, _p(msg, ctypes.c_uint8))
    assert rc == 0
    return msg


def tg_layer_decode_accumulate(cfg: Config, off, msgs):
    off, nseg = _offsets(off)
    arr = (ctypes.POINTER(ctypes.c_uint8) * len(msgs))(*[_p(m, ctypes.c_uint8) for m in msgs])
    avg = np.zeros(cfg.n, dtype=np.float32)
    lib().or_tg_layer_decode_accumulate(ctypes.byref(cfg.c()), _p(off, ctypes.c_int64), nseg, arr, len(msgs),
                                        _p(avg, ctypes.c_float))
    return avg
