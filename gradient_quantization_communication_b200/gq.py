"""Python binding of the C ABI in ``include/gq.h`` (``libgq.so``): argument marshalling only.

Every function keeps the C name.  Tensors are passed as ``data_ptr()``; the stream defaults to
torch's current CUDA stream.  There is no fallback: if ``libgq.so`` is missing the import of the
library fails with an error that says how to build it.
"""
import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgq.so")

GQ_QSGD, GQ_TERNGRAD, GQ_BINGRAD_B, GQ_BINGRAD_PB, GQ_ORQ, GQ_QSGD_NEAREST, GQ_SIGNSGD, GQ_QSGD_L2, GQ_TERNGRAD_LAYER = range(9)
GQ_OK, GQ_ERR_INVALID, GQ_ERR_UNSUPPORTED, GQ_ERR_CUDA, GQ_ERR_NONFINITE, GQ_ERR_NOMEM, GQ_ERR_TIMEOUT = 0, 1, 2, 3, 4, 5, 6
GQ_MAX_WORKERS = 64
GQ_FORMAT_DENSE, GQ_FORMAT_BASE_S = 0, 1
SCHEMES = {"qsgd": GQ_QSGD, "terngrad": GQ_TERNGRAD, "bingrad_b": GQ_BINGRAD_B,
           "bingrad_pb": GQ_BINGRAD_PB, "orq": GQ_ORQ, "qsgd_nearest": GQ_QSGD_NEAREST, "signsgd": GQ_SIGNSGD,
           "qsgd_l2": GQ_QSGD_L2, "terngrad_layer": GQ_TERNGRAD_LAYER}


class gq_config_t(ctypes.Structure):
    _fields_ = [("scheme", ctypes.c_int32), ("levels", ctypes.c_int32), ("bucket", ctypes.c_int32),
                ("workers", ctypes.c_int32), ("error_feedback", ctypes.c_int32),
                ("clip_sigma", ctypes.c_float), ("seed", ctypes.c_uint64), ("n", ctypes.c_int64)]


class GQError(RuntimeError):
    def __init__(self, status, what):
        super().__init__("%s: %s (status %d)" % (what, gq_status_string(status), status))
        self.status = status


_lib = None


def lib():
    """The loaded libgq.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libgq.so is not built (%s); run gradient_quantization_communication_b200/build.py"
                              % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        vp, sz = ctypes.c_void_p, ctypes.c_size_t
        cfgp = ctypes.POINTER(gq_config_t)
        L.gq_config_check.argtypes = [cfgp]
        L.gq_message_layout.argtypes = [cfgp, ctypes.POINTER(sz), ctypes.POINTER(sz), ctypes.POINTER(sz)]
        L.gq_plan_create.argtypes = [cfgp, ctypes.POINTER(vp)]
        L.gq_plan_destroy.argtypes = [vp]
        L.gq_encode.argtypes = [vp, ctypes.c_uint32, ctypes.c_uint64, vp, vp, vp, vp]
        L.gq_decode_accumulate.argtypes = [vp, ctypes.POINTER(vp), ctypes.c_int, vp, vp]
        L.gq_fused_step.argtypes = [vp, ctypes.c_uint64, ctypes.POINTER(vp), ctypes.POINTER(vp),
                                    ctypes.POINTER(vp), vp, vp]
        L.gq_quant_error.argtypes = [vp, ctypes.c_uint32, ctypes.c_uint64, vp, vp, vp, vp]
        L.gq_quant_error_noalloc.argtypes = [cfgp, ctypes.c_uint32, ctypes.c_uint64, vp, vp, vp, vp]
        L.gq_plan_status.argtypes = [vp, vp]
        L.gq_plan_set_segments.argtypes = [vp, ctypes.POINTER(ctypes.c_int64), ctypes.c_int]
        L.gq_plan_set_format.argtypes = [vp, ctypes.c_int]
        L.gq_plan_message_layout.argtypes = [vp, ctypes.POINTER(sz), ctypes.POINTER(sz), ctypes.POINTER(sz)]
        L.gq_selftest_bounded_wait.argtypes = [vp, ctypes.c_int64, vp]
        L.gq_entropy_layout.argtypes = [cfgp, ctypes.POINTER(sz), ctypes.POINTER(sz), ctypes.POINTER(sz)]
        L.gq_entropy_pack.argtypes = [cfgp, vp, vp, vp]
        L.gq_entropy_unpack.argtypes = [cfgp, vp, vp, vp]
        L.gq_elias_layout.argtypes = [cfgp, ctypes.POINTER(sz), ctypes.POINTER(sz), ctypes.POINTER(sz),
                                      ctypes.POINTER(sz)]
        L.gq_elias_used_bytes.argtypes = [cfgp, ctypes.c_uint64, ctypes.POINTER(sz)]
        L.gq_elias_pack.argtypes = [cfgp, vp, vp, vp]
        L.gq_elias_unpack.argtypes = [cfgp, vp, vp, vp]
        L.gq_status_string.argtypes = [ctypes.c_int]
        L.gq_status_string.restype = ctypes.c_char_p
        L.gq_version.restype = ctypes.c_char_p
        for f in ("gq_config_check", "gq_message_layout", "gq_plan_create", "gq_plan_destroy", "gq_encode",
                  "gq_decode_accumulate", "gq_fused_step", "gq_quant_error", "gq_quant_error_noalloc",
                  "gq_plan_status", "gq_plan_set_segments", "gq_plan_message_layout", "gq_plan_set_format",
                  "gq_selftest_bounded_wait", "gq_entropy_layout", "gq_entropy_pack",
                  "gq_entropy_unpack", "gq_elias_layout", "gq_elias_used_bytes", "gq_elias_pack",
                  "gq_elias_unpack"):
            getattr(L, f).restype = ctypes.c_int
        _lib = L
    return _lib


# ---------------------------------------------------------------------------------------------
# marshalling helpers
# ---------------------------------------------------------------------------------------------
def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _ptr_array(xs):
    if xs is None:
        return None
    return (ctypes.c_void_p * len(xs))(*[_ptr(x) for x in xs])


def _check(st, what):
    if st != GQ_OK:
        raise GQError(st, what)


def gq_config(scheme, levels=0, bucket=512, workers=1, error_feedback=True, clip_sigma=0.0, seed=0, n=0):
    if isinstance(scheme, str):
        scheme = SCHEMES[scheme]
    return gq_config_t(scheme, levels, bucket, workers, int(bool(error_feedback)), clip_sigma, seed, n)


# ---------------------------------------------------------------------------------------------
# the C entry points
# ---------------------------------------------------------------------------------------------
def gq_config_check(cfg):
    return lib().gq_config_check(ctypes.byref(cfg))


def gq_message_layout(cfg):
    b, c, l = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().gq_message_layout(ctypes.byref(cfg), ctypes.byref(b), ctypes.byref(c), ctypes.byref(l)),
           "gq_message_layout")
    return b.value, c.value, l.value


def gq_plan_create(cfg):
    h = ctypes.c_void_p()
    _check(lib().gq_plan_create(ctypes.byref(cfg), ctypes.byref(h)), "gq_plan_create")
    return h


def gq_plan_destroy(plan):
    _check(lib().gq_plan_destroy(plan), "gq_plan_destroy")


def gq_encode(plan, worker, step, grad, residual, msg, stream=None):
    _check(lib().gq_encode(plan, worker, step, _ptr(grad), _ptr(residual), _ptr(msg), _stream(stream)), "gq_encode")


def gq_decode_accumulate(plan, msgs, avg, stream=None):
    _check(lib().gq_decode_accumulate(plan, _ptr_array(msgs), len(msgs), _ptr(avg), _stream(stream)),
           "gq_decode_accumulate")


def gq_fused_step(plan, step, grads, residuals, msgs, avg, stream=None):
    _check(lib().gq_fused_step(plan, step, _ptr_array(grads), _ptr_array(residuals), _ptr_array(msgs), _ptr(avg),
                               _stream(stream)), "gq_fused_step")


def gq_quant_error(plan, worker, step, grad, residual, out, stream=None):
    _check(lib().gq_quant_error(plan, worker, step, _ptr(grad), _ptr(residual), _ptr(out), _stream(stream)),
           "gq_quant_error")


def gq_quant_error_noalloc(cfg, worker, step, grad, residual, out, stream=None):
    _check(lib().gq_quant_error_noalloc(ctypes.byref(cfg), worker, step, _ptr(grad), _ptr(residual), _ptr(out),
                                        _stream(stream)), "gq_quant_error_noalloc")


def gq_plan_set_segments(plan, offsets):
    arr = (ctypes.c_int64 * len(offsets))(*[int(x) for x in offsets])
    _check(lib().gq_plan_set_segments(plan, arr, len(offsets) - 1), "gq_plan_set_segments")


def gq_plan_set_format(plan, fmt):
    _check(lib().gq_plan_set_format(plan, int(fmt)), "gq_plan_set_format")


def gq_plan_message_layout(plan):
    b, c, l = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().gq_plan_message_layout(plan, ctypes.byref(b), ctypes.byref(c), ctypes.byref(l)),
           "gq_plan_message_layout")
    return b.value, c.value, l.value


def gq_plan_status(plan, stream=None):
    return lib().gq_plan_status(plan, _stream(stream))


def gq_selftest_bounded_wait(plan, limit_ns, stream=None):
    _check(lib().gq_selftest_bounded_wait(plan, int(limit_ns), _stream(stream)), "gq_selftest_bounded_wait")


def gq_entropy_layout(cfg):
    b, c, l = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().gq_entropy_layout(ctypes.byref(cfg), ctypes.byref(b), ctypes.byref(c), ctypes.byref(l)),
           "gq_entropy_layout")
    return b.value, c.value, l.value


def gq_entropy_pack(cfg, msg, emsg, stream=None):
    _check(lib().gq_entropy_pack(ctypes.byref(cfg), _ptr(msg), _ptr(emsg), _stream(stream)), "gq_entropy_pack")


def gq_entropy_unpack(cfg, emsg, msg, stream=None):
    _check(lib().gq_entropy_unpack(ctypes.byref(cfg), _ptr(emsg), _ptr(msg), _stream(stream)), "gq_entropy_unpack")


def gq_elias_layout(cfg):
    """(capacity bytes, offsets_off, tables_off, stream_off)."""
    v = [ctypes.c_size_t() for _ in range(4)]
    _check(lib().gq_elias_layout(ctypes.byref(cfg), *[ctypes.byref(x) for x in v]), "gq_elias_layout")
    return tuple(x.value for x in v)


def gq_elias_used_bytes(cfg, stream_bits):
    b = ctypes.c_size_t()
    _check(lib().gq_elias_used_bytes(ctypes.byref(cfg), int(stream_bits), ctypes.byref(b)), "gq_elias_used_bytes")
    return b.value


def gq_elias_pack(cfg, msg, emsg, stream=None):
    _check(lib().gq_elias_pack(ctypes.byref(cfg), _ptr(msg), _ptr(emsg), _stream(stream)), "gq_elias_pack")


def gq_elias_unpack(cfg, emsg, msg, stream=None):
    _check(lib().gq_elias_unpack(ctypes.byref(cfg), _ptr(emsg), _ptr(msg), _stream(stream)), "gq_elias_unpack")


def gq_status_string(status):
    return lib().gq_status_string(status).decode()


def gq_version():
    return lib().gq_version().decode()


class Plan:
    """Owner of a gq_plan_t (destroyed on close / exit of a ``with`` block)."""

    def __init__(self, cfg, segments=None, fmt=GQ_FORMAT_DENSE):
        """segments: the tensors' offsets (nseg + 1 values) for GQ_TERNGRAD_LAYER; fmt: the
        message format (GQ_FORMAT_BASE_S: base-s messages written and read directly)."""
        self.cfg = cfg
        self.handle = gq_plan_create(cfg)
        if segments is not None:
            gq_plan_set_segments(self.handle, segments)
        if fmt != GQ_FORMAT_DENSE:
            gq_plan_set_format(self.handle, fmt)
        if cfg.scheme == GQ_TERNGRAD_LAYER and segments is None:
            self.msg_bytes = self.codes_off = self.levels_off = None
        else:
            self.msg_bytes, self.codes_off, self.levels_off = gq_plan_message_layout(self.handle)

    def close(self):
        if self.handle:
            gq_plan_destroy(self.handle)
            self.handle = None

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
