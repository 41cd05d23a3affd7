"""Python binding of libmoa's C ABI (``include/moa.h``) -- argument marshalling only.

Every function named ``moa_*`` here calls the C entry point of the same name
through ctypes.  Device buffers are passed as torch CUDA tensors (their
``data_ptr()``) or raw integer addresses; PyTorch supplies device memory and
streams, nothing else: all attention arithmetic runs in libmoa's kernels.
A missing ``libmoa.so`` raises at first use -- there is no fallback.
"""

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoa.so")

MOA_OK, MOA_ERR_INVALID_ARG, MOA_ERR_CAPACITY, MOA_ERR_WORKSPACE = 0, 1, 2, 3
MOA_ERR_UNSUPPORTED, MOA_ERR_CUDA, MOA_ERR_TIMEOUT, MOA_ERR_HOST = 4, 5, 6, 7
MOA_F32, MOA_BF16 = 0, 1
MOA_OP_PREFILL, MOA_OP_DECODE = 0, 1

EXPORTS = (
    "moa_status_string", "moa_rules_eval", "moa_kv_bytes", "moa_kv_header_bytes", "moa_kv_alloc",
    "moa_kv_free", "moa_kv_append", "moa_kv_positions", "moa_kv_set_positions", "moa_kv_layout",
    "moa_workspace_bytes", "moa_workspace_init", "moa_workspace_check", "moa_prefill",
    "moa_prefill_schedule", "moa_decode", "moa_decode_append", "moa_decode_static_ws", "moa_stream_read", "moa_chunk_workspace_bytes",
    "moa_prefill_chunk", "moa_prefill_stall_test", "moa_kv_bytes_sink", "moa_kv_alloc_sink", "moa_prefill_sink",
    "moa_workspace_bytes_sink", "moa_decode_sink", "moa_decode_append_sink",
)


class MoaError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__("%s: %s" % (where, _status_name(status)))


_lib = None


def load():
    """Load libmoa.so (once) and declare the C signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError("libmoa.so is not built: run `python -m heterogeneous_sliding_window_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, sz, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
    P = ctypes.POINTER
    sig = {
        "moa_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "moa_rules_eval": (ctypes.c_int, [P(ctypes.c_double), P(ctypes.c_double), i32, i64, i32, P(i32)]),
        "moa_kv_bytes": (ctypes.c_int, [i32, i32, i32, ctypes.c_int, P(i32), P(sz)]),
        "moa_kv_header_bytes": (ctypes.c_int, [i32, P(sz)]),
        "moa_kv_alloc": (ctypes.c_int, [vp, sz, i32, i32, i32, ctypes.c_int, P(i32), vp, P(vp)]),
        "moa_kv_free": (ctypes.c_int, [vp]),
        "moa_kv_append": (ctypes.c_int, [vp, vp, vp, i32, vp]),
        "moa_kv_positions": (ctypes.c_int, [vp, P(i64), vp]),
        "moa_kv_set_positions": (ctypes.c_int, [vp, P(i64), vp]),
        "moa_kv_layout": (ctypes.c_int, [vp, P(vp), P(i64)]),
        "moa_workspace_bytes": (ctypes.c_int, [ctypes.c_int, i32, i32, i64, i32, P(i32), P(sz)]),
        "moa_workspace_init": (ctypes.c_int, [vp, sz, vp]),
        "moa_workspace_check": (ctypes.c_int, [vp, vp]),
        "moa_prefill": (ctypes.c_int, [vp, vp, vp, vp, i32, i32, i32, i64, i32, ctypes.c_int, P(i32), f32,
                                       vp, sz, vp, vp]),
        "moa_prefill_schedule": (ctypes.c_int, [i32, i32, i64, P(i32), i32, P(i32), i64, P(i64)]),
        "moa_decode": (ctypes.c_int, [vp, vp, vp, i32, P(i32), f32, vp, sz, vp]),
        "moa_decode_append": (ctypes.c_int, [vp, vp, vp, vp, vp, i32, P(i32), f32, vp, sz, vp]),
        "moa_decode_static_ws": (ctypes.c_int, [vp, vp, vp, i32, P(i32), f32, vp]),
        "moa_stream_read": (ctypes.c_int, [vp, sz, vp, vp]),
        "moa_prefill_stall_test": (ctypes.c_int, [vp, vp, vp, vp, vp, sz, vp]),
        "moa_chunk_workspace_bytes": (ctypes.c_int, [vp, i32, i32, P(i32), P(sz)]),
        "moa_prefill_chunk": (ctypes.c_int, [vp, vp, vp, vp, vp, i32, i32, P(i32), f32, vp, sz, vp]),
        "moa_kv_bytes_sink": (ctypes.c_int, [i32, i32, i32, ctypes.c_int, P(i32), P(i32), P(sz)]),
        "moa_kv_alloc_sink": (ctypes.c_int, [vp, sz, i32, i32, i32, ctypes.c_int, P(i32), P(i32), vp, P(vp)]),
        "moa_prefill_sink": (ctypes.c_int, [vp, vp, vp, vp, i32, i32, i32, i64, i32, ctypes.c_int, P(i32), P(i32),
                                            f32, vp, sz, vp, vp]),
        "moa_workspace_bytes_sink": (ctypes.c_int, [ctypes.c_int, i32, i32, i64, i32, P(i32), P(i32), P(sz)]),
        "moa_decode_sink": (ctypes.c_int, [vp, vp, vp, i32, P(i32), P(i32), f32, vp, sz, vp]),
        "moa_decode_append_sink": (ctypes.c_int, [vp, vp, vp, vp, vp, i32, P(i32), P(i32), f32, vp, sz, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def _status_name(s):
    try:
        return load().moa_status_string(int(s)).decode()
    except Exception:  # pragma: no cover
        return "status %d" % s


def _check(status, where):
    if status != MOA_OK:
        raise MoaError(status, where)


def _ptr(x):
    """Device address of a torch tensor, an int, or None."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s):
    """cudaStream_t of a torch stream / int; None -> torch's current stream."""
    if s is None:
        import torch
        if torch.cuda.is_available():
            return torch.cuda.current_stream().cuda_stream
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _i32(arr):
    a = np.ascontiguousarray(np.asarray(arr, dtype=np.int32))
    return a, a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


def _dtype(dt):
    if dt in (MOA_F32, MOA_BF16):
        return dt
    return {"f32": MOA_F32, "bf16": MOA_BF16}[dt]


# ---- span rule --------------------------------------------------------------
def moa_rules_eval(alpha, beta, N, block):
    a = np.ascontiguousarray(np.asarray(alpha, dtype=np.float64))
    b = np.ascontiguousarray(np.asarray(beta, dtype=np.float64))
    if a.shape != b.shape or a.ndim != 1:
        raise ValueError("alpha and beta must be 1-D of equal length")
    out = np.zeros(a.shape[0], dtype=np.int32)
    dp = ctypes.POINTER(ctypes.c_double)
    _check(load().moa_rules_eval(a.ctypes.data_as(dp), b.ctypes.data_as(dp), a.shape[0], int(N), int(block),
                                 out.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))), "moa_rules_eval")
    return out.tolist()


# ---- KV cache ---------------------------------------------------------------
def moa_kv_bytes(B, Hkv, d, dtype, capacity):
    cap, cp = _i32(capacity)
    out = ctypes.c_size_t()
    _check(load().moa_kv_bytes(B, Hkv, d, _dtype(dtype), cp, ctypes.byref(out)), "moa_kv_bytes")
    return out.value


def moa_kv_header_bytes(B):
    out = ctypes.c_size_t()
    _check(load().moa_kv_header_bytes(B, ctypes.byref(out)), "moa_kv_header_bytes")
    return out.value


def moa_kv_alloc(buf, nbytes, B, Hkv, d, dtype, capacity, stream=None):
    cap, cp = _i32(capacity)
    h = ctypes.c_void_p()
    _check(load().moa_kv_alloc(_ptr(buf), nbytes, B, Hkv, d, _dtype(dtype), cp, _stream(stream),
                               ctypes.byref(h)), "moa_kv_alloc")
    return h


def moa_kv_free(handle):
    _check(load().moa_kv_free(handle), "moa_kv_free")


def moa_kv_append(handle, k, v, n_tok, stream=None):
    _check(load().moa_kv_append(handle, _ptr(k), _ptr(v), int(n_tok), _stream(stream)), "moa_kv_append")


def moa_kv_positions(handle, B, stream=None):
    t = (ctypes.c_int64 * B)()
    _check(load().moa_kv_positions(handle, t, _stream(stream)), "moa_kv_positions")
    return list(t)


def moa_kv_set_positions(handle, t, stream=None):
    arr = (ctypes.c_int64 * len(t))(*[int(x) for x in t])
    _check(load().moa_kv_set_positions(handle, arr, _stream(stream)), "moa_kv_set_positions")


def moa_kv_layout(handle, Hkv):
    data = ctypes.c_void_p()
    goff = (ctypes.c_int64 * (Hkv + 1))()
    _check(load().moa_kv_layout(handle, ctypes.byref(data), goff), "moa_kv_layout")
    return data.value, list(goff)


# ---- workspace --------------------------------------------------------------
def moa_workspace_bytes(op, B, Hq, N, d, spans):
    sp, spp = _i32(spans)
    out = ctypes.c_size_t()
    _check(load().moa_workspace_bytes(op, B, Hq, int(N), d, spp, ctypes.byref(out)), "moa_workspace_bytes")
    return out.value


def moa_workspace_init(ws, nbytes, stream=None):
    _check(load().moa_workspace_init(_ptr(ws), nbytes, _stream(stream)), "moa_workspace_init")


def moa_workspace_check(ws, stream=None):
    _check(load().moa_workspace_check(_ptr(ws), _stream(stream)), "moa_workspace_check")


# ---- attention --------------------------------------------------------------
def moa_prefill(q, k, v, o, B, Hq, Hkv, N, d, dtype, spans, scale, ws=None, ws_bytes=0, fill=None,
                stream=None):
    sp, spp = _i32(spans)
    _check(load().moa_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, Hq, Hkv, int(N), d, _dtype(dtype), spp,
                              float(scale), _ptr(ws), ws_bytes, fill, _stream(stream)), "moa_prefill")


def moa_prefill_schedule(B, Hq, N, spans, n_ctas):
    sp, spp = _i32(spans)
    n = ctypes.c_int64()
    _check(load().moa_prefill_schedule(B, Hq, int(N), spp, int(n_ctas), None, 0, ctypes.byref(n)),
           "moa_prefill_schedule")
    out = np.zeros((n.value, 7), dtype=np.int32)
    _check(load().moa_prefill_schedule(B, Hq, int(N), spp, int(n_ctas),
                                       out.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), n.value,
                                       ctypes.byref(n)), "moa_prefill_schedule")
    return out


def moa_decode(handle, q, o, Hq, spans, scale, ws, ws_bytes, stream=None):
    sp, spp = _i32(spans)
    _check(load().moa_decode(handle, _ptr(q), _ptr(o), Hq, spp, float(scale), _ptr(ws), ws_bytes,
                             _stream(stream)), "moa_decode")


def moa_decode_append(handle, q, k, v, o, Hq, spans, scale, ws, ws_bytes, stream=None):
    sp, spp = _i32(spans)
    _check(load().moa_decode_append(handle, _ptr(q), _ptr(k), _ptr(v), _ptr(o), Hq, spp, float(scale), _ptr(ws),
                                    ws_bytes, _stream(stream)), "moa_decode_append")


def moa_decode_static_ws(handle, q, o, Hq, spans, scale, stream=None):
    """moa_decode for callers that cannot allocate: scratch is libmoa's own 8 MiB device array."""
    sp, spp = _i32(spans)
    _check(load().moa_decode_static_ws(handle, _ptr(q), _ptr(o), Hq, spp, float(scale), _stream(stream)),
           "moa_decode_static_ws")


def moa_chunk_workspace_bytes(handle, Hq, n, spans):
    sp, spp = _i32(spans)
    out = ctypes.c_size_t(0)
    _check(load().moa_chunk_workspace_bytes(handle, Hq, n, spp, ctypes.byref(out)), "moa_chunk_workspace_bytes")
    return out.value


def moa_prefill_chunk(handle, q, k, v, o, Hq, n, spans, scale, ws, ws_bytes, stream=None):
    """The n new tokens of every sequence attend to the cache's window and themselves, then are appended."""
    sp, spp = _i32(spans)
    _check(load().moa_prefill_chunk(handle, _ptr(q), _ptr(k), _ptr(v), _ptr(o), Hq, n, spp, float(scale),
                                    _ptr(ws), int(ws_bytes), _stream(stream)), "moa_prefill_chunk")


def moa_prefill_stall_test(q, k, v, o, ws, ws_bytes, stream=None):
    """Launch the prefill kernel with its work units withheld (its bounded waits run out after 2 s)."""
    _check(load().moa_prefill_stall_test(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(ws), int(ws_bytes),
                                         _stream(stream)), "moa_prefill_stall_test")


def moa_stream_read(buf, nbytes, out, stream=None):
    """Read-only bandwidth probe: checksum of `nbytes` at `buf` into the device uint64 `out`."""
    _check(load().moa_stream_read(_ptr(buf), int(nbytes), _ptr(out), _stream(stream)), "moa_stream_read")


# ---- band plus global tokens ------------------------------------------------
def moa_kv_bytes_sink(B, Hkv, d, dtype, capacity, sink_capacity):
    cap, cp = _i32(capacity)
    sk, skp = _i32(sink_capacity)
    out = ctypes.c_size_t()
    _check(load().moa_kv_bytes_sink(B, Hkv, d, _dtype(dtype), cp, skp, ctypes.byref(out)), "moa_kv_bytes_sink")
    return out.value


def moa_kv_alloc_sink(buf, nbytes, B, Hkv, d, dtype, capacity, sink_capacity, stream=None):
    cap, cp = _i32(capacity)
    sk, skp = _i32(sink_capacity)
    h = ctypes.c_void_p()
    _check(load().moa_kv_alloc_sink(_ptr(buf), nbytes, B, Hkv, d, _dtype(dtype), cp, skp, _stream(stream),
                                    ctypes.byref(h)), "moa_kv_alloc_sink")
    return h


def moa_prefill_sink(q, k, v, o, B, Hq, Hkv, N, d, dtype, spans, sinks, scale, ws=None, ws_bytes=0, fill=None,
                     stream=None):
    sp, spp = _i32(spans)
    sk, skp = _i32(sinks)
    _check(load().moa_prefill_sink(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, Hq, Hkv, int(N), d, _dtype(dtype), spp,
                                   skp, float(scale), _ptr(ws), ws_bytes, fill, _stream(stream)), "moa_prefill_sink")


def moa_workspace_bytes_sink(op, B, Hq, N, d, spans, sinks):
    sp, spp = _i32(spans)
    sk, skp = _i32(sinks)
    out = ctypes.c_size_t()
    _check(load().moa_workspace_bytes_sink(op, B, Hq, int(N), d, spp, skp, ctypes.byref(out)),
           "moa_workspace_bytes_sink")
    return out.value


def moa_decode_sink(handle, q, o, Hq, spans, sinks, scale, ws, ws_bytes, stream=None):
    sp, spp = _i32(spans)
    sk, skp = _i32(sinks)
    _check(load().moa_decode_sink(handle, _ptr(q), _ptr(o), Hq, spp, skp, float(scale), _ptr(ws), ws_bytes,
                                  _stream(stream)), "moa_decode_sink")


def moa_decode_append_sink(handle, q, k, v, o, Hq, spans, sinks, scale, ws, ws_bytes, stream=None):
    sp, spp = _i32(spans)
    sk, skp = _i32(sinks)
    _check(load().moa_decode_append_sink(handle, _ptr(q), _ptr(k), _ptr(v), _ptr(o), Hq, spp, skp, float(scale),
                                         _ptr(ws), ws_bytes, _stream(stream)), "moa_decode_append_sink")


# ---- conveniences over torch-owned device memory ------------------------------
class KVCache:
    """A ring-buffer cache whose device buffer is a torch uint8 tensor."""

    def __init__(self, B, Hkv, d, dtype, capacity, device="cuda", stream=None, sink_capacity=None):
        import torch
        self.B, self.Hkv, self.d, self.dtype = B, Hkv, d, _dtype(dtype)
        self.capacity = [int(c) for c in capacity]
        self.sink_capacity = None if sink_capacity is None else [int(c) for c in sink_capacity]
        if self.sink_capacity is None:
            self.nbytes = moa_kv_bytes(B, Hkv, d, self.dtype, self.capacity)
        else:
            self.nbytes = moa_kv_bytes_sink(B, Hkv, d, self.dtype, self.capacity, self.sink_capacity)
        self.buf = torch.empty(self.nbytes + 256, dtype=torch.uint8, device=device)
        base = self.buf.data_ptr()
        self.ptr = (base + 255) // 256 * 256
        if self.sink_capacity is None:
            self.handle = moa_kv_alloc(self.ptr, self.nbytes, B, Hkv, d, self.dtype, self.capacity, stream)
        else:
            self.handle = moa_kv_alloc_sink(self.ptr, self.nbytes, B, Hkv, d, self.dtype, self.capacity,
                                            self.sink_capacity, stream)

    def append(self, k, v, stream=None):
        moa_kv_append(self.handle, k, v, k.shape[2], stream)

    def positions(self, stream=None):
        return moa_kv_positions(self.handle, self.B, stream)

    def set_positions(self, t, stream=None):
        moa_kv_set_positions(self.handle, t, stream)

    def layout(self):
        return moa_kv_layout(self.handle, self.Hkv)

    def data_bytes(self):
        """The data region as a torch uint8 view (for checks and synthetic fills)."""
        hdr = moa_kv_header_bytes(self.B)
        off = self.ptr - self.buf.data_ptr()
        return self.buf[off + hdr: off + self.nbytes]

    def header_bytes_view(self):
        off = self.ptr - self.buf.data_ptr()
        return self.buf[off: off + moa_kv_header_bytes(self.B)]

    def close(self):
        if self.handle:
            moa_kv_free(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class Workspace:
    """Workspace for one op as a torch uint8 tensor (256-byte aligned), zeroed once."""

    def __init__(self, op, B, Hq, N, d, spans, device="cuda", stream=None):
        import torch
        self.nbytes = moa_workspace_bytes(op, B, Hq, N, d, spans)
        self.buf = torch.empty(self.nbytes + 256, dtype=torch.uint8, device=device)
        self.ptr = (self.buf.data_ptr() + 255) // 256 * 256
        moa_workspace_init(self.ptr, self.nbytes, stream)
