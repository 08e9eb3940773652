"""Python binding of libunweight (lossless BF16 weight compression fused with the matmul).

Argument marshalling only: every step of the computation runs in the CUDA
library ``libunweight.so`` built in this directory (``python
decode_gemm_b200/build.py``).  Importing this package fails loudly when the
library is missing; there is no Python or CPU fallback.

The functions carry the names of the C ABI in ``include/unweight.h``.  Tensors
are ``torch`` tensors on the GPU (device memory and streams come from torch);
host arrays are ``numpy`` arrays.  A device tensor goes to the library as its
data pointer, as in the C ABI: it must be contiguous, on the handle's device
and at least as large as the header states for that argument (nothing here
checks its size).  Every call raises :class:`UwError` when the library returns
a status other than ``UW_OK``.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libunweight.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python decode_gemm_b200/build.py` "
        "(nvcc, sm_100a). There is no fallback implementation.")

lib = C.CDLL(LIB_PATH)

# ----------------------------------------------------------------- constants --
UW_OK, UW_ERR_ARG, UW_ERR_SHAPE, UW_ERR_FORMAT, UW_ERR_UNSUPPORTED = 0, 1, 2, 3, 4
UW_ERR_OOM, UW_ERR_CUDA, UW_ERR_DEVICE, UW_ERR_TIMEOUT, UW_ERR_WORKSPACE = 5, 6, 7, 8, 9
UW_ERR_IO = 10
UW_PIPE_AUTO, UW_PIPE_FULL, UW_PIPE_EXP, UW_PIPE_PALETTE_RT, UW_PIPE_PALETTE_DIRECT = 0, 1, 2, 3, 4
UW_PIPE_HUFFMAN_DIRECT = 5   # the Huffman-direct product (M <= DOT_MAX_M)
DOT_MAX_M = 8     # tokens the Huffman-direct product serves per call
PIPELINES = {"full": UW_PIPE_FULL, "exp": UW_PIPE_EXP, "palette_rt": UW_PIPE_PALETTE_RT,
             "palette_direct": UW_PIPE_PALETTE_DIRECT}


class uw_encode_opts(C.Structure):
    _fields_ = [("max_code_len", C.c_int32), ("chunk_syms", C.c_int32),
                ("prepare_direct", C.c_int32), ("reserved", C.c_int32)]


class uw_format(C.Structure):
    _fields_ = [
        ("N", C.c_int64), ("K", C.c_int64),
        ("max_code_len", C.c_int32), ("chunk_syms", C.c_int32),
        ("code_len", C.c_uint8 * 256), ("palette", C.c_uint8 * 16),
        ("n_words", C.c_int64), ("words", C.POINTER(C.c_uint32)),
        ("n_chunks", C.c_int64), ("chunk_off", C.POINTER(C.c_uint32)),
        ("sm", C.POINTER(C.c_uint8)),
        ("n_esc_words", C.c_int64), ("esc_bits", C.POINTER(C.c_uint32)),
        ("n_esc_groups", C.c_int64), ("esc_off", C.POINTER(C.c_uint32)),
        ("n_esc_rows", C.c_int64), ("esc_exp", C.POINTER(C.c_uint8)),
    ]


class uw_stats_t(C.Structure):
    _fields_ = [
        ("N", C.c_int64), ("K", C.c_int64),
        ("bits_per_exponent", C.c_double), ("entropy_bits", C.c_double),
        ("top16_coverage", C.c_double),
        ("n_rows", C.c_int64), ("n_escape_rows", C.c_int64),
        ("max_len_used", C.c_int32), ("n_symbols", C.c_int32),
        ("bytes_stream", C.c_int64), ("bytes_offsets", C.c_int64), ("bytes_sm", C.c_int64),
        ("bytes_escape", C.c_int64), ("bytes_palette_idx", C.c_int64),
        ("bytes_huffman_bundle", C.c_int64), ("bytes_palette_bundle", C.c_int64),
    ]

    def as_dict(self):
        return {name: getattr(self, name) for name, _ in self._fields_}


class uw_gemm_config(C.Structure):
    _fields_ = [("pipeline", C.c_int32), ("tile_n", C.c_int32), ("stages", C.c_int32),
                ("gemm_ctas", C.c_int32), ("decode_ctas", C.c_int32), ("halves", C.c_int32),
                ("pair", C.c_int32), ("gemv", C.c_int32)]

    def as_dict(self):
        return {k: getattr(self, k) for k in ("pipeline", "tile_n", "stages", "gemm_ctas",
                                               "decode_ctas", "halves", "pair", "gemv")}


class uw_mlp_layer(C.Structure):
    _fields_ = [("gate", C.c_void_p), ("up", C.c_void_p), ("down", C.c_void_p)]


class uw_mlp_opts(C.Structure):
    _fields_ = [("overlap", C.c_int32), ("decode_ctas", C.c_int32), ("gemm_ctas", C.c_int32),
                ("reserved", C.c_int32)]

    def as_dict(self):
        return {k: getattr(self, k) for k in ("overlap", "decode_ctas", "gemm_ctas")}


_vp, _i32, _i64, _sz = C.c_void_p, C.c_int32, C.c_int64, C.c_size_t
_SIGS = {
    "uw_status_str": ([C.c_int], C.c_char_p),
    "uw_abi_version": ([], C.c_int),
    "uw_default_encode_opts": ([C.POINTER(uw_encode_opts)], None),
    "uw_encode_host": ([_vp, _i64, _i64, C.POINTER(uw_encode_opts), C.POINTER(_vp)], C.c_int),
    "uw_host_view": ([_vp, C.POINTER(uw_format)], C.c_int),
    "uw_host_free": ([_vp], None),
    "uw_validate_format": ([C.POINTER(uw_format)], C.c_int),
    "uw_host_stats": ([_vp, C.POINTER(uw_stats_t)], C.c_int),
    "uw_host_save": ([_vp, C.c_char_p], C.c_int),
    "uw_host_load": ([C.c_char_p, C.POINTER(_vp)], C.c_int),
    "uw_load": ([C.c_char_p, C.POINTER(uw_encode_opts), _vp, C.POINTER(_vp)], C.c_int),
    "uw_upload": ([C.POINTER(uw_format), C.POINTER(uw_encode_opts), _vp, C.POINTER(_vp)], C.c_int),
    "uw_encode": ([_vp, _i64, _i64, C.POINTER(uw_encode_opts), _vp, C.POINTER(_vp)], C.c_int),
    "uw_free": ([_vp], C.c_int),
    "uw_set_stream": ([_vp, _vp], C.c_int),
    "uw_stats": ([_vp, C.POINTER(uw_stats_t)], C.c_int),
    "uw_workspace_bytes": ([_vp, _i32, _i64, C.POINTER(_sz)], C.c_int),
    "uw_set_workspace": ([_vp, _vp, _sz], C.c_int),
    "uw_alloc_workspace": ([_vp, _sz], C.c_int),
    "uw_decode_full": ([_vp, _vp], C.c_int),
    "uw_decode_exp": ([_vp, _vp], C.c_int),
    "uw_decode_rows": ([_vp, _vp, _i64, _vp], C.c_int),
    "uw_transcode_palette": ([_vp, _vp], C.c_int),
    "uw_gemm": ([_vp, _vp, _vp, _i64, C.c_int], C.c_int),
    "uw_gemm_f32": ([_vp, _vp, _vp, _i64, C.c_int], C.c_int),
    "uw_gemm_ex": ([_vp, _vp, _vp, _i64, C.POINTER(uw_gemm_config), _i32], C.c_int),
    "uw_autotune": ([C.POINTER(_vp), _i32, C.POINTER(_i64), _i32, C.c_char_p], C.c_int),
    "uw_load_profile": ([C.POINTER(_vp), _i32, C.c_char_p], C.c_int),
    "uw_get_choice": ([_vp, _i64, C.POINTER(uw_gemm_config)], C.c_int),
    "uw_last_device_status": ([_vp], C.c_int),
    "uw_trace_enable": ([_vp, _i32], C.c_int),
    "uw_gemm_palette_noalloc": ([_vp, _vp, _vp, _i64, _i32], C.c_int),
    "uw_swiglu": ([_vp, _vp, _vp, _i64, _vp], C.c_int),
    "uw_mlp_workspace_bytes": ([C.POINTER(uw_mlp_layer), _i32, _i64, C.POINTER(uw_mlp_opts),
                                C.POINTER(_sz)], C.c_int),
    "uw_mlp_forward": ([C.POINTER(uw_mlp_layer), _i32, _vp, _vp, _i64, _vp, _sz, _vp, _vp,
                        C.POINTER(uw_mlp_opts)], C.c_int),
    "uw_mlp_forward_record": ([C.POINTER(uw_mlp_layer), _i32, _vp, _vp, _i64, _vp, _sz, _vp,
                               _vp, C.POINTER(uw_mlp_opts), _vp], C.c_int),
    "uw_mlp_tune_split": ([C.POINTER(uw_mlp_layer), _i32, _vp, _vp, _i64, _vp, _sz, _vp, _vp,
                           C.POINTER(uw_mlp_opts)], C.c_int),
    "uw_trace_read": ([_vp, C.POINTER(_i32), C.POINTER(C.c_float), _i32, C.POINTER(_i32)], C.c_int),
}
for _name, (_args, _res) in _SIGS.items():
    _f = getattr(lib, _name)
    _f.argtypes = _args
    _f.restype = _res

EXPORTED = tuple(_SIGS)


class UwError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = int(status)
        super().__init__(f"{what}: {uw_status_str(status)} ({status})")


def uw_status_str(status: int) -> str:
    return lib.uw_status_str(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != UW_OK:
        raise UwError(status, what)


def default_opts(**kw) -> uw_encode_opts:
    o = uw_encode_opts()
    lib.uw_default_encode_opts(C.byref(o))
    for k, v in kw.items():
        setattr(o, k, int(v))
    return o


def _stream_ptr(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def _dptr(t) -> int:
    return int(t.data_ptr())


# ------------------------------------------------------------------ host side --

class HostEncoded:
    """Host-side encoding (``uw_encode_host``); numpy views via :meth:`arrays`."""

    def __init__(self, ptr):
        self._ptr = _vp(ptr)
        # (module globals may be gone when __del__ runs at interpreter exit)
        self._free, self._null = lib.uw_host_free, _vp(0)

    @property
    def ptr(self):
        return self._ptr

    def view(self) -> uw_format:
        f = uw_format()
        _check(lib.uw_host_view(self._ptr, C.byref(f)), "uw_host_view")
        return f

    def arrays(self) -> dict:
        return format_arrays(self.view())

    def stats(self) -> dict:
        s = uw_stats_t()
        _check(lib.uw_host_stats(self._ptr, C.byref(s)), "uw_host_stats")
        return s.as_dict()

    def __del__(self):
        ptr, free = getattr(self, "_ptr", None), getattr(self, "_free", None)
        if ptr is not None and ptr.value and free is not None:
            free(ptr)
            self._ptr = self._null


def uw_encode_host(w: np.ndarray, opts: uw_encode_opts | None = None) -> HostEncoded:
    w = np.ascontiguousarray(w, dtype=np.uint16)
    n, k = w.shape
    out = _vp()
    _check(lib.uw_encode_host(w.ctypes.data, n, k, C.byref(opts) if opts else None,
                              C.byref(out)), "uw_encode_host")
    return HostEncoded(out.value)


def format_arrays(f: uw_format) -> dict:
    """Copy every array of a format view into numpy."""
    def arr(ptr, n, dt):
        n = int(n)
        if n == 0:
            return np.zeros(0, dt)
        return np.ctypeslib.as_array(ptr, shape=(n,)).copy().astype(dt)
    return dict(
        N=f.N, K=f.K, max_code_len=f.max_code_len, chunk_syms=f.chunk_syms,
        code_len=np.array(f.code_len[:], np.uint8), palette=np.array(f.palette[:], np.uint8),
        words=arr(f.words, f.n_words, np.uint32),
        chunk_off=arr(f.chunk_off, f.n_chunks + 1, np.uint32),
        sm=arr(f.sm, f.N * f.K, np.uint8),
        esc_bits=arr(f.esc_bits, f.n_esc_words, np.uint32),
        esc_off=arr(f.esc_off, f.n_esc_groups + 1, np.uint32),
        esc_exp=arr(f.esc_exp, f.n_esc_rows * 64, np.uint8),
    )


class FormatBuffers:
    """A ``uw_format`` that points into numpy arrays it keeps alive."""

    def __init__(self, N, K, max_code_len, chunk_syms, code_len, palette, words, chunk_off, sm,
                 esc_bits, esc_off, esc_exp):
        self._keep = []

        def ptr(a, ct):
            a = np.ascontiguousarray(a)
            self._keep.append(a)
            return a.ctypes.data_as(C.POINTER(ct))

        f = uw_format()
        f.N, f.K = int(N), int(K)
        f.max_code_len, f.chunk_syms = int(max_code_len), int(chunk_syms)
        f.code_len[:] = [int(x) for x in np.asarray(code_len, np.uint8)]
        f.palette[:] = [int(x) for x in np.asarray(palette, np.uint8)]
        words = np.asarray(words, np.uint32)
        f.n_words, f.words = words.size, ptr(words, C.c_uint32)
        chunk_off = np.asarray(chunk_off, np.uint32)
        f.n_chunks, f.chunk_off = chunk_off.size - 1, ptr(chunk_off, C.c_uint32)
        f.sm = ptr(np.asarray(sm, np.uint8).reshape(-1), C.c_uint8)
        esc_bits = np.asarray(esc_bits, np.uint32).reshape(-1)
        f.n_esc_words, f.esc_bits = esc_bits.size, ptr(esc_bits, C.c_uint32)
        esc_off = np.asarray(esc_off, np.uint32)
        f.n_esc_groups, f.esc_off = esc_off.size - 1, ptr(esc_off, C.c_uint32)
        esc_exp = np.asarray(esc_exp, np.uint8).reshape(-1)
        f.n_esc_rows = esc_exp.size // 64
        f.esc_exp = ptr(esc_exp if esc_exp.size else np.zeros(64, np.uint8), C.c_uint8)
        self.fmt = f


def uw_validate_format(fmt: uw_format) -> int:
    """Returns the status code (does not raise): UW_OK or an error."""
    return int(lib.uw_validate_format(C.byref(fmt)))


# ---------------------------------------------------------------- device side --

class Handle:
    """A device-resident encoded matrix (``uw_handle_t``)."""

    def __init__(self, ptr, N, K):
        self._ptr = _vp(ptr)
        self.N, self.K = int(N), int(K)
        self._ws = None  # torch tensor kept alive while registered
        # (module globals may be gone when __del__ runs at interpreter exit)
        self._free, self._null = lib.uw_free, _vp(0)

    @property
    def ptr(self):
        return self._ptr

    def stats(self) -> dict:
        s = uw_stats_t()
        _check(lib.uw_stats(self._ptr, C.byref(s)), "uw_stats")
        return s.as_dict()

    def free(self):
        ptr = getattr(self, "_ptr", None)
        if ptr is not None and ptr.value:
            self._free(ptr)
            self._ptr = self._null

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass


def uw_host_save(h: HostEncoded, path: str) -> None:
    """Write a host encoding to a bundle file (see include/unweight.h)."""
    _check(lib.uw_host_save(h.ptr, os.fsencode(path)), "uw_host_save")


def uw_host_load(path: str) -> HostEncoded:
    """Read a bundle file into a host encoding (checksummed and validated)."""
    out = _vp()
    _check(lib.uw_host_load(os.fsencode(path), C.byref(out)), "uw_host_load")
    return HostEncoded(out.value)


def uw_load(path: str, opts: uw_encode_opts | None = None, stream=None) -> Handle:
    """A bundle file straight to the device (uw_host_load + uw_upload)."""
    out = _vp()
    _check(lib.uw_load(os.fsencode(path), C.byref(opts) if opts else None,
                       _vp(_stream_ptr(stream)), C.byref(out)), "uw_load")
    h = Handle(out.value, 0, 0)
    st = h.stats()
    h.N, h.K = int(st["N"]), int(st["K"])
    return h


def uw_upload(fmt: uw_format, opts: uw_encode_opts | None = None, stream=None) -> Handle:
    out = _vp()
    _check(lib.uw_upload(C.byref(fmt), C.byref(opts) if opts else None,
                         _vp(_stream_ptr(stream)), C.byref(out)), "uw_upload")
    return Handle(out.value, fmt.N, fmt.K)


def uw_encode(w: np.ndarray, opts: uw_encode_opts | None = None, stream=None) -> Handle:
    w = np.ascontiguousarray(w, dtype=np.uint16)
    n, k = w.shape
    out = _vp()
    _check(lib.uw_encode(w.ctypes.data, n, k, C.byref(opts) if opts else None,
                         _vp(_stream_ptr(stream)), C.byref(out)), "uw_encode")
    return Handle(out.value, n, k)


def uw_free(h: Handle) -> None:
    h.free()


def uw_set_stream(h: Handle, stream=None) -> None:
    _check(lib.uw_set_stream(h.ptr, _vp(_stream_ptr(stream))), "uw_set_stream")


def uw_stats(h: Handle) -> dict:
    return h.stats()


def uw_workspace_bytes(h: Handle, pipeline: int, M: int) -> int:
    out = _sz()
    _check(lib.uw_workspace_bytes(h.ptr, int(pipeline), int(M), C.byref(out)),
           "uw_workspace_bytes")
    return int(out.value)


def uw_set_workspace(h: Handle, ws) -> None:
    """Register a caller-owned device buffer (a torch tensor; kept alive here)."""
    if ws is None:
        _check(lib.uw_set_workspace(h.ptr, None, 0), "uw_set_workspace")
        h._ws = None
        return
    nbytes = ws.numel() * ws.element_size()
    _check(lib.uw_set_workspace(h.ptr, _vp(_dptr(ws)), nbytes), "uw_set_workspace")
    h._ws = ws


def uw_alloc_workspace(h: Handle, nbytes: int) -> None:
    _check(lib.uw_alloc_workspace(h.ptr, int(nbytes)), "uw_alloc_workspace")


def uw_decode_full(h: Handle, w_out) -> None:
    _check(lib.uw_decode_full(h.ptr, _vp(_dptr(w_out))), "uw_decode_full")


def uw_decode_exp(h: Handle, e_out) -> None:
    _check(lib.uw_decode_exp(h.ptr, _vp(_dptr(e_out))), "uw_decode_exp")


def uw_transcode_palette(h: Handle, idx_out) -> None:
    _check(lib.uw_transcode_palette(h.ptr, _vp(_dptr(idx_out))), "uw_transcode_palette")


def uw_decode_rows(h: Handle, rows, out) -> None:
    """BF16 rows `rows` (device int64 tensor) of the encoded matrix into `out`
    ([len(rows), K] on the device): an embedding lookup on compressed weights."""
    _check(lib.uw_decode_rows(h.ptr, _vp(_dptr(rows)), int(rows.numel()), _vp(_dptr(out))),
           "uw_decode_rows")


def uw_gemm(h: Handle, X, Y, M: int, pipeline: int = UW_PIPE_AUTO) -> None:
    _check(lib.uw_gemm(h.ptr, _vp(_dptr(X)), _vp(_dptr(Y)), int(M), int(pipeline)), "uw_gemm")


def uw_gemm_f32(h: Handle, X, Y, M: int, pipeline: int = UW_PIPE_AUTO) -> None:
    _check(lib.uw_gemm_f32(h.ptr, _vp(_dptr(X)), _vp(_dptr(Y)), int(M), int(pipeline)),
           "uw_gemm_f32")


def gemm_config(pipeline: int, tile_n: int = 0, stages: int = 0, gemm_ctas: int = 0,
                decode_ctas: int = 0, halves: int = 0, pair: int = 0,
                gemv: int = 0) -> uw_gemm_config:
    """A variant: gemv = 1 selects the CUDA-core matrix-vector kernel (M <= 2),
    0 the tensor-core GEMM."""
    c = uw_gemm_config()
    c.pipeline, c.tile_n, c.stages = int(pipeline), int(tile_n), int(stages)
    c.gemm_ctas, c.decode_ctas, c.halves = int(gemm_ctas), int(decode_ctas), int(halves)
    c.pair, c.gemv = int(pair), int(gemv)
    return c


def uw_gemm_ex(h: Handle, X, Y, M: int, cfg: uw_gemm_config, out_f32: bool) -> None:
    _check(lib.uw_gemm_ex(h.ptr, _vp(_dptr(X)), _vp(_dptr(Y)), int(M), C.byref(cfg),
                          1 if out_f32 else 0), "uw_gemm_ex")


def uw_gemm_palette_noalloc(h: Handle, X, Y, M: int, out_f32: bool = False) -> None:
    """Pipeline-4 matmul that allocates nothing (split-K scratch is a fixed
    array inside the library); M <= 64.  See include/unweight.h."""
    _check(lib.uw_gemm_palette_noalloc(h.ptr, _vp(_dptr(X)), _vp(_dptr(Y)), int(M),
                                       1 if out_f32 else 0), "uw_gemm_palette_noalloc")


def uw_swiglu(g, u, h, n: int | None = None, stream=None) -> None:
    n = g.numel() if n is None else int(n)
    _check(lib.uw_swiglu(_vp(_dptr(g)), _vp(_dptr(u)), _vp(_dptr(h)), n,
                         _vp(_stream_ptr(stream))), "uw_swiglu")


def mlp_layers(layers):
    """[(gate, up, down) Handles] -> ctypes array of uw_mlp_layer."""
    arr = (uw_mlp_layer * len(layers))()
    for i, (g, u, d) in enumerate(layers):
        arr[i].gate, arr[i].up, arr[i].down = g.ptr.value, u.ptr.value, d.ptr.value
    return arr


def mlp_opts(overlap=False, decode_ctas=0, gemm_ctas=0) -> uw_mlp_opts:
    o = uw_mlp_opts()
    o.overlap, o.decode_ctas, o.gemm_ctas = int(bool(overlap)), int(decode_ctas), int(gemm_ctas)
    return o


def uw_mlp_workspace_bytes(layers, M: int, opts: uw_mlp_opts | None = None) -> int:
    arr = mlp_layers(layers)
    out = _sz()
    _check(lib.uw_mlp_workspace_bytes(arr, len(layers), int(M), C.byref(opts) if opts else None,
                                      C.byref(out)), "uw_mlp_workspace_bytes")
    return int(out.value)


def uw_mlp_forward(layers, X, Y, M: int, ws, opts: uw_mlp_opts | None = None, stream=None,
                   side_stream=None) -> None:
    arr = mlp_layers(layers)
    nbytes = ws.numel() * ws.element_size()
    side = _vp(_stream_ptr(side_stream)) if side_stream is not None else None
    _check(lib.uw_mlp_forward(arr, len(layers), _vp(_dptr(X)), _vp(_dptr(Y)), int(M),
                              _vp(_dptr(ws)), nbytes, _vp(_stream_ptr(stream)), side,
                              C.byref(opts) if opts else None), "uw_mlp_forward")


def uw_mlp_forward_record(layers, X, Y, M: int, ws, act, opts: uw_mlp_opts | None = None,
                          stream=None, side_stream=None) -> None:
    """uw_mlp_forward, also writing each layer's g, u, h and output into act
    (device, per layer M*(3F + D) BF16 values in that order)."""
    arr = mlp_layers(layers)
    nbytes = ws.numel() * ws.element_size()
    side = _vp(_stream_ptr(side_stream)) if side_stream is not None else None
    _check(lib.uw_mlp_forward_record(arr, len(layers), _vp(_dptr(X)), _vp(_dptr(Y)), int(M),
                                     _vp(_dptr(ws)), nbytes, _vp(_stream_ptr(stream)), side,
                                     C.byref(opts) if opts else None, _vp(_dptr(act))),
           "uw_mlp_forward_record")


def uw_mlp_tune_split(layers, X, Y, M: int, ws, stream=None, side_stream=None) -> uw_mlp_opts:
    arr = mlp_layers(layers)
    best = uw_mlp_opts()
    nbytes = ws.numel() * ws.element_size()
    _check(lib.uw_mlp_tune_split(arr, len(layers), _vp(_dptr(X)), _vp(_dptr(Y)), int(M),
                                 _vp(_dptr(ws)), nbytes, _vp(_stream_ptr(stream)),
                                 _vp(_stream_ptr(side_stream)), C.byref(best)),
           "uw_mlp_tune_split")
    return best


def uw_autotune(handles, Ms, profile_out_json: str | None = None) -> None:
    arr = (_vp * len(handles))(*[h.ptr for h in handles])
    ms = (_i64 * len(Ms))(*[int(m) for m in Ms])
    _check(lib.uw_autotune(arr, len(handles), ms, len(Ms),
                           profile_out_json.encode() if profile_out_json else None), "uw_autotune")


def uw_load_profile(handles, profile_json: str) -> None:
    arr = (_vp * len(handles))(*[h.ptr for h in handles])
    _check(lib.uw_load_profile(arr, len(handles), profile_json.encode()), "uw_load_profile")


def uw_get_choice(h: Handle, M: int) -> dict:
    c = uw_gemm_config()
    _check(lib.uw_get_choice(h.ptr, int(M), C.byref(c)), "uw_get_choice")
    return c.as_dict()


KERNEL_KINDS = ("decode_full", "decode_exp", "transcode", "gemm_bf16", "gemm_exp",
                "gemm_palette", "splitk_fixup", "gemv_bf16", "gemv_exp", "gemv_palette",
                "decode_dot")


def uw_trace_enable(h: Handle, enable: bool = True) -> None:
    _check(lib.uw_trace_enable(h.ptr, 1 if enable else 0), "uw_trace_enable")


def uw_trace_read(h: Handle, capacity: int = 16384):
    """[(kernel kind name, milliseconds)] of the launches traced since the last read."""
    kinds = (_i32 * capacity)()
    ms = (C.c_float * capacity)()
    n = _i32()
    _check(lib.uw_trace_read(h.ptr, kinds, ms, capacity, C.byref(n)), "uw_trace_read")
    return [(KERNEL_KINDS[kinds[i]], float(ms[i])) for i in range(min(n.value, capacity))]


def uw_last_device_status(h: Handle) -> int:
    """Synchronises the handle's stream; returns (does not raise) the device status."""
    return int(lib.uw_last_device_status(h.ptr))
