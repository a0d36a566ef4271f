"""ctypes binding of libmla.so: argument marshalling only.

Every step of the decode runs in the CUDA library; this module turns torch
tensors into the C ABI's pointers, sizes and structs (include/mla.h),
allocates outputs / workspace with torch, and raises on any non-zero return
code.  ``load()`` raises if the library has not been built: there is no
fallback path.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmla.so")

MLA_DTYPE_BF16, MLA_DTYPE_F32 = 0, 1
PATH_AUTO, PATH_SM100, PATH_GENERIC = 0, 1, 2
STATUS_BAD_POS, STATUS_BAD_SEQLEN, STATUS_TIMEOUT = 1, 2, 4
NUM_EVENTS = 6
EV_START, EV_ABSORB_DONE, EV_ATTEND_BEGIN, EV_ATTEND_END, EV_COMBINE_DONE, EV_END = range(6)
ERRORS = {-1: "MLA_ERR_ARG", -2: "MLA_ERR_SHAPE", -3: "MLA_ERR_ALIGN", -4: "MLA_ERR_CUDA",
          -5: "MLA_ERR_TIMEOUT", -6: "MLA_ERR_DEVICE", -7: "MLA_ERR_WORKSPACE", -8: "MLA_ERR_UNSUPPORTED"}

# Every symbol the header declares (checked by the CPU test suite).
EXPORTS = ["mla_append_cache", "mla_workspace_bytes", "mla_decode", "mla_decode_ex", "mla_absorb_query",
           "mla_attend_latent", "mla_project_out", "mla_device_status", "mla_last_error", "mla_last_path",
           "mla_version", "mla_decode_no_alloc", "mla_append_from_hidden", "mla_append_from_hidden_workspace_bytes",
           "mla_output_projection", "mla_output_projection_workspace_bytes"]


class Dims(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int32), ("d_c", ctypes.c_int32), ("d_r", ctypes.c_int32),
                ("d_n", ctypes.c_int32), ("d_v", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("rope_base", ctypes.c_float), ("softmax_scale", ctypes.c_float)]


class Cache(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("B", ctypes.c_int32), ("T_max", ctypes.c_int32),
                ("stride_b", ctypes.c_int64), ("stride_t", ctypes.c_int64)]


class Opts(ctypes.Structure):
    _fields_ = [("path", ctypes.c_int32), ("num_pairs", ctypes.c_int32), ("overhead_tiles", ctypes.c_int32),
                ("min_tiles", ctypes.c_int32), ("n_events", ctypes.c_int32),
                ("events", ctypes.POINTER(ctypes.c_void_p)), ("wait_limit_ns", ctypes.c_int64),
                ("withhold_tile", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class MLAError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"{ERRORS.get(code, code)}: {msg}")
        self.code = code


_P = ctypes.c_void_p
_I = ctypes.c_int32
_SIGS = {
    "mla_append_cache": ([ctypes.POINTER(Dims), _P, _P, _P, _I, _I, ctypes.POINTER(Cache), _P], ctypes.c_int),
    "mla_workspace_bytes": ([ctypes.POINTER(Dims), _I, _I], ctypes.c_size_t),
    "mla_decode": ([ctypes.POINTER(Dims), _P, _P, _P, _P, ctypes.POINTER(Cache), _P, _I, _I, _P, _P,
                    ctypes.c_size_t, _P], ctypes.c_int),
    "mla_decode_ex": ([ctypes.POINTER(Dims), _P, _P, _P, _P, ctypes.POINTER(Cache), _P, _I, _I, _P, _P,
                       ctypes.c_size_t, ctypes.POINTER(Opts), _P], ctypes.c_int),
    "mla_decode_no_alloc": ([ctypes.POINTER(Dims), _P, _P, _P, _P, ctypes.POINTER(Cache), _P, _I, _I, _P, _P],
                            ctypes.c_int),
    "mla_absorb_query": ([ctypes.POINTER(Dims), _P, _P, _P, _P, _I, _I, _P, ctypes.POINTER(Opts), _P], ctypes.c_int),
    "mla_attend_latent": ([ctypes.POINTER(Dims), _P, ctypes.POINTER(Cache), _P, _I, _I, _P, _P, ctypes.c_size_t,
                           ctypes.POINTER(Opts), _P], ctypes.c_int),
    "mla_project_out": ([ctypes.POINTER(Dims), _P, _P, _I, _P, ctypes.POINTER(Opts), _P], ctypes.c_int),
    "mla_append_from_hidden_workspace_bytes": ([ctypes.POINTER(Dims), _I, _I, _I], ctypes.c_size_t),
    "mla_append_from_hidden": ([ctypes.POINTER(Dims), _P, _P, _P, _P, _I, _I, _I, ctypes.POINTER(Cache), _P,
                                ctypes.c_size_t, _P], ctypes.c_int),
    "mla_output_projection_workspace_bytes": ([ctypes.POINTER(Dims), _I, _I], ctypes.c_size_t),
    "mla_output_projection": ([ctypes.POINTER(Dims), _P, _P, _I, _I, _P, _P, ctypes.c_size_t, _P], ctypes.c_int),
    "mla_device_status": ([_P, ctypes.POINTER(_I)], ctypes.c_int),
    "mla_last_error": ([], ctypes.c_char_p),
    "mla_last_path": ([], ctypes.c_char_p),
    "mla_version": ([], ctypes.c_int),
}


def _torch_dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return MLA_DTYPE_BF16
    if t.dtype == torch.float32:
        return MLA_DTYPE_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t: torch.Tensor, name: str, dtype=None, ndim=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")


class Library:
    def __init__(self, path: str = LIB_PATH):
        if not os.path.exists(path):
            raise FileNotFoundError(f"{path} is missing: build it with "
                                    "`python -m latent_compressed_attention_absorbed_b200.build`")
        self.path = path
        self.lib = ctypes.CDLL(path)
        for name, (args, res) in _SIGS.items():
            f = getattr(self.lib, name)
            f.argtypes = args
            f.restype = res

    # ------------------------------------------------------------------ helpers
    def _check(self, rc: int):
        if rc != 0:
            raise MLAError(rc, self.lib.mla_last_error().decode())

    @staticmethod
    def dims(H, d_c, d_r, d_n, d_v, dtype, rope_base=10000.0, softmax_scale=0.0) -> Dims:
        code = dtype if isinstance(dtype, int) else _torch_dtype_code(torch.empty(0, dtype=dtype))
        return Dims(H, d_c, d_r, d_n, d_v, code, rope_base, softmax_scale)

    @staticmethod
    def cache_desc(cache: torch.Tensor) -> Cache:
        """[B][T_max][row] with unit stride along the row; the other two strides
        are passed on (a view of a larger buffer: padded rows, or a subset of a
        larger batch), and the library checks them."""
        if not cache.is_cuda:
            raise ValueError("cache must be a CUDA tensor")
        if cache.dim() != 3:
            raise ValueError(f"cache must have 3 dims, got {tuple(cache.shape)}")
        if cache.stride(2) != 1:
            raise ValueError("cache rows must be contiguous (unit stride along the last dimension)")
        return Cache(cache.data_ptr(), cache.shape[0], cache.shape[1], cache.stride(0), cache.stride(1))

    @staticmethod
    def opts(path=PATH_AUTO, num_pairs=0, overhead_tiles=-1, min_tiles=0, events=None, wait_limit_ns=0,
             withhold_tile=0) -> Opts:
        """``events``: MLA_NUM_EVENTS recorded torch.cuda.Event objects (stage timing).
        ``wait_limit_ns`` / ``withhold_tile``: see mla_decode_opts_t (the latter is a test hook)."""
        o = Opts(path, num_pairs, overhead_tiles, min_tiles, 0, None, wait_limit_ns, withhold_tile, 0)
        if events is not None:
            arr = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
            o.events = ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p))
            o.n_events = len(events)
            o._keep = arr  # keep the array alive as long as the options
        return o

    def last_path(self) -> str:
        return self.lib.mla_last_path().decode()

    def version(self) -> int:
        return self.lib.mla_version()

    # ------------------------------------------------------------------ entry points
    def workspace_bytes(self, dims: Dims, B: int, q_len: int) -> int:
        return int(self.lib.mla_workspace_bytes(ctypes.byref(dims), B, q_len))

    def append_cache(self, dims: Dims, cache: torch.Tensor, c_kv: torch.Tensor, k_rope: torch.Tensor,
                     pos: torch.Tensor, stream=None):
        """Rows pos[b]+i of cache[b] <- [c_kv[b,i] || RoPE(k_rope[b,i], pos[b]+i)]."""
        _need(c_kv, "c_kv", ndim=3)
        _need(k_rope, "k_rope", ndim=3)
        _need(pos, "pos", dtype=torch.int32, ndim=1)
        B, n_tok = c_kv.shape[0], c_kv.shape[1]
        cd = self.cache_desc(cache)
        self._check(self.lib.mla_append_cache(ctypes.byref(dims), _ptr(c_kv), _ptr(k_rope), _ptr(pos), B, n_tok,
                                              ctypes.byref(cd), _stream(stream)))

    def decode(self, dims: Dims, q_nope, q_rope, W_UK, W_UV, cache, seqlens, out=None, workspace=None,
               opts: Optional[Opts] = None, stream=None):
        """One absorbed-MLA decode step; returns out [B, q_len, H, d_v]."""
        for t, n in ((q_nope, "q_nope"), (q_rope, "q_rope"), (W_UK, "W_UK"), (W_UV, "W_UV")):
            _need(t, n)
        _need(seqlens, "seqlens", dtype=torch.int32, ndim=1)
        B, q_len = q_nope.shape[0], q_nope.shape[1]
        if out is None:
            out = torch.empty((B, q_len, dims.H, dims.d_v), dtype=q_nope.dtype, device=q_nope.device)
        if workspace is None:
            workspace = torch.empty(max(self.workspace_bytes(dims, B, q_len), 16), dtype=torch.uint8,
                                    device=q_nope.device)
        cd = self.cache_desc(cache)
        o = opts if opts is not None else self.opts()
        self._check(self.lib.mla_decode_ex(ctypes.byref(dims), _ptr(q_nope), _ptr(q_rope), _ptr(W_UK), _ptr(W_UV),
                                           ctypes.byref(cd), _ptr(seqlens), B, q_len, _ptr(out), _ptr(workspace),
                                           workspace.numel(), ctypes.byref(o), _stream(stream)))
        return out

    def decode_no_alloc(self, dims: Dims, q_nope, q_rope, W_UK, W_UV, cache, seqlens, out=None, stream=None):
        """Same step as decode() using the library's static device scratch (no workspace argument)."""
        for t, n in ((q_nope, "q_nope"), (q_rope, "q_rope"), (W_UK, "W_UK"), (W_UV, "W_UV")):
            _need(t, n)
        _need(seqlens, "seqlens", dtype=torch.int32, ndim=1)
        B, q_len = q_nope.shape[0], q_nope.shape[1]
        if out is None:
            out = torch.empty((B, q_len, dims.H, dims.d_v), dtype=q_nope.dtype, device=q_nope.device)
        cd = self.cache_desc(cache)
        self._check(self.lib.mla_decode_no_alloc(ctypes.byref(dims), _ptr(q_nope), _ptr(q_rope), _ptr(W_UK),
                                                 _ptr(W_UV), ctypes.byref(cd), _ptr(seqlens), B, q_len, _ptr(out),
                                                 _stream(stream)))
        return out

    def absorb_query(self, dims: Dims, q_nope, q_rope, W_UK, seqlens, out=None, opts=None, stream=None):
        B, q_len = q_nope.shape[0], q_nope.shape[1]
        if out is None:
            out = torch.empty((B, q_len, dims.H, dims.d_c + dims.d_r), dtype=q_nope.dtype, device=q_nope.device)
        o = opts if opts is not None else self.opts()
        self._check(self.lib.mla_absorb_query(ctypes.byref(dims), _ptr(q_nope), _ptr(q_rope), _ptr(W_UK),
                                              _ptr(seqlens), B, q_len, _ptr(out), ctypes.byref(o), _stream(stream)))
        return out

    def attend_latent(self, dims: Dims, q_hat, cache, seqlens, out=None, workspace=None, opts=None, stream=None):
        B, q_len = q_hat.shape[0], q_hat.shape[1]
        if out is None:
            out = torch.empty((B, q_len, dims.H, dims.d_c), dtype=q_hat.dtype, device=q_hat.device)
        if workspace is None:
            workspace = torch.empty(max(self.workspace_bytes(dims, B, q_len), 16), dtype=torch.uint8,
                                    device=q_hat.device)
        cd = self.cache_desc(cache)
        o = opts if opts is not None else self.opts()
        self._check(self.lib.mla_attend_latent(ctypes.byref(dims), _ptr(q_hat), ctypes.byref(cd), _ptr(seqlens), B,
                                               q_len, _ptr(out), _ptr(workspace), workspace.numel(), ctypes.byref(o),
                                               _stream(stream)))
        return out

    def project_out(self, dims: Dims, o_lat, W_UV, out=None, opts=None, stream=None):
        rows = o_lat.shape[0] * o_lat.shape[1]
        if out is None:
            out = torch.empty((o_lat.shape[0], o_lat.shape[1], dims.H, dims.d_v), dtype=o_lat.dtype,
                              device=o_lat.device)
        o = opts if opts is not None else self.opts()
        self._check(self.lib.mla_project_out(ctypes.byref(dims), _ptr(o_lat), _ptr(W_UV), rows, _ptr(out),
                                             ctypes.byref(o), _stream(stream)))
        return out

    def append_from_hidden(self, dims: Dims, cache: torch.Tensor, x: torch.Tensor, W_A: torch.Tensor,
                           gamma: torch.Tensor, pos: torch.Tensor, workspace=None, stream=None):
        """Rows pos[b]+i of cache[b] <- [RMSNorm_gamma(W_DKV x[b,i]) || RoPE(W_KR x[b,i], pos[b]+i)];
        W_A = [W_DKV; W_KR] as [d_c + d_r, d_model]."""
        _need(x, "x", ndim=3)
        _need(W_A, "W_A", ndim=2)
        _need(gamma, "gamma", ndim=1)
        _need(pos, "pos", dtype=torch.int32, ndim=1)
        B, n_tok, d_model = x.shape
        if workspace is None:
            n = self.lib.mla_append_from_hidden_workspace_bytes(ctypes.byref(dims), B, n_tok, d_model)
            workspace = torch.empty(max(int(n), 16), dtype=torch.uint8, device=x.device)
        cd = self.cache_desc(cache)
        self._check(self.lib.mla_append_from_hidden(ctypes.byref(dims), _ptr(x), _ptr(W_A), _ptr(gamma), _ptr(pos),
                                                    B, n_tok, d_model, ctypes.byref(cd), _ptr(workspace),
                                                    workspace.numel(), _stream(stream)))

    def output_projection(self, dims: Dims, attn_out: torch.Tensor, W_O: torch.Tensor, y=None, workspace=None,
                          stream=None):
        """y[r] = W_O attn_out[r] with attn_out viewed as [rows, H * d_v]; W_O is [d_model, H * d_v]."""
        _need(attn_out, "attn_out")
        _need(W_O, "W_O", ndim=2)
        width = dims.H * dims.d_v
        rows, d_model = attn_out.numel() // width, W_O.shape[0]
        if y is None:
            y = torch.empty((rows, d_model), dtype=attn_out.dtype, device=attn_out.device)
        if workspace is None:
            n = self.lib.mla_output_projection_workspace_bytes(ctypes.byref(dims), rows, d_model)
            workspace = torch.empty(max(int(n), 16), dtype=torch.uint8, device=attn_out.device)
        self._check(self.lib.mla_output_projection(ctypes.byref(dims), _ptr(attn_out), _ptr(W_O), rows, d_model,
                                                   _ptr(y), _ptr(workspace), workspace.numel(), _stream(stream)))
        return y

    def device_status(self, stream=None) -> int:
        """Synchronises the stream, returns and clears the device status bits."""
        v = ctypes.c_int32(0)
        rc = self.lib.mla_device_status(_stream(stream), ctypes.byref(v))
        if rc not in (0, -6):
            self._check(rc)
        return int(v.value)


_lock = threading.Lock()
_lib: Optional[Library] = None


def load(path: str = LIB_PATH) -> Library:
    """The CUDA library (loaded once).  Raises if it is not built."""
    global _lib
    with _lock:
        if _lib is None:
            _lib = Library(path)
        return _lib
