"""ctypes binding of the C ABI in ``include/fs_stream.h`` -- argument marshalling only.

Functions keep the C names (``fs_stream_create`` ...). ``Stream`` is a small
convenience wrapper that takes torch tensors, checks dtype/layout/device, and
passes their device pointers and torch's current CUDA stream to the library.
Every step of the path runs in the library's CUDA kernels; if the library is
missing, ``load()`` raises -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib", "libfsstream.so")

FS_OK = 0
FS_ERR_ARG = -1
FS_ERR_STATE = -2
FS_ERR_CUDA = -3
FS_ERR_DEVICE_TIMEOUT = -4
FS_ERR_OOM = -5
FS_ERR_RANGE = -6
FS_STATE_EXPECT_PREFILL = 0
FS_STATE_PREFILLED = 1
FS_STATE_STREAMING = 2
FS_MAX_VERIFY_TOKENS = 256
FS_MAX_TAIL_TOKENS = 1024

# Every symbol the header declares, with (restype, argtypes).
_P = ctypes.c_void_p
_I = ctypes.c_int


class fs_stream_info_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "views", "frames", "tok_per_frame", "text_len", "H", "Hkv", "d", "window_len", "step_tokens",
        "state", "insert_tokens", "query_tokens", "head")] + [
        ("steps", ctypes.c_longlong), ("cache_bytes", ctypes.c_longlong), ("launches", ctypes.c_longlong),
        ("tail_tokens", ctypes.c_int), ("rebase_every", ctypes.c_int)]


SIGNATURES = {
    "fs_stream_create": (_I, [ctypes.POINTER(_P), _I, _I, _I, _I, _I, _I, _I, ctypes.c_float]),
    "fs_stream_destroy": (_I, [_P]),
    "fs_stream_set_stream": (_I, [_P, _P]),
    "fs_stream_reset": (_I, [_P]),
    "fs_stream_insert": (_I, [_P, _P, _P]),
    "fs_stream_insert_batch": (_I, [ctypes.POINTER(_P), _I, ctypes.POINTER(_P), ctypes.POINTER(_P)]),
    "fs_stream_append": (_I, [_P, _P, _P, _I]),
    "fs_stream_insert_proj": (_I, [_P, _P, _P, _I]),
    "fs_stream_attend": (_I, [_P, _P, _P]),
    "fs_stream_attend_ext": (_I, [_P, _P, _P, _P, _I, _P]),
    "fs_stream_attend_ext_static": (_I, [_P, _P, _P, _P, _I, _P]),
    "fs_frame_attend": (_I, [_P, _P, _P, _P, _I, _I, _I, _P]),
    "fs_stream_step_host": (_I, [_P, _P, _P, _P, _P]),
    "fs_stream_sync": (_I, [_P]),
    "fs_stream_info": (_I, [_P, ctypes.POINTER(fs_stream_info_t)]),
    "fs_stream_debug_export": (_I, [_P, _P, _P, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32)]),
    "fs_stream_debug_wait_probe": (_I, [_P, _I]),
    "fs_stream_last_error": (ctypes.c_char_p, [_P]),
    "fs_last_error": (ctypes.c_char_p, []),
}

_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the library (once) and set every function's signature."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library not built: {path} (run python -m streaming_kv_cache_stream_b200.build)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


class FsError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"[{code}] {msg}")
        self.code = code


def _check(rc: int, handle=None) -> None:
    if rc != FS_OK:
        lib = load()
        msg = lib.fs_stream_last_error(handle) if handle else lib.fs_last_error()
        raise FsError(rc, (msg or b"").decode())


def _ptr(t, dtype_name="bfloat16"):
    import torch

    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch tensor")
    if not t.is_cuda:
        raise ValueError("tensor must be on a CUDA device")
    if str(t.dtype) != f"torch.{dtype_name}":
        raise TypeError(f"tensor must be {dtype_name}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


class Stream:
    """One layer's streaming KV cache on the current CUDA device.

    Mirrors the C calls: ``insert(K_new, V_new)``, ``attend(Q, out)``,
    ``attend_ext(Q_x, K_x, V_x, out)``; tensors are contiguous bf16 CUDA tensors
    shaped as the header documents. Work is enqueued on torch's current stream.
    """

    def __init__(self, views, frames, tok_per_frame, text_len, H, Hkv, d, rope_base=10000.0):
        lib = load()
        h = ctypes.c_void_p()
        _check(lib.fs_stream_create(ctypes.byref(h), views, frames, tok_per_frame, text_len, H, Hkv, d,
                                    float(rope_base)))
        self._lib, self.handle = lib, h
        self._bound = None  # the cudaStream_t last passed to fs_stream_set_stream
        self.views, self.frames, self.tok_per_frame, self.text_len = views, frames, tok_per_frame, text_len
        self.H, self.Hkv, self.d = H, Hkv, d

    def close(self):
        if self.handle:
            self._lib.fs_stream_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _bind_stream(self):
        import torch

        cur = torch.cuda.current_stream().cuda_stream
        if cur != self._bound:
            _check(self._lib.fs_stream_set_stream(self.handle, ctypes.c_void_p(cur)), self.handle)
            self._bound = cur

    def info(self) -> fs_stream_info_t:
        i = fs_stream_info_t()
        _check(self._lib.fs_stream_info(self.handle, ctypes.byref(i)), self.handle)
        return i

    def reset(self):
        _check(self._lib.fs_stream_reset(self.handle), self.handle)

    def insert(self, K_new, V_new):
        self._bind_stream()
        _check(self._lib.fs_stream_insert(self.handle, _ptr(K_new), _ptr(V_new)), self.handle)

    def insert_proj(self, X, W):
        """fs_stream_insert_proj: X [tokens, d_model], W [2*Hkv*d, d_model] bf16."""
        if X.dim() != 2 or W.dim() != 2 or W.shape[1] != X.shape[1] or W.shape[0] != 2 * self.Hkv * self.d:
            raise ValueError("X must be [tokens, d_model] and W [2*Hkv*d, d_model]")
        self._bind_stream()
        _check(self._lib.fs_stream_insert_proj(self.handle, _ptr(X), _ptr(W), int(X.shape[1])), self.handle)

    def append(self, K_acc, V_acc):
        """Persist accepted tokens [n, Hkv, d] bf16 at the end of the decode tail."""
        self._bind_stream()
        _check(self._lib.fs_stream_append(self.handle, _ptr(K_acc), _ptr(V_acc), int(K_acc.shape[0])), self.handle)

    def attend(self, Q, out):
        """Q bf16 [tokens, H, d] -> out fp32 [tokens, H, d]."""
        self._bind_stream()
        _check(self._lib.fs_stream_attend(self.handle, _ptr(Q), _ptr(out, "float32")), self.handle)

    def attend_ext(self, Q_x, K_x, V_x, out):
        self._bind_stream()
        _check(self._lib.fs_stream_attend_ext(self.handle, _ptr(Q_x), _ptr(K_x), _ptr(V_x), int(Q_x.shape[0]),
                                              _ptr(out, "float32")), self.handle)

    def attend_ext_static(self, Q_x, K_x, V_x, out):
        """attend_ext with the split-KV partials in the library's fixed device array (no allocation)."""
        self._bind_stream()
        _check(self._lib.fs_stream_attend_ext_static(self.handle, _ptr(Q_x), _ptr(K_x), _ptr(V_x),
                                                     int(Q_x.shape[0]), _ptr(out, "float32")), self.handle)

    def frame_attend(self, Q, K, V, out):
        """Encoder attention over each view's newest frame: Q [views*n, H, d],
        K/V [views*n, Hkv, d] bf16 -> out fp32 [views*n, H, d]."""
        self._bind_stream()
        _check(self._lib.fs_frame_attend(self.handle, _ptr(Q), _ptr(K), _ptr(V), int(Q.shape[1]), int(K.shape[1]),
                                         int(Q.shape[2]), _ptr(out, "float32")), self.handle)

    def step_host(self, K_new_h, V_new_h, Q_h, out_h):
        """Host-buffer step: numpy/torch CPU buffers (pinned for asynchrony)."""
        self._bind_stream()

        def hp(x):
            if hasattr(x, "data_ptr"):
                return ctypes.c_void_p(x.data_ptr())
            return ctypes.c_void_p(x.ctypes.data)
        _check(self._lib.fs_stream_step_host(self.handle, hp(K_new_h), hp(V_new_h), hp(Q_h), hp(out_h)),
               self.handle)

    def sync(self):
        _check(self._lib.fs_stream_sync(self.handle), self.handle)

    def debug_export(self):
        """Host copies: K, V [Hkv][rows][d] bf16 bits (uint16), pos[rows], frame_id[rows]."""
        import numpy as np

        i = self.info()
        rows = i.window_len + i.tail_tokens
        K = np.empty((self.Hkv, rows, self.d), dtype=np.uint16)
        V = np.empty_like(K)
        pos = np.empty(rows, dtype=np.int32)
        fid = np.empty(rows, dtype=np.int32)
        _check(self._lib.fs_stream_debug_export(
            self.handle, ctypes.c_void_p(K.ctypes.data), ctypes.c_void_p(V.ctypes.data),
            pos.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), fid.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))),
            self.handle)
        return dict(K=K, V=V, pos=pos, frame_id=fid)


def insert_batch(streams, K_list, V_list):
    """fs_stream_insert_batch: one kv_stream_insert launch for every layer's
    handle (streams[i] gets K_list[i], V_list[i]); torch's current stream."""
    import torch

    n = len(streams)
    if not (n == len(K_list) == len(V_list)) or n == 0:
        raise ValueError("need one K and one V per stream")
    lib = load()
    for s in streams:
        s._bind_stream()
    hs = (_P * n)(*[s.handle.value for s in streams])
    ks = (_P * n)(*[_ptr(k).value for k in K_list])
    vs = (_P * n)(*[_ptr(v).value for v in V_list])
    _check(lib.fs_stream_insert_batch(hs, n, ks, vs), streams[0].handle)
