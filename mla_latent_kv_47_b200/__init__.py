"""Python binding of the B200 MLA latent-KV library (libmla_b200.so).

Argument marshalling only: every step of the MLA path runs in the library's
CUDA kernels.  PyTorch supplies device memory and the current stream.  The
library must be built (``python -m mla_latent_kv_47_b200.build``); importing
this module without it raises, there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmla_b200.so")

MLA_BF16, MLA_FP32 = 0, 1
CACHE_DTYPE, CACHE_E4M3 = 0, 1
STATUS = {0: "MLA_OK", -1: "MLA_ERR_INVALID_ARG", -2: "MLA_ERR_UNSUPPORTED", -3: "MLA_ERR_MISALIGNED",
          -4: "MLA_ERR_WORKSPACE", -5: "MLA_ERR_CUDA", -6: "MLA_ERR_DEVICE_FAULT"}
FAULT_CAPACITY, FAULT_WAIT_TIMEOUT, FAULT_PLAN, FAULT_RANGE = 1, 2, 4, 8
WS_CQ, WS_QC, WS_QLAT, WS_OLAT, WS_O, WS_CKV_RAW = range(6)

EXPORTS = ("mla_workspace_bytes", "mla_cache_append", "mla_decode", "mla_prefill",
           "mla_get_device_status", "mla_status_string", "mla_workspace_offset", "mla_set_attention_events",
           "mla_decode_static", "mla_kernel_launches", "mla_check_wait_timeout")


class MLAError(RuntimeError):
    def __init__(self, code, where):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)} ({status_string(code)})")


class Dims(ctypes.Structure):
    _fields_ = [("d_model", ctypes.c_int), ("n_h", ctypes.c_int), ("d_h", ctypes.c_int), ("d_R", ctypes.c_int),
                ("d_c", ctypes.c_int), ("d_cq", ctypes.c_int), ("rope_base", ctypes.c_double),
                ("dtype", ctypes.c_int), ("yarn_s", ctypes.c_double), ("yarn_alpha", ctypes.c_double),
                ("yarn_beta", ctypes.c_double), ("yarn_L0", ctypes.c_double), ("cache_format", ctypes.c_int)]


WEIGHT_FIELDS = ("W_DQ", "W_UQ", "W_QR", "W_DKV", "W_UK", "W_UV", "W_KR", "W_O", "g_kv", "g_q")


class Weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in WEIGHT_FIELDS]


class Cache(ctypes.Structure):
    _fields_ = [("base", ctypes.c_void_p), ("seq_start", ctypes.c_void_p), ("capacity", ctypes.c_void_p),
                ("n_rows", ctypes.c_int64), ("block_table", ctypes.c_void_p), ("block_size", ctypes.c_int32),
                ("max_blocks", ctypes.c_int32)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m mla_latent_kv_47_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    P = ctypes.POINTER
    lib.mla_workspace_bytes.argtypes = [P(Dims), i32, i32]
    lib.mla_workspace_bytes.restype = sz
    lib.mla_workspace_offset.argtypes = [P(Dims), i32, i32, i32]
    lib.mla_workspace_offset.restype = sz
    lib.mla_cache_append.argtypes = [P(Dims), P(Weights), vp, i32, vp, vp, P(Cache), vp, sz, vp]
    lib.mla_cache_append.restype = i32
    lib.mla_decode.argtypes = [P(Dims), P(Weights), vp, i32, P(Cache), vp, vp, vp, sz, vp]
    lib.mla_decode.restype = i32
    lib.mla_prefill.argtypes = [P(Dims), P(Weights), vp, i32, i32, P(Cache), i32, vp, vp, sz, vp]
    lib.mla_prefill.restype = i32
    lib.mla_get_device_status.argtypes = [vp, vp, P(i32)]
    lib.mla_get_device_status.restype = i32
    lib.mla_status_string.argtypes = [i32]
    lib.mla_status_string.restype = ctypes.c_char_p
    lib.mla_decode_static.argtypes = [P(Dims), P(Weights), vp, i32, P(Cache), vp, vp, vp]
    lib.mla_decode_static.restype = i32
    lib.mla_kernel_launches.argtypes = []
    lib.mla_kernel_launches.restype = ctypes.c_ulonglong
    lib.mla_check_wait_timeout.argtypes = [vp, vp]
    lib.mla_check_wait_timeout.restype = i32
    lib.mla_set_attention_events.argtypes = [vp, vp]
    lib.mla_set_attention_events.restype = None
    return lib


_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        _LIB = _load()
    return _LIB


def __getattr__(name):
    # `lib` is loaded on first use, so the build script can import this package
    # before the library exists.  A missing library raises ImportError here.
    if name == "lib":
        return _lib()
    raise AttributeError(name)


def status_string(code: int) -> str:
    return _lib().mla_status_string(int(code)).decode()


def make_dims(d) -> Dims:
    """ctypes dims from any object with the fields of synth.Dims (and, for
    YaRN, a `yarn` = (s, alpha, beta, L0) attribute)."""
    y = getattr(d, "yarn", None) or (0.0, 0.0, 0.0, 0.0)
    fmt = {"dtype": CACHE_DTYPE, "e4m3": CACHE_E4M3}[getattr(d, "cache", "dtype")]
    return Dims(d.d_model, d.n_h, d.d_h, d.d_R, d.d_c, d.d_cq, float(d.rope_base),
                MLA_FP32 if getattr(d, "dtype", "bf16") == "fp32" else MLA_BF16, *[float(v) for v in y], fmt)


def cache_row_bytes(dims: Dims) -> int:
    """Bytes of one cache row (the layouts of mla_cache_format)."""
    if dims.cache_format == CACHE_E4M3:
        return dims.d_c + 2 * dims.d_R + 16
    return (dims.d_c + dims.d_R) * (4 if dims.dtype == MLA_FP32 else 2)


def _ptr(t):
    if t is None:
        return None
    assert t.is_cuda and t.is_contiguous(), "device tensors must be contiguous CUDA tensors"
    return t.data_ptr()


def make_weights(W: dict) -> Weights:
    """Device weight tensors by name (the RMSNorm gains g_kv / g_q are optional).
    The returned struct holds the tensors, so their memory lives as long as it does."""
    w = Weights(*[_ptr(W.get(n)) for n in WEIGHT_FIELDS])
    w._tensors = [W.get(n) for n in WEIGHT_FIELDS]
    return w


def make_cache(base, seq_start=None, capacity=None, block_table=None, block_size=0) -> Cache:
    """base: [n_rows, d_c + d_R] device tensor; seq_start int64 [n_seq] (contiguous layout) or
    block_table int32 [n_seq, max_blocks] with block_size rows per page (paged layout);
    capacity int32 [n_seq] or None."""
    assert seq_start is None or seq_start.dtype == torch.int64
    assert capacity is None or capacity.dtype == torch.int32
    if block_table is not None:
        assert block_table.dtype == torch.int32 and block_table.dim() == 2
        c = Cache(_ptr(base), _ptr(seq_start), _ptr(capacity), int(base.shape[0]), _ptr(block_table),
                  int(block_size), int(block_table.shape[1]))
    else:
        c = Cache(_ptr(base), _ptr(seq_start), _ptr(capacity), int(base.shape[0]), None, 0, 0)
    c._tensors = (base, seq_start, capacity, block_table)  # the struct keeps the memory it points to alive
    return c


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(code, where):
    if code != 0:
        raise MLAError(code, where)


def workspace_bytes(dims: Dims, max_batch: int, max_tokens: int) -> int:
    return int(_lib().mla_workspace_bytes(ctypes.byref(dims), int(max_batch), int(max_tokens)))


def workspace_offset(dims: Dims, batch: int, which: int) -> int:
    return int(_lib().mla_workspace_offset(ctypes.byref(dims), int(batch), 0, int(which)))


def workspace_offset_tokens(dims: Dims, max_tokens: int, which: int) -> int:
    """Offset of an append / prefill intermediate (WS_CKV_RAW) for up to max_tokens tokens."""
    return int(_lib().mla_workspace_offset(ctypes.byref(dims), 1, int(max_tokens), int(which)))


def alloc_workspace(dims: Dims, max_batch: int, max_tokens: int, device="cuda") -> torch.Tensor:
    n = workspace_bytes(dims, max_batch, max_tokens)
    if n == 0:
        raise MLAError(-2, "mla_workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def cache_append(dims, weights, h, seq_idx, pos, cache, workspace, stream=None):
    assert seq_idx.dtype == torch.int32 and pos.dtype == torch.int32
    _check(_lib().mla_cache_append(ctypes.byref(dims), ctypes.byref(weights), _ptr(h), int(h.shape[0]),
                                _ptr(seq_idx), _ptr(pos), ctypes.byref(cache), _ptr(workspace),
                                workspace.numel(), _stream(stream)), "mla_cache_append")


def decode(dims, weights, h, cache, seqlen, u, workspace, stream=None):
    assert seqlen.dtype == torch.int32 and u.dtype == torch.float32
    _check(_lib().mla_decode(ctypes.byref(dims), ctypes.byref(weights), _ptr(h), int(h.shape[0]),
                          ctypes.byref(cache), _ptr(seqlen), _ptr(u), _ptr(workspace), workspace.numel(),
                          _stream(stream)), "mla_decode")


def prefill(dims, weights, h, start_pos, cache, seq, u, workspace, stream=None):
    assert u.dtype == torch.float32
    _check(_lib().mla_prefill(ctypes.byref(dims), ctypes.byref(weights), _ptr(h), int(h.shape[0]), int(start_pos),
                           ctypes.byref(cache), int(seq), _ptr(u), _ptr(workspace), workspace.numel(),
                           _stream(stream)), "mla_prefill")


def decode_static(dims, weights, h, cache, seqlen, u, stream=None):
    """mla_decode without a workspace: the library's static device scratch is used."""
    assert seqlen.dtype == torch.int32 and u.dtype == torch.float32
    _check(_lib().mla_decode_static(ctypes.byref(dims), ctypes.byref(weights), _ptr(h), int(h.shape[0]),
                                    ctypes.byref(cache), _ptr(seqlen), _ptr(u), _stream(stream)),
           "mla_decode_static")


def check_wait_timeout(workspace, stream=None):
    """Runs the library's bounded-wait self-check (about 2 s on the GPU)."""
    _check(_lib().mla_check_wait_timeout(_ptr(workspace), _stream(stream)), "mla_check_wait_timeout")


def device_status(workspace, stream=None):
    """(status code, fault bits); synchronises the stream and clears the word."""
    detail = ctypes.c_int(0)
    code = _lib().mla_get_device_status(_ptr(workspace), _stream(stream), ctypes.byref(detail))
    return int(code), int(detail.value)


def set_attention_events(begin=None, end=None):
    """Bracket the attention kernel of the next calls with two torch.cuda.Event objects (None clears)."""
    _lib().mla_set_attention_events(ctypes.c_void_p(begin.cuda_event) if begin is not None else None,
                                 ctypes.c_void_p(end.cuda_event) if end is not None else None)


def kernel_launches() -> int:
    """Kernels launched by the library so far in this process (diagnostic)."""
    return int(_lib().mla_kernel_launches())
