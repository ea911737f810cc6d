"""ctypes binding of libswa.so (include/swa.h), same names as the C ABI.

Argument marshalling only: every step of the attention path runs in the CUDA
kernels behind the C ABI.  PyTorch supplies device memory and the current
stream.  There is no fallback: if libswa.so is missing or a call fails, this
module raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libswa.so")

WINDOW_FULL = -1

SWA_OK = 0
STATUS_NAMES = {0: "SWA_OK", 1: "SWA_ERR_INVALID_ARG", 2: "SWA_ERR_UNSUPPORTED", 3: "SWA_ERR_WORKSPACE",
                4: "SWA_ERR_CUDA"}

# every function include/swa.h declares
SYMBOLS = ("swa_rope_qk", "swa_prefill_workspace_size", "swa_attn_prefill", "swa_decode_workspace_size",
           "swa_attn_decode", "swa_kv_cache_bytes", "swa_status_string", "swa_last_error_detail",
           "swa_device_error", "swa_version", "swa_attn_decode_no_alloc", "swa_prefill_chunk_workspace_size",
           "swa_attn_prefill_chunk", "swa_decode_mq_workspace_size", "swa_attn_decode_mq")

# bytes of the static device array behind swa_attn_decode_no_alloc
NO_ALLOC_SCRATCH_BYTES = 16 * 1024 * 1024


class SwaError(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {detail}")
        self.status = status
        self.detail = detail


class _Params(ctypes.Structure):
    _fields_ = [
        ("num_q_heads", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("window", ctypes.c_int32),
        ("rope_theta", ctypes.c_double),
        ("rotary_dim", ctypes.c_int32),
        ("softmax_scale", ctypes.c_float),
        ("inv_freq", ctypes.POINTER(ctypes.c_double)),
    ]


@dataclass(frozen=True)
class LayerParams:
    """swa_layer_params: window -1 = full causal; rope_theta 0 = no RoPE;
    softmax_scale <= 0 = 1/sqrt(head_dim); inv_freq = rotary_dim/2 angular
    frequencies replacing rope_theta^(-2k/rotary_dim) (a caller-scaled RoPE),
    or None."""

    num_q_heads: int
    num_kv_heads: int
    head_dim: int = 128
    window: int = WINDOW_FULL
    rope_theta: float = 10000.0
    rotary_dim: int = 128
    softmax_scale: float = 0.0
    inv_freq: tuple = None

    def c(self) -> _Params:
        """The swa_layer_params struct, built once per (immutable) instance."""
        prm = self.__dict__.get("_c")
        if prm is not None:
            return prm
        freq = None
        if self.inv_freq is not None:
            if len(self.inv_freq) != self.rotary_dim // 2:
                raise ValueError(f"inv_freq holds {len(self.inv_freq)} values, rotary_dim/2 = {self.rotary_dim // 2}")
            freq = (ctypes.c_double * len(self.inv_freq))(*map(float, self.inv_freq))
        prm = _Params(self.num_q_heads, self.num_kv_heads, self.head_dim, self.window, float(self.rope_theta),
                      self.rotary_dim, float(self.softmax_scale),
                      None if freq is None else ctypes.cast(freq, ctypes.POINTER(ctypes.c_double)))
        prm._freq = freq  # the table lives as long as the struct that points to it
        object.__setattr__(self, "_c", prm)  # not a field: equality and hashing ignore it
        return prm


_lib = None


def load(path: str = LIB_PATH):
    """Load libswa.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m full_gqa_attention_swa_b200.build`")
    lib = ctypes.CDLL(path)
    P = ctypes.POINTER(_Params)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    lib.swa_rope_qk.argtypes = [P, i32, i32, vp, vp, vp, i32, vp, vp, vp, i32, vp]
    lib.swa_rope_qk.restype = ctypes.c_int
    lib.swa_prefill_workspace_size.argtypes = [P, i32, i32]
    lib.swa_prefill_workspace_size.restype = sz
    lib.swa_attn_prefill.argtypes = [P, i32, i32, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.swa_attn_prefill.restype = ctypes.c_int
    lib.swa_decode_workspace_size.argtypes = [P, i32, i32]
    lib.swa_decode_workspace_size.restype = sz
    lib.swa_attn_decode.argtypes = [P, i32, vp, vp, vp, vp, i32, vp, i32, vp, vp, sz, vp]
    lib.swa_attn_decode.restype = ctypes.c_int
    lib.swa_kv_cache_bytes.argtypes = [P, i64, i64]
    lib.swa_kv_cache_bytes.restype = i64
    lib.swa_status_string.argtypes = [ctypes.c_int]
    lib.swa_status_string.restype = ctypes.c_char_p
    lib.swa_last_error_detail.argtypes = []
    lib.swa_last_error_detail.restype = ctypes.c_char_p
    lib.swa_device_error.argtypes = [ctypes.POINTER(ctypes.c_int32), i32]
    lib.swa_device_error.restype = ctypes.c_int
    lib.swa_version.argtypes = []
    lib.swa_version.restype = ctypes.c_char_p
    lib.swa_attn_decode_no_alloc.argtypes = [P, i32, vp, vp, vp, vp, i32, vp, i32, vp, vp]
    lib.swa_attn_decode_no_alloc.restype = ctypes.c_int
    lib.swa_prefill_chunk_workspace_size.argtypes = [P, i32, i32, i32]
    lib.swa_prefill_chunk_workspace_size.restype = sz
    lib.swa_attn_prefill_chunk.argtypes = [P, i32, i32, i32, vp, vp, vp, vp, vp, vp, i32, vp, vp, sz, vp]
    lib.swa_attn_prefill_chunk.restype = ctypes.c_int
    lib.swa_decode_mq_workspace_size.argtypes = [P, i32, i32, i32]
    lib.swa_decode_mq_workspace_size.restype = sz
    lib.swa_attn_decode_mq.argtypes = [P, i32, i32, vp, vp, vp, vp, vp, vp, i32, vp, i32, vp, vp, sz, vp]
    lib.swa_attn_decode_mq.restype = ctypes.c_int
    _lib = lib
    return lib


def _check(status: int):
    if status != SWA_OK:
        detail = load().swa_last_error_detail().decode()
        raise SwaError(status, detail)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream):
    """The cudaStream_t to launch on: the given stream, else the current
    stream of the current device (read as a raw handle, without building a
    torch.cuda.Stream object)."""
    if stream is not None:
        return ctypes.c_void_p(stream.cuda_stream)
    if _raw_stream is not None:
        return ctypes.c_void_p(_raw_stream(torch.cuda.current_device()))
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _need(t, name, dtype, shape=None):
    if t is None:
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be on a CUDA device")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _device(*tensors, stream=None):
    """The one CUDA device every given tensor lives on.  The call runs with
    it current (and on its current stream unless one is given): the library
    takes plain pointers, and a pointer into another GPU's memory would reach
    a kernel as an invalid address."""
    devs = {t.device for t in tensors if t is not None}
    if len(devs) != 1:
        raise ValueError(f"tensors must all be on one CUDA device, got {sorted(str(d) for d in devs)}")
    dev = devs.pop()
    if stream is not None and stream.device != dev:
        raise ValueError(f"stream is on {stream.device}, tensors on {dev}")
    return dev


class _Current:
    """Context that makes a CUDA device current only when it is not already
    (the common case costs one device query, not a device switch)."""

    __slots__ = ("dev", "prev")

    def __init__(self, dev):
        self.dev = dev
        self.prev = None

    def __enter__(self):
        cur = torch.cuda.current_device()
        if cur != self.dev.index:
            self.prev = cur
            torch.cuda.set_device(self.dev)
        return self

    def __exit__(self, *exc):
        if self.prev is not None:
            torch.cuda.set_device(self.prev)
        return False


def version() -> str:
    return load().swa_version().decode()


def kv_cache_bytes(layer: LayerParams, batch: int, context: int) -> int:
    return int(load().swa_kv_cache_bytes(ctypes.byref(layer.c()), batch, context))


def rope_qk(layer: LayerParams, q=None, k=None, pos=None, pos0: int = 0, v=None, k_cache=None, v_cache=None,
            stream=None):
    """swa_rope_qk: rotate q [B,S,Hq,D] / k [B,S,Hkv,D] in place at pos [B,S]
    (int32) or pos0 + s; optionally append rotated k and v to the cache
    [B,Hkv,C,D]."""
    ref = q if q is not None else k
    if ref is None:
        return
    B, S = ref.shape[0], ref.shape[1]
    D = layer.head_dim
    _need(q, "q", torch.bfloat16, None if q is None else (B, S, layer.num_q_heads, D))
    _need(k, "k", torch.bfloat16, None if k is None else (B, S, layer.num_kv_heads, D))
    _need(v, "v", torch.bfloat16, None if v is None else (B, S, layer.num_kv_heads, D))
    _need(pos, "pos", torch.int32, None if pos is None else (B, S))
    C = 0
    if k_cache is not None:
        C = k_cache.shape[2]
        _need(k_cache, "k_cache", torch.bfloat16, (B, layer.num_kv_heads, C, D))
        _need(v_cache, "v_cache", torch.bfloat16, (B, layer.num_kv_heads, C, D))
    with _Current(_device(q, k, pos, v, k_cache, v_cache, stream=stream)):
        _check(load().swa_rope_qk(ctypes.byref(layer.c()), B, S, _ptr(q), _ptr(k), _ptr(pos), int(pos0), _ptr(v),
                                  _ptr(k_cache), _ptr(v_cache), C, _stream(stream)))


def prefill_workspace_size(layer: LayerParams, B: int, S: int) -> int:
    return int(load().swa_prefill_workspace_size(ctypes.byref(layer.c()), B, S))


def attn_prefill(layer: LayerParams, q, k, v, gate=None, out=None, workspace=None, stream=None):
    """swa_attn_prefill on un-rotated q [B,S,Hq,D], k/v [B,S,Hkv,D] (bf16);
    gate [B,S,Hq] fp32 or None.  Returns out [B,S,Hq,D] bf16."""
    B, S = q.shape[0], q.shape[1]
    D = layer.head_dim
    _need(q, "q", torch.bfloat16, (B, S, layer.num_q_heads, D))
    _need(k, "k", torch.bfloat16, (B, S, layer.num_kv_heads, D))
    _need(v, "v", torch.bfloat16, (B, S, layer.num_kv_heads, D))
    _need(gate, "gate", torch.float32, (B, S, layer.num_q_heads))
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", torch.bfloat16, (B, S, layer.num_q_heads, D))
    need = prefill_workspace_size(layer, B, S)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with _Current(_device(q, k, v, gate, out, workspace, stream=stream)):
        _check(load().swa_attn_prefill(ctypes.byref(layer.c()), B, S, _ptr(q), _ptr(k), _ptr(v), _ptr(gate),
                                       _ptr(out), _ptr(workspace), nbytes, _stream(stream)))
    return out


def prefill_chunk_workspace_size(layer: LayerParams, B: int, S: int, pos0: int) -> int:
    return int(load().swa_prefill_chunk_workspace_size(ctypes.byref(layer.c()), B, S, pos0))


def attn_prefill_chunk(layer: LayerParams, pos0: int, q, k, v, gate, k_cache, v_cache, out=None, workspace=None,
                       stream=None):
    """swa_attn_prefill_chunk: new tokens at positions pos0 .. pos0+S-1 (q
    [B,S,Hq,D], k/v [B,S,Hkv,D] bf16, not rotated; gate [B,S,Hq] fp32 or None)
    against the KV cache [B,Hkv,C,D] holding positions < pos0; appends the
    chunk to the cache.  Returns out [B,S,Hq,D] bf16."""
    B, S = q.shape[0], q.shape[1]
    D = layer.head_dim
    C = k_cache.shape[2]
    _need(q, "q", torch.bfloat16, (B, S, layer.num_q_heads, D))
    _need(k, "k", torch.bfloat16, (B, S, layer.num_kv_heads, D))
    _need(v, "v", torch.bfloat16, (B, S, layer.num_kv_heads, D))
    _need(gate, "gate", torch.float32, (B, S, layer.num_q_heads))
    _need(k_cache, "k_cache", torch.bfloat16, (B, layer.num_kv_heads, C, D))
    _need(v_cache, "v_cache", torch.bfloat16, (B, layer.num_kv_heads, C, D))
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", torch.bfloat16, (B, S, layer.num_q_heads, D))
    need = prefill_chunk_workspace_size(layer, B, S, pos0)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with _Current(_device(q, k, v, gate, k_cache, v_cache, out, workspace, stream=stream)):
        _check(load().swa_attn_prefill_chunk(ctypes.byref(layer.c()), B, S, int(pos0), _ptr(q), _ptr(k), _ptr(v),
                                             _ptr(gate), _ptr(k_cache), _ptr(v_cache), C, _ptr(out), _ptr(workspace),
                                             nbytes, _stream(stream)))
    return out


def decode_workspace_size(layer: LayerParams, B: int, max_len: int) -> int:
    return int(load().swa_decode_workspace_size(ctypes.byref(layer.c()), B, max_len))


def attn_decode(layer: LayerParams, q, gate, k_cache, v_cache, seq_lens, max_len: int, out=None, workspace=None,
                stream=None):
    """swa_attn_decode: q [B,Hq,D] (rotated), gate [B,Hq] fp32 or None, caches
    [B,Hkv,C,D], seq_lens [B] int32 (device, counts the current token).
    Returns out [B,Hq,D] bf16."""
    B = q.shape[0]
    D = layer.head_dim
    C = k_cache.shape[2]
    _need(q, "q", torch.bfloat16, (B, layer.num_q_heads, D))
    _need(gate, "gate", torch.float32, (B, layer.num_q_heads))
    _need(k_cache, "k_cache", torch.bfloat16, (B, layer.num_kv_heads, C, D))
    _need(v_cache, "v_cache", torch.bfloat16, (B, layer.num_kv_heads, C, D))
    _need(seq_lens, "seq_lens", torch.int32, (B,))
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", torch.bfloat16, (B, layer.num_q_heads, D))
    need = decode_workspace_size(layer, B, max_len)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with _Current(_device(q, gate, k_cache, v_cache, seq_lens, out, workspace, stream=stream)):
        _check(load().swa_attn_decode(ctypes.byref(layer.c()), B, _ptr(q), _ptr(gate), _ptr(k_cache), _ptr(v_cache), C,
                                      _ptr(seq_lens), int(max_len), _ptr(out), _ptr(workspace), nbytes,
                                      _stream(stream)))
    return out


def decode_mq_workspace_size(layer: LayerParams, B: int, T: int, max_len: int) -> int:
    return int(load().swa_decode_mq_workspace_size(ctypes.byref(layer.c()), B, T, max_len))


def attn_decode_mq(layer: LayerParams, q, gate, k_new, v_new, k_cache, v_cache, seq_lens, max_len: int, out=None,
                   workspace=None, stream=None):
    """swa_attn_decode_mq: T new tokens per sequence in one call.  q [B,T,Hq,D]
    and k_new [B,T,Hkv,D] already rotated, v_new [B,T,Hkv,D], gate [B,T,Hq]
    fp32 or None; the caches [B,Hkv,C,D] hold the L - T earlier tokens only;
    seq_lens [B] int32 (device) counts the new tokens.  Returns out [B,T,Hq,D]."""
    B, T = q.shape[0], q.shape[1]
    D = layer.head_dim
    C = k_cache.shape[2]
    _need(q, "q", torch.bfloat16, (B, T, layer.num_q_heads, D))
    _need(gate, "gate", torch.float32, (B, T, layer.num_q_heads))
    _need(k_new, "k_new", torch.bfloat16, (B, T, layer.num_kv_heads, D))
    _need(v_new, "v_new", torch.bfloat16, (B, T, layer.num_kv_heads, D))
    _need(k_cache, "k_cache", torch.bfloat16, (B, layer.num_kv_heads, C, D))
    _need(v_cache, "v_cache", torch.bfloat16, (B, layer.num_kv_heads, C, D))
    _need(seq_lens, "seq_lens", torch.int32, (B,))
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", torch.bfloat16, (B, T, layer.num_q_heads, D))
    need = decode_mq_workspace_size(layer, B, T, max_len)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with _Current(_device(q, gate, k_new, v_new, k_cache, v_cache, seq_lens, out, workspace, stream=stream)):
        _check(load().swa_attn_decode_mq(ctypes.byref(layer.c()), B, T, _ptr(q), _ptr(gate), _ptr(k_new), _ptr(v_new),
                                         _ptr(k_cache), _ptr(v_cache), C, _ptr(seq_lens), int(max_len), _ptr(out),
                                         _ptr(workspace), nbytes, _stream(stream)))
    return out


def attn_decode_no_alloc(layer: LayerParams, q, gate, k_cache, v_cache, seq_lens, max_len: int, out,
                         stream=None):
    """swa_attn_decode_no_alloc: attn_decode without a workspace, for callers
    that cannot allocate device memory; the split-K partials live in a static
    device array of NO_ALLOC_SCRATCH_BYTES inside libswa.so.  `out` must be
    given (this call allocates nothing).  Calls that overlap on the GPU race
    on the shared array."""
    B = q.shape[0]
    D = layer.head_dim
    C = k_cache.shape[2]
    _need(q, "q", torch.bfloat16, (B, layer.num_q_heads, D))
    _need(gate, "gate", torch.float32, (B, layer.num_q_heads))
    _need(k_cache, "k_cache", torch.bfloat16, (B, layer.num_kv_heads, C, D))
    _need(v_cache, "v_cache", torch.bfloat16, (B, layer.num_kv_heads, C, D))
    _need(seq_lens, "seq_lens", torch.int32, (B,))
    _need(out, "out", torch.bfloat16, (B, layer.num_q_heads, D))
    with _Current(_device(q, gate, k_cache, v_cache, seq_lens, out, stream=stream)):
        _check(load().swa_attn_decode_no_alloc(ctypes.byref(layer.c()), B, _ptr(q), _ptr(gate), _ptr(k_cache),
                                               _ptr(v_cache), C, _ptr(seq_lens), int(max_len), _ptr(out),
                                               _stream(stream)))
    return out


def device_error(reset: bool = True) -> int:
    """swa_device_error: synchronise and read (optionally clear) the device
    error word; 0 means no kernel gave up on a wait."""
    code = ctypes.c_int32(0)
    _check(load().swa_device_error(ctypes.byref(code), 1 if reset else 0))
    return int(code.value)
