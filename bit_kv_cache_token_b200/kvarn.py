"""Thin ctypes binding of libkvarn.so (the C ABI declared in include/kvarn.h).

Argument marshalling only: every step of the quantiser and of decode
attention runs in the CUDA kernels behind the C ABI.  PyTorch supplies device
memory and the current stream.  If the library is missing this module raises;
there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvarn.so")

KVARN_OK = 0
KVARN_EINVAL = -1
KVARN_EUNSUPPORTED = -2
KVARN_EWORKSPACE = -3
KVARN_ECUDA = -4
KVARN_STATUS_CAPACITY = 1
KVARN_STATUS_NONFINITE = 2
KVARN_STATUS_LENGTH = 4
KVARN_STATUS_TIMEOUT = 8
KVARN_F32 = 0
KVARN_BF16 = 1

# every extern "C" symbol declared in include/kvarn.h
EXPORTED = (
    "kvarn_record_bytes", "kvarn_cache_bytes", "kvarn_decode_workspace_bytes", "kvarn_quantize_blocks",
    "kvarn_append_token", "kvarn_decode_attention", "kvarn_dequantize", "kvarn_strerror",
    "kvarn_decode_attention_noalloc", "kvarn_token_errors", "kvarn_decode_attention_multi",
    "kvarn_decode_selftest_timeout",
)


class KvarnError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {strerror(code)} ({code})")
        self.code = code


class kvarn_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "num_seqs", "num_kv_heads", "head_dim", "block_tokens", "group", "hadamard", "sweeps", "max_blocks",
        "dtype")]


class kvarn_cache(ctypes.Structure):
    _fields_ = [("k_records", ctypes.c_void_p), ("v_records", ctypes.c_void_p), ("k_tail", ctypes.c_void_p),
                ("v_tail", ctypes.c_void_p), ("n_tokens", ctypes.c_void_p), ("arrive", ctypes.c_void_p),
                ("status", ctypes.c_void_p)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libkvarn.so; raise if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m bit_kv_cache_token_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, S, F, V = ctypes.POINTER, ctypes.c_int, ctypes.c_size_t, ctypes.c_float, ctypes.c_void_p
        L.kvarn_record_bytes.argtypes = [P(kvarn_config)]
        L.kvarn_record_bytes.restype = S
        L.kvarn_cache_bytes.argtypes = [P(kvarn_config), I]
        L.kvarn_cache_bytes.restype = S
        L.kvarn_decode_workspace_bytes.argtypes = [P(kvarn_config), I]
        L.kvarn_decode_workspace_bytes.restype = S
        L.kvarn_quantize_blocks.argtypes = [P(kvarn_config), V, V, I, I, P(kvarn_cache), V, V, V]
        L.kvarn_append_token.argtypes = [P(kvarn_config), V, V, P(kvarn_cache), V]
        L.kvarn_decode_attention.argtypes = [P(kvarn_config), V, I, F, P(kvarn_cache), I, V, V, S, V]
        L.kvarn_dequantize.argtypes = [P(kvarn_config), P(kvarn_cache), I, I, I, V, V, V]
        L.kvarn_decode_attention_noalloc.argtypes = [P(kvarn_config), V, I, F, P(kvarn_cache), I, V, V]
        L.kvarn_token_errors.argtypes = [P(kvarn_config), V, V, I, I, P(kvarn_cache), V, V, V]
        L.kvarn_decode_attention_multi.argtypes = [P(kvarn_config), V, I, I, F, P(kvarn_cache), I, V, V, S, V]
        L.kvarn_decode_selftest_timeout.argtypes = [P(kvarn_config), V, I, P(kvarn_cache), I, V, V, S, V]
        L.kvarn_strerror.argtypes = [I]
        L.kvarn_strerror.restype = ctypes.c_char_p
        for name in ("kvarn_quantize_blocks", "kvarn_append_token", "kvarn_decode_attention", "kvarn_dequantize",
                     "kvarn_decode_attention_noalloc"):
            getattr(L, name).restype = I
        _lib = L
    return _lib


def strerror(code: int) -> str:
    return lib().kvarn_strerror(int(code)).decode()


def _check(rc: int, where: str):
    if rc != KVARN_OK:
        raise KvarnError(rc, where)


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _torch_dtype(code: int):
    return torch.bfloat16 if code == KVARN_BF16 else torch.float32


@dataclass
class Config:
    """Python mirror of kvarn_config (defaults: 128-token blocks, group 32, 4 sweeps)."""
    num_seqs: int
    num_kv_heads: int
    head_dim: int
    max_blocks: int
    hadamard: int = -1  # -1: head_dim, or 32 when head_dim is not a power of two
    sweeps: int = 4
    dtype: int = KVARN_BF16
    block_tokens: int = 128
    group: int = 32

    def c(self) -> kvarn_config:
        hb = self.hadamard
        if hb < 0:
            hb = self.head_dim if (self.head_dim & (self.head_dim - 1)) == 0 else 32
        return kvarn_config(self.num_seqs, self.num_kv_heads, self.head_dim, self.block_tokens, self.group, hb,
                            self.sweeps, self.max_blocks, self.dtype)

    @property
    def hb(self) -> int:
        return self.c().hadamard

    @property
    def torch_dtype(self):
        return _torch_dtype(self.dtype)


def record_bytes(cfg: Config) -> int:
    c = cfg.c()
    return int(lib().kvarn_record_bytes(ctypes.byref(c)))


def cache_bytes(cfg: Config, part: int) -> int:
    c = cfg.c()
    return int(lib().kvarn_cache_bytes(ctypes.byref(c), int(part)))


def decode_workspace_bytes(cfg: Config, num_q_heads: int) -> int:
    c = cfg.c()
    return int(lib().kvarn_decode_workspace_bytes(ctypes.byref(c), int(num_q_heads)))


class KVCache:
    """Device buffers of one layer's cache, allocated with torch (caller-owned, as the C ABI expects)."""

    def __init__(self, cfg: Config, device="cuda"):
        self.cfg = cfg
        S, H, D, T = cfg.num_seqs, cfg.num_kv_heads, cfg.head_dim, cfg.block_tokens
        rb = record_bytes(cfg)
        if rb == 0:
            raise KvarnError(KVARN_EINVAL, "kvarn_record_bytes")
        self.k_records = torch.zeros(S, H, cfg.max_blocks, rb, dtype=torch.uint8, device=device)
        self.v_records = torch.zeros_like(self.k_records)
        self.k_tail = torch.zeros(S, H, T, D, dtype=cfg.torch_dtype, device=device)
        self.v_tail = torch.zeros_like(self.k_tail)
        self.n_tokens = torch.zeros(S, dtype=torch.int32, device=device)
        self.arrive = torch.zeros(S, dtype=torch.int32, device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)

    def struct(self) -> kvarn_cache:
        return kvarn_cache(*(ctypes.c_void_p(t.data_ptr()) for t in (
            self.k_records, self.v_records, self.k_tail, self.v_tail, self.n_tokens, self.arrive, self.status)))


def _need(t, name, dtype=None, shape=None):
    """The C ABI takes bare pointers: dtype, shape and layout are checked here, before any launch
    (the device is checked last, by _on_device, once every shape is known to be right)."""
    if t is None:
        raise ValueError(f"{name} is required")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _on_device(**tensors):
    """Every tensor must live on the current CUDA device: the library launches on the current device (its
    stream, its SM count, and for the no-alloc decode its own copy of the static workspace)."""
    cur = None
    for name, t in tensors.items():
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if cur is None:
            cur = torch.cuda.current_device()
        if t.device.index != cur:
            raise ValueError(f"{name} is on cuda:{t.device.index} but the current device is cuda:{cur}; "
                             f"call inside torch.cuda.device({t.device.index})")


def _need_cache(cfg: Config, cache: KVCache):
    """The cache's buffers must have the sizes cfg implies (the kernels index them from cfg)."""
    S, H, D, T = cfg.num_seqs, cfg.num_kv_heads, cfg.head_dim, cfg.block_tokens
    rec = (S, H, cfg.max_blocks, record_bytes(cfg))
    for name in ("k_records", "v_records"):
        _need(getattr(cache, name), f"cache.{name}", torch.uint8, rec)
    for name in ("k_tail", "v_tail"):
        _need(getattr(cache, name), f"cache.{name}", cfg.torch_dtype, (S, H, T, D))
    for name in ("n_tokens", "arrive"):
        _need(getattr(cache, name), f"cache.{name}", torch.int32, (S,))
    _need(cache.status, "cache.status", torch.int32, (1,))


def quantize_blocks(cfg: Config, k, v, cache: KVCache, first_block: int = 0, debug: bool = False, stream=None):
    """kvarn_quantize_blocks: k, v [S, Hkv, T, D] -> records (+ tail).  Returns (debug_k, debug_v) if debug."""
    if k is None or k.dim() != 4:
        raise ValueError("k must be a 4-d tensor [S, Hkv, T, D]")
    T = k.shape[2]
    _need(k, "k", cfg.torch_dtype, (cfg.num_seqs, cfg.num_kv_heads, T, cfg.head_dim))
    _need(v, "v", cfg.torch_dtype, k.shape)
    _need_cache(cfg, cache)
    _on_device(k=k, v=v, cache=cache.k_records)
    dk = dv = None
    if debug:
        nb = T // cfg.block_tokens
        per = cfg.block_tokens + cfg.head_dim + 2 * cfg.block_tokens * (cfg.head_dim // cfg.group)
        dk = torch.empty(cfg.num_seqs * cfg.num_kv_heads * nb * per + 4, dtype=torch.float32, device=k.device)
        dv = torch.empty_like(dk)
    c, cs = cfg.c(), cache.struct()
    _check(lib().kvarn_quantize_blocks(ctypes.byref(c), _ptr(k), _ptr(v), int(T), int(first_block), ctypes.byref(cs),
                                       _ptr(dk), _ptr(dv), _stream(stream)), "kvarn_quantize_blocks")
    return (dk, dv) if debug else None


def append_token(cfg: Config, k, v, cache: KVCache, stream=None):
    """kvarn_append_token: k, v [S, Hkv, D]."""
    _need(k, "k", cfg.torch_dtype, (cfg.num_seqs, cfg.num_kv_heads, cfg.head_dim))
    _need(v, "v", cfg.torch_dtype, k.shape)
    _need_cache(cfg, cache)
    _on_device(k=k, v=v, cache=cache.k_records)
    c, cs = cfg.c(), cache.struct()
    _check(lib().kvarn_append_token(ctypes.byref(c), _ptr(k), _ptr(v), ctypes.byref(cs), _stream(stream)),
           "kvarn_append_token")


def decode_workspace(cfg: Config, num_q_heads: int, device="cuda"):
    nbytes = decode_workspace_bytes(cfg, num_q_heads)
    if nbytes == 0:
        raise KvarnError(KVARN_EINVAL, "kvarn_decode_workspace_bytes")
    return torch.zeros(nbytes, dtype=torch.uint8, device=device)


def decode_attention(cfg: Config, q, cache: KVCache, max_tokens: int, out=None, workspace=None,
                     softmax_scale: float = 0.0, stream=None):
    """kvarn_decode_attention: q [S, Hq, D] -> out [S, Hq, D] fp32."""
    if q is None or q.dim() != 3:
        raise ValueError("q must be a 3-d tensor [S, Hq, D]")
    Hq = q.shape[1]
    _need(q, "q", cfg.torch_dtype, (cfg.num_seqs, Hq, cfg.head_dim))
    _need_cache(cfg, cache)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    _need(out, "out", torch.float32, q.shape)
    _on_device(q=q, out=out, cache=cache.k_records, workspace=workspace)
    if workspace is None:
        workspace = decode_workspace(cfg, Hq, q.device)
    c, cs = cfg.c(), cache.struct()
    _check(lib().kvarn_decode_attention(ctypes.byref(c), _ptr(q), int(Hq), float(softmax_scale), ctypes.byref(cs),
                                        int(max_tokens), _ptr(out), _ptr(workspace), int(workspace.numel() * workspace.element_size()),
                                        _stream(stream)), "kvarn_decode_attention")
    return out


def decode_attention_noalloc(cfg: Config, q, cache: KVCache, max_tokens: int, out, softmax_scale: float = 0.0,
                             stream=None):
    """kvarn_decode_attention_noalloc: like decode_attention, with the library's own static workspace.

    `out` must be given (this path allocates nothing); calls that overlap on the GPU race."""
    if q is None or q.dim() != 3:
        raise ValueError("q must be a 3-d tensor [S, Hq, D]")
    _need(q, "q", cfg.torch_dtype, (cfg.num_seqs, q.shape[1], cfg.head_dim))
    _need(out, "out", torch.float32, q.shape)
    _need_cache(cfg, cache)
    _on_device(q=q, out=out, cache=cache.k_records)
    c, cs = cfg.c(), cache.struct()
    _check(lib().kvarn_decode_attention_noalloc(ctypes.byref(c), _ptr(q), int(q.shape[1]), float(softmax_scale),
                                                ctypes.byref(cs), int(max_tokens), _ptr(out), _stream(stream)),
           "kvarn_decode_attention_noalloc")
    return out


def decode_attention_multi(cfg: Config, q, cache: KVCache, max_tokens: int, out=None, workspace=None,
                           softmax_scale: float = 0.0, stream=None):
    """kvarn_decode_attention_multi: q [S, Q, Hq, D] (the last Q tokens of each sequence) -> out fp32, same shape."""
    if q is None or q.dim() != 4:
        raise ValueError("q must be a 4-d tensor [S, Q, Hq, D]")
    S, Q, Hq, D = q.shape
    _need(q, "q", cfg.torch_dtype, (cfg.num_seqs, Q, Hq, cfg.head_dim))
    _need_cache(cfg, cache)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    _need(out, "out", torch.float32, q.shape)
    _on_device(q=q, out=out, cache=cache.k_records, workspace=workspace)
    if workspace is None:
        workspace = decode_workspace(cfg, Q * Hq, q.device)
    c, cs = cfg.c(), cache.struct()
    _check(lib().kvarn_decode_attention_multi(ctypes.byref(c), _ptr(q), int(Hq), int(Q), float(softmax_scale),
                                              ctypes.byref(cs), int(max_tokens), _ptr(out), _ptr(workspace),
                                              int(workspace.numel() * workspace.element_size()), _stream(stream)),
           "kvarn_decode_attention_multi")
    return out


def decode_selftest_timeout(cfg: Config, q, cache: KVCache, max_tokens: int, stream=None):
    """kvarn_decode_selftest_timeout: decode with every first K copy withheld and 1 ms waits; returns the output
    (not meaningful) -- the caller checks KVARN_STATUS_TIMEOUT in cache.status."""
    if q is None or q.dim() != 3:
        raise ValueError("q must be a 3-d tensor [S, Hq, D]")
    Hq = q.shape[1]
    _need(q, "q", cfg.torch_dtype, (cfg.num_seqs, Hq, cfg.head_dim))
    _need_cache(cfg, cache)
    _on_device(q=q, cache=cache.k_records)
    out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    workspace = decode_workspace(cfg, Hq, q.device)
    c, cs = cfg.c(), cache.struct()
    _check(lib().kvarn_decode_selftest_timeout(ctypes.byref(c), _ptr(q), int(Hq), ctypes.byref(cs), int(max_tokens),
                                               _ptr(out), _ptr(workspace), int(workspace.numel() * workspace.element_size()), _stream(stream)),
           "kvarn_decode_selftest_timeout")
    return out


def token_errors(cfg: Config, k, v, cache: KVCache, first_block: int = 0, stream=None):
    """kvarn_token_errors -> (err_k, err_v) fp32 [S, Hkv, T_total, 2]: per token (|‖x^‖/‖x‖ - 1|, 1 - cos)
    of the records from first_block on against the original rows k, v [S, Hkv, T_total, D]."""
    if k is None or k.dim() != 4:
        raise ValueError("k must be a 4-d tensor [S, Hkv, T, D]")
    n = k.shape[2]
    _need(k, "k", cfg.torch_dtype, (cfg.num_seqs, cfg.num_kv_heads, n, cfg.head_dim))
    _need(v, "v", cfg.torch_dtype, k.shape)
    _need_cache(cfg, cache)
    _on_device(k=k, v=v, cache=cache.k_records)
    ek = torch.empty(k.shape[0], k.shape[1], n, 2, dtype=torch.float32, device=k.device)
    ev = torch.empty_like(ek)
    c, cs = cfg.c(), cache.struct()
    _check(lib().kvarn_token_errors(ctypes.byref(c), _ptr(k), _ptr(v), int(n), int(first_block), ctypes.byref(cs),
                                    _ptr(ek), _ptr(ev), _stream(stream)), "kvarn_token_errors")
    return ek, ev


def dequantize(cfg: Config, cache: KVCache, first_block: int, num_blocks: int, rotated: bool = False, stream=None):
    """kvarn_dequantize -> (k_out, v_out) fp32 [S, Hkv, num_blocks*T, D]."""
    _need_cache(cfg, cache)
    _on_device(cache=cache.k_records)
    shape = (cfg.num_seqs, cfg.num_kv_heads, num_blocks * cfg.block_tokens, cfg.head_dim)
    ko = torch.empty(shape, dtype=torch.float32, device=cache.k_records.device)
    vo = torch.empty_like(ko)
    c, cs = cfg.c(), cache.struct()
    _check(lib().kvarn_dequantize(ctypes.byref(c), ctypes.byref(cs), int(first_block), int(num_blocks),
                                  1 if rotated else 0, _ptr(ko), _ptr(vo), _stream(stream)), "kvarn_dequantize")
    return ko, vo


def debug_split(cfg: Config, dbg, num_blocks_total: int):
    """View a debug buffer as dict(r [B,T], c [B,D], s [B,T,D/G], m [B,T,D/G]) over B = S*Hkv*nb blocks."""
    T, D, NG = cfg.block_tokens, cfg.head_dim, cfg.head_dim // cfg.group
    per = T + D + 2 * T * NG
    a = dbg[: num_blocks_total * per].view(num_blocks_total, per)
    return dict(r=a[:, :T], c=a[:, T:T + D], s=a[:, T + D:T + D + T * NG].reshape(-1, T, NG),
                m=a[:, T + D + T * NG:].reshape(-1, T, NG))
