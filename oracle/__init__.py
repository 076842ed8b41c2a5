"""Plain fp64 CPU oracle for the KVarN hot path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it and
shares no code with it.

The arithmetic lives in ``kvarn_oracle.c`` (plain C, fp64, explicit
definitions).  This module only loads the shared object and marshals numpy
arrays.  Sources: the paper "KVarN: Variance-Normalized KV-Cache Quantization
Mitigates Error Accumulation in Reasoning Tasks" -- abstract (Hadamard
rotation, then a variance normalisation with a token scale and a channel scale for K and V,
2-bit), and the rndamp.com article, section "How It Works" items 1-2 and
section "Numbers" (the second scale fused into dequantisation).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvarn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libkvarn_oracle.so")
_lib = None

_dp = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_u8p = np.ctypeslib.ndpointer(dtype=np.uint8, flags="C_CONTIGUOUS")


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-D_GNU_SOURCE", "-ffp-contract=off", "-fno-fast-math",
             "-fPIC", "-shared", "-pthread", _SRC, "-o", _LIB_PATH, "-lm"])
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        L.kvo_hadamard_matrix.argtypes = [ctypes.c_int, _dp]
        L.kvo_rotate.argtypes = [_dp, ctypes.c_int, ctypes.c_int, _dp]
        L.kvo_normalize.argtypes = [_dp, ctypes.c_int, ctypes.c_int, ctypes.c_int, _dp, _dp]
        L.kvo_quantize_block.argtypes = [_dp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, _dp, _dp, _dp, _dp, _dp, _dp, _u8p]
        L.kvo_f16_bits.argtypes = [ctypes.c_double]
        L.kvo_f16_bits.restype = ctypes.c_uint16
        L.kvo_f16_value.argtypes = [ctypes.c_uint16]
        L.kvo_f16_value.restype = ctypes.c_double
        L.kvo_record_bytes.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int]
        L.kvo_record_bytes.restype = ctypes.c_size_t
        L.kvo_pack_record.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, _u8p, _dp, _dp, _dp,
                                      _dp, _u8p]
        L.kvo_unpack_record.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, _u8p, _u8p, _dp, _dp,
                                        _dp, _dp]
        L.kvo_dequantize_record.argtypes = [_u8p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_int, _dp]
        L.kvo_attention.argtypes = [_dp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, _dp, _dp,
                                    ctypes.c_double, _dp]
        L.kvo_quantize_many.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                                        ctypes.c_int]
        L.kvo_quantize_many.restype = ctypes.c_int
        _lib = L
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


# ---------------------------------------------------------------- rotation
def hadamard_matrix(n: int) -> np.ndarray:
    """Unnormalised Sylvester Hadamard matrix H_n (n x n)."""
    H = np.empty((n, n), dtype=np.float64)
    lib().kvo_hadamard_matrix(n, H)
    return H


def rotate(x, hb: int) -> np.ndarray:
    """Rotate every row of x (..., D): blockdiag(H_hb)/sqrt(hb) applied along the last axis."""
    x = _f64(x)
    D = x.shape[-1]
    flat = x.reshape(-1, D)
    out = np.empty_like(flat)
    for i in range(flat.shape[0]):
        row = np.ascontiguousarray(flat[i])
        o = np.empty(D, dtype=np.float64)
        lib().kvo_rotate(row, D, hb, o)
        out[i] = o
    return out.reshape(x.shape)


# ----------------------------------------------------------- normalisation
def normalize(Xrot, sweeps: int):
    """Dual-axis variance normalisation of a rotated T x D block -> (r[T], c[D])."""
    X = _f64(Xrot)
    T, D = X.shape
    r = np.empty(T, dtype=np.float64)
    c = np.empty(D, dtype=np.float64)
    lib().kvo_normalize(X, T, D, sweeps, r, c)
    return r, c


# ---------------------------------------------------------------- quantise
def quantize_block(X, hb: int, sweeps: int = 4, group: int = 32) -> dict:
    """Quantise one T x D block.  Returns dict with xrot, r, c, s, m, v, codes (all fp64 except codes)."""
    X = _f64(X)
    T, D = X.shape
    ng = D // group
    out = dict(
        xrot=np.empty((T, D)), r=np.empty(T), c=np.empty(D), s=np.empty((T, ng)), m=np.empty((T, ng)),
        v=np.empty((T, D)), codes=np.empty((T, D), dtype=np.uint8))
    lib().kvo_quantize_block(X, T, D, hb, sweeps, group, out["xrot"], out["r"], out["c"], out["s"], out["m"],
                             out["v"], out["codes"])
    return out


# --------------------------------------------------------------- binary16
def f16_bits(x: float) -> int:
    return int(lib().kvo_f16_bits(float(x)))


def f16_value(bits: int) -> float:
    return float(lib().kvo_f16_value(int(bits)))


# ------------------------------------------------------------------ records
# Code layouts of a record: NATURAL (token-major, any T), K_ORDER / V_ORDER (the
# fragment orders the library writes for K and V blocks of 128 tokens).
NATURAL, K_ORDER, V_ORDER = 0, 1, 2


def record_bytes(T: int, D: int, group: int = 32) -> int:
    return int(lib().kvo_record_bytes(T, D, group))


def pack_record(q: dict, layout: int = NATURAL, group: int = 32) -> np.ndarray:
    codes = np.ascontiguousarray(q["codes"], dtype=np.uint8)
    T, D = codes.shape
    rec = np.empty(record_bytes(T, D, group), dtype=np.uint8)
    lib().kvo_pack_record(T, D, group, layout, codes, _f64(q["r"]), _f64(q["c"]), _f64(q["s"]), _f64(q["m"]), rec)
    return rec


def unpack_record(rec, T: int, D: int, layout: int = NATURAL, group: int = 32) -> dict:
    rec = np.ascontiguousarray(rec, dtype=np.uint8)
    ng = D // group
    out = dict(codes=np.empty((T, D), dtype=np.uint8), r=np.empty(T), c=np.empty(D), s=np.empty((T, ng)),
               m=np.empty((T, ng)))
    lib().kvo_unpack_record(T, D, group, layout, rec, out["codes"], out["r"], out["c"], out["s"], out["m"])
    return out


def dequantize_record(rec, T: int, D: int, hb: int, rotated: bool = False, layout: int = NATURAL,
                      group: int = 32) -> np.ndarray:
    rec = np.ascontiguousarray(rec, dtype=np.uint8)
    out = np.empty((T, D), dtype=np.float64)
    lib().kvo_dequantize_record(rec, T, D, group, layout, hb, 1 if rotated else 0, out)
    return out


# ------------------------------------------------------ error decomposition
def magnitude_direction_errors(x, xhat) -> np.ndarray:
    """Per row of x and its reconstruction xhat (..., D): (|norm(xhat)/norm(x) - 1|, 1 - cos(xhat, x)) in fp64.

    The split the KVarN article draws ("The Problem"; "How It Works"): error in a token's magnitude versus error
    in its direction.  A zero row of x gives (0, 0); a zero xhat of a nonzero x gives (1, 1).
    """
    x = _f64(x)
    xhat = _f64(xhat)
    nx = np.sqrt(np.sum(x * x, axis=-1))
    ny = np.sqrt(np.sum(xhat * xhat, axis=-1))
    dot = np.sum(x * xhat, axis=-1)
    with np.errstate(divide="ignore", invalid="ignore"):
        mag = np.where(nx > 0, np.abs(ny / nx - 1.0), 0.0)
        dirr = np.where(nx > 0, np.where(ny > 0, 1.0 - dot / (nx * ny), 1.0), 0.0)
    return np.stack([mag, dirr], axis=-1)


def record_token_errors(x, rec, T: int, D: int, hb: int, layout: int = NATURAL) -> np.ndarray:
    """(T, 2) magnitude / direction errors of the T original rows x against their record (original basis)."""
    return magnitude_direction_errors(x, dequantize_record(rec, T, D, hb, False, layout))


# ---------------------------------------------------------------- attention
def attention(q, K, V, scale: float) -> np.ndarray:
    """q (Hq, D); K, V (Hkv, L, D) -> out (Hq, D) by explicit softmax in fp64."""
    q = _f64(q)
    K = _f64(K)
    V = _f64(V)
    Hq, D = q.shape
    Hkv, L, _ = K.shape
    out = np.empty((Hq, D), dtype=np.float64)
    lib().kvo_attention(q, Hq, Hkv, D, L, K, V, float(scale), out)
    return out


def decode_from_cache(q, k_records, v_records, k_tail, v_tail, n_tokens: int, T: int, hb: int,
                      scale: float, group: int = 32, layouts=None) -> np.ndarray:
    """Decode attention for one sequence from packed records plus the residual tail.

    q (Hq, D); k_records/v_records (Hkv, nblk_capacity, record_bytes) uint8; k_tail/v_tail (Hkv, T, D) values
    as stored (any float dtype, widened exactly).  The first n_tokens // T blocks are dequantised to the
    original basis, followed by n_tokens % T tail tokens; then explicit softmax attention.  layouts =
    (K layout, V layout); by default the library's K_ORDER / V_ORDER for T = 128, NATURAL otherwise.
    """
    if layouts is None:
        layouts = (K_ORDER, V_ORDER) if T == 128 else (NATURAL, NATURAL)
    q = _f64(q)
    Hq, D = q.shape
    Hkv = k_records.shape[0]
    nblk, ntail = n_tokens // T, n_tokens % T
    K = np.empty((Hkv, n_tokens, D))
    V = np.empty((Hkv, n_tokens, D))
    for h in range(Hkv):
        for b in range(nblk):
            K[h, b * T:(b + 1) * T] = dequantize_record(k_records[h, b], T, D, hb, False, layouts[0], group)
            V[h, b * T:(b + 1) * T] = dequantize_record(v_records[h, b], T, D, hb, False, layouts[1], group)
        K[h, nblk * T:] = np.asarray(k_tail[h, :ntail], dtype=np.float64)
        V[h, nblk * T:] = np.asarray(v_tail[h, :ntail], dtype=np.float64)
    return attention(q, K, V, scale)


def decode_multi_from_cache(q, k_records, v_records, k_tail, v_tail, n_tokens: int, T: int, hb: int,
                            scale: float, group: int = 32, layouts=None) -> np.ndarray:
    """Decode for the last Q tokens of one sequence at once: q (Q, Hq, D) -> out (Q, Hq, D).

    The cache holds n_tokens tokens (blocks dequantised to the original basis, then the tail as stored); query i
    sits at position n_tokens - Q + i and attends positions 0 .. n_tokens - Q + i (causal), by explicit softmax.
    A query before position 0 gets zeros.
    """
    if layouts is None:
        layouts = (K_ORDER, V_ORDER) if T == 128 else (NATURAL, NATURAL)
    q = _f64(q)
    Q, Hq, D = q.shape
    Hkv = k_records.shape[0]
    nblk, ntail = n_tokens // T, n_tokens % T
    K = np.empty((Hkv, n_tokens, D))
    V = np.empty((Hkv, n_tokens, D))
    for h in range(Hkv):
        for b in range(nblk):
            K[h, b * T:(b + 1) * T] = dequantize_record(k_records[h, b], T, D, hb, False, layouts[0], group)
            V[h, b * T:(b + 1) * T] = dequantize_record(v_records[h, b], T, D, hb, False, layouts[1], group)
        K[h, nblk * T:] = np.asarray(k_tail[h, :ntail], dtype=np.float64)
        V[h, nblk * T:] = np.asarray(v_tail[h, :ntail], dtype=np.float64)
    out = np.zeros((Q, Hq, D))
    for i in range(Q):
        visible = n_tokens - Q + i + 1
        if visible > 0:
            out[i] = attention(q[i], K[:, :visible], V[:, :visible], scale)
    return out


# ------------------------------------------------------------ bulk, threads
def quantize_many(x: np.ndarray, dtype: str, T: int, D: int, hb: int, sweeps: int = 4, group: int = 32,
                  nthreads: int = 1, layout: int = NATURAL):
    """Quantise consecutive T x D blocks of a raw fp32 / bf16 (as uint16) array on nthreads threads.

    Returns (records uint8 [nunits, record_bytes], threads used).
    """
    x = np.ascontiguousarray(x)
    code = {"f32": 0, "bf16": 1}[dtype]
    nunits = x.size // (T * D)
    rb = record_bytes(T, D, group)
    recs = np.empty((nunits, rb), dtype=np.uint8)
    used = lib().kvo_quantize_many(x.ctypes.data, code, nunits, T, D, hb, sweeps, group, layout,
                                   recs.ctypes.data, nthreads)
    return recs, used
