"""Helpers for the GPU-vs-oracle parity tests: parse record bytes with numpy and apply the
parity contract.

Contract (codes, scales, decode):
  * codes bit-exact, except elements whose oracle pre-rounding level v lies within 1e-5 of a
    rounding boundary k + 1/2; those are counted and must still be one of the two adjacent codes;
  * unrounded fp32 r_t, c_d, s, m within 1e-5 relative of the oracle's fp64 values;
  * stored binary16 scales equal to the binary16 rounding of the oracle value, except where that
    value lies within 1e-5 relative of a binary16 rounding midpoint (counted);
  * decode output within 2e-3 max-abs of the oracle's result on the same dequantised cache.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

WINDOW = 1e-5
SCALE_RTOL = 1e-5
DECODE_ATOL = 2e-3


def code_bit_index(T: int, D: int, layout: int) -> np.ndarray:
    """Bit index of each (token, channel) code inside the code area, from the record format in kvarn.h."""
    t = np.arange(T)[:, None]
    d = np.arange(D)[None, :]
    if layout == oracle.NATURAL:
        return (t * D // 4 + d // 4) * 8 + 2 * (d % 4)
    if layout == oracle.K_ORDER:
        F = D // 64
        u, n, lane, half, q = t // 16, (t % 16) // 8, 4 * (t % 8) + (d % 8) // 2, d % 2, d // 8
        word = np.where(q < 8 * F, n * F + q // 8, 2 * F)
        pos = np.where(q < 8 * F, q % 8, q - 8 * F + 4 * n)
        return ((u * 32 + lane) * (D // 32) + word) * 32 + 16 * half + 2 * pos
    j, lane, half, a = d // 8, 4 * (d % 8) + (t % 8) // 2, t % 2, (t % 32) // 8
    word, pos = a // 2, 4 * (a % 2) + t // 32
    return ((j * 32 + lane) * 2 + word) * 32 + 16 * half + 2 * pos


def view_record(rec, T: int, D: int, layout: int, G: int = 32) -> dict:
    rec = np.ascontiguousarray(np.asarray(rec, dtype=np.uint8))
    nc, ng = T * D // 4, D // G
    bits = code_bit_index(T, D, layout)
    codes = (rec[bits // 8] >> (bits % 8)) & 3
    so = nc
    mo = so + T * ng * 2
    ro = mo + T * ng * 2
    s = rec[so:mo].view(np.float16).reshape(T, ng)
    m = rec[mo:ro].view(np.float16).reshape(T, ng)
    r = rec[ro:ro + 2 * T].view(np.float16)
    c = rec[ro + 2 * T:ro + 2 * T + 2 * D].view(np.float16)
    pad = rec[ro + 2 * T + 2 * D:]
    return dict(codes=codes.astype(np.uint8), s=s.copy(), m=m.copy(), r=r.copy(), c=c.copy(), pad=pad.copy())


def near_f16_midpoint(x, window: float = None) -> np.ndarray:
    """True where x lies within `window` (default 1e-5) relative of a binary16 rounding midpoint."""
    window = WINDOW if window is None else window
    x = np.asarray(x, dtype=np.float64)
    h = x.astype(np.float16)
    bits = h.view(np.uint16).astype(np.int32)
    out = np.zeros(x.shape, dtype=bool)
    for step in (-1, 1):
        nb = np.clip(bits + step * np.where(x < 0, -1, 1), 0, 0xFFFF).astype(np.uint16)
        nbv = nb.view(np.float16).astype(np.float64)
        mid = 0.5 * (h.astype(np.float64) + nbv)
        out |= np.abs(x - mid) <= window * np.abs(x)
    return out


def near_boundary(v, s, window: float = None) -> np.ndarray:
    window = WINDOW if window is None else window
    frac = np.asarray(v) - np.floor(v)
    return (np.abs(frac - 0.5) < window) & (np.repeat(np.asarray(s), np.asarray(v).shape[-1] // np.asarray(s).shape[-1],
                                                       axis=-1) > 0)


def check_block(rec, dbg: dict | None, oq: dict, T: int, D: int, layout: int, rtol: float = None,
                window: float = None) -> dict:
    """Compare one GPU record (+ optional fp32 debug scales) against an oracle quantize_block result.

    rtol (scales) and window (codes, binary16 midpoints) default to the contract's 1e-5; a looser value is only
    for blocks whose scales are ill-conditioned in fp32, with the reason stated where it is used."""
    rtol = SCALE_RTOL if rtol is None else rtol
    window = WINDOW if window is None else window
    g = view_record(rec, T, D, layout)
    stats = dict(elements=T * D, boundary=0, code_flips=0, f16_flips=0, max_rel=0.0)
    # codes
    nb = near_boundary(oq["v"], oq["s"], window)
    mism = g["codes"] != oq["codes"]
    bad = mism & ~nb
    assert not bad.any(), f"{int(bad.sum())} code mismatches outside the rounding window, e.g. at " \
                          f"{np.argwhere(bad)[:5].tolist()} v={oq['v'][bad][:5]}"
    assert np.all(np.abs(g["codes"].astype(int) - oq["codes"].astype(int)) <= 1)
    stats["boundary"] = int(nb.sum())
    stats["code_flips"] = int(mism.sum())
    # unrounded fp32 scales
    if dbg is not None:
        for key in ("r", "c", "s", "m"):
            o = np.asarray(oq[key], dtype=np.float64)
            gv = np.asarray(dbg[key], dtype=np.float64).reshape(o.shape)
            err = np.abs(gv - o)
            tol = rtol * np.abs(o)
            ok = (err <= tol) | ((o == 0) & (err == 0))
            nzo = o != 0
            if nzo.any():
                stats["max_rel"] = max(stats["max_rel"], float(np.max(err[nzo] / np.abs(o[nzo]))))
            assert ok.all(), f"{key}: max rel err {np.max(err / np.maximum(np.abs(o), 1e-300)):.3e}"
    # stored binary16 scales
    for key in ("r", "c", "s", "m"):
        o = np.asarray(oq[key], dtype=np.float64)
        expect = o.astype(np.float16)
        got = g[key].reshape(o.shape)
        diff = expect.view(np.uint16) != got.view(np.uint16)
        near = near_f16_midpoint(o, max(window, rtol))
        assert not (diff & ~near).any(), f"binary16 {key} differs away from a midpoint at " \
                                         f"{np.argwhere(diff & ~near)[:5].tolist()}"
        stats["f16_flips"] += int(diff.sum())
    assert np.all(g["pad"] == 0)
    return stats


def oracle_records(x: np.ndarray, hb: int, sweeps: int = 4, layout: int = oracle.K_ORDER):
    """Oracle quantisation of x [..., nblk*T, D] (float64) -> (records [..., nblk, rb], list of dicts)."""
    T = 128
    *lead, L, D = x.shape
    nb = L // T
    flat = x.reshape(-1, L, D)
    recs = np.zeros((flat.shape[0], nb, oracle.record_bytes(T, D)), dtype=np.uint8)
    qs = []
    for i in range(flat.shape[0]):
        for b in range(nb):
            q = oracle.quantize_block(flat[i, b * T:(b + 1) * T], hb, sweeps)
            recs[i, b] = oracle.pack_record(q, layout)
            qs.append(q)
    return recs.reshape(*lead, nb, -1), qs


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()
