"""Host-side checks of the C ABI: the library loads, exports what include/kvarn.h declares, sizes are
right and malformed arguments are rejected before anything is launched (no GPU needed)."""
import ctypes
import os
import re

import pytest

from bit_kv_cache_token_b200 import kvarn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "kvarn.h")).read()
    return sorted(set(re.findall(r"KVARN_API\s+[\w\s\*]*?\b(kvarn_\w+)\s*\(", src)))


def test_header_declares_what_binding_lists():
    assert _declared() == sorted(kvarn.EXPORTED)


def test_library_exports_every_declared_symbol():
    L = kvarn.lib()
    for name in _declared():
        assert hasattr(L, name), name


@pytest.mark.parametrize("D,raw", [(64, 2048 + 1024 + 256 + 128), (96, 3072 + 1536 + 256 + 192),
                                   (128, 4096 + 2048 + 256 + 256)])
def test_record_bytes(D, raw):
    cfg = kvarn.Config(2, 3, D, 5)
    rb = kvarn.record_bytes(cfg)
    assert rb == (raw + 127) // 128 * 128
    assert kvarn.cache_bytes(cfg, 0) == 2 * 3 * 5 * rb
    assert kvarn.cache_bytes(cfg, 1) == 2 * 3 * 128 * D * 2
    assert kvarn.cache_bytes(cfg, 2) == 8 and kvarn.cache_bytes(cfg, 3) == 8 and kvarn.cache_bytes(cfg, 4) == 4
    assert kvarn.cache_bytes(cfg, 9) == 0


def test_workspace_bytes():
    cfg = kvarn.Config(8, 8, 128, 256)
    ws = kvarn.decode_workspace_bytes(cfg, 32)
    # tickets (64 units, padded to 256 B) + one partial per (warp, unit) segment, at most 148 SMs x 12 warps
    # + 64, + four tail-slot partials per unit; a partial is 4 heads x (m, l, pad, pad, o[128]) fp32.  Without a
    # GPU the library assumes 148 SMs.
    assert ws == 256 + (148 * 12 + 64 + 4 * 64) * 4 * 132 * 4
    assert kvarn.decode_workspace_bytes(cfg, 12) == 0  # not a multiple of the kv heads


def test_strerror_covers_codes():
    for code in (0, -1, -2, -3, -4):
        assert kvarn.strerror(code)
    assert "unknown" in kvarn.strerror(17)


def _call_quant(cfg: kvarn.kvarn_config, cache=None, k=16, v=16, T=128, first=0):
    cs = cache if cache is not None else kvarn.kvarn_cache(16, 32, 48, 64, 80, 96, 112)
    return kvarn.lib().kvarn_quantize_blocks(ctypes.byref(cfg), ctypes.c_void_p(k), ctypes.c_void_p(v), T, first,
                                             ctypes.byref(cs), None, None, None)


@pytest.mark.parametrize("field,value,code", [
    ("head_dim", 160, kvarn.KVARN_EUNSUPPORTED), ("head_dim", 100, kvarn.KVARN_EINVAL),
    ("block_tokens", 64, kvarn.KVARN_EUNSUPPORTED), ("group", 16, kvarn.KVARN_EUNSUPPORTED),
    ("group", 48, kvarn.KVARN_EINVAL), ("hadamard", 16, kvarn.KVARN_EUNSUPPORTED),
    ("hadamard", 48, kvarn.KVARN_EINVAL), ("hadamard", 256, kvarn.KVARN_EINVAL),
    ("sweeps", -1, kvarn.KVARN_EINVAL), ("sweeps", 17, kvarn.KVARN_EINVAL), ("dtype", 7, kvarn.KVARN_EINVAL),
    ("num_seqs", 0, kvarn.KVARN_EINVAL), ("num_kv_heads", 0, kvarn.KVARN_EINVAL), ("max_blocks", -1, kvarn.KVARN_EINVAL),
])
def test_bad_config_rejected_on_host(field, value, code):
    cfg = kvarn.Config(1, 1, 128, 4, hadamard=32).c()
    setattr(cfg, field, value)
    assert _call_quant(cfg) == code


def test_bad_pointers_and_sizes_rejected_on_host():
    cfg = kvarn.Config(1, 1, 128, 4).c()
    assert _call_quant(cfg, k=0) == kvarn.KVARN_EINVAL              # null input
    assert _call_quant(cfg, k=24) == kvarn.KVARN_EINVAL             # misaligned input
    assert _call_quant(cfg, T=-1) == kvarn.KVARN_EINVAL
    assert _call_quant(cfg, T=5 * 128) == kvarn.KVARN_EINVAL        # more blocks than max_blocks
    assert _call_quant(cfg, T=2 * 128, first=3) == kvarn.KVARN_EINVAL
    bad = kvarn.kvarn_cache(16, 32, 48, 64, 0, 96, 112)             # n_tokens missing
    assert _call_quant(cfg, cache=bad) == kvarn.KVARN_EINVAL
    bad = kvarn.kvarn_cache(17, 32, 48, 64, 80, 96, 112)            # misaligned records
    assert _call_quant(cfg, cache=bad) == kvarn.KVARN_EINVAL


def test_append_needs_arrival_counters():
    cfg = kvarn.Config(1, 1, 128, 4).c()
    cs = kvarn.kvarn_cache(16, 32, 48, 64, 80, 0, 112)
    rc = kvarn.lib().kvarn_append_token(ctypes.byref(cfg), ctypes.c_void_p(16), ctypes.c_void_p(32), ctypes.byref(cs),
                                        None)
    assert rc == kvarn.KVARN_EINVAL


def _call_decode(cfg, Hq=4, max_tokens=100, ws=256, ws_bytes=10 ** 9, scale=0.0, q=16, out=32):
    cs = kvarn.kvarn_cache(16, 32, 48, 64, 80, 96, 112)
    return kvarn.lib().kvarn_decode_attention(ctypes.byref(cfg), ctypes.c_void_p(q), Hq, scale, ctypes.byref(cs),
                                              max_tokens, ctypes.c_void_p(out), ctypes.c_void_p(ws), ws_bytes, None)


def test_decode_argument_errors():
    cfg = kvarn.Config(1, 2, 128, 4).c()
    assert _call_decode(cfg, Hq=3) == kvarn.KVARN_EINVAL             # not a multiple of Hkv
    assert _call_decode(cfg, Hq=6) == kvarn.KVARN_EUNSUPPORTED       # GQA 3
    assert _call_decode(cfg, Hq=32) == kvarn.KVARN_EUNSUPPORTED      # GQA 16
    assert _call_decode(cfg, max_tokens=4 * 128 + 128) == kvarn.KVARN_EINVAL  # beyond capacity
    assert _call_decode(cfg, ws_bytes=100) == kvarn.KVARN_EWORKSPACE
    assert _call_decode(cfg, ws=0) == kvarn.KVARN_EWORKSPACE
    assert _call_decode(cfg, q=0) == kvarn.KVARN_EINVAL
    assert _call_decode(cfg, scale=float("nan")) == kvarn.KVARN_EINVAL


def test_dequantize_range_checked():
    cfg = kvarn.Config(1, 1, 128, 4).c()
    cs = kvarn.kvarn_cache(16, 32, 48, 64, 80, 96, 112)
    L = kvarn.lib()
    assert L.kvarn_dequantize(ctypes.byref(cfg), ctypes.byref(cs), 3, 2, 0, None, None, None) == kvarn.KVARN_EINVAL
    assert L.kvarn_dequantize(ctypes.byref(cfg), ctypes.byref(cs), -1, 1, 0, None, None, None) == kvarn.KVARN_EINVAL


def test_grid_overflow_rejected_on_host():
    """One CTA per (sequence, kv head, block): a call whose grid would not fit an int is refused."""
    cfg = kvarn.Config(1 << 12, 1 << 12, 128, 1 << 20).c()  # 2^24 units
    assert _call_quant(cfg, T=128 * 127) == kvarn.KVARN_EINVAL   # 2^24 x 128 CTAs
    cs = kvarn.kvarn_cache(16, 32, 48, 64, 80, 96, 112)
    L = kvarn.lib()
    assert L.kvarn_dequantize(ctypes.byref(cfg), ctypes.byref(cs), 0, 128, 0, None, None, None) == kvarn.KVARN_EINVAL
    assert L.kvarn_token_errors(ctypes.byref(cfg), ctypes.c_void_p(16), ctypes.c_void_p(32), 128 * 128, 0,
                                ctypes.byref(cs), ctypes.c_void_p(48), ctypes.c_void_p(64), None) == kvarn.KVARN_EINVAL


def test_binding_checks_shapes_before_launch():
    """The binding refuses tensors whose shape, dtype or cache sizes do not follow the config, on the host."""
    import torch
    cfg = kvarn.Config(2, 2, 128, 4)
    cache = kvarn.KVCache(cfg, device="cpu")
    k = torch.zeros(2, 2, 256, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="shape"):
        kvarn.quantize_blocks(cfg, k[:, :, :, :64].contiguous(), k[:, :, :, :64].contiguous(), cache)
    with pytest.raises(ValueError, match="shape"):
        kvarn.quantize_blocks(cfg, k, k[:1].contiguous(), cache)
    with pytest.raises(ValueError, match="bfloat16"):
        kvarn.quantize_blocks(cfg, k.float(), k.float(), cache)
    with pytest.raises(ValueError, match="contiguous"):
        kvarn.quantize_blocks(cfg, k.transpose(1, 0), k.transpose(1, 0), cache)
    with pytest.raises(ValueError, match="CUDA"):  # well-formed, but not on the device
        kvarn.quantize_blocks(cfg, k, k, cache)
    other = kvarn.KVCache(kvarn.Config(2, 2, 128, 8), device="cpu")  # more blocks than cfg says
    with pytest.raises(ValueError, match="cache.k_records"):
        kvarn.quantize_blocks(cfg, k, k, other)
    with pytest.raises(ValueError, match="shape"):
        kvarn.append_token(cfg, k[:, :, 0, :96].contiguous(), k[:, :, 0, :96].contiguous(), cache)
    q = torch.zeros(2, 8, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="shape"):
        kvarn.decode_attention(cfg, q, cache, 256, out=torch.zeros(2, 8, 64))
    with pytest.raises(ValueError, match="shape"):
        kvarn.decode_attention(cfg, q[:1].contiguous(), cache, 256)
    with pytest.raises(ValueError, match="4-d"):
        kvarn.decode_attention_multi(cfg, q, cache, 256)
    with pytest.raises(ValueError, match="shape"):
        kvarn.token_errors(cfg, k, k[:, :, :128].contiguous(), cache)
    with pytest.raises(ValueError, match="cache.k_tail"):
        kvarn.dequantize(kvarn.Config(2, 2, 128, 4, dtype=kvarn.KVARN_F32), cache, 0, 1)
