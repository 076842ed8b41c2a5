"""Decode through the allocation-free entry point (library-held static workspace).

Callers that cannot allocate device memory where they run decode use
kvarn_decode_attention_noalloc.  It must give the same result as
kvarn_decode_attention with a caller workspace, call after call, because the
static array keeps whatever the previous call left in it.  This file is named
so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

from bit_kv_cache_token_b200 import kvarn, synth

pytestmark = pytest.mark.gpu


def test_noalloc_decode_matches_workspace_decode_twice_in_a_row():
    S, H, Hq, D, L = 2, 4, 16, 128, 1111
    cfg = kvarn.Config(S, H, D, max_blocks=10)
    cache = kvarn.KVCache(cfg)
    k, v = synth.layer_kv(123, 0, S, H, L, D, device="cuda")
    kvarn.quantize_blocks(cfg, k, v, cache)
    for call in range(2):
        q = synth.queries(200 + call, S, Hq, D, device="cuda")
        ref = kvarn.decode_attention(cfg, q, cache, max_tokens=L)
        out = torch.full_like(ref, float("nan"))
        kvarn.decode_attention_noalloc(cfg, q, cache, L, out)
        torch.cuda.synchronize()
        assert int(cache.status.item()) == 0
        # the same kernel on the same inputs, and decode is deterministic: bit-identical
        assert torch.equal(out, ref)


def test_noalloc_rejects_a_workspace_beyond_the_static_size():
    # 2048 (sequence, kv head) pairs at GQA 8: ~25 MB of partials (two 4 KB slots per pair, one per warp)
    cfg = kvarn.Config(256, 8, 128, max_blocks=1)
    assert kvarn.decode_workspace_bytes(cfg, 64) > 16 << 20
    cache = kvarn.KVCache(cfg)
    q = torch.zeros(256, 64, 128, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(q.shape, dtype=torch.float32, device="cuda")
    with pytest.raises(kvarn.KvarnError) as e:
        kvarn.decode_attention_noalloc(cfg, q, cache, 0, out)
    assert e.value.code == kvarn.KVARN_EWORKSPACE
