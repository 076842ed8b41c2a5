"""Parity at the full benchmark sizes, on sampled outputs the oracle computes one by one.

* Bulk quantisation of the Llama-3-8B-shaped prefill (batch 32 x 32 layers x 8 kv heads x 8192 tokens,
  head_dim 128, bf16, K token sigma 0.7), in the single launch the benchmark times: 256 seeded random blocks and the
  first and last, K and V, against the oracle (codes outside the 1e-5 rounding window and binary16 scales away from a rounding midpoint, exact).
* One Qwen3-4B-shaped decode layer at a 32K context (batch 8, 32 q / 8 kv heads), built as the benchmark builds
  it: bulk prefill, then appended tokens (one of them quantises block 254), decode at context 32705 with the
  benchmark's max_tokens.  Sampled (sequence, kv head) pairs get oracle-packed records on the same
  inputs; their outputs must match the oracle on that cache within 2e-3.
* One Phi-3-mini-shaped MHA layer (batch 16, 32 heads, head_dim 96, 3 x 32 Hadamard, 16284 tokens with a tail).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from bit_kv_cache_token_b200 import kvarn, synth
from parity_util import DECODE_ATOL, check_block, to_f64

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def test_llama_bulk_quantise_full_size_sampled():
    nseq, H, T, D = 32 * 32, 8, 8192, 128
    cfg = kvarn.Config(nseq, H, D, max_blocks=T // 128)
    k = torch.empty(nseq, H, T, D, dtype=torch.bfloat16, device="cuda")
    v = torch.empty_like(k)
    for i in range(0, nseq, 32):  # one layer of the batch at a time, as the benchmark generates it
        kk, vv = synth.layer_kv(5, i // 32, 32, H, T, D, n_outliers=4, sigma_k=0.7, device="cuda")
        k[i:i + 32] = kk
        v[i:i + 32] = vv
        del kk, vv
    cache = kvarn.KVCache(cfg)
    kvarn.quantize_blocks(cfg, k, v, cache)
    torch.cuda.synchronize()
    assert int(cache.status.item()) == 0
    rng = np.random.default_rng(0)
    picks = [(int(rng.integers(nseq)), int(rng.integers(H)), int(rng.integers(T // 128))) for _ in range(256)]
    picks += [(0, 0, 0), (nseq - 1, H - 1, T // 128 - 1)]
    for s, h, b in picks:
        for tensor, x, recs, lay in ((0, k, cache.k_records, oracle.K_ORDER), (1, v, cache.v_records, oracle.V_ORDER)):
            xb = to_f64(x[s, h, b * 128:(b + 1) * 128])
            oq = oracle.quantize_block(xb, 128, 4)
            check_block(recs[s, h, b].cpu().numpy(), None, oq, 128, D, lay)


def _bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def _decode_layer(S, H, Hq, D, hb, ctx, appended, seed, n_out, max_blocks, max_tokens, fixed=None, samples=4,
                  layer=0):
    """Prefill ctx tokens in bulk, append the rest one at a time, decode; compare sampled units with the oracle."""
    total = ctx + appended
    cfg = kvarn.Config(S, H, D, max_blocks=max_blocks, hadamard=hb)
    k, v = synth.layer_kv(seed, layer, S, H, total, D, n_outliers=n_out, outlier_channels=fixed, device="cuda")
    cache = kvarn.KVCache(cfg)
    kvarn.quantize_blocks(cfg, k[:, :, :ctx].contiguous(), v[:, :, :ctx].contiguous(), cache)
    for t in range(ctx, total):
        kvarn.append_token(cfg, k[:, :, t].contiguous(), v[:, :, t].contiguous(), cache)
    torch.cuda.synchronize()
    assert cache.n_tokens.tolist() == [total] * S and int(cache.status.item()) == 0
    nb = total // 128
    rng = np.random.default_rng(seed)
    units = sorted({(int(rng.integers(S)), int(rng.integers(H))) for _ in range(samples)} | {(S - 1, H - 1)})
    krec_o, vrec_o = {}, {}
    for s, h in units:  # the sampled units' records come from the oracle, on the same inputs
        kr = np.zeros((max_blocks, cache.k_records.shape[-1]), np.uint8)
        vr = np.zeros_like(kr)
        kr[:nb] = oracle.quantize_many(_bf16_bits(k[s, h, :nb * 128]), "bf16", 128, D, hb, nthreads=8,
                                       layout=oracle.K_ORDER)[0]
        vr[:nb] = oracle.quantize_many(_bf16_bits(v[s, h, :nb * 128]), "bf16", 128, D, hb, nthreads=8,
                                       layout=oracle.V_ORDER)[0]
        for b in sorted({0, ctx // 128 - 1, nb - 1}):  # what the GPU wrote: bulk path, and append path last
            for x, recs, lay in ((k, cache.k_records, oracle.K_ORDER), (v, cache.v_records, oracle.V_ORDER)):
                oq = oracle.quantize_block(to_f64(x[s, h, b * 128:(b + 1) * 128]), hb, 4)
                check_block(recs[s, h, b].cpu().numpy(), None, oq, 128, D, lay)
        krec_o[(s, h)], vrec_o[(s, h)] = kr, vr
        cache.k_records[s, h] = torch.from_numpy(kr).cuda()
        cache.v_records[s, h] = torch.from_numpy(vr).cuda()
    q = synth.queries(seed + 1, S, Hq, D, device="cuda")
    out = kvarn.decode_attention(cfg, q, cache, max_tokens=max_tokens).cpu().numpy()
    grp = Hq // H
    kt, vt = to_f64(cache.k_tail.cpu()), to_f64(cache.v_tail.cpu())
    qd = to_f64(q.cpu())
    worst = 0.0
    for s, h in units:
        ref = oracle.decode_from_cache(qd[s, h * grp:(h + 1) * grp], krec_o[(s, h)][None], vrec_o[(s, h)][None],
                                       kt[s, h:h + 1], vt[s, h:h + 1], total, 128, hb, 1 / math.sqrt(D))
        worst = max(worst, float(np.max(np.abs(out[s, h * grp:(h + 1) * grp] - ref))))
    assert np.all(np.isfinite(out))
    assert worst <= DECODE_ATOL, worst
    return worst


def test_qwen_decode_layer_32k_sampled():
    # context 32705 as in the benchmark's probe sub-step; block 254 quantised by the append path, 65 tail tokens
    print("max abs err", _decode_layer(8, 8, 32, 128, 128, 32512, 193, 2, 4, max_blocks=256, max_tokens=32768))


@pytest.mark.parametrize("total,layer", [(1024, 0), (1151, 35), (4153, 0), (32768, 35)])
def test_qwen_decode_at_checkpoint_contexts(total, layer):
    """The Qwen3-4B-shaped batch (8 sequences, 8 kv / 32 q heads) at the checkpoint contexts, first and last layer:
    bulk prefill of the whole blocks but the last, the rest appended token by token."""
    ctx = (total // 128 - 1) * 128 if total >= 256 else 0
    err = _decode_layer(8, 8, 32, 128, 128, ctx, total - ctx, 40 + layer, 4, max_blocks=256, max_tokens=total,
                        samples=2, layer=layer)
    print(total, layer, "max abs err", err)


def test_phi_mha_decode_layer_16k_sampled():
    print("max abs err", _decode_layer(16, 32, 32, 96, 32, 16384 - 200, 100, 4, 4, max_blocks=128, max_tokens=16384,
                                       fixed=(31, 32, 63, 64)))


def test_qwen_batch1_decode_in_the_benchmark_launch():
    """The batch-1 Qwen3-4B shape as the benchmark launches it (context 4153, max_tokens 4224): fewer items than
    warps, so every block of a unit sits on its own warp and the merge gathers the partials of exactly those
    warps (37 of them, a CTA merge), not of the span between the first and the last."""
    err = _decode_layer(1, 8, 32, 128, 128, 4096 - 128, 128 + 57, 21, 4, max_blocks=64, max_tokens=4224, samples=3)
    print("max abs err", err)


def test_single_unit_long_context_merges_by_warp():
    """One (sequence, kv head) over 16421 tokens: 133 partials (129 block items of which 128 hold blocks, and 4
    tail slots), more than the CTA merge holds in shared memory, so the completing warp merges them alone."""
    err = _decode_layer(1, 1, 4, 128, 128, 16384 - 128, 128 + 37, 23, 4, max_blocks=129, max_tokens=16512, samples=1)
    print("max abs err", err)
