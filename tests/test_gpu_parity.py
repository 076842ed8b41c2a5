"""GPU parity: the CUDA path through the C ABI against the fp64 oracle, element by element.

Inputs come from bit_kv_cache_token_b200.synth (seeded); expected values only from oracle/.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from bit_kv_cache_token_b200 import kvarn, synth
from parity_util import DECODE_ATOL, check_block, oracle_records, to_f64, view_record

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _cfg(S, H, D, max_blocks, dtype, hb=-1, sweeps=4):
    return kvarn.Config(S, H, D, max_blocks, hadamard=hb, sweeps=sweeps,
                        dtype=kvarn.KVARN_F32 if dtype == torch.float32 else kvarn.KVARN_BF16)


QCASES = [
    # name, S, H, D, T, dtype, hb, sweeps, n_outliers, sigma_k, fixed outliers, seed
    ("c0_tiny", 1, 1, 64, 256, torch.float32, 64, 4, 2, 0.5, None, 0),
    ("c1_qwen", 1, 8, 128, 512, torch.bfloat16, 128, 4, 4, 0.5, None, 1),
    ("c3_llama", 2, 2, 128, 256, torch.bfloat16, 128, 4, 4, 0.7, None, 3),
    ("c4_phi", 1, 4, 96, 256, torch.bfloat16, 32, 4, 4, 0.5, (31, 32, 63, 64), 4),
    ("d128_hb32", 1, 2, 128, 256, torch.bfloat16, 32, 4, 4, 0.5, None, 5),
    ("d128_hb64", 1, 2, 128, 256, torch.float32, 64, 4, 4, 0.5, None, 6),
    ("d128_nohad", 1, 2, 128, 256, torch.bfloat16, 0, 4, 4, 0.5, None, 7),
    ("d128_sweeps0", 1, 2, 128, 256, torch.bfloat16, 128, 0, 4, 0.5, None, 8),
    ("d128_sweeps1", 1, 2, 128, 256, torch.bfloat16, 128, 1, 4, 0.5, None, 9),
    ("d64_hb32_bf16", 2, 1, 64, 256, torch.bfloat16, 32, 4, 2, 0.5, None, 10),
    ("d96_nohad_f32", 1, 2, 96, 128, torch.float32, 0, 4, 4, 0.5, (31, 32, 63, 64), 11),
]


def _inputs(S, H, D, T, dtype, n_out, sigma, fixed, seed):
    return synth.layer_kv(seed, 0, S, H, T, D, n_outliers=n_out, sigma_k=sigma, outlier_channels=fixed, dtype=dtype)


@pytest.mark.parametrize("case", QCASES, ids=[c[0] for c in QCASES])
def test_quantize_blocks_matches_oracle(case):
    name, S, H, D, T, dtype, hb, sweeps, n_out, sigma, fixed, seed = case
    k, v = _inputs(S, H, D, T, dtype, n_out, sigma, fixed, seed)
    nb = T // 128
    cfg = _cfg(S, H, D, nb + 1, dtype, hb, sweeps)
    cache = kvarn.KVCache(cfg)
    dk, dv = kvarn.quantize_blocks(cfg, k.to(DEV), v.to(DEV), cache, first_block=1, debug=True)
    torch.cuda.synchronize()
    assert int(cache.status.item()) == 0
    assert cache.n_tokens.tolist() == [128 + T] * S
    totals = dict(boundary=0, code_flips=0, f16_flips=0, elements=0)
    for tensor, x, dbg, recs in ((0, k, dk, cache.k_records), (1, v, dv, cache.v_records)):
        dd = kvarn.debug_split(cfg, dbg.cpu(), S * H * nb)
        xs = to_f64(x)
        recs = recs.cpu().numpy()
        for s in range(S):
            for h in range(H):
                for b in range(nb):
                    oq = oracle.quantize_block(xs[s, h, b * 128:(b + 1) * 128], hb, sweeps)
                    i = (s * H + h) * nb + b
                    st = check_block(recs[s, h, 1 + b], {kk: dd[kk][i].numpy() for kk in "rcsm"}, oq, 128, D,
                                     oracle.V_ORDER if tensor else oracle.K_ORDER)
                    for kk in totals:
                        totals[kk] += st[kk]
    print(name, totals)
    # the rounding window is rare: far below 1e-3 of the elements
    assert totals["code_flips"] <= max(3, totals["elements"] * 1e-4)


# Blocks whose tokens share a large common part: the zero-variance guard, the shifted variances (row and column
# mean/std of 30 and more) and the gauge steps that keep r, c, s and m inside binary16.
#
# Tolerance.  Where every token is (nearly) the same vector, or one channel dominates every token, the column step
# sees z_td = X_td / r_t whose spread across tokens is made of differences of r_t of relative size d (1e-3 down to
# 1e-5 here): the fp32 rounding of r_t (2^-24) then moves c_d by about 2^-24 / d, 1e-4 to 1e-2 relative, however
# the sums are formed.  Those cases ("ill") are checked for what stays well defined: the status word, binary16
# range, codes within one level, scales within 3e-2, and a reconstruction r c (s code + m) within one
# quantisation step of the oracle's.  The uniform-offset cases, whose rows and columns are well conditioned at
# mean/std 30 and 50, and exact copies keep the contract's 1e-5.
CCASES = [
    # name, kind, amount, channel, D, dtype, hb, ill-conditioned
    ("identical_hb128", "identical", 0.0, 0, 128, torch.bfloat16, 128, False),
    ("identical_noise1e-2_hb128", "identical", 1e-2, 0, 128, torch.bfloat16, 128, True),
    ("identical_noise1e-2_nohad", "identical", 1e-2, 0, 128, torch.bfloat16, 0, True),
    ("identical_noise1e-4_f32_d64", "identical", 1e-4, 0, 64, torch.float32, 64, True),
    ("dc100_ch0_hb128", "dc", 100.0, 0, 128, torch.bfloat16, 128, True),
    ("dc1000_ch77_hb128", "dc", 1000.0, 77, 128, torch.bfloat16, 128, True),
    ("dc1000_ch0_nohad", "dc", 1000.0, 0, 128, torch.bfloat16, 0, True),
    ("dc100_ch50_nohad_d96", "dc", 100.0, 50, 96, torch.bfloat16, 0, True),
    ("offset50_nohad", "offset", 50.0, 0, 128, torch.bfloat16, 0, False),
    ("offset30_hb32_f32", "offset", 30.0, 0, 128, torch.float32, 32, False),
]


@pytest.mark.parametrize("case", CCASES, ids=[c[0] for c in CCASES])
def test_common_component_blocks_match_oracle(case):
    name, kind, amount, ch, D, dtype, hb, ill = case
    rtol, window = (3e-2, 0.1) if ill else (None, None)
    S, H, T = 1, 2, 256
    k, v = synth.common_component_kv(17, kind, S, H, T, D, amount, ch, dtype=dtype)
    nb = T // 128
    cfg = _cfg(S, H, D, nb, dtype, hb, 4)
    cache = kvarn.KVCache(cfg)
    dk, dv = kvarn.quantize_blocks(cfg, k.to(DEV), v.to(DEV), cache, debug=True)
    torch.cuda.synchronize()
    assert int(cache.status.item()) == 0, "a stored scale left binary16"
    worst = 0.0
    for tensor, x, dbg, recs in ((0, k, dk, cache.k_records), (1, v, dv, cache.v_records)):
        dd = kvarn.debug_split(cfg, dbg.cpu(), S * H * nb)
        xs = to_f64(x)
        recs = recs.cpu().numpy()
        for h in range(H):
            for b in range(nb):
                oq = oracle.quantize_block(xs[0, h, b * 128:(b + 1) * 128], hb, 4)
                i = h * nb + b
                layout = oracle.V_ORDER if tensor else oracle.K_ORDER
                st = check_block(recs[0, h, b], {kk: dd[kk][i].numpy() for kk in "rcsm"}, oq, 128, D, layout,
                                 rtol=rtol, window=window)
                worst = max(worst, st["max_rel"])
                if ill:
                    xg = oracle.dequantize_record(recs[0, h, b], 128, D, hb, True, layout)
                    xo = oracle.dequantize_record(oracle.pack_record(oq, layout), 128, D, hb, True, layout)
                    step = (oq["r"][:, None] * oq["c"][None, :]) * np.repeat(oq["s"], 32, axis=1)
                    assert np.all(np.abs(xg - xo) <= 1.05 * step + 1e-3 * np.abs(xo) + 1e-30), name
                if kind == "identical" and amount == 0.0:
                    assert np.all(dd["c"][i].numpy() == 1.0)
    print(name, "largest relative scale error", worst)


def test_ragged_prefill_fills_tail_and_length():
    S, H, D, T = 2, 2, 128, 300
    k, v = _inputs(S, H, D, T, torch.bfloat16, 4, 0.5, None, 12)
    cfg = _cfg(S, H, D, 4, torch.bfloat16)
    cache = kvarn.KVCache(cfg)
    kvarn.quantize_blocks(cfg, k.to(DEV), v.to(DEV), cache, first_block=1)
    torch.cuda.synchronize()
    assert cache.n_tokens.tolist() == [128 + 300] * S
    assert torch.equal(cache.k_tail[:, :, :44].cpu(), k[:, :, 256:300])
    assert torch.equal(cache.v_tail[:, :, :44].cpu(), v[:, :, 256:300])
    # block slot 0 untouched, slots 1..2 written
    assert int(cache.k_records[:, :, 0].abs().sum()) == 0 and int(cache.k_records[:, :, 3].abs().sum()) == 0
    assert int(cache.k_records[:, :, 1:3].sum()) > 0


def test_empty_prefill_sets_length():
    cfg = _cfg(3, 1, 64, 4, torch.float32)
    cache = kvarn.KVCache(cfg)
    e = torch.empty(3, 1, 0, 64, device=DEV)
    kvarn.quantize_blocks(cfg, e, e, cache, first_block=2)
    torch.cuda.synchronize()
    assert cache.n_tokens.tolist() == [256] * 3


@pytest.mark.parametrize("D,dtype,hb", [(128, torch.bfloat16, 128), (96, torch.bfloat16, 32), (64, torch.float32, 64)])
def test_append_is_bit_identical_to_bulk(D, dtype, hb):
    S, H, N = 2, 3, 300
    k, v = _inputs(S, H, D, N, dtype, 4, 0.5, None, 13)
    cfg = _cfg(S, H, D, 3, dtype, hb)
    bulk = kvarn.KVCache(cfg)
    kvarn.quantize_blocks(cfg, k.to(DEV), v.to(DEV), bulk)
    app = kvarn.KVCache(cfg)
    kd, vd = k.to(DEV), v.to(DEV)
    for t in range(N):
        kvarn.append_token(cfg, kd[:, :, t].contiguous(), vd[:, :, t].contiguous(), app)
    torch.cuda.synchronize()
    assert app.n_tokens.tolist() == [N] * S
    assert int(app.arrive.abs().sum()) == 0
    assert torch.equal(app.k_records[:, :, :2], bulk.k_records[:, :, :2])
    assert torch.equal(app.v_records[:, :, :2], bulk.v_records[:, :, :2])
    assert torch.equal(app.k_tail[:, :, :N % 128], bulk.k_tail[:, :, :N % 128])
    assert torch.equal(app.v_tail[:, :, :N % 128], bulk.v_tail[:, :, :N % 128])
    assert int(app.status.item()) == 0


def test_append_capacity_sets_status_and_stops():
    S, H, D = 1, 2, 64
    cfg = _cfg(S, H, D, 1, torch.float32, 64)
    cache = kvarn.KVCache(cfg)
    k, v = _inputs(S, H, D, 256, torch.float32, 2, 0.5, None, 14)
    kd, vd = k.to(DEV), v.to(DEV)
    for t in range(255):
        kvarn.append_token(cfg, kd[:, :, t].contiguous(), vd[:, :, t].contiguous(), cache)
    torch.cuda.synchronize()
    assert cache.n_tokens.tolist() == [255] and int(cache.status.item()) == 0
    kvarn.append_token(cfg, kd[:, :, 255].contiguous(), vd[:, :, 255].contiguous(), cache)
    torch.cuda.synchronize()
    assert cache.n_tokens.tolist() == [255]
    assert int(cache.status.item()) & kvarn.KVARN_STATUS_CAPACITY


def test_scale_beyond_binary16_sets_nonfinite_status():
    """Token scales r_t near 1e6 exceed the binary16 range (65504): the quantiser flags the status word."""
    S, H, D = 1, 1, 128
    cfg = _cfg(S, H, D, 1, torch.float32, 128)
    cache = kvarn.KVCache(cfg)
    k, v = _inputs(S, H, D, 128, torch.float32, 4, 0.5, None, 15)
    kd, vd = k.to(DEV), v.to(DEV)
    kvarn.quantize_blocks(cfg, kd, vd, cache)
    torch.cuda.synchronize()
    assert int(cache.status.item()) == 0
    kvarn.quantize_blocks(cfg, (kd * 1e6).contiguous(), vd, cache)
    torch.cuda.synchronize()
    assert int(cache.status.item()) & kvarn.KVARN_STATUS_NONFINITE


def _oracle_cache(cfg, k, v, L, hb, sweeps=4):
    """Fill a GPU cache with ORACLE-packed records and the raw tail; return (cache, krec, vrec) numpy."""
    S, H, D = cfg.num_seqs, cfg.num_kv_heads, cfg.head_dim
    nb, nt = L // 128, L % 128
    kx, vx = to_f64(k[:, :, :nb * 128]), to_f64(v[:, :, :nb * 128])
    cache = kvarn.KVCache(cfg)
    rb = cache.k_records.shape[-1]
    krec = np.zeros((S, H, cfg.max_blocks, rb), dtype=np.uint8)
    vrec = np.zeros_like(krec)
    if nb:
        krec[:, :, :nb] = oracle_records(kx, hb, sweeps, oracle.K_ORDER)[0]
        vrec[:, :, :nb] = oracle_records(vx, hb, sweeps, oracle.V_ORDER)[0]
    cache.k_records.copy_(torch.from_numpy(krec))
    cache.v_records.copy_(torch.from_numpy(vrec))
    cache.k_tail[:, :, :nt] = k[:, :, nb * 128:L].to(DEV)
    cache.v_tail[:, :, :nt] = v[:, :, nb * 128:L].to(DEV)
    cache.n_tokens.fill_(L)
    return cache, krec, vrec


def _oracle_decode(q, krec, vrec, ktail, vtail, L, hb, scale):
    S = q.shape[0]
    return np.stack([oracle.decode_from_cache(q[s], krec[s], vrec[s], ktail[s], vtail[s], L, 128, hb, scale)
                     for s in range(S)])


DCASES = [
    # name, S, H, Hq, D, dtype, L, hb
    ("c0_256", 1, 1, 1, 64, torch.float32, 256, 64),
    ("c0_300", 1, 1, 1, 64, torch.float32, 300, 64),
    ("c1_qwen_4153", 1, 8, 32, 128, torch.bfloat16, 4153, 128),
    ("tail_only", 2, 2, 8, 128, torch.bfloat16, 57, 128),
    ("one_token", 2, 2, 8, 128, torch.bfloat16, 1, 128),
    ("empty", 2, 2, 8, 128, torch.bfloat16, 0, 128),
    ("boundary_256", 2, 2, 8, 128, torch.bfloat16, 256, 128),
    ("tail_127", 1, 2, 4, 128, torch.bfloat16, 383, 128),
    ("c4_phi_mha", 2, 4, 4, 96, torch.bfloat16, 1000, 32),
    ("gqa2_d64", 2, 2, 4, 64, torch.bfloat16, 700, 64),
    ("gqa8", 1, 1, 8, 128, torch.bfloat16, 900, 128),
    ("nohad", 1, 2, 8, 128, torch.bfloat16, 600, 0),
]


@pytest.mark.parametrize("case", DCASES, ids=[c[0] for c in DCASES])
def test_decode_matches_oracle_on_same_cache(case):
    name, S, H, Hq, D, dtype, L, hb = case
    Lgen = max(L, 1)
    k, v = _inputs(S, H, D, Lgen, dtype, 4, 0.5, None, 20 + len(name))
    q = synth.queries(30 + len(name), S, Hq, D, dtype=dtype)
    cfg = _cfg(S, H, D, max(L // 128, 1) + 1, dtype, hb)
    cache, krec, vrec = _oracle_cache(cfg, k, v, L, hb)
    out = kvarn.decode_attention(cfg, q.to(DEV), cache, max_tokens=L)
    torch.cuda.synchronize()
    assert int(cache.status.item()) == 0
    scale = 1 / math.sqrt(D)
    ref = _oracle_decode(to_f64(q), krec, vrec, to_f64(cache.k_tail.cpu()), to_f64(cache.v_tail.cpu()), L, hb, scale)
    got = out.cpu().numpy()
    err = np.max(np.abs(got - ref)) if got.size else 0.0
    print(name, "max abs err", err)
    assert np.all(np.isfinite(got))
    assert err <= DECODE_ATOL
    if L == 0:
        assert np.all(got == 0)


def test_decode_respects_per_sequence_lengths_and_max_tokens():
    S, H, Hq, D = 3, 2, 4, 128
    k, v = _inputs(S, H, D, 700, torch.bfloat16, 4, 0.5, None, 40)
    q = synth.queries(41, S, Hq, D)
    cfg = _cfg(S, H, D, 6, torch.bfloat16)
    cache, krec, vrec = _oracle_cache(cfg, k, v, 700, 128)
    lens = [700, 129, 0]
    for s, L in enumerate(lens):  # shorter sequences: same records, smaller n_tokens, tail rebuilt
        nb = L // 128
        cache.k_tail[s, :, :L % 128] = k[s, :, nb * 128:L].to(DEV)
        cache.v_tail[s, :, :L % 128] = v[s, :, nb * 128:L].to(DEV)
    cache.n_tokens.copy_(torch.tensor(lens, dtype=torch.int32))
    out = kvarn.decode_attention(cfg, q.to(DEV), cache, max_tokens=700).cpu().numpy()
    kt, vt = to_f64(cache.k_tail.cpu()), to_f64(cache.v_tail.cpu())
    for s, L in enumerate(lens):
        ref = oracle.decode_from_cache(to_f64(q)[s], krec[s], vrec[s], kt[s], vt[s], L, 128, 128, 1 / math.sqrt(D))
        assert np.max(np.abs(out[s] - ref)) <= DECODE_ATOL
    # a length above max_tokens is flagged
    kvarn.decode_attention(cfg, q.to(DEV), cache, max_tokens=600)
    torch.cuda.synchronize()
    assert int(cache.status.item()) & kvarn.KVARN_STATUS_LENGTH


def test_gqa_equals_repeated_mha_on_gpu():
    S, H, D, L = 2, 2, 128, 500
    k, v = _inputs(S, H, D, L, torch.bfloat16, 4, 0.5, None, 50)
    q = synth.queries(51, S, 4 * H, D).to(DEV)
    cfg = _cfg(S, H, D, 4, torch.bfloat16)
    cache = kvarn.KVCache(cfg)
    kvarn.quantize_blocks(cfg, k.to(DEV), v.to(DEV), cache)
    out_gqa = kvarn.decode_attention(cfg, q, cache, max_tokens=L)
    cfg4 = _cfg(S, 4 * H, D, 4, torch.bfloat16)
    rep = kvarn.KVCache(cfg4)
    rep.k_records.copy_(cache.k_records.repeat_interleave(4, dim=1))
    rep.v_records.copy_(cache.v_records.repeat_interleave(4, dim=1))
    rep.k_tail.copy_(cache.k_tail.repeat_interleave(4, dim=1))
    rep.v_tail.copy_(cache.v_tail.repeat_interleave(4, dim=1))
    rep.n_tokens.copy_(cache.n_tokens)
    out_mha = kvarn.decode_attention(cfg4, q, rep, max_tokens=L)
    torch.cuda.synchronize()
    assert torch.allclose(out_gqa, out_mha, rtol=0, atol=1e-5)


@pytest.mark.parametrize("D,hb,dtype", [(128, 128, torch.bfloat16), (96, 32, torch.float32), (64, 0, torch.float32)])
def test_dequantize_matches_oracle(D, hb, dtype):
    S, H, L = 1, 2, 256
    k, v = _inputs(S, H, D, L, dtype, 4, 0.5, None, 60)
    cfg = _cfg(S, H, D, 2, dtype, hb)
    cache, krec, vrec = _oracle_cache(cfg, k, v, L, hb)
    for rotated in (True, False):
        ko, vo = kvarn.dequantize(cfg, cache, 0, 2, rotated=rotated)
        ko, vo = ko.cpu().numpy(), vo.cpu().numpy()
        for h in range(H):
            for b in range(2):
                for got, rec, lay in ((ko, krec, oracle.K_ORDER), (vo, vrec, oracle.V_ORDER)):
                    ref = oracle.dequantize_record(rec[0, h, b], 128, D, hb, rotated, lay)
                    np.testing.assert_allclose(got[0, h, b * 128:(b + 1) * 128], ref, rtol=2e-6,
                                               atol=2e-6 * np.abs(ref).max())


def test_closed_form_on_gpu():
    """Paired rank-one checkerboard, rotation off: r_t = a_t GM(b), c_d = b_d / GM(b) (GM = geometric mean),
    codes 0/3 by sign."""
    T, D = 128, 128
    rng = np.random.default_rng(3)
    a = np.repeat(np.exp(rng.standard_normal(T // 2) * 0.5), 2)
    b = np.repeat(np.exp(rng.standard_normal(D // 2) * 0.5), 2)
    sign = (-1.0) ** np.add.outer(np.arange(T), np.arange(D))
    X = torch.tensor(np.outer(a, b) * sign, dtype=torch.float32)
    cfg = _cfg(1, 1, D, 1, torch.float32, 0)
    cache = kvarn.KVCache(cfg)
    dk, _ = kvarn.quantize_blocks(cfg, X[None, None].to(DEV).contiguous(), X[None, None].to(DEV).contiguous(), cache,
                                  debug=True)
    dd = kvarn.debug_split(cfg, dk.cpu(), 1)
    gm = math.exp(np.mean(np.log(b)))
    np.testing.assert_allclose(dd["r"][0].numpy(), a * gm, rtol=1e-5)
    np.testing.assert_allclose(dd["c"][0].numpy(), b / gm, rtol=1e-5)
    g = view_record(cache.k_records[0, 0, 0].cpu().numpy(), T, D, oracle.K_ORDER)
    np.testing.assert_array_equal(g["codes"], np.where(sign > 0, 3, 0))
    g = view_record(cache.v_records[0, 0, 0].cpu().numpy(), T, D, oracle.V_ORDER)
    np.testing.assert_array_equal(g["codes"], np.where(sign > 0, 3, 0))


def test_checkerboard_fixed_point_on_gpu():
    sign = torch.tensor((-1.0) ** np.add.outer(np.arange(128), np.arange(64)), dtype=torch.float32)
    cfg = _cfg(1, 1, 64, 1, torch.float32, 0)
    cache = kvarn.KVCache(cfg)
    x = sign[None, None].to(DEV).contiguous()
    dk, _ = kvarn.quantize_blocks(cfg, x, x, cache, debug=True)
    dd = kvarn.debug_split(cfg, dk.cpu(), 1)
    assert torch.all(dd["r"] == 1) and torch.all(dd["c"] == 1)


def test_power_of_two_token_scaling_is_exact_on_gpu():
    k, v = _inputs(1, 1, 128, 128, torch.float32, 4, 0.5, None, 70)
    k2 = k.clone()
    k2[0, 0, 5] *= 2.0 ** 6
    k2[0, 0, 90] *= 2.0 ** -4
    cfg = _cfg(1, 1, 128, 1, torch.float32, 128)
    c1, c2 = kvarn.KVCache(cfg), kvarn.KVCache(cfg)
    d1, _ = kvarn.quantize_blocks(cfg, k.to(DEV), v.to(DEV), c1, debug=True)
    d2, _ = kvarn.quantize_blocks(cfg, k2.to(DEV), v.to(DEV), c2, debug=True)
    a, b = kvarn.debug_split(cfg, d1.cpu(), 1), kvarn.debug_split(cfg, d2.cpu(), 1)
    r = a["r"].clone()
    r[0, 5] *= 2.0 ** 6
    r[0, 90] *= 2.0 ** -4
    assert torch.equal(b["r"], r) and torch.equal(b["c"], a["c"]) and torch.equal(b["s"], a["s"])
    ga = view_record(c1.k_records[0, 0, 0].cpu().numpy(), 128, 128, oracle.K_ORDER)
    gb = view_record(c2.k_records[0, 0, 0].cpu().numpy(), 128, 128, oracle.K_ORDER)
    assert np.array_equal(ga["codes"], gb["codes"])


def test_zero_rows_on_gpu():
    k, v = _inputs(1, 1, 128, 128, torch.float32, 4, 0.5, None, 71)
    k[0, 0, 7] = 0.0
    cfg = _cfg(1, 1, 128, 1, torch.float32, 128)
    cache = kvarn.KVCache(cfg)
    dk, _ = kvarn.quantize_blocks(cfg, k.to(DEV), v.to(DEV), cache, debug=True)
    dd = kvarn.debug_split(cfg, dk.cpu(), 1)
    assert float(dd["r"][0, 7]) == 1.0 and torch.all(dd["s"][0, 7] == 0)
    oq = oracle.quantize_block(to_f64(k[0, 0]), 128, 4)
    check_block(cache.k_records[0, 0, 0].cpu().numpy(), {kk: dd[kk][0].numpy() for kk in "rcsm"}, oq, 128, 128,
                oracle.K_ORDER)


def test_kernels_are_deterministic():
    S, H, D, L = 2, 4, 128, 1000
    k, v = _inputs(S, H, D, L, torch.bfloat16, 4, 0.5, None, 80)
    q = synth.queries(81, S, 4 * H, D).to(DEV)
    cfg = _cfg(S, H, D, 8, torch.bfloat16)
    outs = []
    for _ in range(2):
        cache = kvarn.KVCache(cfg)
        kvarn.quantize_blocks(cfg, k.to(DEV), v.to(DEV), cache)
        outs.append((cache.k_records.clone(), cache.v_records.clone(),
                     kvarn.decode_attention(cfg, q, cache, max_tokens=L).clone()))
    torch.cuda.synchronize()
    for x, y in zip(*outs):
        assert torch.equal(x, y)


def test_end_to_end_gpu_quantize_and_decode_vs_oracle():
    """GPU quantise + GPU decode against oracle quantise + oracle decode on the same inputs."""
    S, H, Hq, D, L = 1, 4, 16, 128, 1111
    k, v = _inputs(S, H, D, L, torch.bfloat16, 4, 0.5, None, 90)
    q = synth.queries(91, S, Hq, D)
    cfg = _cfg(S, H, D, 9, torch.bfloat16)
    cache = kvarn.KVCache(cfg)
    kvarn.quantize_blocks(cfg, k.to(DEV), v.to(DEV), cache)
    out = kvarn.decode_attention(cfg, q.to(DEV), cache, max_tokens=L).cpu().numpy()
    ocache, krec, vrec = _oracle_cache(cfg, k, v, L, 128)
    ref = _oracle_decode(to_f64(q), krec, vrec, to_f64(ocache.k_tail.cpu()), to_f64(ocache.v_tail.cpu()), L, 128,
                         1 / math.sqrt(D))
    assert np.max(np.abs(out - ref)) <= DECODE_ATOL


def test_hadamard_absorbed_mode_on_gpu():
    """Rotation folded into the inputs: hadamard 0 on K, V, q rotated beforehand (fp32) gives the oracle's
    hadamard-0 result on those inputs, and, rotated back, the standard mode's output."""
    S, H, Hq, D, L = 2, 2, 8, 128, 3 * 128 + 41
    k, v = _inputs(S, H, D, L, torch.float32, 4, 0.5, None, 77)
    q = synth.queries(78, S, Hq, D, dtype=torch.float32)
    kr = torch.from_numpy(oracle.rotate(to_f64(k), D)).float()
    vr = torch.from_numpy(oracle.rotate(to_f64(v), D)).float()
    qr = torch.from_numpy(oracle.rotate(to_f64(q), D)).float()
    outs = {}
    for name, (kk, vv, qq, hb) in {"std": (k, v, q, D), "abs": (kr, vr, qr, 0)}.items():
        cfg = _cfg(S, H, D, 4, torch.float32, hb)
        cache = kvarn.KVCache(cfg)
        kvarn.quantize_blocks(cfg, kk.to(DEV), vv.to(DEV), cache)
        outs[name] = kvarn.decode_attention(cfg, qq.to(DEV), cache, max_tokens=L).cpu().numpy()
        assert int(cache.status.item()) == 0
    # parity of the absorbed mode itself: the oracle with hadamard 0 on the same fp32 inputs
    ocfg = _cfg(S, H, D, 4, torch.float32, 0)
    _, krec, vrec = _oracle_cache(ocfg, kr, vr, L, 0)
    nb = L // 128
    ktail = np.zeros((S, H, 128, D)); vtail = np.zeros((S, H, 128, D))
    ktail[:, :, :L - nb * 128] = to_f64(kr[:, :, nb * 128:])
    vtail[:, :, :L - nb * 128] = to_f64(vr[:, :, nb * 128:])
    ref = _oracle_decode(to_f64(qr), krec, vrec, ktail, vtail, L, 0, 1 / math.sqrt(D))
    assert np.max(np.abs(outs["abs"] - ref)) <= DECODE_ATOL
    # rotated back, the standard mode's output
    back = oracle.rotate(outs["abs"].astype(np.float64), D)
    assert np.max(np.abs(back - outs["std"])) <= DECODE_ATOL


@pytest.mark.parametrize("D,hb,sweeps,dtype", [(128, 128, 4, torch.bfloat16), (128, 0, 4, torch.bfloat16),
                                               (128, 128, 0, torch.bfloat16), (128, 0, 0, torch.bfloat16),
                                               (96, 32, 4, torch.float32), (64, 64, 1, torch.float32)])
def test_token_errors_match_oracle(D, hb, sweeps, dtype):
    """Per-token magnitude / direction errors on the GPU against the oracle's, on the records the GPU wrote."""
    S, H, T = 2, 2, 256
    k, v = _inputs(S, H, D, T, dtype, 4, 0.5, (31, 32, 63, 64) if D == 96 else None, 60 + D + hb + sweeps)
    cfg = _cfg(S, H, D, 2, dtype, hb, sweeps)
    cache = kvarn.KVCache(cfg)
    kd, vd = k.to(DEV), v.to(DEV)
    kvarn.quantize_blocks(cfg, kd, vd, cache)
    ek, ev = kvarn.token_errors(cfg, kd, vd, cache)
    torch.cuda.synchronize()
    for x, recs, err, lay in ((k, cache.k_records, ek, oracle.K_ORDER), (v, cache.v_records, ev, oracle.V_ORDER)):
        xs, rs, es = to_f64(x), recs.cpu().numpy(), err.cpu().numpy()
        for s in range(S):
            for h in range(H):
                for b in range(2):
                    ref = oracle.record_token_errors(xs[s, h, b * 128:(b + 1) * 128], rs[s, h, b], 128, D, hb, lay)
                    np.testing.assert_allclose(es[s, h, b * 128:(b + 1) * 128], ref, rtol=1e-4, atol=2e-5)


MQCASES = [
    # name, S, H, Hq, Q, D, L, dtype, hb
    ("gqa4_q2_tail41", 2, 2, 8, 2, 128, 3 * 128 + 41, torch.bfloat16, 128),
    ("gqa4_q2_crosses_block", 2, 2, 8, 2, 128, 3 * 128, torch.bfloat16, 128),
    ("gqa4_q2_block_edge", 1, 2, 8, 2, 128, 3 * 128 + 1, torch.bfloat16, 128),
    ("gqa2_q4_crosses_block", 1, 2, 4, 4, 128, 2 * 128 + 2, torch.bfloat16, 128),
    ("mha_q8_d96", 1, 4, 4, 8, 96, 2 * 128 + 3, torch.bfloat16, 32),
    ("gqa8_q1", 1, 1, 8, 1, 128, 300, torch.bfloat16, 128),
    ("q2_before_start", 2, 1, 4, 2, 64, 1, torch.float32, 64),
]


@pytest.mark.parametrize("case", MQCASES, ids=[c[0] for c in MQCASES])
def test_multi_query_decode_matches_oracle(case):
    name, S, H, Hq, Q, D, L, dtype, hb = case
    k, v = _inputs(S, H, D, max(L, 1), dtype, 4, 0.5, (31, 32, 63, 64) if D == 96 else None, 300 + len(name))
    q = synth.queries(301 + len(name), S * Q, Hq, D, dtype=dtype).reshape(S, Q, Hq, D)
    cfg = _cfg(S, H, D, L // 128 + 1, dtype, hb)
    cache, krec, vrec = _oracle_cache(cfg, k, v, L, hb)
    out = kvarn.decode_attention_multi(cfg, q.to(DEV), cache, max_tokens=L).cpu().numpy()
    assert int(cache.status.item()) == 0
    kt, vt, qd = to_f64(cache.k_tail.cpu()), to_f64(cache.v_tail.cpu()), to_f64(q)
    ref = np.stack([oracle.decode_multi_from_cache(qd[s], krec[s], vrec[s], kt[s], vt[s], L, 128, hb,
                                                   1 / math.sqrt(D)) for s in range(S)])
    err = float(np.max(np.abs(out - ref)))
    print(name, "max abs err", err)
    assert np.all(np.isfinite(out)) and err <= DECODE_ATOL
    if Q == 1:  # one query is the single-token decode, bit for bit
        single = kvarn.decode_attention(cfg, q[:, 0].contiguous().to(DEV), cache, max_tokens=L).cpu().numpy()
        np.testing.assert_array_equal(out[:, 0], single)


def test_multi_query_rows_beyond_eight_are_unsupported():
    cfg = _cfg(1, 1, 128, 2, torch.bfloat16)
    cache = kvarn.KVCache(cfg)
    q = torch.zeros(1, 4, 4, 128, dtype=torch.bfloat16, device=DEV)  # 4 queries x GQA 4 = 16 rows
    with pytest.raises(kvarn.KvarnError) as e:
        kvarn.decode_attention_multi(cfg, q, cache, max_tokens=128, workspace=kvarn.decode_workspace(cfg, 8, DEV))
    assert e.value.code == kvarn.KVARN_EUNSUPPORTED


def test_decode_many_short_sequences():
    """1024 (sequence, kv head) units of 300 tokens: more items than warps, so warp ranges cross units and
    partials merge warp by warp.  Sampled units against the oracle decoding the records the GPU wrote."""
    S, H, Hq, D, L = 128, 8, 32, 128, 300
    k, v = synth.layer_kv(700, 0, S, H, L, D, n_outliers=4, device=DEV)
    q = synth.queries(701, S, Hq, D, device=DEV)
    cfg = _cfg(S, H, D, 3, torch.bfloat16)
    cache = kvarn.KVCache(cfg)
    kvarn.quantize_blocks(cfg, k, v, cache)
    out = kvarn.decode_attention(cfg, q, cache, max_tokens=L).cpu().numpy()
    torch.cuda.synchronize()
    assert int(cache.status.item()) == 0 and np.all(np.isfinite(out))
    rng = np.random.default_rng(702)
    kr, vr = cache.k_records.cpu().numpy(), cache.v_records.cpu().numpy()
    kt, vt, qd = to_f64(cache.k_tail.cpu()), to_f64(cache.v_tail.cpu()), to_f64(q.cpu())
    for s in sorted({int(x) for x in rng.integers(0, S, 6)} | {0, S - 1}):
        ref = oracle.decode_from_cache(qd[s], kr[s], vr[s], kt[s], vt[s], L, 128, 128, 1 / math.sqrt(D))
        assert np.max(np.abs(out[s] - ref)) <= DECODE_ATOL


def test_bounded_wait_ends_with_timeout_status_and_leaves_context_usable():
    """A staged record that never arrives (the self-test withholds each warp's first K copy, 1 ms limit) ends the
    launch with KVARN_STATUS_TIMEOUT instead of a hang; a normal decode afterwards gives its usual result."""
    S, H, Hq, D, L = 2, 2, 8, 128, 1000
    k, v = _inputs(S, H, D, L, torch.bfloat16, 4, 0.5, None, 800)
    q = synth.queries(801, S, Hq, D).to(DEV)
    cfg = _cfg(S, H, D, L // 128 + 1, torch.bfloat16)
    cache = kvarn.KVCache(cfg)
    kvarn.quantize_blocks(cfg, k.to(DEV), v.to(DEV), cache)
    ref = kvarn.decode_attention(cfg, q, cache, max_tokens=L).cpu()
    torch.cuda.synchronize()
    assert int(cache.status.item()) == 0
    kvarn.decode_selftest_timeout(cfg, q, cache, max_tokens=L)
    torch.cuda.synchronize()
    assert int(cache.status.item()) & kvarn.KVARN_STATUS_TIMEOUT
    cache.status.zero_()
    again = kvarn.decode_attention(cfg, q, cache, max_tokens=L).cpu()
    torch.cuda.synchronize()
    assert int(cache.status.item()) == 0
    assert torch.equal(again, ref)
