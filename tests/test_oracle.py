"""Pins for the CPU oracle: each test checks it against something other than itself.

Sources: "KVarN: Variance-Normalized KV-Cache Quantization Mitigates Error
Accumulation in Reasoning Tasks" -- abstract (Hadamard rotation, dual-scaling
variance normalisation over both axes, 2-bit) and the rndamp.com article,
"How It Works" items 1-2, "Numbers" (second scale fused into dequantisation).
The pages print no worked example, so the pins are closed forms, invariants,
library routines and brute force.
"""
import math

import numpy as np
import pytest
import scipy.linalg
import torch

import oracle
from bit_kv_cache_token_b200 import synth


# ------------------------------------------------------------------ rotation
@pytest.mark.parametrize("n", [2, 4, 32, 64, 128])
def test_hadamard_is_sylvester_and_orthogonal(n):
    H = oracle.hadamard_matrix(n)
    np.testing.assert_array_equal(H, scipy.linalg.hadamard(n).astype(np.float64))
    np.testing.assert_array_equal(H @ H.T, n * np.eye(n))


@pytest.mark.parametrize("D,hb", [(64, 64), (128, 128), (96, 32), (128, 32), (128, 64)])
def test_rotation_matches_library_blockdiag(D, hb):
    rng = np.random.default_rng(D + hb)
    x = rng.standard_normal((5, D))
    H = scipy.linalg.hadamard(hb) / math.sqrt(hb)
    M = scipy.linalg.block_diag(*([H] * (D // hb)))
    np.testing.assert_allclose(oracle.rotate(x, hb), x @ M.T, rtol=0, atol=1e-12)
    # orthogonal and self-inverse
    np.testing.assert_allclose(np.linalg.norm(oracle.rotate(x, hb), axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    np.testing.assert_allclose(oracle.rotate(oracle.rotate(x, hb), hb), x, atol=1e-12)


def test_rotation_off_is_identity():
    x = np.random.default_rng(1).standard_normal((3, 64))
    np.testing.assert_array_equal(oracle.rotate(x, 0), x)


@pytest.mark.parametrize("D,hb", [(64, 64), (128, 128), (96, 32)])
def test_joint_rotation_preserves_dot_products(D, hb):
    rng = np.random.default_rng(7)
    q = rng.standard_normal((4, D))
    k = rng.standard_normal((9, D)) * np.exp(rng.standard_normal(D))
    np.testing.assert_allclose(oracle.rotate(q, hb) @ oracle.rotate(k, hb).T, q @ k.T, rtol=0, atol=1e-12 * D)


# ------------------------------------------------------------ normalisation
def _config0_k(seed=0):
    k, v = synth.layer_kv(seed, 0, 1, 1, 256, 64, n_outliers=2, dtype=torch.float32)
    return k[0, 0].double().numpy(), v[0, 0].double().numpy()


@pytest.mark.parametrize("which", ["k", "v"])
def test_variance_uniform_after_four_sweeps(which):
    """Rows and columns of Y = Xrot / (r c) end within 1e-3 of uniform variance."""
    kk, vv = _config0_k(0)
    X = kk if which == "k" else vv
    for b in range(2):
        Xb = oracle.rotate(X[b * 128:(b + 1) * 128], 64)
        r, c = oracle.normalize(Xb, 4)
        Y = Xb / (r[:, None] * c[None, :])
        col = Y.var(axis=0)
        row = Y.var(axis=1)
        np.testing.assert_allclose(col, 1.0, rtol=0, atol=1e-12)  # the last step is a column step
        assert np.max(np.abs(row / row.mean() - 1.0)) <= 1e-3
        # one sweep leaves the rows visibly less uniform than four (the iteration is doing work)
        r1, c1 = oracle.normalize(Xb, 1)
        row1 = (Xb / (r1[:, None] * c1[None, :])).var(axis=1)
        assert np.max(np.abs(row1 / row1.mean() - 1.0)) > np.max(np.abs(row / row.mean() - 1.0))


def _paired_rank_one(T=16, D=64, seed=3):
    rng = np.random.default_rng(seed)
    a = np.repeat(np.exp(rng.standard_normal(T // 2)), 2)
    b = np.repeat(np.exp(rng.standard_normal(D // 2)), 2)
    sign = (-1.0) ** np.add.outer(np.arange(T), np.arange(D))
    return a, b, np.outer(a, b) * sign


@pytest.mark.parametrize("sweeps", [1, 2, 4])
def test_closed_form_paired_rank_one(sweeps):
    """X_td = a_t b_d (-1)^(t+d), a and b positive and paired, rotation off:
    r_t = a_t GM(b), c_d = b_d / GM(b) (GM = geometric mean) after the first sweep and at every later
    one, Y = +-1 and the codes are 0 / 3 by the sign pattern.  Without the gauge step the split would
    be r_t = a_t RMS(b), c_d = b_d / RMS(b): the product r_t c_d = a_t b_d is the same either way."""
    a, b, X = _paired_rank_one()
    gm = math.exp(np.mean(np.log(b)))
    r, c = oracle.normalize(X, sweeps)
    np.testing.assert_allclose(r, a * gm, rtol=1e-13)
    np.testing.assert_allclose(c, b / gm, rtol=1e-13)
    np.testing.assert_allclose(np.outer(r, c), np.outer(a, b), rtol=1e-13)
    q = oracle.quantize_block(X, hb=0, sweeps=sweeps, group=32)
    sign = (-1.0) ** np.add.outer(np.arange(16), np.arange(64))
    np.testing.assert_array_equal(q["codes"], np.where(sign > 0, 3, 0))
    np.testing.assert_allclose(q["m"], -1.0, rtol=1e-13)
    np.testing.assert_allclose(q["s"], 2.0 / 3.0, rtol=1e-13)


def test_checkerboard_is_fixed_point():
    sign = (-1.0) ** np.add.outer(np.arange(128), np.arange(64))
    r, c = oracle.normalize(sign, 4)
    np.testing.assert_array_equal(r, np.ones(128))
    np.testing.assert_array_equal(c, np.ones(64))


@pytest.mark.parametrize("hb", [0, 64])
def test_power_of_two_token_scaling_is_exact(hb):
    """Scaling token t by 2^k scales r_t by exactly 2^k and changes nothing else (bit-exact)."""
    X, _ = _config0_k(1)
    X = X[:128]
    X2 = X.copy()
    X2[5] *= 2.0 ** 7
    X2[77] *= 2.0 ** -3
    q1 = oracle.quantize_block(X, hb=hb, sweeps=4)
    q2 = oracle.quantize_block(X2, hb=hb, sweeps=4)
    expect_r = q1["r"].copy()
    expect_r[5] *= 2.0 ** 7
    expect_r[77] *= 2.0 ** -3
    np.testing.assert_array_equal(q2["r"], expect_r)
    np.testing.assert_array_equal(q2["c"], q1["c"])
    np.testing.assert_array_equal(q2["codes"], q1["codes"])
    np.testing.assert_array_equal(q2["s"], q1["s"])
    np.testing.assert_array_equal(q2["m"], q1["m"])


def test_zero_rows_and_columns_get_unit_scale():
    """A zero row or column has zero variance, takes scale 1 and stays out of the gauge step: the other channel
    scales have geometric mean 1 on their own.  The zero row codes to 0 with s = m = 0."""
    X = np.random.default_rng(2).standard_normal((128, 64))
    X[3] = 0.0
    X[:, 10] = 0.0
    r, c = oracle.normalize(X, 4)
    assert r[3] == 1.0 and c[10] == 1.0
    assert abs(np.mean(np.log(np.delete(c, 10)))) < 1e-14
    q = oracle.quantize_block(X, hb=0, sweeps=4)
    assert np.all(q["codes"][3] == 0) and np.all(q["s"][3] == 0.0) and np.all(q["m"][3] == 0.0)


def _population_std(x):
    return float(np.sqrt(np.mean((x - x.mean()) ** 2)))


@pytest.mark.parametrize("hb", [0, 128])
def test_identical_tokens_give_token_std_and_unit_channel_scales(hb):
    """128 copies of one token: every column of X / r is constant, so every c_d = 1 exactly (zero variance, and
    the gauge of all-ones is 1) and r_t is the population std of the rotated token.  Scaling copies by powers of
    two scales their r_t by the same power and leaves c = 1."""
    x = np.random.default_rng(12).standard_normal(128) * np.exp(np.random.default_rng(13).standard_normal(128))
    X = np.tile(x, (128, 1))
    q = oracle.quantize_block(X, hb=hb, sweeps=4)
    np.testing.assert_array_equal(q["c"], np.ones(128))
    np.testing.assert_allclose(q["r"], _population_std(oracle.rotate(x, hb)), rtol=1e-14)
    p = 2.0 ** np.random.default_rng(14).integers(-6, 7, size=128)
    q2 = oracle.quantize_block(X * p[:, None], hb=hb, sweeps=4)
    np.testing.assert_array_equal(q2["c"], np.ones(128))
    np.testing.assert_array_equal(q2["r"], q["r"] * p)
    np.testing.assert_array_equal(q2["codes"], q["codes"])


def _common_component_blocks():
    """Blocks whose tokens share a large common part: near-identical tokens, and a DC offset on one channel."""
    rng = np.random.default_rng(15)
    x = rng.standard_normal(128) * np.exp(rng.standard_normal(128))
    base = rng.standard_normal((128, 128))
    out = [("identical+1e-2", np.tile(x, (128, 1)) + 1e-2 * base),
           ("identical+1e-4", np.tile(x, (128, 1)) + 1e-4 * base)]
    for off in (100.0, 1000.0):
        for ch in (0, 77):
            X = base.copy()
            X[:, ch] += off
            out.append((f"dc{off:g}@{ch}", X))
    return out


@pytest.mark.parametrize("hb", [0, 128])
def test_common_component_keeps_scales_in_binary16(hb):
    """On blocks with a large common token component every stored scale (r, c, s, m) is a finite, nonzero (r, c)
    binary16 number -- the iteration without the gauge step drives r and c to 1e7..1e14 and 1e-10..1e-19 on these
    blocks -- the channel scales of the columns that vary have geometric mean 1 and those columns of
    Y = X / (r c) have unit variance (a column that no longer varies keeps scale 1), and no stored |Y| reaches
    2^14."""
    for name, X in _common_component_blocks():
        Xb = oracle.rotate(X, hb)
        r, c = oracle.normalize(Xb, 4)
        Y = Xb / (r[:, None] * c[None, :])
        flat = c == 1.0  # zero-variance columns (variance below 2^-40 of the mean square) keep scale 1
        assert np.all(Y[:, flat].var(axis=0) <= 2.0 ** -30 * np.mean(Y[:, flat] ** 2, axis=0)), name
        assert abs(np.mean(np.log(c[~flat]))) < 1e-13, name
        np.testing.assert_allclose(Y[:, ~flat].var(axis=0), 1.0, rtol=0, atol=1e-9, err_msg=name)
        q = oracle.quantize_block(X, hb=hb, sweeps=4)
        for key in ("r", "c", "s", "m"):
            h = np.array([oracle.f16_value(oracle.f16_bits(v)) for v in np.ravel(q[key])])
            assert np.all(np.isfinite(h)), (name, key, np.abs(q[key]).max())
            if key in ("r", "c"):
                assert np.all(h > 0), (name, key, q[key].min())
        Ys = q["xrot"] / (q["r"][:, None] * q["c"][None, :])
        assert np.abs(Ys).max() < 2.0 ** 14, name


@pytest.mark.parametrize("A,k", [(1000.0, 0), (100000.0, 3), (3.0e6, 8)])
def test_token_gauge_closed_form(A, k):
    """X_td = A + (-1)^(t+d), rotation off: r = c = 1 exactly (every row and column is A +- 1), so Y = X.  Once
    max |Y| = A + 1 reaches 2^14 the token gauge moves 2^k, k = floor(log2(A + 1)) - 13, into every r_t: r = 2^k,
    m = (A - 1) / 2^k, s = 2 / (3 2^k), and the codes stay 3 / 0 by the sign pattern."""
    sign = (-1.0) ** np.add.outer(np.arange(128), np.arange(64))
    X = A + sign
    r, c = oracle.normalize(X, 4)
    np.testing.assert_array_equal(r, np.ones(128))
    np.testing.assert_array_equal(c, np.ones(64))
    q = oracle.quantize_block(X, hb=0, sweeps=4)
    assert k == max(0, math.floor(math.log2(A + 1)) - 13)
    np.testing.assert_array_equal(q["r"], np.full(128, 2.0 ** k))
    np.testing.assert_array_equal(q["c"], np.ones(64))
    np.testing.assert_array_equal(q["m"], np.full((128, 2), (A - 1) / 2.0 ** k))
    np.testing.assert_allclose(q["s"], 2.0 / (3 * 2.0 ** k), rtol=1e-15)
    np.testing.assert_array_equal(q["codes"], np.where(sign > 0, 3, 0))


def test_gauge_moves_only_a_common_factor():
    """Against the iteration written without the gauge step (a plain numpy loop, central variance): the products
    r_t c_d agree and the gauged channel scales are the ungauged ones divided by their geometric mean."""
    X, _ = _config0_k(4)
    Xb = oracle.rotate(X[:128], 64)
    c0 = np.ones(64)
    for _ in range(4):
        r0 = (Xb / c0).std(axis=1)
        c0 = (Xb / r0[:, None]).std(axis=0)
    r, c = oracle.normalize(Xb, 4)
    np.testing.assert_allclose(np.outer(r, c), np.outer(r0, c0), rtol=1e-12)
    np.testing.assert_allclose(c, c0 / math.exp(np.mean(np.log(c0))), rtol=1e-12)


def test_zero_sweeps_is_plain_group_rtn():
    X = np.random.default_rng(4).standard_normal((128, 64))
    r, c = oracle.normalize(X, 0)
    assert np.all(r == 1.0) and np.all(c == 1.0)


# --------------------------------------------------------------------- codec
def test_grid_values_round_trip_exactly():
    """Values on the 2-bit grid {m + k s} with binary16-exact m, s come back exactly."""
    rng = np.random.default_rng(5)
    T, D = 128, 64
    m = rng.integers(-64, 64, size=(T, 2)) / 16.0
    s = rng.integers(1, 32, size=(T, 2)) / 32.0
    k = rng.integers(0, 4, size=(T, D))
    k[:, 0], k[:, 1], k[:, 32], k[:, 33] = 0, 3, 0, 3  # every group spans the full grid
    X = m.repeat(32, axis=1) + k * s.repeat(32, axis=1)
    q = oracle.quantize_block(X, hb=0, sweeps=0)
    np.testing.assert_array_equal(q["codes"], k)
    rec = oracle.pack_record(q)
    np.testing.assert_array_equal(oracle.dequantize_record(rec, T, D, hb=0), X)


def test_codes_are_the_nearest_level():
    """Brute force: the code is the nearest of the four levels m + k s (ties excluded)."""
    X, _ = _config0_k(2)
    q = oracle.quantize_block(X[:128], hb=64, sweeps=4)
    Y = q["xrot"] / (q["r"][:, None] * q["c"][None, :])
    lv = q["m"].repeat(32, axis=1)[..., None] + np.arange(4) * q["s"].repeat(32, axis=1)[..., None]
    best = np.argmin(np.abs(Y[..., None] - lv), axis=-1)
    tie = np.abs(q["v"] - np.floor(q["v"]) - 0.5) < 1e-9
    assert np.array_equal(best[~tie], q["codes"][~tie])
    assert q["codes"].max() == 3 and q["codes"].min() == 0


def test_dequantisation_error_is_at_most_half_a_step():
    X, _ = _config0_k(3)
    q = oracle.quantize_block(X[128:], hb=64, sweeps=4)
    rec = oracle.pack_record(q)
    u = oracle.unpack_record(rec, 128, 64)
    Xr_hat = oracle.dequantize_record(rec, 128, 64, hb=64, rotated=True)
    step = (u["r"][:, None] * u["c"][None, :]) * u["s"].repeat(32, axis=1)
    # error of RTN with the unrounded scales, plus what binary16 rounding of r, c, s, m may add
    slack = 4 * 2.0 ** -11 * np.abs(q["xrot"]) + 2 * 2.0 ** -11 * np.abs(
        u["r"][:, None] * u["c"][None, :] * u["m"].repeat(32, axis=1))
    assert np.all(np.abs(Xr_hat - q["xrot"]) <= 0.5 * step + slack + 1e-12)
    # the unrotated dequantisation is the rotated one rotated back
    np.testing.assert_allclose(oracle.dequantize_record(rec, 128, 64, hb=64), oracle.rotate(Xr_hat, 64), atol=1e-12)


def test_binary16_rounding_matches_numpy():
    rng = np.random.default_rng(6)
    xs = np.concatenate([
        rng.standard_normal(4000) * np.exp(rng.uniform(-25, 12, 4000)),
        [0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e6, -1e6, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26,
         2.0 ** -14, 2.0 ** -14 * (1 - 2.0 ** -11), 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, float("inf")]])
    with np.errstate(over="ignore"):  # values beyond 65520 round to infinity on purpose
        for x in xs:
            assert oracle.f16_bits(x) == int(np.array(x, dtype=np.float64).astype(np.float16).view(np.uint16)), x
    for bits in list(range(0, 0x7C01, 37)) + [0x8001, 0xBC00, 0x7BFF]:
        assert oracle.f16_value(bits) == float(np.array(bits, dtype=np.uint16).view(np.float16))


def test_record_bit_layout():
    T, D = 128, 64
    codes = np.zeros((T, D), dtype=np.uint8)
    codes[0, :4] = [0, 1, 2, 3]
    codes[1, 4:8] = [3, 2, 1, 0]
    q = dict(codes=codes, r=np.full(T, 2.0), c=np.full(D, 0.5), s=np.full((T, 2), 0.25), m=np.full((T, 2), -1.0))
    rec = oracle.pack_record(q, oracle.NATURAL)
    assert len(rec) == oracle.record_bytes(T, D) == 3456  # 2048 + 512 + 512 + 256 + 128, already 128-aligned
    assert rec[0] == 0xE4 and rec[1] == 0 and rec[16 + 1] == 0x1B
    assert np.all(np.frombuffer(rec[2048:2560].tobytes(), dtype=np.float16) == 0.25)
    assert np.all(np.frombuffer(rec[2560:3072].tobytes(), dtype=np.float16) == -1.0)
    assert np.all(np.frombuffer(rec[3072:3328].tobytes(), dtype=np.float16) == 2.0)
    assert np.all(np.frombuffer(rec[3328:3456].tobytes(), dtype=np.float16) == 0.5)
    assert oracle.record_bytes(128, 128) == 6656 and oracle.record_bytes(128, 96) == 5120


def _one_hot_site(layout, D, t, d):
    """(word index, bit) where the code of (t, d) lands, found by packing a single 1."""
    codes = np.zeros((128, D), dtype=np.uint8)
    codes[t, d] = 1
    q = dict(codes=codes, r=np.ones(128), c=np.ones(D), s=np.zeros((128, D // 32)), m=np.zeros((128, D // 32)))
    words = oracle.pack_record(q, layout)[:32 * D].view(np.uint32)
    (w,) = np.nonzero(words)
    assert len(w) == 1
    return int(w[0]), int(words[w[0]]).bit_length() - 1


@pytest.mark.parametrize("layout", [oracle.K_ORDER, oracle.V_ORDER])
@pytest.mark.parametrize("D", [64, 96, 128])
def test_fragment_layouts_are_permutations_with_pairs(layout, D):
    rng = np.random.default_rng(D + layout)
    codes = rng.integers(0, 4, size=(128, D)).astype(np.uint8)
    q = dict(codes=codes, r=np.ones(128), c=np.ones(D), s=np.ones((128, D // 32)), m=np.zeros((128, D // 32)))
    rec = oracle.pack_record(q, layout)
    np.testing.assert_array_equal(oracle.unpack_record(rec, 128, D, layout)["codes"], codes)
    full = dict(q, codes=np.full((128, D), 3, dtype=np.uint8))
    assert np.all(oracle.pack_record(full, layout)[:32 * D] == 0xFF)  # every code bit used exactly once
    # the two codes an AND extracts as one binary16 pair sit at bit b and b + 16 of the same word:
    # K pairs channels (k, k+1) of one token, V pairs tokens (t, t+1) of one channel
    for t, d in [(0, 0), (37, 18), (127, D - 2), (64, 40), (90, 66 % D)]:
        if layout == oracle.K_ORDER:
            d -= d % 2
            a, b = _one_hot_site(layout, D, t, d), _one_hot_site(layout, D, t, d + 1)
        else:
            t -= t % 2
            a, b = _one_hot_site(layout, D, t, d), _one_hot_site(layout, D, t + 1, d)
        assert a[0] == b[0] and b[1] == a[1] + 16 and a[1] < 16


# ----------------------------------------------------------------- attention
def _sdpa(q, K, V, scale):
    """Library reference: torch scaled_dot_product_attention in fp64, kv heads repeated."""
    Hq, Hkv = q.shape[0], K.shape[0]
    rep = Hq // Hkv
    Kt = torch.from_numpy(np.repeat(K, rep, axis=0))
    Vt = torch.from_numpy(np.repeat(V, rep, axis=0))
    qt = torch.from_numpy(q)[:, None, :]
    o = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt, scale=scale)
    return o[:, 0, :].numpy()


@pytest.mark.parametrize("Hq,Hkv", [(1, 1), (4, 1), (8, 2)])
def test_attention_brute_force_16_tokens(Hq, Hkv):
    rng = np.random.default_rng(8)
    D, L = 64, 16
    q = rng.standard_normal((Hq, D))
    K = rng.standard_normal((Hkv, L, D)) * 2
    V = rng.standard_normal((Hkv, L, D))
    out = oracle.attention(q, K, V, 1 / math.sqrt(D))
    np.testing.assert_allclose(out, _sdpa(q, K, V, 1 / math.sqrt(D)), rtol=0, atol=1e-12)


def test_gqa_equals_repeated_mha():
    rng = np.random.default_rng(9)
    q = rng.standard_normal((8, 32))
    K = rng.standard_normal((2, 20, 32))
    V = rng.standard_normal((2, 20, 32))
    a = oracle.attention(q, K, V, 0.3)
    b = oracle.attention(q, np.repeat(K, 4, axis=0), np.repeat(V, 4, axis=0), 0.3)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-14)


def test_attention_is_rotation_invariant_in_scores():
    rng = np.random.default_rng(10)
    q = rng.standard_normal((2, 64))
    K = rng.standard_normal((1, 30, 64))
    V = rng.standard_normal((1, 30, 64))
    a = oracle.attention(q, K, V, 0.125)
    b = oracle.attention(oracle.rotate(q, 64), oracle.rotate(K, 64), V, 0.125)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


@pytest.mark.parametrize("n_tokens", [0, 5, 8, 13, 16])
def test_decode_from_cache_brute_force(n_tokens):
    """16-token cache, 8-token blocks: two packed blocks, one block + tail, tail only, empty."""
    rng = np.random.default_rng(11)
    T, D, Hkv, Hq = 8, 64, 2, 4
    Kx = rng.standard_normal((Hkv, 16, D)) * 3
    Vx = rng.standard_normal((Hkv, 16, D))
    q = rng.standard_normal((Hq, D))
    nb = n_tokens // T
    krec = np.zeros((Hkv, 2, oracle.record_bytes(T, D)), dtype=np.uint8)
    vrec = np.zeros_like(krec)
    Khat = np.zeros((Hkv, n_tokens, D))
    Vhat = np.zeros((Hkv, n_tokens, D))
    for h in range(Hkv):
        for b in range(nb):
            krec[h, b] = oracle.pack_record(oracle.quantize_block(Kx[h, b * T:(b + 1) * T], 64, 4))
            vrec[h, b] = oracle.pack_record(oracle.quantize_block(Vx[h, b * T:(b + 1) * T], 64, 4))
            Khat[h, b * T:(b + 1) * T] = oracle.dequantize_record(krec[h, b], T, D, 64)
            Vhat[h, b * T:(b + 1) * T] = oracle.dequantize_record(vrec[h, b], T, D, 64)
        Khat[h, nb * T:] = Kx[h, nb * T:n_tokens]
        Vhat[h, nb * T:] = Vx[h, nb * T:n_tokens]
    ktail = np.zeros((Hkv, T, D))
    vtail = np.zeros((Hkv, T, D))
    ktail[:, :n_tokens - nb * T] = Kx[:, nb * T:n_tokens]
    vtail[:, :n_tokens - nb * T] = Vx[:, nb * T:n_tokens]
    out = oracle.decode_from_cache(q, krec, vrec, ktail, vtail, n_tokens, T, 64, 1 / 8)
    if n_tokens == 0:
        assert np.all(out == 0)
    else:
        np.testing.assert_allclose(out, _sdpa(q, Khat, Vhat, 1 / 8), rtol=0, atol=1e-12)


# ------------------------------------------------------------ threaded bulk
def test_quantize_many_matches_single_blocks():
    k, _ = synth.layer_kv(0, 0, 1, 2, 256, 64, n_outliers=2, dtype=torch.bfloat16)
    raw = k.contiguous().view(torch.int16).numpy().view(np.uint16)
    recs, used = oracle.quantize_many(raw, "bf16", 128, 64, 64, nthreads=3)
    assert used == 3 and recs.shape == (4, 3456)
    kd = k.double().numpy().reshape(4, 128, 64)
    for u in range(4):
        np.testing.assert_array_equal(recs[u], oracle.pack_record(oracle.quantize_block(kd[u], 64, 4)))


def test_hadamard_absorbed_mode_identity():
    """Rotation folded into the inputs (hadamard 0 on pre-rotated K, V, q) is the same encoding, and its output is
    the rotated output of the standard mode (the rotation is orthogonal and its own inverse)."""
    rng = np.random.default_rng(31)
    T, D, Hkv, Hq, n = 8, 64, 1, 2, 19  # two 8-token blocks and a 3-token tail
    Kx = rng.standard_normal((Hkv, 24, D)) * np.exp(rng.standard_normal(D))
    Vx = rng.standard_normal((Hkv, 24, D))
    q = rng.standard_normal((Hq, D))
    Kr, Vr, qr = oracle.rotate(Kx, D), oracle.rotate(Vx, D), oracle.rotate(q, D)
    nb = n // T
    rb = oracle.record_bytes(T, D)
    recs = {}
    for name, X, hb in (("std", (Kx, Vx), D), ("abs", (Kr, Vr), 0)):
        kr = np.zeros((Hkv, nb, rb), dtype=np.uint8)
        vr = np.zeros_like(kr)
        for b in range(nb):
            kr[0, b] = oracle.pack_record(oracle.quantize_block(X[0][0, b * T:(b + 1) * T], hb, 4))
            vr[0, b] = oracle.pack_record(oracle.quantize_block(X[1][0, b * T:(b + 1) * T], hb, 4))
        recs[name] = (kr, vr)
    # the rotation inside the quantiser equals the rotation done beforehand: identical records
    np.testing.assert_array_equal(recs["std"][0], recs["abs"][0])
    np.testing.assert_array_equal(recs["std"][1], recs["abs"][1])
    tail = lambda X: np.concatenate([X[:, nb * T:n], np.zeros((Hkv, T - (n - nb * T), D))], axis=1)
    out_std = oracle.decode_from_cache(q, *recs["std"], tail(Kx), tail(Vx), n, T, D, 1 / 8)
    out_abs = oracle.decode_from_cache(qr, *recs["abs"], tail(Kr), tail(Vr), n, T, 0, 1 / 8)
    np.testing.assert_allclose(oracle.rotate(out_abs, D), out_std, rtol=0, atol=1e-12)


def test_error_split_closed_forms():
    """Magnitude / direction split: a scaled copy has only a magnitude error, an orthogonal one only a direction
    error of 1, and a rotation of both rows changes neither."""
    rng = np.random.default_rng(41)
    x = rng.standard_normal((5, 64))
    a = np.array([0.5, 1.0, 1.25, 2.0, 3.0])
    e = oracle.magnitude_direction_errors(x, x * a[:, None])
    np.testing.assert_allclose(e[:, 0], np.abs(a - 1), rtol=0, atol=1e-14)
    np.testing.assert_allclose(e[:, 1], 0.0, rtol=0, atol=1e-14)
    y = rng.standard_normal((5, 64))
    y -= (np.sum(x * y, axis=1) / np.sum(x * x, axis=1))[:, None] * x  # orthogonal to x
    e = oracle.magnitude_direction_errors(x, y)
    np.testing.assert_allclose(e[:, 1], 1.0, rtol=0, atol=1e-12)
    np.testing.assert_allclose(e[:, 0], np.abs(np.linalg.norm(y, axis=1) / np.linalg.norm(x, axis=1) - 1),
                               rtol=1e-13)
    z = x + 0.1 * rng.standard_normal((5, 64))
    np.testing.assert_allclose(oracle.magnitude_direction_errors(oracle.rotate(x, 64), oracle.rotate(z, 64)),
                               oracle.magnitude_direction_errors(x, z), rtol=0, atol=1e-12)
    np.testing.assert_array_equal(oracle.magnitude_direction_errors(np.zeros((1, 8)), np.ones((1, 8))), [[0, 0]])


def test_record_errors_vanish_on_the_grid_and_grow_without_normalisation():
    """Values on the 2-bit grid reconstruct exactly (zero error); on the synthetic K the two-stage encoding
    (rotation + normalisation) leaves a smaller mean magnitude error than plain group RTN."""
    rng = np.random.default_rng(5)
    T, D = 128, 64
    m = rng.integers(-64, 64, size=(T, 2)) / 16.0
    s = rng.integers(1, 32, size=(T, 2)) / 32.0
    k = rng.integers(0, 4, size=(T, D))
    k[:, 0], k[:, 1], k[:, 32], k[:, 33] = 0, 3, 0, 3
    X = m.repeat(32, axis=1) + k * s.repeat(32, axis=1)
    rec = oracle.pack_record(oracle.quantize_block(X, hb=0, sweeps=0))
    np.testing.assert_allclose(oracle.record_token_errors(X, rec, T, D, 0), 0.0, rtol=0, atol=1e-14)
    K, _ = _config0_k(3)
    K = K[:128]
    err = {}
    for name, hb, sw in (("kvarn", 64, 4), ("rtn", 0, 0)):
        rec = oracle.pack_record(oracle.quantize_block(K, hb, sw))
        err[name] = oracle.record_token_errors(K, rec, T, D, hb).mean(axis=0)
    assert err["kvarn"][0] < err["rtn"][0]


def test_multi_query_decode_is_causal_single_decodes():
    """Q queries at once equal Q single-token decodes, each over the cache truncated after its own position; the
    last query sees the whole cache."""
    rng = np.random.default_rng(51)
    T, D, Hkv, Hq, Q, n = 8, 64, 1, 2, 3, 17  # blocks 0-1 packed, one tail token; queries at positions 14, 15, 16
    Kx = rng.standard_normal((Hkv, 24, D))
    Vx = rng.standard_normal((Hkv, 24, D))
    q = rng.standard_normal((Q, Hq, D))
    krec = np.stack([[oracle.pack_record(oracle.quantize_block(Kx[0, b * T:(b + 1) * T], 64, 4)) for b in range(2)]])
    vrec = np.stack([[oracle.pack_record(oracle.quantize_block(Vx[0, b * T:(b + 1) * T], 64, 4)) for b in range(2)]])
    ktail = np.zeros((Hkv, T, D)); vtail = np.zeros((Hkv, T, D))
    ktail[:, 0] = Kx[:, 16]; vtail[:, 0] = Vx[:, 16]
    out = oracle.decode_multi_from_cache(q, krec, vrec, ktail, vtail, n, T, 64, 0.125)
    np.testing.assert_allclose(out[Q - 1], oracle.decode_from_cache(q[Q - 1], krec, vrec, ktail, vtail, n, T, 64, 0.125),
                               rtol=0, atol=1e-13)
    Khat = np.concatenate([oracle.dequantize_record(krec[0, b], T, D, 64) for b in range(2)] + [Kx[0, 16:17]])
    Vhat = np.concatenate([oracle.dequantize_record(vrec[0, b], T, D, 64) for b in range(2)] + [Vx[0, 16:17]])
    for i in range(Q):
        pos = n - Q + i
        ref = oracle.attention(q[i], Khat[None, :pos + 1], Vhat[None, :pos + 1], 0.125)
        np.testing.assert_allclose(out[i], ref, rtol=0, atol=1e-13)
    # a query before position 0 gets zeros
    z = oracle.decode_multi_from_cache(q, krec[:, :0], vrec[:, :0], ktail, vtail, 2, T, 64, 0.125)
    assert np.all(z[0] == 0) and not np.all(z[2] == 0)
