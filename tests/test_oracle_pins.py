"""Pins of the CPU oracle against facts that do not come from the oracle itself:
closed forms, invariants, special cases that reduce to a textbook result or a library
routine, and brute force on tiny inputs.  CPU only."""
import math
import os

import numpy as np
import pytest

import oracle as O
from block_diffusion_decoding_denoising_b200 import gen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bits(x):
    return gen.bf16_bits(np.asarray(x, dtype=np.float64))


# ------------------------------------------------------------------ number formats
def test_round_bf16_matches_independent_bit_trick():
    # gen.bf16_bits rounds through float32 with an integer carry trick; the oracle rounds a
    # double with frexp/nearbyint.  For float32-representable inputs they must agree.
    x = gen.normal_np(5, 4000, 3.0).astype(np.float32).astype(np.float64)
    x = np.concatenate([x, [1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 1e-40, 3e38]])
    ref = gen.bf16_to_f64(gen.bf16_bits(x))
    got = np.array([O.round_bf16(v) for v in x])
    np.testing.assert_array_equal(got, ref)


def test_round_bf16_ties_to_even():
    assert O.round_bf16(1.0 + 2 ** -8) == 1.0                 # tie -> even mantissa
    assert O.round_bf16(1.0 + 3 * 2 ** -8) == 1.0 + 2 ** -6   # tie -> even (up)
    assert O.round_bf16(1.0 + 2 ** -8 + 2 ** -20) == 1.0 + 2 ** -7


def _golden_table(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                rows.append(line.split())
    return rows


def test_e2m1_grid_roundtrip():
    for code, val in _golden_table("e2m1_grid.txt"):
        code, val = int(code, 0), float(val)
        assert O.e2m1_value(code) == val
        assert O.e2m1_encode(val) == code or val == 0.0


def test_e2m1_ties_and_saturation():
    # midpoints between grid neighbours go to the even code (even mantissa bit)
    assert O.e2m1_value(O.e2m1_encode(0.25)) == 0.0
    assert O.e2m1_value(O.e2m1_encode(0.75)) == 1.0
    assert O.e2m1_value(O.e2m1_encode(1.25)) == 1.0
    assert O.e2m1_value(O.e2m1_encode(1.75)) == 2.0
    assert O.e2m1_value(O.e2m1_encode(2.5)) == 2.0
    assert O.e2m1_value(O.e2m1_encode(3.5)) == 4.0
    assert O.e2m1_value(O.e2m1_encode(5.0)) == 4.0
    assert O.e2m1_value(O.e2m1_encode(-5.1)) == -6.0
    assert O.e2m1_value(O.e2m1_encode(100.0)) == 6.0
    assert O.e2m1_value(O.e2m1_encode(-0.26)) == -0.5


def test_e4m3_golden_encodings():
    for b, val in _golden_table("e4m3_values.txt"):
        b, val = int(b, 0), float(val)
        assert O.e4m3_value(b) == val
        assert O.e4m3_bits(val) == b
        assert O.e4m3_round(np.float32(val)) == val


def test_e4m3_all_codes_roundtrip_and_saturate():
    for b in range(0x7F):  # 0x7F is NaN in the fn variant
        v = O.e4m3_value(b)
        assert O.e4m3_bits(v) == b
        assert O.e4m3_round(np.float32(v)) == v
    assert O.e4m3_round(1e6) == 448.0
    assert O.e4m3_round(460.0) == 448.0
    # halfway between 1.0 and 1.125 -> even (1.0); between 1.125 and 1.25 -> 1.25
    assert O.e4m3_round(1.0625) == 1.0
    assert O.e4m3_round(1.1875) == 1.25


def test_nvfp4_exact_on_grid_blocks():
    # a block whose values are e2m1 grid points times a power-of-two scale is reproduced
    # Tensor scale S = 2^-10 exactly (global amax 6 * 448 * 2^-10), block scales are e4m3
    # values (448 for block 0, powers of two elsewhere), elements are e2m1 grid points.
    grid = np.array([O.e2m1_value(c) for c in range(16)])
    rng = np.random.default_rng(1)
    blocks = np.stack([grid[rng.permutation(16)] for _ in range(8)])
    blocks[:, 0] = 6.0  # every block reaches the top of the grid
    sig = np.array([448.0, 1.0, 2.0, 0.5, 64.0, 2.0 ** -6, 2.0 ** -9, 8.0])
    w = (blocks * sig[:, None] * 2.0 ** -10).reshape(4, 32)
    codes, scales, S = O.nvfp4_quantize(w)
    assert S == 2.0 ** -10
    np.testing.assert_array_equal([O.e4m3_value(b) for b in scales.reshape(-1)], sig)
    dq = O.nvfp4_dequant(codes, scales, S, 4, 32)
    np.testing.assert_array_equal(dq, w)


def test_nvfp4_idempotent_and_error_bound():
    w = gen.normal_np(3, 64 * 128, 0.02).reshape(64, 128).astype(np.float32)
    codes, scales, S = O.nvfp4_quantize(w)
    dq = O.nvfp4_dequant(codes, scales, S, 64, 128)
    # idempotent: quantizing the dequantized tensor reproduces it
    c2, s2, S2 = O.nvfp4_quantize(dq.astype(np.float32))
    dq2 = O.nvfp4_dequant(c2, s2, S2, 64, 128)
    np.testing.assert_allclose(dq2, dq, rtol=0, atol=1e-12 * np.abs(dq).max())
    # error bound: at most half of the largest e2m1 step (1.0, between 4 and 6) x sigma x S,
    # plus the fp32 rounding of the final product
    sig = np.array([O.e4m3_value(b) for b in scales.reshape(-1)]).reshape(64, 8)
    bound = np.repeat(sig, 16, axis=1) * S * 1.0 * (1 + 1e-6) + 1e-12
    assert np.all(np.abs(dq - w) <= bound)
    # and relative to the block amax the error is at most 1/6 + e4m3 rounding
    assert np.abs(dq - w).max() <= np.abs(w).max() / 6 * 1.1


# ------------------------------------------------------------------ row statistics
def test_rowstats_uniform_row_closed_form():
    V = 151936
    st = O.rowstats(np.zeros((2, V)), mask_id=-1)
    assert abs(st["entropy"][0] - math.log(V)) < 1e-9
    assert abs(st["maxprob"][0] - 1.0 / V) < 1e-15
    assert st["argmax"][0] == 0          # ties -> lowest id
    assert abs(st["lse"][0] - math.log(V)) < 1e-9


def test_rowstats_mask_exclusion():
    V = 512
    st = O.rowstats(np.zeros((1, V)), mask_id=V - 1)
    assert abs(st["entropy"][0] - math.log(V - 1)) < 1e-12
    l = np.zeros((1, V))
    l[0, V - 1] = 50.0                   # the mask id never wins
    st = O.rowstats(l, mask_id=V - 1)
    assert st["argmax"][0] != V - 1 and abs(st["maxprob"][0] - 1.0 / (V - 1)) < 1e-15


def test_rowstats_one_hot_dominant_and_sum_to_one():
    V = 1000
    l = gen.normal_np(7, 3 * V, 1.0).reshape(3, V)
    l[1, 123] = 80.0
    st = O.rowstats(l)
    assert st["argmax"][1] == 123 and abs(st["maxprob"][1] - 1.0) < 1e-12
    assert st["entropy"][1] < 1e-20
    # probabilities from lse sum to one, entropy matches scipy's definition
    from scipy.stats import entropy as sp_entropy
    p = np.exp(l - st["lse"][:, None])
    np.testing.assert_allclose(p.sum(1), 1.0, atol=1e-12)
    np.testing.assert_allclose(st["entropy"], sp_entropy(p, axis=1), rtol=1e-10)
    np.testing.assert_allclose(st["maxprob"], p.max(1), rtol=1e-12)
    np.testing.assert_array_equal(st["argmax"], l.argmax(1))


def test_rowstats_shift_invariance():
    l = gen.normal_np(8, 2 * 777, 2.0).reshape(2, 777)
    a, b = O.rowstats(l), O.rowstats(l + 13.25)
    np.testing.assert_allclose(a["entropy"], b["entropy"], rtol=1e-10)
    np.testing.assert_allclose(a["maxprob"], b["maxprob"], rtol=1e-10)
    np.testing.assert_array_equal(a["argmax"], b["argmax"])


# ------------------------------------------------------------------ LM head and P @ E
def test_lmhead_one_hot_p_reproduces_embedding_row():
    V, d = 300, 64
    E = bits(gen.normal_np(9, V * d, 0.02).reshape(V, d))
    x = gen.normal_np(10, 2 * d).reshape(2, d)
    P = np.zeros((2, V))
    P[0, 17] = 1.0
    P[1, 299] = 1.0
    out = O.lmhead(x, E, p_given=P)
    Ef = gen.bf16_to_f64(E)
    np.testing.assert_array_equal(out["s"][0], Ef[17])
    np.testing.assert_array_equal(out["s"][1], Ef[299])


def test_lmhead_uniform_p_gives_column_mean_and_logits_match_matmul():
    V, d = 256, 32
    E = bits(gen.normal_np(11, V * d, 0.5).reshape(V, d))
    Ef = gen.bf16_to_f64(E)
    x = np.zeros((1, d))           # zero hidden state -> uniform softmax
    out = O.lmhead(x, E)
    np.testing.assert_allclose(out["s"][0], Ef.mean(0), rtol=1e-12, atol=1e-15)
    x2 = gen.normal_np(12, 3 * d).reshape(3, d)
    out2 = O.lmhead(x2, E, want_logits=True)
    np.testing.assert_allclose(out2["logits"], x2 @ Ef.T, rtol=1e-12, atol=1e-12)
    p = np.exp(out2["logits"] - out2["lse"][:, None])
    np.testing.assert_allclose(out2["s"], p @ Ef, rtol=1e-10, atol=1e-14)


def test_lmhead_nvfp4_uses_the_dequantized_embedding():
    # NVFP4 E: a one-hot P reproduces the dequantized row (s = P E with E = q sigma S), and
    # with grid-representable x and E the logits are their exact product
    V, d = 96, 64
    Eg = _on_grid_rows(V, d, 21)
    codes, scales, S = O.nvfp4_quantize(Eg.astype(np.float32))
    Eq = dict(codes=codes, scales=scales, tscale=S, rows=V, cols=d)
    x = _on_grid_rows(2, d, 22)
    P = np.zeros((2, V))
    P[0, 5] = 1.0
    P[1, 95] = 1.0
    out = O.lmhead(x, Eq, p_given=P, act_fp4=True, want_logits=True)
    np.testing.assert_array_equal(out["s"][0], Eg[5])
    np.testing.assert_array_equal(out["s"][1], Eg[95])
    np.testing.assert_array_equal(out["logits"], x @ Eg.T)
    ref = O.rowstats(x @ Eg.T)
    np.testing.assert_array_equal(out["argmax"], ref["argmax"])
    np.testing.assert_allclose(out["lse"], ref["lse"], rtol=1e-12)


# ------------------------------------------------------------------ layers
def test_linear_exact_on_integers_and_matches_matmul():
    W = bits(np.arange(-6, 6, dtype=np.float64).reshape(3, 4))
    x = np.array([[1.0, 2.0, -3.0, 4.0]])
    np.testing.assert_array_equal(O.linear(x, W), x @ gen.bf16_to_f64(W).T)
    W2 = bits(gen.normal_np(13, 40 * 24).reshape(40, 24))
    x2 = gen.normal_np(14, 5 * 24).reshape(5, 24)
    np.testing.assert_allclose(O.linear(x2, W2), x2 @ gen.bf16_to_f64(W2).T, rtol=1e-12, atol=1e-12)


def _on_grid_rows(rows, cols, seed):
    """Rows whose 16-element blocks are e2m1 grid points x an e4m3 block scale x 2^-10, with a
    block at 6 x 448 x 2^-10 in every row: the NVFP4 round trip reproduces them exactly
    (row scale 2^-10, block scales exact)."""
    grid = np.array([O.e2m1_value(c) for c in range(16)])
    rng = np.random.default_rng(seed)
    sig_choices = np.array([448.0, 1.0, 2.0, 0.5, 64.0, 2.0 ** -6, 8.0, 16.0])
    out = np.zeros((rows, cols))
    for r in range(rows):
        for b in range(cols // 16):
            blk = grid[rng.integers(0, 16, 16)]
            blk[0] = 6.0
            sig = 448.0 if b == 0 else sig_choices[rng.integers(0, len(sig_choices))]
            out[r, b * 16:(b + 1) * 16] = blk * sig * 2.0 ** -10
    return out


def test_linear_nvfp4_exact_on_grid_operands():
    # weights and activations both exactly representable: the NVFP4 linear is the exact
    # fp64 product of the two (activation row scales, block scales and codes all exact)
    K, N = 64, 24
    w = _on_grid_rows(N, K, 7)
    codes, scales, S = O.nvfp4_quantize(w.astype(np.float32))
    assert S == 2.0 ** -10
    Wq = dict(codes=codes, scales=scales, tscale=S, rows=N, cols=K)
    x = _on_grid_rows(3, K, 8)
    np.testing.assert_array_equal(O.linear(x, Wq, act_fp4=True), x @ w.T)
    # weights alone: the activations stay fp64
    xr = gen.normal_np(9, 3 * K).reshape(3, K)
    np.testing.assert_allclose(O.linear(xr, Wq, act_fp4=False), xr @ w.T, rtol=1e-13, atol=1e-15)


def test_linear_nvfp4_quantizes_each_activation_row_by_itself():
    # act_fp4 = quantize every row with its own row scale, then the product with the
    # dequantized weights (a second row scaled by 2^20 changes nothing in the first)
    K, N = 64, 16
    w = gen.normal_np(10, N * K, 0.02).reshape(N, K).astype(np.float32)
    codes, scales, S = O.nvfp4_quantize(w)
    Wq = dict(codes=codes, scales=scales, tscale=S, rows=N, cols=K)
    wd = O.nvfp4_dequant(codes, scales, S, N, K)
    x = gen.normal_np(11, 2 * K).reshape(2, K)
    x[1] *= 2.0 ** 20
    xq = np.stack([O.nvfp4_dequant(*O.nvfp4_quantize(x[t:t + 1].astype(np.float32)), 1, K)[0] for t in range(2)])
    np.testing.assert_allclose(O.linear(x, Wq, act_fp4=True), xq @ wd.T, rtol=1e-12, atol=0)


def test_rmsnorm_constant_vector():
    g = bits(np.linspace(0.5, 2.0, 16))
    for c in (3.0, -0.25):
        out = O.rmsnorm(np.full((1, 16), c), g, 1e-12)
        np.testing.assert_allclose(out[0], np.sign(c) * gen.bf16_to_f64(g), rtol=1e-9)


def test_rope_identity_at_zero_norm_preserving_and_closed_form():
    x = gen.normal_np(15, 32)
    np.testing.assert_array_equal(O.rope(x, 0, 10000.0), x)
    y = O.rope(x, 1234, 10000.0)
    assert abs(np.linalg.norm(y) - np.linalg.norm(x)) < 1e-12
    # hd = 2: theta_0 = 1, so position p rotates (1, 0) by p radians
    np.testing.assert_allclose(O.rope(np.array([1.0, 0.0]), 5, 1e6), [math.cos(5), math.sin(5)],
                               rtol=1e-14)
    # pairing is (j, j + hd/2): for hd = 4 the second pair uses theta_1 = base^-1/2
    z = O.rope(np.array([0.0, 1.0, 0.0, 0.0]), 3, 100.0)
    np.testing.assert_allclose(z, [0.0, math.cos(0.3), 0.0, math.sin(0.3)], atol=1e-15)


def _attn_bruteforce_scipy(q, kc, vc, pos0, causal):
    from scipy.special import softmax
    nq, Hq, hd = q.shape
    Hkv = kc.shape[0]
    out = np.zeros_like(q)
    for i in range(nq):
        for h in range(Hq):
            g = h * Hkv // Hq
            n = pos0 + i + 1 if causal else pos0 + nq
            s = kc[g, :n] @ q[i, h] / math.sqrt(hd)
            out[i, h] = softmax(s) @ vc[g, :n]
    return out


@pytest.mark.parametrize("causal", [False, True])
def test_attention_matches_scipy_bruteforce(causal):
    nq, Hq, Hkv, hd, L, mc = 5, 4, 2, 16, 11, 24
    q = gen.normal_np(16, nq * Hq * hd).reshape(nq, Hq, hd)
    kc = gen.normal_np(17, Hkv * mc * hd).reshape(Hkv, mc, hd)
    vc = gen.normal_np(18, Hkv * mc * hd).reshape(Hkv, mc, hd)
    np.testing.assert_allclose(O.attention(q, kc, vc, L, causal),
                               _attn_bruteforce_scipy(q, kc, vc, L, causal), rtol=1e-12, atol=1e-12)


def test_attention_special_cases():
    hd = 8
    q = gen.normal_np(19, hd).reshape(1, 1, hd)
    kc = gen.normal_np(20, 4 * hd).reshape(1, 4, hd)
    vc = gen.normal_np(21, 4 * hd).reshape(1, 4, hd)
    # L = 0, one query: the only key is its own, the output is its value
    np.testing.assert_allclose(O.attention(q, kc, vc, 0)[0, 0], vc[0, 0], rtol=1e-15)
    # identical keys: uniform weights, output is the mean of the values
    kc2 = np.repeat(kc[:, :1], 4, axis=1)
    np.testing.assert_allclose(O.attention(q, kc2, vc, 3)[0, 0], vc[0].mean(0), rtol=1e-12)
    # causal: the first query of a prefill sees only key 0
    q3 = gen.normal_np(22, 3 * hd).reshape(3, 1, hd)
    np.testing.assert_allclose(O.attention(q3, kc, vc, 0, causal=True)[0, 0], vc[0, 0], rtol=1e-15)


def test_attention_gqa_with_equal_heads_is_mha():
    nq, H, hd, mc = 3, 2, 8, 10
    q = gen.normal_np(23, nq * H * hd).reshape(nq, H, hd)
    kc = gen.normal_np(24, H * mc * hd).reshape(H, mc, hd)
    vc = gen.normal_np(25, H * mc * hd).reshape(H, mc, hd)
    full = O.attention(q, kc, vc, 4)
    for h in range(H):
        single = O.attention(q[:, h:h + 1], kc[h:h + 1], vc[h:h + 1], 4)
        np.testing.assert_allclose(full[:, h], single[:, 0], rtol=1e-14)


# ------------------------------------------------------------------ commit rule
def test_commit_threshold_min1_and_topk():
    mp = np.array([0.3, 0.95, 0.2, 0.91, 0.5])
    am = np.arange(5) + 100
    n, tok, com = O.commit(mp, am, 0.9, 0, 0, np.full(5, -1), np.zeros(5))
    assert n == 2 and list(com) == [0, 1, 0, 1, 0] and tok[1] == 101 and tok[3] == 103
    n, tok, com = O.commit(mp, am, 0.99, 0, 0, np.full(5, -1), np.zeros(5))
    assert n == 1 and list(com) == [0, 1, 0, 0, 0]
    # min-1 ties -> lowest position; already committed positions are skipped
    n, tok, com = O.commit(np.array([0.4, 0.4, 0.9]), am[:3], 0.95, 0, 0, np.full(3, -1),
                           np.array([0, 0, 1]))
    assert n == 1 and list(com) == [1, 0, 1]
    n, tok, com = O.commit(mp, am, 0.0, 1, 2, np.full(5, -1), np.zeros(5))
    assert n == 2 and list(com) == [0, 1, 0, 1, 0]
    n, tok, com = O.commit(np.full(5, 0.1), am, 0.0, 1, 3, np.full(5, -1), np.zeros(5))
    assert list(com) == [1, 1, 1, 0, 0]


# ------------------------------------------------------------------ model level
@pytest.fixture(scope="module")
def tiny():
    cfg, w = gen.tiny_model(seed=0)
    return cfg, w


def _rounds(cfg, w, tau, mode, k):
    m = O.OracleModel(cfg, w)
    m.prefill(gen.prompt_np(cfg, 32))
    return m.decode_block(32, tau, mode, k)


def test_block_rounds_tau_above_one_commit_one_per_round(tiny):
    cfg, w = tiny
    r, _ = _rounds(cfg, w, 1.5, 0, 0)
    assert r == cfg["block_size"]


def test_block_rounds_tau_nonpositive_single_round(tiny):
    cfg, w = tiny
    r, _ = _rounds(cfg, w, 0.0, 0, 0)
    assert r == 1


@pytest.mark.parametrize("k", [1, 3, 8])
def test_block_rounds_fixed_k(tiny, k):
    cfg, w = tiny
    r, _ = _rounds(cfg, w, 0.0, 1, k)
    assert r == math.ceil(cfg["block_size"] / k)


@pytest.mark.parametrize("std", [0.02, 0.125])
def test_round_invariants_monotone_commits_and_residual_rows(std):
    cfg, w = gen.tiny_model(seed=0, std=std)
    B, d = cfg["block_size"], cfg["d"]
    m = O.OracleModel(cfg, w)
    m.prefill(gen.prompt_np(cfg, 32))
    tok = np.full(B, cfg["mask_id"], np.int32)
    com = np.zeros(B, np.uint8)
    s = np.zeros((B, d))
    rnd = 0
    while not com.all():
        n, st, stats = m.round(tok, com, s, rnd, 32, 0.9, 0, 0)
        assert n >= 1
        assert np.all(st["committed"] >= com)                       # never shrinks
        assert np.all(st["tokens"][com == 1] == tok[com == 1])       # committed tokens stay
        assert np.all(st["s"][st["committed"] == 1] == 0.0)          # committed rows carry no residual
        assert np.all(np.abs(st["s"][st["committed"] == 0]).sum(1) > 0)
        assert np.all(stats["argmax"] != cfg["mask_id"])
        assert st["round"] == rnd + 1
        tok, com, s, rnd = st["tokens"], st["committed"], st["s"], st["round"]
        assert rnd <= B
    if std > 0.1:
        # distinct positions: some rounds commit several positions by threshold
        assert rnd < B


def test_generate_deterministic_and_shapes(tiny):
    cfg, w = tiny
    prompt = gen.prompt_np(cfg, 32)
    outs = []
    for _ in range(2):
        m = O.OracleModel(cfg, w)
        nb, out, rpb = m.generate(prompt, 32, 0.9, 0, 0)
        assert nb == 4 and np.all(rpb >= 1) and np.all(rpb <= cfg["block_size"])
        assert np.all((out >= 0) & (out < cfg["vocab"] - 1))
        outs.append((out.copy(), rpb.copy()))
    np.testing.assert_array_equal(outs[0][0], outs[1][0])
    np.testing.assert_array_equal(outs[0][1], outs[1][1])


def _zero(wmat):
    return np.zeros_like(wmat)


def test_zero_layer_outputs_reduce_to_embedding_head(tiny):
    # With W_o = W_down = 0 every layer adds nothing to the residual stream, so the
    # logits are RMSNorm(E[x]) E^T, whose argmax is x itself for random embeddings.
    cfg, w = tiny
    w2 = dict(w)
    w2["layers"] = [dict(l, w_o=_zero(l["w_o"]), w_down=_zero(l["w_down"])) for l in w["layers"]]
    m = O.OracleModel(cfg, w2, act_round=False)
    toks = np.array([3, 77, 200, 5, 9, 400, 13, 21], np.int32)
    xf = m.forward(toks, None, 0)
    st = O.lmhead(xf, w["embed"], mask_id=cfg["mask_id"])
    np.testing.assert_array_equal(st["argmax"], toks)
    E = gen.bf16_to_f64(w["embed"])
    ref = E[toks] / np.sqrt((E[toks] ** 2).mean(1, keepdims=True) + cfg["rms_eps"])
    np.testing.assert_allclose(xf, ref, rtol=1e-12)


def test_adapter_adds_w_a_times_s(tiny):
    # W_a = identity and s = E[y]: the input row is E[x] + E[y] (residual self-conditioning)
    cfg, w = tiny
    d = cfg["d"]
    w2 = dict(w)
    w2["w_adapter"] = bits(np.eye(d))
    w2["layers"] = [dict(l, w_o=_zero(l["w_o"]), w_down=_zero(l["w_down"])) for l in w["layers"]]
    m = O.OracleModel(cfg, w2, act_round=False)
    E = gen.bf16_to_f64(w["embed"])
    toks = np.array([3, 77], np.int32)
    s = np.stack([E[150], E[151]])
    xf = m.forward(toks, s, 0)
    h = E[toks] + s
    ref = h / np.sqrt((h ** 2).mean(1, keepdims=True) + cfg["rms_eps"])
    np.testing.assert_allclose(xf, ref, rtol=1e-12)


def test_kv_cache_prefill_vs_block_of_one(tiny):
    # A block of one token at position P attending to [0, P] is the last row of a causal
    # prefill of P + 1 tokens: both must write identical K/V rows, and the prefill of the
    # first P tokens must not depend on token P (causality).
    cfg, w = tiny
    prompt = gen.prompt_np(cfg, 20)
    a = O.OracleModel(cfg, w, act_round=False)
    a.prefill(prompt)
    b = O.OracleModel(cfg, w, act_round=False)
    b.prefill(prompt[:19])
    b.forward(prompt[19:], None, 19, want_xf=False)
    np.testing.assert_allclose(a.kc[:, :, :20], b.kc[:, :, :20], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(a.vc[:, :, :20], b.vc[:, :, :20], rtol=1e-12, atol=1e-14)
    c = O.OracleModel(cfg, w, act_round=False)
    p2 = prompt.copy()
    p2[19] = (p2[19] + 1) % 500
    c.prefill(p2)
    np.testing.assert_array_equal(a.kc[:, :, :19], c.kc[:, :, :19])


def test_block_attention_is_bidirectional(tiny):
    # changing the last token of a block changes the hidden state of its first position
    cfg, w = tiny
    m = O.OracleModel(cfg, w, act_round=False)
    m.prefill(gen.prompt_np(cfg, 16))
    t1 = np.array([1, 2, 3, 4, 5, 6, 7, 8], np.int32)
    t2 = t1.copy()
    t2[-1] = 300
    x1 = m.forward(t1, None, 16)
    x2 = m.forward(t2, None, 16)
    assert np.abs(x1[0] - x2[0]).max() > 1e-6


# ---------------------------------------------------------------- NVFP4 rounding margins
def _lmhead_qmargin(rows):
    """qmargin of orc_lmhead's activation quantization for the given x rows (d = 32)."""
    x = np.array(rows, np.float64)
    B, d = x.shape
    E = gen.bf16_bits(gen.normal_np(99, 8 * d, 0.1).reshape(8, d))
    Ef = (E.astype(np.uint32) << np.uint32(16)).view(np.float32)
    codes, scales, S = O.nvfp4_quantize(Ef)
    q = {"codes": codes, "scales": scales, "tscale": S, "rows": 8, "cols": d}
    return O.lmhead(x, q, act_fp4=True)["qmargin"], O.lmhead(x, q, act_fp4=False)["qmargin"]


def test_qmargin_pins():
    """Rows whose quantization decisions sit at known distances from the rounding boundaries
    (the e2m1 midpoints 0.25 .. 5 and the e4m3 midpoints (k + 1/2) q):
      row 0: block 0 on the e2m1 grid with amax/(6S) = 448 (saturated, 16/432 above the
             midpoint 432), block 1 on the grid with block scale 96 (4 below the midpoint
             100; e2m1 values sit at least 1/7 from a midpoint) -> 16/432;
      row 1: block 1 scaled to put amax/(6S) on the e4m3 midpoint 100 -> ~0;
      row 2: one element exactly on the e2m1 midpoint 2.5 -> ~0."""
    grid = [6, 4, 3, 2, 1.5, 1, 0.5, 0, -6, -4, -3, -2, -1.5, -1, -0.5, 0]
    b0 = np.array(grid, np.float64)
    r0 = np.concatenate([b0, b0 * 96.0 / 448.0])
    r1 = np.concatenate([b0, b0 * 100.0 / 448.0])
    b2 = b0.copy()
    b2[1] = 2.5
    r2 = np.concatenate([b2, b0 * 96.0 / 448.0])
    qm, qm_off = _lmhead_qmargin([r0, r1, r2])
    assert abs(qm[0] - 16.0 / 432.0) < 1e-5, qm
    assert qm[1] < 1e-5 and qm[2] < 1e-5, qm
    assert np.all(np.isinf(qm_off))


# ------------------------------------------------------------------ layer composition
# Closed forms of one pre-norm layer (reading R6) with structured weights: scaled identity
# and permutation blocks make every sub-block's output a formula in the input row, so that
# a slip in the forward pass's composition (silu on the wrong operand, a sigmoid for the
# SiLU, the gate and up rows exchanged, the wrong norm gain, RoPE applied to v or missing
# on q, the q/k/v rows taken in the wrong order, W_o transposed, a dropped residual) moves
# the result far outside the rounding error of the fp64 oracle.
def _closed_form_layer_setup(tiny):
    cfg, w = tiny
    d, F, hd = cfg["d"], cfg["ffn"], cfg["head_dim"]
    ga = 0.5 + 0.25 * (np.arange(d) % 4)           # attn_norm gains (bf16-exact)
    gm = 2.0 - 0.25 * (np.arange(d) % 5)           # mlp_norm gains
    gf = 1.0 + 0.125 * (np.arange(d) % 3)          # final_norm gains
    lw = dict(w["layers"][0], attn_norm=bits(ga), mlp_norm=bits(gm))
    w2 = dict(w, final_norm=bits(gf))
    return cfg, w2, lw, ga, gm, gf


def _rms(x, g, eps):
    return x / np.sqrt(np.mean(x * x) + eps) * g


def _silu(x):
    return x / (1.0 + np.exp(-x))


def test_pin_mlp_sub_block_closed_form(tiny):
    # W_qkv = 0: q = k = v = 0, the attention output is the mean of zero values, so W_o
    # (left random) adds nothing and the MLP sees RMSNorm(E[x]) * g_mlp.  With
    # W_gate = a [I 0], W_up = b [P 0] (P a permutation) and W_down = c [I 0]:
    #   h = E[x] + c * silu(a xn) * (b xn[pi]),  xf = RMSNorm(h) * g_final.
    cfg, w2, lw, ga, gm, gf = _closed_form_layer_setup(tiny)
    d, F = cfg["d"], cfg["ffn"]
    a, b, c = 2.0, 1.5, 0.75
    pi = (np.arange(d) * 7 + 3) % d                 # a permutation of 0..d-1 (7 is odd, d = 64)
    Wg = np.zeros((F, d)); Wg[np.arange(d), np.arange(d)] = a
    Wu = np.zeros((F, d)); Wu[np.arange(d), pi] = b
    Wd = np.zeros((d, F)); Wd[np.arange(d), np.arange(d)] = c
    lw.update(w_qkv=bits(np.zeros((cfg["n_q_heads"] + 2 * cfg["n_kv_heads"]) * cfg["head_dim"] * d)
                         .reshape(-1, d)), w_gate=bits(Wg), w_up=bits(Wu), w_down=bits(Wd))
    w2["layers"] = [lw]
    m = O.OracleModel(cfg, w2, act_round=False)
    E = gen.bf16_to_f64(w2["embed"])
    toks = np.array([3, 77, 200, 5], np.int32)
    xf = m.forward(toks, None, 7)
    eps = cfg["rms_eps"]
    for i, t in enumerate(toks):
        xn = _rms(E[t], gm, eps)
        h = E[t] + c * _silu(a * xn) * (b * xn[pi])
        np.testing.assert_allclose(xf[i], _rms(h, gf, eps), rtol=1e-11, atol=1e-13)
    # the gate and up roles are not interchangeable here: silu(u) * g is far away
    xn = _rms(E[toks[0]], gm, eps)
    swapped = _rms(E[toks[0]] + c * _silu(b * xn[pi]) * (a * xn), gf, eps)
    assert np.abs(swapped - xf[0]).max() > 1e-3


def _rope_np(x, pos, base):
    """NeoX rotate-half rotation of one head vector (pairs j, j + hd/2)."""
    half = len(x) // 2
    th = base ** (-2.0 * np.arange(half) / len(x))
    c, s = np.cos(pos * th), np.sin(pos * th)
    return np.concatenate([x[:half] * c - x[half:] * s, x[:half] * s + x[half:] * c])


def test_pin_attention_sub_block_closed_form(tiny):
    # One block token at position p over an injected prefix of p keys (layer 0, one kv head
    # shared by both q heads).  Structured W_qkv rows (q heads, then the k head, then the v
    # head), each reading a different slice of xn = RMSNorm(E[x]) * g_attn:
    #   q0 = al xn[0:32], q1 = be xn[32:64], k = xn[16:48], v = ga_ xn[perm]
    # RoPE rotates q0, q1 and k at position p, not v.  W_o is a scaled cyclic shift
    # ((W_o o)[n] = de o[(n+1) % 64]) and W_down = 0, so
    #   h = E[x] + de shift(concat(o0, o1)),  o_h = softmax(rope(q_h) . K / sqrt(32)) V
    # with K, V the injected rows followed by the block's own (rope(k), v).
    cfg, w2, lw, ga, gm, gf = _closed_form_layer_setup(tiny)
    d, hd, F = cfg["d"], cfg["head_dim"], cfg["ffn"]
    Hq, Hkv = cfg["n_q_heads"], cfg["n_kv_heads"]
    assert (Hq, Hkv, hd, d) == (2, 1, 32, 64)
    al, be, ga_, de = 1.5, 0.75, 2.0, 0.5
    perm = (np.arange(hd) * 5 + 11) % d
    Wqkv = np.zeros(((Hq + 2 * Hkv) * hd, d))
    Wqkv[np.arange(32), np.arange(32)] = al
    Wqkv[32 + np.arange(32), 32 + np.arange(32)] = be
    Wqkv[64 + np.arange(32), 16 + np.arange(32)] = 1.0
    Wqkv[96 + np.arange(32), perm] = ga_
    Wo = np.zeros((d, Hq * hd))
    Wo[np.arange(d), (np.arange(d) + 1) % d] = de
    lw.update(w_qkv=bits(Wqkv), w_o=bits(Wo), w_down=bits(np.zeros((d, F))))
    w2["layers"] = [lw]
    m = O.OracleModel(cfg, w2, act_round=False)
    p, base, eps = 3, cfg["rope_theta"], cfg["rms_eps"]
    Kp = gen.normal_np(61, p * hd).reshape(p, hd)
    Vp = gen.normal_np(62, p * hd).reshape(p, hd)
    m.kc[0, 0, :p] = Kp
    m.vc[0, 0, :p] = Vp
    tok = 123
    xf = m.forward(np.array([tok], np.int32), None, p)
    E = gen.bf16_to_f64(w2["embed"])
    xn = _rms(E[tok], ga, eps)
    q = [_rope_np(al * xn[0:32], p, base), _rope_np(be * xn[32:64], p, base)]
    k = _rope_np(xn[16:48], p, base)
    v = ga_ * xn[perm]
    # the block's K/V rows in the cache: k rotated, v as projected
    np.testing.assert_allclose(m.kc[0, 0, p], k, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(m.vc[0, 0, p], v, rtol=1e-12, atol=1e-14)
    K = np.vstack([Kp, k])
    V = np.vstack([Vp, v])
    o = []
    for qh in q:
        sc = K @ qh / np.sqrt(hd)
        e = np.exp(sc - sc.max())
        o.append(e @ V / e.sum())
    oc = np.concatenate(o)
    h = E[tok] + de * oc[(np.arange(d) + 1) % d]
    np.testing.assert_allclose(xf[0], _rms(h, gf, eps), rtol=1e-11, atol=1e-13)
    # unrotated queries (a plausible slip) give a visibly different row
    o_bad = []
    for qh in (al * xn[0:32], be * xn[32:64]):
        sc = K @ qh / np.sqrt(hd)
        e = np.exp(sc - sc.max())
        o_bad.append(e @ V / e.sum())
    ob = np.concatenate(o_bad)
    bad = _rms(E[tok] + de * ob[(np.arange(d) + 1) % d], gf, eps)
    assert np.abs(bad - xf[0]).max() > 1e-4


# ------------------------------------------------------------------ FP8 KV cache (reading R13)
def test_kv_fp8_rows_on_the_e4m3_grid_round_trip():
    # rows made of golden e4m3 values (OCP OFP8 E4M3, tests/golden/e4m3_values.txt) times a
    # power of two, with 448 present: the scale is exactly that power of two and every value
    # and code comes back unchanged
    table = [(int(b, 0), float(v)) for b, v in _golden_table("e4m3_values.txt")]
    vals = np.array([v for _, v in table] + [448.0])
    signs = np.where(np.arange(len(vals)) % 3 == 1, -1.0, 1.0)
    for p2 in (2.0 ** -7, 1.0, 2.0 ** 5):
        row = np.resize(vals * signs, 32) * p2
        row[5] = 448.0 * p2
        codes, scales, out = O.kv_quantize(row)
        assert scales[0] == np.float32(p2)
        np.testing.assert_array_equal(out[0], row)
        for c, x in zip(codes[0], row / p2):
            assert O.e4m3_value(int(c) & 0x7F) == abs(x) and (int(c) >> 7) == (1 if x < 0 else 0)


def test_kv_fp8_idempotent_error_bound_saturation_and_zero_rows():
    x = gen.normal_np(91, 8 * 128, 1.7).reshape(8, 128)
    x[3] *= 1e-3
    x[5] = 0.0
    codes, scales, out = O.kv_quantize(x)
    for r in range(8):
        if r == 5:
            assert scales[r] == 0.0 and np.all(codes[r] == 0) and np.all(out[r] == 0.0)
            continue
        s = float(scales[r])
        assert s == np.float32(np.float32(np.abs(x[r]).max()) / np.float32(448.0))
        j = int(np.argmax(np.abs(x[r])))
        assert int(codes[r][j]) & 0x7F == 0x7E  # the amax element is +-448 * s
        # e4m3 keeps 4 significant bits: relative error at most 2^-4 in the normal range, and at
        # most half the subnormal quantum (2^-10 * s) below it
        err = np.abs(out[r] - x[r])
        assert np.all(err <= np.maximum(np.abs(x[r]) * 2.0 ** -4, 2.0 ** -10 * s) * (1 + 1e-6))
        c2, s2, out2 = O.kv_quantize(out[r])
        np.testing.assert_array_equal(out2[0], out[r])


def test_pin_kv_fp8_applies_to_k_and_v_rows_only(tiny):
    # the structured attention sub-block above with an FP8 KV cache: the cached K and V rows are
    # the quantized closed forms, and the attention reads those stored values
    cfg, w2, lw, ga, gm, gf = _closed_form_layer_setup(tiny)
    cfg = dict(cfg, kv_fmt=1)
    d, hd, F = cfg["d"], cfg["head_dim"], cfg["ffn"]
    perm = (np.arange(hd) * 5 + 11) % d
    Wqkv = np.zeros((4 * hd, d))
    Wqkv[np.arange(32), np.arange(32)] = 1.5
    Wqkv[32 + np.arange(32), 32 + np.arange(32)] = 0.75
    Wqkv[64 + np.arange(32), 16 + np.arange(32)] = 1.0
    Wqkv[96 + np.arange(32), perm] = 2.0
    Wo = np.zeros((d, 2 * hd))
    Wo[np.arange(d), np.arange(d)] = 1.0
    lw.update(w_qkv=bits(Wqkv), w_o=bits(Wo), w_down=bits(np.zeros((d, F))))
    w2["layers"] = [lw]
    m = O.OracleModel(cfg, w2, act_round=False)
    p, base, eps, tok = 3, cfg["rope_theta"], cfg["rms_eps"], 123
    Kp = O.kv_quantize(gen.normal_np(63, p * hd).reshape(p, hd))[2]
    Vp = O.kv_quantize(gen.normal_np(64, p * hd).reshape(p, hd))[2]
    m.kc[0, 0, :p] = Kp
    m.vc[0, 0, :p] = Vp
    xf = m.forward(np.array([tok], np.int32), None, p)
    E = gen.bf16_to_f64(w2["embed"])
    xn = _rms(E[tok], ga, eps)
    k = O.kv_quantize(_rope_np(xn[16:48], p, base))[2][0]
    v = O.kv_quantize(2.0 * xn[perm])[2][0]
    np.testing.assert_array_equal(m.kc[0, 0, p], k)
    np.testing.assert_array_equal(m.vc[0, 0, p], v)
    q = [_rope_np(1.5 * xn[0:32], p, base), _rope_np(0.75 * xn[32:64], p, base)]  # q not quantized
    K, V = np.vstack([Kp, k]), np.vstack([Vp, v])
    o = []
    for qh in q:
        sc = K @ qh / np.sqrt(hd)
        e = np.exp(sc - sc.max())
        o.append(e @ V / e.sum())
    np.testing.assert_allclose(xf[0], _rms(E[tok] + np.concatenate(o), gf, eps), rtol=1e-11, atol=1e-13)


# ------------------------------------------------------------------ routed-expert MLP (R14)
def _bits_f32(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def _moe(E, k, F, d, seed, router_std=0.3, w_std=0.2, fp4=False):
    rng = np.random.default_rng(seed)
    gate = gen.bf16_bits(rng.normal(0, w_std, (E * F, d)))
    up = gen.bf16_bits(rng.normal(0, w_std, (E * F, d)))
    down = gen.bf16_bits(rng.normal(0, w_std, (d, E * F)))
    if fp4:
        def q(w):
            c, s, S = O.nvfp4_quantize(_bits_f32(w))
            return {"codes": c, "scales": s, "tscale": S, "rows": w.shape[0], "cols": w.shape[1]}
        gate, up, down = q(gate), q(up), q(down)
    return dict(n_experts=E, top_k=k, ffn_expert=F, w_router=gen.bf16_bits(rng.normal(0, router_std, (E, d))),
                norm=gen.bf16_bits(np.ones(d)), gate=gate, up=up, down=down)


def test_pin_moe_uniform_router_takes_the_lowest_indices_with_equal_weights():
    """All router logits equal (W_r = 0): every expert has probability 1/E, so the top-k rule
    with ties to the lower index selects experts 0..k-1, each with weight 1/k."""
    moe = _moe(6, 3, 16, 32, seed=1)
    moe["w_router"] = np.zeros_like(moe["w_router"])
    r = O.moe_mlp(np.random.default_rng(2).normal(0, 1, (4, 32)), moe, act_fp4=False)
    assert np.array_equal(r["idx"], np.tile(np.arange(3, dtype=np.int32), (4, 1)))
    np.testing.assert_array_equal(r["w"], np.full((4, 3), 1.0 / 3.0))
    np.testing.assert_array_equal(r["logits"], 0.0)


def test_pin_moe_expert_permutation_invariance():
    """Relabelling the experts (router rows, gate/up row blocks and down column blocks
    permuted together) leaves the output unchanged and maps the selections through the
    permutation: catches an expert slice or a router row read at the wrong index."""
    E, k, F, d, T = 5, 2, 16, 32, 6
    moe = _moe(E, k, F, d, seed=3)
    h = np.random.default_rng(4).normal(0, 1, (T, d))
    perm = np.array([3, 0, 4, 1, 2])
    pm = dict(moe)
    pm["w_router"] = moe["w_router"][perm]
    rows = np.concatenate([np.arange(e * F, (e + 1) * F) for e in perm])
    pm["gate"] = moe["gate"][rows]
    pm["up"] = moe["up"][rows]
    pm["down"] = moe["down"][:, rows]
    a = O.moe_mlp(h, moe, act_fp4=False)
    b = O.moe_mlp(h, pm, act_fp4=False)
    np.testing.assert_allclose(b["h_out"], a["h_out"], rtol=1e-12, atol=1e-12)
    # new expert j is old expert perm[j]
    assert np.array_equal(perm[b["idx"]], a["idx"])
    np.testing.assert_allclose(b["w"], a["w"], rtol=1e-12)


def test_pin_moe_scaled_identity_experts_closed_form():
    """Experts G_e = a_e I, U_e = b_e I, D_e = c_e I (d = F, bf16-exact scalars) make every
    expert elementwise: out = h + sum_e w_e c_e silu(a_e x) b_e x with x = RMSNorm(h).  With a
    router that puts one expert far ahead (k = 1) the weight is exactly 1; with W_r = 0 and
    k = 2 the weights are 1/2 on experts 0 and 1."""
    E, d = 3, 16
    a = np.array([0.5, 1.0, 2.0])
    b = np.array([1.0, -0.5, 0.25])
    c = np.array([2.0, 1.0, -1.0])
    I = np.eye(d)
    gate = gen.bf16_bits(np.concatenate([a[e] * I for e in range(E)]))
    up = gen.bf16_bits(np.concatenate([b[e] * I for e in range(E)]))
    down = gen.bf16_bits(np.concatenate([c[e] * I for e in range(E)], axis=1))
    h = np.random.default_rng(5).normal(0, 1, (2, d))
    x = h / np.sqrt(np.mean(h ** 2, axis=1, keepdims=True) + 1e-6)
    silu = lambda v: v / (1.0 + np.exp(-v))
    # router: expert 2 far ahead for every row (logit 8 * sum(x) with x summed ... use a
    # router row of +1 on coordinate 0 scaled by the sign of x_0 so its logit is large)
    wr = np.zeros((E, d))
    for_row = np.sign(x[:, 0])
    assert np.all(for_row == for_row[0])
    wr[2, 0] = 64.0 * for_row[0]
    moe = dict(n_experts=E, top_k=1, ffn_expert=d, w_router=gen.bf16_bits(wr), norm=gen.bf16_bits(np.ones(d)),
               gate=gate, up=up, down=down)
    r = O.moe_mlp(h, moe, act_fp4=False)
    assert np.array_equal(r["idx"][:, 0], [2, 2])
    np.testing.assert_array_equal(r["w"], 1.0)
    want = h + c[2] * silu(a[2] * x) * b[2] * x
    np.testing.assert_allclose(r["h_out"], want, rtol=1e-12, atol=1e-12)
    moe["w_router"] = gen.bf16_bits(np.zeros((E, d)))
    moe["top_k"] = 2
    r = O.moe_mlp(h, moe, act_fp4=False)
    want = h + 0.5 * sum(c[e] * silu(a[e] * x) * b[e] * x for e in (0, 1))
    np.testing.assert_allclose(r["h_out"], want, rtol=1e-12, atol=1e-12)


def test_pin_moe_single_expert_nvfp4_is_the_dense_mlp():
    """E = k = 1 with NVFP4 weights: the weight is exactly 1, so the sub-block is the dense
    NVFP4 MLP built from the pinned linear (each input row quantized, R8):
    h + Q(silu(Q(x) G^T) * Q(x) U^T) D^T."""
    F, d = 64, 64
    moe = _moe(1, 1, F, d, seed=6, fp4=True)
    h = np.random.default_rng(7).normal(0, 1, (5, d))
    r = O.moe_mlp(h, moe, act_fp4=True)
    x = O.rmsnorm(h, moe["norm"], 1e-6)
    g = O.linear(x, moe["gate"], act_fp4=True)
    u = O.linear(x, moe["up"], act_fp4=True)
    act = g / (1.0 + np.exp(-g)) * u
    want = h + O.linear(act, moe["down"], act_fp4=True)
    np.testing.assert_allclose(r["h_out"], want, rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(r["w"], 1.0)
