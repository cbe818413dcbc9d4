"""Per-kernel parity of the CUDA path (through the C ABI) against the CPU oracle, on
seeded inputs: the tensor-core GEMM, block-diffusion attention (the attention sweep
shapes), the fused LM head with row statistics and P E (the single-round LM-head
workload), the residual adapter, the commit rule and the NVFP4 quantizer."""
import numpy as np
import pytest

import oracle as O
from block_diffusion_decoding_denoising_b200 import gen
from helpers import (RTOL_BF16, assert_close, bf16_f64, from_torch_bf16, rel_err, to_torch_bf16,
                     unambiguous_argmax)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from block_diffusion_decoding_denoising_b200 import build, dlm
    build.build()
    dlm.lib()
    return dlm


def _bits(seed, shape, std=1.0):
    return gen.bf16_bits(gen.normal_np(seed, int(np.prod(shape)), std).reshape(shape))


# ------------------------------------------------------------------ GEMM
GEMM_SHAPES = [(32, 6144, 2560), (32, 2560, 9728), (8, 200, 320), (5, 64, 64), (33, 300, 1000),
               (100, 384, 192), (200, 256, 512), (256, 130, 128), (1, 128, 64), (64, 19456, 256)]


@pytest.mark.parametrize("T,N,K", GEMM_SHAPES)
def test_gemm_tcgen05_parity(lib, T, N, K):
    xb = _bits(100 + T, (T, K))
    wb = _bits(200 + N, (N, K), 0.02)
    y = lib.gemm_bf16(to_torch_bf16(xb), to_torch_bf16(wb)).cpu().numpy().astype(np.float64)
    ref = O.linear(bf16_f64(xb), wb)
    # identical bf16 operands: only the fp32 accumulation order differs
    assert_close(y, ref, 1e-3, "gemm %dx%dx%d" % (T, N, K))


@pytest.mark.parametrize("T,N,K", [(32, 6144, 2560), (8, 200, 320), (100, 384, 192), (128, 512, 1024)])
def test_gemm_split_activation_parity(lib, T, N, K):
    """x carried as a bf16 pair hi + lo: the GEMM must match the fp64 product with x
    exact to about 16 significant bits, far tighter than a single bf16 rounding."""
    import torch
    x = gen.normal_np(300 + T, T * K).reshape(T, K).astype(np.float32)
    wb = _bits(400 + N, (N, K), 0.02)
    y = lib.gemm_bf16x2(torch.from_numpy(x).cuda(), to_torch_bf16(wb)).cpu().numpy()
    ref = O.linear(x.astype(np.float64), wb)
    e = assert_close(y, ref, 5e-5, "split gemm %dx%dx%d" % (T, N, K))
    # a single bf16 rounding of x would be two orders of magnitude worse
    xb = gen.bf16_bits(x.astype(np.float64))
    assert rel_err(O.linear(bf16_f64(xb), wb), ref) > 20 * e


# ------------------------------------------------------------------ attention
def _attn_case(lib, B, L, Hq=32, Hkv=8, hd=128, causal=False, rows=None, seed=0):
    import torch
    q, k, v = gen.attention_inputs_torch(B, L, Hq, Hkv, hd, seed=seed)
    o = lib.bd_attention(q, k, v, L, causal=causal)
    torch.cuda.synchronize()
    qf = bf16_f64(from_torch_bf16(q))
    kf = bf16_f64(from_torch_bf16(k))
    vf = bf16_f64(from_torch_bf16(v))
    of = bf16_f64(from_torch_bf16(o))
    if rows is None:
        ref = O.attention(qf, kf, vf, L, causal)
        return of, ref
    # sampled query rows: non-causal queries all see keys [0, L + B), so a subset of
    # rows is evaluated at pos0 = L + B - len(rows) with the same key range
    sel = np.array(rows)
    ref = O.attention(qf[sel], kf, vf, L + B - len(sel), False)
    return of[sel], ref


@pytest.mark.parametrize("B", [4, 16, 32, 64])
@pytest.mark.parametrize("L", [1024, 4096])
def test_attention_sweep_full(lib, B, L):
    got, ref = _attn_case(lib, B, L)
    assert_close(got, ref, RTOL_BF16, "attention B=%d L=%d" % (B, L))


@pytest.mark.parametrize("B", [4, 16, 32, 64])
@pytest.mark.parametrize("L", [16384, 65536])
def test_attention_sweep_sampled_rows(lib, B, L):
    rows = sorted({0, B // 2, B - 1})
    got, ref = _attn_case(lib, B, L, rows=rows)
    assert_close(got, ref, RTOL_BF16, "attention B=%d L=%d rows %s" % (B, L, rows))


def test_attention_empty_prefix_and_tiny_heads(lib):
    got, ref = _attn_case(lib, 8, 0, Hq=2, Hkv=1, hd=32)
    assert_close(got, ref, RTOL_BF16, "L=0 tiny heads")
    got, ref = _attn_case(lib, 1, 0, Hq=4, Hkv=4, hd=64)
    assert_close(got, ref, RTOL_BF16, "one query, MHA")


@pytest.mark.parametrize("T,L", [(100, 37), (256, 0), (64, 300)])
def test_attention_causal_prefill(lib, T, L):
    got, ref = _attn_case(lib, T, L, Hq=8, Hkv=2, hd=128, causal=True)
    assert_close(got, ref, RTOL_BF16, "causal T=%d L=%d" % (T, L))


# ------------------------------------------------------------------ attention on an FP8 KV cache
def _fp8_attn_case(lib, B, L, Hq=32, Hkv=8, hd=128, causal=False, rows=None, seed=0):
    """K and V quantized per row by the oracle's FP8 KV quantizer (reading R13); the GPU reads
    the codes and scales, the oracle attends over the stored values."""
    import torch
    q, k, v = gen.attention_inputs_torch(B, L, Hq, Hkv, hd, seed=seed)
    mc = k.shape[1]
    mc4 = (mc + 3) // 4 * 4
    kf = bf16_f64(from_torch_bf16(k))
    vf = bf16_f64(from_torch_bf16(v))
    kc, ks, kq = O.kv_quantize(kf.reshape(-1, hd))
    vc, vs, vq = O.kv_quantize(vf.reshape(-1, hd))

    def dev(codes, scales):
        c = np.zeros((Hkv, mc4, hd), np.uint8)
        sc = np.zeros((Hkv, mc4), np.float32)
        c[:, :mc] = codes.reshape(Hkv, mc, hd)
        sc[:, :mc] = scales.reshape(Hkv, mc)
        return torch.from_numpy(c).cuda(), torch.from_numpy(sc).cuda()

    kcd, ksd = dev(kc, ks)
    vcd, vsd = dev(vc, vs)
    o = lib.bd_attention_fp8(q, kcd, ksd, vcd, vsd, L, causal=causal)
    torch.cuda.synchronize()
    qf = bf16_f64(from_torch_bf16(q))
    of = bf16_f64(from_torch_bf16(o))
    kq, vq = kq.reshape(Hkv, mc, hd), vq.reshape(Hkv, mc, hd)
    if rows is None:
        return of, O.attention(qf, kq, vq, L, causal)
    sel = np.array(rows)
    return of[sel], O.attention(qf[sel], kq, vq, L + B - len(sel), False)


@pytest.mark.parametrize("B,L", [(32, 1024), (64, 4096), (4, 2048), (1, 0), (16, 300)])
def test_attention_fp8_kv(lib, B, L):
    got, ref = _fp8_attn_case(lib, B, L)
    assert_close(got, ref, RTOL_BF16, "fp8 attention B=%d L=%d" % (B, L))


@pytest.mark.parametrize("B,L", [(32, 16384), (4, 65536)])
def test_attention_fp8_kv_sampled_rows(lib, B, L):
    rows = sorted({0, B // 2, B - 1})
    got, ref = _fp8_attn_case(lib, B, L, rows=rows)
    assert_close(got, ref, RTOL_BF16, "fp8 attention B=%d L=%d rows" % (B, L))


@pytest.mark.parametrize("T,L,Hq,Hkv,hd", [(100, 37, 8, 2, 128), (24, 0, 4, 4, 64), (16, 20, 2, 1, 32)])
def test_attention_fp8_kv_causal_and_head_dims(lib, T, L, Hq, Hkv, hd):
    got, ref = _fp8_attn_case(lib, T, L, Hq=Hq, Hkv=Hkv, hd=hd, causal=True)
    assert_close(got, ref, RTOL_BF16, "fp8 causal T=%d L=%d hd=%d" % (T, L, hd))


# ------------------------------------------------------------------ LM head + row stats + P E
def _check_stats(st, ref, what, logits=None):
    for k in ("m", "lse", "maxprob", "entropy"):
        assert_close(st[k].cpu().numpy(), ref[k], RTOL_BF16, "%s %s" % (what, k))
    am = st["argmax"].cpu().numpy()
    ok = np.ones(len(am), bool) if logits is None else unambiguous_argmax(logits)
    assert np.array_equal(am[ok], ref["argmax"][ok]), what + " argmax"


@pytest.mark.parametrize("B,V,d,mask", [(8, 1000, 192, 999), (3, 520, 64, -1), (32, 4096, 256, 4095)])
def test_lmhead_small(lib, B, V, d, mask):
    xb = _bits(11, (B, d))
    Eb = _bits(12, (V, d), 0.1)
    st = lib.lmhead_rowstats(to_torch_bf16(xb), to_torch_bf16(Eb), mask_id=mask)
    ref = O.lmhead(bf16_f64(xb), Eb, mask_id=mask, want_logits=True)
    _check_stats(st, ref, "lmhead", ref["logits"])
    assert_close(st["s"].cpu().numpy(), ref["s"], RTOL_BF16, "s")


def test_lmhead_given_p(lib):
    import torch
    B, V, d = 4, 640, 128
    xb = _bits(13, (B, d))
    Eb = _bits(14, (V, d), 0.1)
    z = np.exp(gen.normal_np(15, B * V, 3.0).reshape(B, V))
    Pb = gen.bf16_bits(z / z.sum(1, keepdims=True))
    st = lib.lmhead_rowstats(to_torch_bf16(xb), to_torch_bf16(Eb), p_given=to_torch_bf16(Pb))
    ref = O.lmhead(bf16_f64(xb), Eb, p_given=bf16_f64(Pb), want_logits=True)
    _check_stats(st, ref, "lmhead given P", ref["logits"])
    assert_close(st["s"].cpu().numpy(), ref["s"], RTOL_BF16, "s = P E")


def test_lmhead_one_hot_p_reproduces_rows_exactly(lib):
    B, V, d = 2, 1024, 256
    xb = _bits(16, (B, d))
    Eb = _bits(17, (V, d), 0.1)
    P = np.zeros((B, V))
    P[0, 5] = 1.0
    P[1, 1000] = 1.0
    st = lib.lmhead_rowstats(to_torch_bf16(xb), to_torch_bf16(Eb), p_given=to_torch_bf16(gen.bf16_bits(P)))
    s = st["s"].cpu().numpy().astype(np.float64)
    np.testing.assert_array_equal(s[0], bf16_f64(Eb)[5])
    np.testing.assert_array_equal(s[1], bf16_f64(Eb)[1000])


def _rescale_case(B, V, d):
    """x = token-dependent mix of features 0 and 1 only, so the logits are set by E[:, 0:2]:
    N(0, 1) plus a +9 bump in the last tile of each multi-tile cluster range, so those
    clusters raise their reference and rescale (the bump exceeds the first tile's max by
    more than 8) with about 5 % of the mass from before the bump: a wrong rescale factor
    is visible at the 2e-2 tolerance."""
    E = gen.normal_np(31, V * d, 0.1).reshape(V, d)
    E[:, 0] = gen.normal_np(32, V, 1.0)
    E[:, 1] = gen.normal_np(33, V, 0.5)
    # the bump goes into the last vocabulary tile of every multi-tile range of the fused
    # kernel's schedule (contiguous tile ranges over min(tiles, 74) clusters)
    n_tiles = (V + 127) // 128
    n_clu = min(n_tiles, 74)
    for c in range(n_clu):
        tb, te = c * n_tiles // n_clu, (c + 1) * n_tiles // n_clu
        if te - tb >= 2 and (te - 1) * 128 + 5 < V:
            E[(te - 1) * 128 + 5, 0] += 9.0
    x = np.zeros((B, d))
    x[:, 0] = 1.0
    x[:, 1] = (np.arange(B) + 1) / 8.0
    return gen.bf16_bits(x), gen.bf16_bits(E)


@pytest.mark.parametrize("B,V,d,mask", [(5, 20000, 512, 19999), (32, 20000, 256, -1), (1, 3000, 768, 7)])
def test_lmhead_fused_rescale_and_ragged(lib, B, V, d, mask):
    """The fused single-pass LM head (d % 256 == 0, B <= 32): reference raised inside a
    cluster, a ragged last vocabulary tile, B < 32, mask exclusion."""
    xb, Eb = _rescale_case(B, V, d)
    st = lib.lmhead_rowstats(to_torch_bf16(xb), to_torch_bf16(Eb), mask_id=mask)
    ref = O.lmhead(bf16_f64(xb), Eb, mask_id=mask, want_logits=True)
    _check_stats(st, ref, "fused lmhead", ref["logits"])
    assert_close(st["s"].cpu().numpy(), ref["s"], RTOL_BF16, "fused s")


def test_lmhead_fused_given_p_multi_tile(lib):
    B, V, d = 7, 20000, 512
    xb = _bits(41, (B, d))
    Eb = _bits(42, (V, d), 0.1)
    z = np.exp(gen.normal_np(43, B * V, 3.0).reshape(B, V))
    Pb = gen.bf16_bits(z / z.sum(1, keepdims=True))
    st = lib.lmhead_rowstats(to_torch_bf16(xb), to_torch_bf16(Eb), mask_id=V - 1, p_given=to_torch_bf16(Pb))
    ref = O.lmhead(bf16_f64(xb), Eb, mask_id=V - 1, p_given=bf16_f64(Pb), want_logits=True)
    _check_stats(st, ref, "fused lmhead given P", ref["logits"])
    assert_close(st["s"].cpu().numpy(), ref["s"], RTOL_BF16, "fused s = P E")


def test_lmhead_single_round_4b_shapes(lib):
    """Single round at 4B-class shapes: B=32, d=2560, V=151936, P_prev given."""
    import torch
    B, d, V = 32, 2560, 151936
    H, E, Wa, P = gen.lmhead_inputs_torch(B, d, V)
    x = H.to(torch.bfloat16)
    st = lib.lmhead_rowstats(x, E, mask_id=V - 1, p_given=P)
    st2 = lib.lmhead_rowstats(x, E, mask_id=V - 1)
    torch.cuda.synchronize()
    xb, Eb, Pb = from_torch_bf16(x), from_torch_bf16(E), from_torch_bf16(P)
    ref = O.lmhead(bf16_f64(xb), Eb, mask_id=V - 1, p_given=bf16_f64(Pb), want_logits=True)
    _check_stats(st, ref, "4b lmhead", ref["logits"])
    assert_close(st["s"].cpu().numpy(), ref["s"], RTOL_BF16, "4b s = P_prev E")
    ref2 = O.lmhead(bf16_f64(xb), Eb, mask_id=V - 1)
    assert_close(st2["s"].cpu().numpy(), ref2["s"], RTOL_BF16, "4b s = softmax E")


# ------------------------------------------------------------------ adapter
@pytest.mark.parametrize("B,d,V", [(32, 2560, 1000), (8, 64, 512)])
def test_adapter_embed(lib, B, d, V):
    import torch
    Eb = _bits(20, (V, d), 0.02)
    Wab = _bits(21, (d, d), 0.02)
    s = gen.normal_np(22, B * d, 0.05).reshape(B, d)
    tok = gen.uniform_tokens_np(23, B, 0, V)
    h0 = lib.adapter_embed(to_torch_bf16(Eb), to_torch_bf16(Wab), torch.from_numpy(tok).cuda(),
                           torch.from_numpy(s.astype(np.float32)).cuda()).cpu().numpy()
    s32 = s.astype(np.float32).astype(np.float64)
    ref = bf16_f64(Eb)[tok] + O.linear(s32, Wab)
    assert_close(h0, ref, 1e-4, "adapter")


# ------------------------------------------------------------------ commit
@pytest.mark.parametrize("case", range(12))
def test_commit_matches_oracle(lib, case):
    import torch
    B, d = [8, 32, 64, 1][case % 4], 16
    rng = np.random.default_rng(case)
    mp = rng.random(B).astype(np.float32)
    if case % 3 == 0:
        mp[: B // 2] = mp[0]  # ties
    am = rng.integers(0, 500, B).astype(np.int32)
    com = (rng.random(B) < 0.3).astype(np.uint8)
    if com.all():
        com[0] = 0
    tok = np.where(com == 1, rng.integers(0, 500, B), 511).astype(np.int32)
    mode = case % 2
    tau = [0.5, 0.95, 1.5, 0.0][case % 4]
    k = [1, 3, 11][case % 3]
    s = np.ones((B, d), np.float32)
    t = {n: torch.from_numpy(v).cuda() for n, v in dict(mp=mp, am=am, tok=tok.copy(), com=com.copy(), s=s).items()}
    rnd = torch.zeros(1, dtype=torch.int32, device="cuda")
    lib.commit(t["mp"], t["am"], t["tok"], t["com"], t["s"], rnd, tau, mode, k)
    n, rtok, rcom = O.commit(mp.astype(np.float64), am, tau, mode, k, tok, com)
    np.testing.assert_array_equal(t["com"].cpu().numpy(), rcom)
    np.testing.assert_array_equal(t["tok"].cpu().numpy(), rtok)
    srow = t["s"].cpu().numpy()
    assert np.all(srow[rcom == 1] == 0) and np.all(srow[rcom == 0] == 1)
    assert int(rnd.item()) == 1


# ------------------------------------------------------------------ NVFP4 quantizer
@pytest.mark.parametrize("rows,cols,std", [(64, 256, 0.02), (9728, 2560, 0.02), (5, 48, 3.0)])
def test_nvfp4_quantizer_bit_exact(lib, rows, cols, std):
    import torch
    wb = _bits(30 + rows, (rows, cols), std)
    codes, scales, ts = lib.nvfp4_quantize(to_torch_bf16(wb))
    torch.cuda.synchronize()
    rc, rs, rS = O.nvfp4_quantize(bf16_f64(wb).astype(np.float32))
    assert np.float32(ts.item()) == np.float32(rS)
    np.testing.assert_array_equal(scales.cpu().numpy(), rs)
    np.testing.assert_array_equal(codes.cpu().numpy(), rc)
