"""NVFP4 weight GEMM (dlm_gemm_nvfp4, block-scaled FP4 tensor cores) against the oracle:
weights quantized by the oracle's codec, activations quantized per row on both sides from
the same fp32 values.  The products of the quantized operands are exact on both sides, so
the results differ only by accumulation order (the contract is rel 6e-2; a tighter bound is
checked too)."""
import numpy as np
import pytest

import oracle as O
from block_diffusion_decoding_denoising_b200 import gen
from helpers import RTOL_NVFP4, assert_close, bf16_f64, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from block_diffusion_decoding_denoising_b200 import build, dlm as D
    build.build()
    D.lib()
    return D


def oracle_q(wb):
    codes, scales, S = O.nvfp4_quantize(bf16_f64(wb).astype(np.float32))
    return {"codes": codes, "scales": scales, "tscale": S, "rows": wb.shape[0], "cols": wb.shape[1]}


def to_device_q(q):
    import torch
    return {"codes": torch.from_numpy(q["codes"]).cuda(), "scales": torch.from_numpy(q["scales"]).cuda(),
            "tscale": q["tscale"], "rows": q["rows"], "cols": q["cols"]}


def run_case(D, T, N, K, seed, std=0.02, x_std=1.0):
    import torch
    wb = gen.bf16_bits(gen.normal_np(gen.tensor_seed(seed, 1), N * K, std).reshape(N, K))
    x = gen.normal_np(gen.tensor_seed(seed, 2), T * K, x_std).reshape(T, K).astype(np.float32)
    q = oracle_q(wb)
    want = O.linear(x.astype(np.float64), q, act_fp4=True)
    got = D.gemm_nvfp4(torch.from_numpy(x).cuda(), to_device_q(q)).cpu().numpy()
    assert_close(got, want, RTOL_NVFP4, "nvfp4 gemm T=%d N=%d K=%d" % (T, N, K))
    err = rel_err(got, want)
    assert err < 1e-3, (T, N, K, err)  # exact products: only the summation order differs
    return err


@pytest.mark.parametrize("T", [1, 5, 17, 32, 33, 48, 64])
@pytest.mark.parametrize("N,K", [(128, 256), (384, 512), (200, 768), (640, 2560)])
def test_gemm_nvfp4_small(lib, T, N, K):
    run_case(lib, T, N, K, seed=T * 1000 + N + K)


@pytest.mark.parametrize("N,K", [(9728, 2560), (2560, 9728)])
@pytest.mark.parametrize("T", [32, 64])
def test_gemm_nvfp4_4b_mlp_shapes(lib, N, K, T):
    err = run_case(lib, T, N, K, seed=7 + T)
    print("nvfp4 %dx%d rel err %.2e" % (N, K, err))


def test_gemm_nvfp4_zero_rows_and_blocks(lib):
    """A zero activation row (row scale 0) gives zero outputs; all-zero weight blocks
    (block scale 0) contribute nothing."""
    import torch
    T, N, K = 4, 256, 512
    wb = gen.bf16_bits(gen.normal_np(3, N * K, 0.02).reshape(N, K))
    wb[:, :64] = 0
    x = gen.normal_np(4, T * K).reshape(T, K).astype(np.float32)
    x[1] = 0.0
    q = oracle_q(wb)
    want = O.linear(x.astype(np.float64), q, act_fp4=True)
    got = lib.gemm_nvfp4(torch.from_numpy(x).cuda(), to_device_q(q)).cpu().numpy()
    assert np.all(got[1] == 0.0)
    assert_close(got, want, RTOL_NVFP4, "zero rows/blocks")


def test_gemm_nvfp4_rejects_bad_shapes(lib):
    import torch
    from block_diffusion_decoding_denoising_b200.dlm import DlmError
    q = to_device_q(oracle_q(gen.bf16_bits(gen.normal_np(5, 128 * 320, 0.02).reshape(128, 320))))
    with pytest.raises(DlmError):
        lib.gemm_nvfp4(torch.zeros((4, 320), device="cuda"), q)  # K % 256 != 0
    q2 = to_device_q(oracle_q(gen.bf16_bits(gen.normal_np(6, 128 * 256, 0.02).reshape(128, 256))))
    with pytest.raises(DlmError):
        lib.gemm_nvfp4(torch.zeros((65, 256), device="cuda"), q2)  # T > 64


# ------------------------------------------------------------------ fused NVFP4 LM head
def _check_lm_stats(st, ref, what, rtol=1e-4):
    from helpers import unambiguous_argmax
    for k in ("m", "lse", "maxprob", "entropy"):
        assert_close(st[k].cpu().numpy(), ref[k], rtol, "%s %s" % (what, k))
    am = st["argmax"].cpu().numpy()
    ok = unambiguous_argmax(ref["logits"])
    assert np.array_equal(am[ok], ref["argmax"][ok]), what + " argmax"


def _lm_case(D, B, V, d, mask, seed, e_std=0.1, bump=False):
    """Logits from the quantized x and E are exact products on both sides (only the
    summation order differs), so the statistics agree far inside the NVFP4 contract; s = P E
    carries P as f16 (relative rounding 2^-11 per weight)."""
    import torch
    E = gen.normal_np(gen.tensor_seed(seed, 1), V * d, e_std).reshape(V, d)
    if bump:  # raise the reference inside a cluster's tile range (see the bf16 rescale case)
        E[:, 0] = gen.normal_np(gen.tensor_seed(seed, 3), V, 1.0)
        n_tiles = (V + 127) // 128
        n_clu = min(n_tiles, 74)
        for c in range(n_clu):
            tb, te = c * n_tiles // n_clu, (c + 1) * n_tiles // n_clu
            if te - tb >= 2 and (te - 1) * 128 + 5 < V:
                E[(te - 1) * 128 + 5, 0] += 9.0
    q = oracle_q(gen.bf16_bits(E))
    x = gen.normal_np(gen.tensor_seed(seed, 2), B * d, 1.0).reshape(B, d).astype(np.float32)
    if bump:
        x[:, 0] = 4.0
    ref = O.lmhead(x.astype(np.float64), q, mask_id=mask, act_fp4=True, want_logits=True)
    st = D.lmhead_rowstats_nvfp4(torch.from_numpy(x).cuda(), to_device_q(q), mask_id=mask)
    torch.cuda.synchronize()
    return st, ref


@pytest.mark.parametrize("B,V,d,mask", [(5, 3000, 512, 7), (32, 20000, 1024, -1), (1, 1000, 2560, 999),
                                        (17, 9600, 1536, 9599)])
def test_lmhead_nvfp4_matches_oracle(lib, B, V, d, mask):
    st, ref = _lm_case(lib, B, V, d, mask, seed=B * 7 + d)
    _check_lm_stats(st, ref, "nvfp4 lmhead")
    s = st["s"].cpu().numpy()
    assert_close(s, ref["s"], RTOL_NVFP4, "nvfp4 s")
    assert rel_err(s, ref["s"]) < 2e-3, rel_err(s, ref["s"])


def test_lmhead_nvfp4_rescale_inside_cluster(lib):
    """A +9 logit bump in the last tile of every multi-tile cluster range raises the running
    reference and rescales the s accumulators."""
    st, ref = _lm_case(lib, 8, 30000, 512, 29999, seed=5, bump=True)
    _check_lm_stats(st, ref, "nvfp4 lmhead rescale")
    s = st["s"].cpu().numpy()
    assert rel_err(s, ref["s"]) < 2e-3, rel_err(s, ref["s"])


def test_lmhead_nvfp4_peaked_softmax_reproduces_dequantized_rows(lib):
    """x_b points along E row a_b with a logit gap of about 60, so P is one-hot in f16 and Z
    is 1 in fp32: s_b must equal the dequantized row E[a_b] = code x sigma x S_E up to one
    fp32 rounding.  Pins the code nibble order, the scale bytes and the layout of the
    dequantized tiles."""
    import torch
    B, V, d = 6, 3000, 512
    E = gen.normal_np(gen.tensor_seed(9, 1), V * d, 0.1).reshape(V, d)
    q = oracle_q(gen.bf16_bits(E))
    Ed = O.nvfp4_dequant(q["codes"], q["scales"], q["tscale"], V, d)
    rows = np.array([0, 1, 777, 1500, 2998, 2999])
    x = np.stack([40.0 * Ed[a] / np.linalg.norm(Ed[a]) for a in rows]).astype(np.float32)
    ref = O.lmhead(x.astype(np.float64), q, act_fp4=True, want_logits=True)
    assert np.array_equal(ref["argmax"], rows)
    gap = np.sort(ref["logits"], 1)
    assert np.all(gap[:, -1] - gap[:, -2] > 40.0)
    st = lib.lmhead_rowstats_nvfp4(torch.from_numpy(x).cuda(), to_device_q(q))
    s = st["s"].cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(s, Ed[rows], rtol=2e-7, atol=1e-12)
    assert np.array_equal(st["argmax"].cpu().numpy(), rows)


def test_lmhead_nvfp4_4b_shapes(lib):
    """B 32, d 2560, V 151936 (the 4B-class vocabulary), mask id V - 1."""
    B, V, d = 32, 151936, 2560
    st, ref = _lm_case(lib, B, V, d, V - 1, seed=11, e_std=0.02)
    _check_lm_stats(st, ref, "nvfp4 lmhead 4b")
    s = st["s"].cpu().numpy()
    err = rel_err(s, ref["s"])
    print("nvfp4 lmhead 4b: s rel err %.2e" % err)
    assert err < 2e-3, err


def test_lmhead_nvfp4_rejects_unsupported_shapes(lib):
    import torch
    from block_diffusion_decoding_denoising_b200.dlm import DlmError
    q = to_device_q(oracle_q(gen.bf16_bits(gen.normal_np(5, 256 * 768, 0.02).reshape(256, 768))))
    with pytest.raises(DlmError):
        lib.lmhead_rowstats_nvfp4(torch.zeros((4, 768), device="cuda"), q)  # d % 512 != 0
    q2 = to_device_q(oracle_q(gen.bf16_bits(gen.normal_np(6, 256 * 512, 0.02).reshape(256, 512))))
    with pytest.raises(DlmError):
        lib.lmhead_rowstats_nvfp4(torch.zeros((33, 512), device="cuda"), q2)  # B > 32
