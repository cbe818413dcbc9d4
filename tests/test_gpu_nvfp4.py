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


@pytest.mark.parametrize("T", [1, 5, 17, 32])
@pytest.mark.parametrize("N,K", [(128, 256), (384, 512), (200, 768), (640, 2560)])
def test_gemm_nvfp4_small(lib, T, N, K):
    run_case(lib, T, N, K, seed=T * 1000 + N + K)


@pytest.mark.parametrize("N,K", [(9728, 2560), (2560, 9728)])
def test_gemm_nvfp4_4b_mlp_shapes(lib, N, K):
    err = run_case(lib, 32, N, K, seed=7)
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
        lib.gemm_nvfp4(torch.zeros((33, 256), device="cuda"), q2)  # T > 32
