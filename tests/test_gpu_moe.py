"""Routed-expert MLP sub-block with NVFP4 experts (dlm_moe_mlp_nvfp4) against the oracle
(reading R14).  Both sides use the oracle codec's NVFP4 weights; the GPU quantizes its
activation rows from fp32 / split-bf16 values, the oracle from fp64 ones, so a few activation
codes may sit on the other side of a rounding boundary: outputs are compared at a tolerance
well inside the NVFP4 contract, the expert choice exactly wherever the router's k-th and
(k+1)-th logits are at least 1e-3 apart, and the weights of the chosen experts at 1e-4."""
import numpy as np
import pytest

import oracle as O
from block_diffusion_decoding_denoising_b200 import gen
from helpers import RTOL_NVFP4, assert_close, bf16_f64, rel_err, to_torch_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def D():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from block_diffusion_decoding_denoising_b200 import build, dlm
    build.build()
    dlm.lib()
    return dlm


def _q(wb):
    c, s, S = O.nvfp4_quantize(bf16_f64(wb).astype(np.float32))
    return {"codes": c, "scales": s, "tscale": S, "rows": wb.shape[0], "cols": wb.shape[1]}


def _dev(q):
    import torch
    return {"codes": torch.from_numpy(q["codes"]).cuda(), "scales": torch.from_numpy(q["scales"]).cuda(),
            "tscale": q["tscale"], "rows": q["rows"], "cols": q["cols"]}


def make_case(E, k, F, d, T, seed, router_std=0.05, zero_router=False):
    s = lambda i: gen.tensor_seed(seed, i)
    wr = np.zeros((E, d)) if zero_router else gen.normal_np(s(1), E * d, router_std).reshape(E, d)
    moe = dict(n_experts=E, top_k=k, ffn_expert=F, w_router=gen.bf16_bits(wr),
               norm=gen.bf16_bits(1.0 + gen.normal_np(s(2), d, 0.1)),
               gate=_q(gen.bf16_bits(gen.normal_np(s(3), E * F * d, 0.05).reshape(E * F, d))),
               up=_q(gen.bf16_bits(gen.normal_np(s(4), E * F * d, 0.05).reshape(E * F, d))),
               down=_q(gen.bf16_bits(gen.normal_np(s(5), d * E * F, 0.05).reshape(d, E * F))))
    h = gen.normal_np(s(6), T * d, 1.0).reshape(T, d).astype(np.float32)
    return moe, h


def run(D, moe, h):
    import torch
    m = D.Moe(moe["n_experts"], moe["top_k"], moe["ffn_expert"], h.shape[1], to_torch_bf16(moe["w_router"]),
              to_torch_bf16(moe["norm"]), _dev(moe["gate"]), _dev(moe["up"]), _dev(moe["down"]))
    out, idx, w = m(torch.from_numpy(h).cuda())
    torch.cuda.synchronize()
    return out.cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy()


def check(D, moe, h, what, tol=2e-2):
    ref = O.moe_mlp(h.astype(np.float64), moe, act_fp4=True)
    out, idx, w = run(D, moe, h)
    k = moe["top_k"]
    srt = -np.sort(-ref["logits"], axis=1)
    clear = np.ones(h.shape[0], bool) if k == moe["n_experts"] else (srt[:, k - 1] - srt[:, k]) >= 1e-3
    assert clear.sum() >= 0.8 * len(clear), "too few rows with a clear expert choice"
    assert np.array_equal(idx[clear], ref["idx"][clear]), what + ": chosen experts"
    np.testing.assert_allclose(w[clear], ref["w"][clear], rtol=1e-4, atol=1e-6, err_msg=what + ": weights")
    assert_close(out, ref["h_out"], RTOL_NVFP4, what + ": h_out")
    e = rel_err(out - h, ref["h_out"] - h)
    print("%s: MLP output rel err %.2e" % (what, e))
    assert e < tol, (what, e)


@pytest.mark.parametrize("E,k,F,d,T", [(4, 2, 64, 256, 5), (16, 4, 128, 512, 32), (64, 8, 64, 1024, 17),
                                       (8, 1, 256, 768, 3), (16, 2, 128, 512, 64)])
def test_moe_matches_oracle(D, E, k, F, d, T):
    moe, h = make_case(E, k, F, d, T, seed=E * 100 + k * 10 + T)
    check(D, moe, h, "moe E=%d k=%d F=%d d=%d T=%d" % (E, k, F, d, T))


def test_moe_uniform_router_chooses_the_first_k_experts(D):
    """W_r = 0: all logits equal, so experts 0..k-1 are chosen with weight 1/k each."""
    moe, h = make_case(8, 3, 64, 256, 6, seed=9, zero_router=True)
    out, idx, w = run(D, moe, h)
    assert np.array_equal(idx, np.tile(np.arange(3, dtype=np.int32), (6, 1)))
    np.testing.assert_allclose(w, 1.0 / 3.0, rtol=1e-6)
    ref = O.moe_mlp(h.astype(np.float64), moe, act_fp4=True)
    assert_close(out, ref["h_out"], RTOL_NVFP4, "uniform router")


def test_moe_4b_width_64_experts(D):
    """The 4B-class width (d 2560), 64 experts of F 512, top-4, 32 rows."""
    moe, h = make_case(64, 4, 512, 2560, 32, seed=77, router_std=0.02)
    check(D, moe, h, "moe 4b width")


def test_moe_rejects_unsupported_shapes(D):
    import torch
    from block_diffusion_decoding_denoising_b200.dlm import DlmError
    moe, h = make_case(4, 2, 64, 256, 4, seed=3)
    with pytest.raises(DlmError):
        run(D, dict(moe, ffn_expert=48), h)  # F % 64 != 0
    with pytest.raises(DlmError):
        run(D, moe, np.zeros((65, 256), np.float32))  # T > 64
