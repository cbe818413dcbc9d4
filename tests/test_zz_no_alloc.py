"""The attention entry point without a scratch argument (dlm_bd_attention_noalloc) against
the scratch-taking one (dlm_bd_attention): same inputs, two calls in a row, results
identical (and so within the bf16 tolerance); calls too large for its fixed scratch are
rejected.  This file is named to be collected last and needs nothing from the other test
files."""
import numpy as np
import pytest

from helpers import RTOL_BF16, assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def D():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from block_diffusion_decoding_denoising_b200 import build, dlm
    build.build()
    dlm.lib()
    return dlm


@pytest.mark.parametrize("T,L,causal", [(32, 2048, False), (4, 700, False), (48, 1000, True)])
def test_noalloc_matches_scratch_entry_twice(D, T, L, causal):
    import torch
    from block_diffusion_decoding_denoising_b200 import gen
    Hq, Hkv, hd = 32, 8, 128
    outs = []
    for call in range(2):  # two calls in a row, different inputs
        q, kc, vc = gen.attention_inputs_torch(T, L, Hq, Hkv, hd, max_ctx=L + T + 16, seed=11 + call)
        want = D.bd_attention(q, kc, vc, L, causal=causal)
        got = D.bd_attention_noalloc(q, kc, vc, L, causal=causal)
        torch.cuda.synchronize()
        assert_close(got.float().cpu().numpy(), want.float().cpu().numpy(), RTOL_BF16, "noalloc call %d" % call)
        # the same kernels with the same split count: identical bits, so a stale or misplaced
        # partial in the shared static array cannot hide inside the tolerance
        assert torch.equal(got, want), "noalloc call %d differs from dlm_bd_attention" % call
        outs.append(got.float().cpu().numpy())
    assert not np.array_equal(outs[0], outs[1])


def test_noalloc_rejects_oversized_call(D):
    import torch
    from block_diffusion_decoding_denoising_b200.dlm import DLM_ENOMEM_WS, DlmError
    # 64 queries x 512 heads of 128 (one split): the partials exceed the 16 MiB array
    T, Hq, Hkv, hd, L = 64, 512, 64, 128, 8192
    q = torch.zeros((T, Hq, hd), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((Hkv, L + T, hd), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(DlmError) as ei:
        D.bd_attention_noalloc(q, kc, kc, L)
    assert ei.value.status == DLM_ENOMEM_WS
