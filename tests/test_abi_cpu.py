"""C-ABI checks that need no GPU: the library loads, exports every function that
include/dlm.h declares, sizes its buffers, and rejects bad arguments before touching
the device."""
import ctypes as C
import os
import re

import pytest

from block_diffusion_decoding_denoising_b200 import build, dlm, gen

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return dlm.lib()


def declared_functions():
    txt = open(os.path.join(ROOT, "include", "dlm.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    names = re.findall(r"\b(dlm_[a-z0-9_]+)\s*\(", txt)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 20
    for n in names:
        assert hasattr(L, n), n


def test_version(L):
    assert b"sm_100a" in L.dlm_version()


def test_workspace_and_kv_sizes(L):
    cfg = dlm.Config.from_dict(gen.config_4b())
    kv = L.dlm_kv_cache_size(C.byref(cfg))
    c = gen.config_4b()
    assert kv == 2 * c["n_layers"] * c["n_kv_heads"] * c["max_ctx"] * c["head_dim"] * 2
    ws = L.dlm_workspace_size(C.byref(cfg))
    assert ws % 256 == 0 and ws > c["block_size"] * c["vocab"] * 6
    tiny = dlm.Config.from_dict(gen.config_tiny())
    assert 0 < L.dlm_workspace_size(C.byref(tiny)) < ws


def test_nvfp4_workspace_keeps_no_bf16_copy_of_e(L):
    # With the fused NVFP4 LM head (B <= 32) the embedding rows and P E read E's codes, so the
    # workspace holds no bf16 copy of E; the unfused head (B = 33) needs one (V x d x 2 bytes).
    def ws(B):
        c = gen.config_4b()
        c["weight_fmt"], c["block_size"] = dlm.WEIGHTS_NVFP4, B
        return L.dlm_workspace_size(C.byref(dlm.Config.from_dict(c)))
    c = gen.config_4b()
    e_bf16 = c["vocab"] * c["d"] * 2
    assert ws(32) < e_bf16 // 2
    assert ws(33) - ws(32) > 0.9 * e_bf16


@pytest.mark.parametrize("field,value", [("d", 65), ("n_kv_heads", 3), ("head_dim", 48), ("block_size", 0),
                                         ("block_size", 65), ("mask_id", 512), ("vocab", 510), ("weight_fmt", 2),
                                         ("rms_eps", 0.0)])
def test_invalid_config_rejected(L, field, value):
    c = gen.config_tiny()
    c[field] = value
    cfg = dlm.Config.from_dict(c)
    assert L.dlm_workspace_size(C.byref(cfg)) == 0
    assert L.dlm_kv_cache_size(C.byref(cfg)) == 0
    out = C.c_void_p()
    w = dlm.Weights()
    st = L.dlm_ctx_create(C.byref(cfg), C.byref(w), C.c_void_p(256), 1 << 30, C.c_void_p(256), 1 << 30,
                          C.byref(out))
    assert st == dlm.DLM_EINVAL and not out.value


def test_ctx_create_argument_checks(L):
    cfg = dlm.Config.from_dict(gen.config_tiny())
    out = C.c_void_p()
    w = dlm.Weights()  # null weight pointers
    assert L.dlm_ctx_create(C.byref(cfg), C.byref(w), C.c_void_p(256), 1 << 30, C.c_void_p(256), 1 << 30,
                            C.byref(out)) == dlm.DLM_EINVAL
    assert L.dlm_ctx_create(C.byref(cfg), None, None, 0, None, 0, C.byref(out)) == dlm.DLM_EINVAL
    assert L.dlm_ctx_create(C.byref(cfg), C.byref(w), None, 0, None, 0, None) == dlm.DLM_EINVAL
    assert L.dlm_ctx_destroy(None) == dlm.DLM_EINVAL
    assert L.dlm_last_error(None) == b"null context"
    assert L.dlm_prefix_len(None) == -1


def test_null_context_calls(L):
    assert L.dlm_round(None, None, 0.9, 0, 1, None) == dlm.DLM_EINVAL
    assert L.dlm_decode_block(None, 0.9, 0, 1, None, None, None) == dlm.DLM_EINVAL
    assert L.dlm_generate(None, None, 0, 0, 0.9, 0, 1, None, None, None, None) == dlm.DLM_EINVAL
    assert L.dlm_prefill(None, None, 0, None) == dlm.DLM_EINVAL
    assert L.dlm_kv_fill(None, None, None) == dlm.DLM_EINVAL
    assert L.dlm_kv_flush(None, None) == dlm.DLM_EINVAL
    assert L.dlm_fill_pending(None) == -1
    assert L.dlm_set_fill_mode(None, dlm.FILL_DEFERRED, None) == dlm.DLM_EINVAL
    assert L.dlm_mlp_block(None, 0, None, None, 1, None) == dlm.DLM_EINVAL
    assert L.dlm_set_prefix_len(None, 0, None) == dlm.DLM_EINVAL


def test_single_op_argument_checks(L):
    p = C.c_void_p(256)
    nan = float("nan")
    # commit: tau NaN, bad mode, k < 1, B out of range
    assert L.dlm_commit(p, p, p, p, p, p, None, 8, 64, nan, 0, 1, None) == dlm.DLM_EINVAL
    assert L.dlm_commit(p, p, p, p, p, p, None, 8, 64, 0.9, 7, 1, None) == dlm.DLM_EINVAL
    assert L.dlm_commit(p, p, p, p, p, p, None, 8, 64, 0.9, 1, 0, None) == dlm.DLM_EINVAL
    assert L.dlm_commit(p, p, p, p, p, p, None, 65, 64, 0.9, 0, 1, None) == dlm.DLM_EINVAL
    # gemm: bad shapes and a scratch that is too small
    assert L.dlm_gemm_bf16(p, p, p, 0, 128, 128, p, 1 << 20, None) == dlm.DLM_EINVAL
    assert L.dlm_gemm_bf16(None, p, p, 8, 128, 128, p, 1 << 20, None) == dlm.DLM_EINVAL
    assert L.dlm_gemm_bf16(p, p, p, 8, 128, 100, p, 1 << 20, None) == dlm.DLM_EINVAL
    assert L.dlm_gemm_bf16(p, p, p, 8, 128, 128, p, 16, None) == dlm.DLM_ENOMEM_WS
    assert L.dlm_gemm_f32(p, p, p, 129, 128, 128, p, 1 << 20, None) == dlm.DLM_EINVAL
    assert L.dlm_gemm_f32(p, p, None, 8, 128, 128, p, 1 << 20, None) == dlm.DLM_EINVAL
    assert L.dlm_gemm_f32(p, p, p, 8, 128, 128, p, 16, None) == dlm.DLM_ENOMEM_WS
    assert L.dlm_gemm_f32_scratch_size(8, 128, 128) > L.dlm_gemm_scratch_size(8, 128, 128)
    assert L.dlm_gemm_f32_scratch_size(129, 128, 128) == 0
    # attention: L + T beyond the cache, bad head dim
    assert L.dlm_bd_attention(p, p, p, p, 8, 100, 4, 2, 128, 64, 0, p, 1 << 20, None) == dlm.DLM_EINVAL
    assert L.dlm_bd_attention(p, p, p, p, 8, 0, 4, 2, 96, 64, 0, p, 1 << 20, None) == dlm.DLM_EINVAL
    assert L.dlm_bd_attention(p, p, p, p, 8, 0, 4, 3, 128, 64, 0, p, 1 << 20, None) == dlm.DLM_EINVAL
    # lm head: null stats
    assert L.dlm_lmhead_rowstats(p, p, 8, 512, 64, -1, None, dlm.RowStats(), p, p, 1 << 30, None) == dlm.DLM_EINVAL
    # nvfp4: cols not a multiple of 16
    assert L.dlm_nvfp4_quantize(p, 4, 40, p, p, p, None) == dlm.DLM_EINVAL


def test_scratch_sizes_grow_with_shape(L):
    a = L.dlm_gemm_scratch_size(32, 6144, 2560)
    b = L.dlm_gemm_scratch_size(256, 6144, 2560)
    assert 0 < a < b
    assert L.dlm_lmhead_scratch_size(32, 151936, 2560) > 32 * 151936 * 6
    assert L.dlm_attention_scratch_size(32, 32, 128, 65600) >= L.dlm_attention_scratch_size(32, 32, 128, 1024)
