"""Python binding of libdlm.so (include/dlm.h): argument marshalling only.

Every step of the decoding path runs in the CUDA library; PyTorch is used only to own
device memory and streams.  Importing this module on a machine without the built
library raises: there is no fallback.
"""
from __future__ import annotations

import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libdlm.so")

DLM_OK, DLM_EINVAL, DLM_ENOMEM_WS, DLM_EKVCAP, DLM_ECUDA, DLM_EROUNDCAP, DLM_ETIMEOUT, DLM_EUNSUPPORTED = range(8)
COMMIT_THRESHOLD, COMMIT_TOPK = 0, 1
FILL_EAGER, FILL_DEFERRED = 0, 1
KV_BF16, KV_FP8 = 0, 1
WEIGHTS_BF16, WEIGHTS_NVFP4 = 0, 1
STATUS_NAMES = {0: "DLM_OK", 1: "DLM_EINVAL", 2: "DLM_ENOMEM_WS", 3: "DLM_EKVCAP", 4: "DLM_ECUDA",
                5: "DLM_EROUNDCAP", 6: "DLM_ETIMEOUT", 7: "DLM_EUNSUPPORTED"}


class DlmError(RuntimeError):
    def __init__(self, status, msg=""):
        super().__init__("%s %s" % (STATUS_NAMES.get(status, status), msg))
        self.status = status


class Config(C.Structure):
    _fields_ = [("n_layers", C.c_int), ("d", C.c_int), ("n_q_heads", C.c_int), ("n_kv_heads", C.c_int),
                ("head_dim", C.c_int), ("ffn", C.c_int), ("vocab", C.c_int), ("mask_id", C.c_int),
                ("max_ctx", C.c_int), ("block_size", C.c_int), ("rope_theta", C.c_float),
                ("rms_eps", C.c_float), ("weight_fmt", C.c_int), ("kv_fmt", C.c_int)]

    @classmethod
    def from_dict(cls, c):
        return cls(c["n_layers"], c["d"], c["n_q_heads"], c["n_kv_heads"], c["head_dim"], c["ffn"],
                   c["vocab"], c["mask_id"], c["max_ctx"], c["block_size"], float(c["rope_theta"]),
                   float(c["rms_eps"]), int(c.get("weight_fmt", 0)), int(c.get("kv_fmt", 0)))


class Nvfp4Matrix(C.Structure):
    _fields_ = [("codes", C.c_void_p), ("scales", C.c_void_p), ("tensor_scale", C.c_float)]


class MoeWeights(C.Structure):
    _fields_ = [("n_experts", C.c_int), ("top_k", C.c_int), ("ffn_expert", C.c_int),
                ("w_router", C.c_void_p), ("mlp_norm", C.c_void_p), ("q_gate", Nvfp4Matrix),
                ("q_up", Nvfp4Matrix), ("q_down", Nvfp4Matrix)]


class LayerWeights(C.Structure):
    _fields_ = [("attn_norm", C.c_void_p), ("w_qkv", C.c_void_p), ("w_o", C.c_void_p),
                ("mlp_norm", C.c_void_p), ("w_gate", C.c_void_p), ("w_up", C.c_void_p),
                ("w_down", C.c_void_p), ("q_gate", Nvfp4Matrix), ("q_up", Nvfp4Matrix),
                ("q_down", Nvfp4Matrix)]


class Weights(C.Structure):
    _fields_ = [("embed", C.c_void_p), ("w_adapter", C.c_void_p), ("final_norm", C.c_void_p),
                ("layers", C.POINTER(LayerWeights)), ("q_embed", Nvfp4Matrix)]


class RowStats(C.Structure):
    _fields_ = [("m", C.c_void_p), ("lse", C.c_void_p), ("maxprob", C.c_void_p), ("entropy", C.c_void_p),
                ("argmax", C.c_void_p)]


class BlockState(C.Structure):
    _fields_ = [("tokens", C.c_void_p), ("committed", C.c_void_p), ("s", C.c_void_p), ("round", C.c_void_p),
                ("status", C.c_void_p), ("stats", RowStats)]


class Timing(C.Structure):
    _fields_ = [("prefill_ms", C.c_double), ("decode_ms", C.c_double), ("n_blocks", C.c_int),
                ("n_rounds", C.c_int)]


_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libdlm.so is not built (run python -m block_diffusion_decoding_denoising_b200.build)")
        L = C.CDLL(LIB_PATH)
        p, i, f, z = C.c_void_p, C.c_int, C.c_float, C.c_size_t
        L.dlm_version.restype = C.c_char_p
        L.dlm_workspace_size.restype = z
        L.dlm_workspace_size.argtypes = [C.POINTER(Config)]
        L.dlm_kv_cache_size.restype = z
        L.dlm_kv_cache_size.argtypes = [C.POINTER(Config)]
        L.dlm_ctx_create.argtypes = [C.POINTER(Config), C.POINTER(Weights), p, z, p, z, C.POINTER(p)]
        L.dlm_ctx_destroy.argtypes = [p]
        L.dlm_last_error.restype = C.c_char_p
        L.dlm_last_error.argtypes = [p]
        L.dlm_prefix_len.argtypes = [p]
        L.dlm_set_prefix_len.argtypes = [p, i, p]
        L.dlm_prefill.argtypes = [p, p, i, p]
        L.dlm_block_init.argtypes = [p, C.POINTER(BlockState), p]
        L.dlm_round.argtypes = [p, C.POINTER(BlockState), f, i, i, p]
        L.dlm_kv_fill.argtypes = [p, p, p]
        L.dlm_kv_flush.argtypes = [p, p]
        L.dlm_fill_pending.argtypes = [p]
        L.dlm_set_fill_mode.argtypes = [p, i, p]
        L.dlm_mlp_block.argtypes = [p, i, p, p, i, p]
        L.dlm_decode_block.argtypes = [p, f, i, i, p, p, p]
        L.dlm_generate.argtypes = [p, p, i, i, f, i, i, p, p, C.POINTER(Timing), p]
        L.dlm_gemm_scratch_size.restype = z
        L.dlm_gemm_scratch_size.argtypes = [i, i, i]
        L.dlm_gemm_bf16.argtypes = [p, p, p, i, i, i, p, z, p]
        L.dlm_gemm_bf16x2.argtypes = [p, p, p, i, i, i, p, z, p]
        L.dlm_split_pad.argtypes = [i]
        L.dlm_gemm_f32_scratch_size.restype = z
        L.dlm_gemm_f32_scratch_size.argtypes = [i, i, i]
        L.dlm_gemm_f32.argtypes = [p, p, p, i, i, i, p, z, p]
        L.dlm_lmhead_scratch_size.restype = z
        L.dlm_lmhead_scratch_size.argtypes = [i, i, i]
        L.dlm_lmhead_rowstats.argtypes = [p, p, i, i, i, i, p, RowStats, p, p, z, p]
        L.dlm_adapter_scratch_size.restype = z
        L.dlm_adapter_scratch_size.argtypes = [i, i]
        L.dlm_adapter_embed.argtypes = [p, p, p, p, p, i, i, p, z, p]
        L.dlm_attention_scratch_size.restype = z
        L.dlm_attention_scratch_size.argtypes = [i, i, i, i]
        L.dlm_bd_attention.argtypes = [p, p, p, p, i, i, i, i, i, i, i, p, z, p]
        L.dlm_bd_attention_noalloc.argtypes = [p, p, p, p, i, i, i, i, i, i, i, p]
        L.dlm_bd_attention_fp8.argtypes = [p, p, p, p, p, p, i, i, i, i, i, i, i, p, z, p]
        L.dlm_commit.argtypes = [p, p, p, p, p, p, p, i, i, f, i, i, p]
        L.dlm_nvfp4_quantize.argtypes = [p, i, i, p, p, p, p]
        L.dlm_moe_prepare_size.restype = z
        L.dlm_moe_prepare_size.argtypes = [i, C.POINTER(MoeWeights)]
        L.dlm_moe_prepare.argtypes = [i, C.POINTER(MoeWeights), p, z, p]
        L.dlm_moe_scratch_size.restype = z
        L.dlm_moe_scratch_size.argtypes = [i, i, C.POINTER(MoeWeights)]
        L.dlm_moe_mlp_nvfp4.argtypes = [p, p, i, i, f, C.POINTER(MoeWeights), p, p, p, p, z, p]
        L.dlm_lmhead_nvfp4_scratch_size.restype = z
        L.dlm_lmhead_nvfp4_scratch_size.argtypes = [i, i, i]
        L.dlm_lmhead_rowstats_nvfp4.argtypes = [p, C.POINTER(Nvfp4Matrix), i, i, i, i, RowStats, p, p, z, p]
        L.dlm_gemm_nvfp4_scratch_size.restype = z
        L.dlm_gemm_nvfp4_scratch_size.argtypes = [i, i, i]
        L.dlm_gemm_nvfp4.argtypes = [p, C.POINTER(Nvfp4Matrix), p, i, i, i, p, z, p]
        L.dlm_debug_set_pdl.argtypes = [i]
        _lib = L
    return _lib


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _addr(t):
    return None if t is None else t.data_ptr()


def _stream(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def _check(st, ctx=None):
    if st != DLM_OK:
        msg = ""
        if ctx is not None:
            m = lib().dlm_last_error(ctx)
            msg = m.decode() if m else ""
        raise DlmError(st, msg)


def set_pdl(on: bool) -> None:
    lib().dlm_debug_set_pdl(int(bool(on)))


# ------------------------------------------------------------------ single operations
def _scratch(nbytes, device):
    import torch
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def gemm_bf16(x, w, stream=None):
    """y[T][N] fp32 = x[T][K] (bf16) @ w[N][K]^T (bf16)."""
    import torch
    T, K = x.shape
    N = w.shape[0]
    y = torch.empty((T, N), dtype=torch.float32, device=x.device)
    n = lib().dlm_gemm_scratch_size(T, N, K)
    sc = _scratch(n, x.device)
    _check(lib().dlm_gemm_bf16(_ptr(x), _ptr(w), _ptr(y), T, N, K, _ptr(sc), n, _stream(stream)))
    return y


def gemm_bf16x2(x, w, stream=None):
    """y[T][N] fp32 = x[T][K] (fp32, split by the library into a bf16 hi + lo pair) @ w[N][K]^T
    (bf16): dlm_gemm_f32."""
    import torch
    T, K = x.shape
    N = w.shape[0]
    y = torch.empty((T, N), dtype=torch.float32, device=x.device)
    n = lib().dlm_gemm_f32_scratch_size(T, N, K)
    if n == 0:
        raise DlmError(DLM_EINVAL, "unsupported gemm shape")
    sc = _scratch(n, x.device)
    _check(lib().dlm_gemm_f32(_ptr(x.contiguous()), _ptr(w), _ptr(y), T, N, K, _ptr(sc), n, _stream(stream)))
    return y


def new_stats(B, device):
    import torch
    st = {k: torch.zeros(B, dtype=torch.float32, device=device) for k in ("m", "lse", "maxprob", "entropy")}
    st["argmax"] = torch.zeros(B, dtype=torch.int32, device=device)
    return st


def _rowstats(st):
    return RowStats(_ptr(st["m"]), _ptr(st["lse"]), _ptr(st["maxprob"]), _ptr(st["entropy"]), _ptr(st["argmax"]))


def lmhead_rowstats(x, E, mask_id=-1, p_given=None, stream=None):
    """Fused LM head: stats of x E^T and s = P E.  x bf16 [B][d] (normalised)."""
    import torch
    B, d = x.shape
    V = E.shape[0]
    st = new_stats(B, x.device)
    s = torch.empty((B, d), dtype=torch.float32, device=x.device)
    n = lib().dlm_lmhead_scratch_size(B, V, d)
    sc = _scratch(n, x.device)
    _check(lib().dlm_lmhead_rowstats(_ptr(x), _ptr(E), B, V, d, int(mask_id), _ptr(p_given), _rowstats(st),
                                     _ptr(s), _ptr(sc), n, _stream(stream)))
    st["s"] = s
    return st


def lmhead_rowstats_nvfp4(x, Eq, mask_id=-1, stream=None):
    """Fused LM head on an NVFP4 embedding: stats of Q(x) E^T and s = P E.  x fp32 [B][d]
    (normalised, quantized per row by the library); Eq a dict with device codes, scales,
    tscale, rows (V) and cols (d)."""
    import torch
    B, d = x.shape
    V = Eq["rows"]
    st = new_stats(B, x.device)
    s = torch.empty((B, d), dtype=torch.float32, device=x.device)
    n = lib().dlm_lmhead_nvfp4_scratch_size(B, V, d)
    if n == 0:
        raise DlmError(DLM_EUNSUPPORTED, "nvfp4 lm head: unsupported shape B=%d V=%d d=%d" % (B, V, d))
    sc = _scratch(n, x.device)
    m = _q_matrix(Eq)
    _check(lib().dlm_lmhead_rowstats_nvfp4(_ptr(x), C.byref(m), B, V, d, int(mask_id), _rowstats(st), _ptr(s),
                                           _ptr(sc), n, _stream(stream)))
    st["s"] = s
    return st


class Moe:
    """A routed-expert MLP sub-block on the device: router bf16 [E][d], norm gain bf16 [d],
    and the experts' NVFP4 stacks gate, up [E F][d] and down [d][E F] (dicts as
    nvfp4_matrix returns), with their scales re-tiled once (dlm_moe_prepare)."""

    def __init__(self, n_experts, top_k, ffn_expert, d, w_router, mlp_norm, q_gate, q_up, q_down, stream=None):
        import torch
        self.d = d
        self._keep = [w_router, mlp_norm, q_gate, q_up, q_down]
        self.w = MoeWeights(n_experts, top_k, ffn_expert, _ptr(w_router).value, _ptr(mlp_norm).value,
                            _q_matrix(q_gate), _q_matrix(q_up), _q_matrix(q_down))
        n = lib().dlm_moe_prepare_size(d, C.byref(self.w))
        if n == 0:
            raise DlmError(DLM_EUNSUPPORTED, "moe: unsupported shape E=%d k=%d F=%d d=%d" %
                           (n_experts, top_k, ffn_expert, d))
        self.tiles = torch.empty(n, dtype=torch.uint8, device=w_router.device)
        _check(lib().dlm_moe_prepare(d, C.byref(self.w), _ptr(self.tiles), n, _stream(stream)))
        self.k = top_k

    def __call__(self, h, eps=1e-6, stream=None):
        """h fp32 [T][d] -> (h_out fp32 [T][d], chosen experts int32 [T][k], weights fp32 [T][k])."""
        import torch
        T, d = h.shape
        out = torch.empty_like(h)
        idx = torch.empty((T, self.k), dtype=torch.int32, device=h.device)
        w = torch.empty((T, self.k), dtype=torch.float32, device=h.device)
        n = lib().dlm_moe_scratch_size(T, d, C.byref(self.w))
        if n == 0:
            raise DlmError(DLM_EUNSUPPORTED, "moe: unsupported rows T=%d d=%d" % (T, d))
        sc = _scratch(n, h.device)
        _check(lib().dlm_moe_mlp_nvfp4(_ptr(h), _ptr(out), T, d, float(eps), C.byref(self.w), _ptr(self.tiles),
                                       _ptr(idx), _ptr(w), _ptr(sc), n, _stream(stream)))
        return out, idx, w


def adapter_embed(E, Wa, tokens, s, stream=None):
    import torch
    B, d = s.shape
    h0 = torch.empty((B, d), dtype=torch.float32, device=s.device)
    n = lib().dlm_adapter_scratch_size(B, d)
    sc = _scratch(n, s.device)
    _check(lib().dlm_adapter_embed(_ptr(E), _ptr(Wa), _ptr(tokens), _ptr(s), _ptr(h0), B, d, _ptr(sc), n,
                                   _stream(stream)))
    return h0


def bd_attention(q, k_cache, v_cache, L, causal=False, stream=None):
    """q bf16 [T][Hq][hd]; caches bf16 [Hkv][max_ctx][hd] -> o bf16 [T][Hq][hd]."""
    import torch
    T, Hq, hd = q.shape
    Hkv, max_ctx, _ = k_cache.shape
    o = torch.empty_like(q)
    n = lib().dlm_attention_scratch_size(T, Hq, hd, max_ctx)
    sc = _scratch(n, q.device)
    _check(lib().dlm_bd_attention(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(o), T, int(L), Hq, Hkv, hd,
                                  max_ctx, int(causal), _ptr(sc), n, _stream(stream)))
    return o


def bd_attention_fp8(q, k_codes, k_scales, v_codes, v_scales, L, causal=False, stream=None):
    """Attention on an FP8 KV cache: codes uint8 [Hkv][max_ctx][hd] (e4m3), scales fp32
    [Hkv][max_ctx] -> o bf16 [T][Hq][hd]."""
    import torch
    T, Hq, hd = q.shape
    Hkv, max_ctx, _ = k_codes.shape
    o = torch.empty_like(q)
    n = lib().dlm_attention_scratch_size(T, Hq, hd, max_ctx)
    sc = _scratch(n, q.device)
    _check(lib().dlm_bd_attention_fp8(_ptr(q), _ptr(k_codes), _ptr(k_scales), _ptr(v_codes), _ptr(v_scales), _ptr(o),
                                      T, int(L), Hq, Hkv, hd, max_ctx, int(causal), _ptr(sc), n, _stream(stream)))
    return o


def bd_attention_noalloc(q, k_cache, v_cache, L, causal=False, o=None, stream=None):
    """bd_attention through the entry point that takes no scratch (library-owned static
    device memory; see dlm_bd_attention_noalloc).  `o` may be given to reuse an output."""
    import torch
    T, Hq, hd = q.shape
    Hkv, max_ctx, _ = k_cache.shape
    if o is None:
        o = torch.empty_like(q)
    _check(lib().dlm_bd_attention_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(o), T, int(L), Hq, Hkv,
                                          hd, max_ctx, int(causal), _stream(stream)))
    return o


def commit(maxprob, argmax, tokens, committed, s, rnd, tau, mode, k, status=None, stream=None):
    B, d = s.shape
    _check(lib().dlm_commit(_ptr(maxprob), _ptr(argmax), _ptr(tokens), _ptr(committed), _ptr(s), _ptr(rnd),
                            _ptr(status), B, d, float(tau), int(mode), int(k), _stream(stream)))


def nvfp4_quantize(w, stream=None):
    """bf16 [rows][cols] -> (codes uint8 [rows][cols/2], scales uint8 [rows][cols/16], tscale fp32 [1])."""
    import torch
    rows, cols = w.shape
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=w.device)
    scales = torch.empty((rows, cols // 16), dtype=torch.uint8, device=w.device)
    ts = torch.empty(1, dtype=torch.float32, device=w.device)
    _check(lib().dlm_nvfp4_quantize(_ptr(w), rows, cols, _ptr(codes), _ptr(scales), _ptr(ts), _stream(stream)))
    return codes, scales, ts


def _q_matrix(q):
    return Nvfp4Matrix(_ptr(q["codes"]).value, _ptr(q["scales"]).value, float(q["tscale"]))


def nvfp4_matrix(w, stream=None):
    """NVFP4 form of a bf16 [rows][cols] weight as a dict(codes, scales, tscale (float), rows, cols)."""
    codes, scales, ts = nvfp4_quantize(w, stream)
    return {"codes": codes, "scales": scales, "tscale": float(ts.item()), "rows": w.shape[0], "cols": w.shape[1]}


def quantize_model(weights: dict, stream=None) -> dict:
    """Adds the NVFP4 matrices an NVFP4 model runs on (q_gate, q_up, q_down per layer and
    q_embed) to a bf16 weight dict, quantized on the device."""
    out = dict(weights)
    out["layers"] = []
    for lw in weights["layers"]:
        l2 = dict(lw)
        for n in ("gate", "up", "down"):
            l2["q_" + n] = nvfp4_matrix(lw["w_" + n], stream)
        out["layers"].append(l2)
    out["q_embed"] = nvfp4_matrix(weights["embed"], stream)
    return out


def gemm_nvfp4(x, q, stream=None):
    """y[T][N] fp32 = Q(x) W^T with W the NVFP4 matrix q (see nvfp4_matrix) and Q the
    per-row NVFP4 quantizer of x (fp32 [T][K])."""
    import torch
    T, K = x.shape
    N = q["rows"]
    y = torch.empty((T, N), dtype=torch.float32, device=x.device)
    n = lib().dlm_gemm_nvfp4_scratch_size(T, N, K)
    if n == 0:
        raise DlmError(DLM_EINVAL, "unsupported nvfp4 gemm shape")
    sc = _scratch(n, x.device)
    m = _q_matrix(q)
    _check(lib().dlm_gemm_nvfp4(_ptr(x), C.byref(m), _ptr(y), T, N, K, _ptr(sc), n, _stream(stream)))
    return y


# ------------------------------------------------------------------ model context
class Model:
    """Owns (through torch) the workspace and the KV cache of one dlm context."""

    def __init__(self, cfg: dict, weights: dict, device="cuda"):
        import torch
        self.cfg_d = dict(cfg)
        self.cfg = Config.from_dict(cfg)
        self.device = torch.device(device)
        self.weights = weights  # keeps tensors alive
        L = lib()
        nl = cfg["n_layers"]
        self._layers = (LayerWeights * max(nl, 1))()
        fp4 = int(cfg.get("weight_fmt", 0)) == WEIGHTS_NVFP4
        empty = Nvfp4Matrix(None, None, 0.0)
        for i, lw in enumerate(weights["layers"]):
            qs = [_q_matrix(lw["q_" + n]) if fp4 else empty for n in ("gate", "up", "down")]
            self._layers[i] = LayerWeights(_ptr(lw["attn_norm"]).value, _ptr(lw["w_qkv"]).value,
                                           _ptr(lw["w_o"]).value, _ptr(lw["mlp_norm"]).value,
                                           _addr(lw.get("w_gate")), _addr(lw.get("w_up")),
                                           _addr(lw.get("w_down")), *qs)
        self._w = Weights(_addr(weights.get("embed")), _ptr(weights["w_adapter"]).value,
                          _ptr(weights["final_norm"]).value, self._layers,
                          _q_matrix(weights["q_embed"]) if fp4 else empty)
        ws = L.dlm_workspace_size(C.byref(self.cfg))
        kv = L.dlm_kv_cache_size(C.byref(self.cfg))
        if ws == 0:
            raise DlmError(DLM_EINVAL, "invalid config")
        self.workspace = torch.empty(ws, dtype=torch.uint8, device=self.device)
        self.kv = torch.zeros(max(kv, 256), dtype=torch.uint8, device=self.device)
        ctx = C.c_void_p()
        _check(L.dlm_ctx_create(C.byref(self.cfg), C.byref(self._w), _ptr(self.workspace), ws, _ptr(self.kv),
                                kv, C.byref(ctx)))
        self.ctx = ctx

    def close(self):
        if self.ctx:
            lib().dlm_ctx_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # KV cache views: [layer][K|V][kv_head][max_ctx][head_dim]
    def kv_view(self):
        """bf16 cache values (DLM_KV_BF16 contexts)."""
        c = self.cfg_d
        assert int(c.get("kv_fmt", 0)) == KV_BF16
        import torch
        n = 2 * c["n_layers"] * c["n_kv_heads"] * c["max_ctx"] * c["head_dim"]
        return self.kv[: 2 * n].view(torch.bfloat16).view(c["n_layers"], 2, c["n_kv_heads"], c["max_ctx"],
                                                          c["head_dim"])

    def kv_view_fp8(self):
        """(codes uint8 [layer][K|V][kv_head][max_ctx][head_dim], scales fp32
        [layer][K|V][kv_head][max_ctx]) of a DLM_KV_FP8 context."""
        import torch
        c = self.cfg_d
        assert int(c.get("kv_fmt", 0)) == KV_FP8
        rows = 2 * c["n_layers"] * c["n_kv_heads"] * c["max_ctx"]
        codes = self.kv[: rows * c["head_dim"]].view(c["n_layers"], 2, c["n_kv_heads"], c["max_ctx"], c["head_dim"])
        scales = self.kv[rows * c["head_dim"]: rows * c["head_dim"] + 4 * rows].view(torch.float32).view(
            c["n_layers"], 2, c["n_kv_heads"], c["max_ctx"])
        return codes, scales

    @property
    def prefix_len(self):
        return lib().dlm_prefix_len(self.ctx)

    def set_prefix_len(self, L, stream=None):
        _check(lib().dlm_set_prefix_len(self.ctx, int(L), _stream(stream)), self.ctx)

    def prefill(self, tokens, stream=None):
        _check(lib().dlm_prefill(self.ctx, _ptr(tokens), int(tokens.numel()), _stream(stream)), self.ctx)

    def new_block_state(self):
        import torch
        B, d = self.cfg.block_size, self.cfg.d
        st = dict(tokens=torch.zeros(B, dtype=torch.int32, device=self.device),
                  committed=torch.zeros(B, dtype=torch.uint8, device=self.device),
                  s=torch.zeros((B, d), dtype=torch.float32, device=self.device),
                  round=torch.zeros(1, dtype=torch.int32, device=self.device),
                  status=torch.zeros(1, dtype=torch.int32, device=self.device))
        st["stats"] = new_stats(B, self.device)
        return st

    @staticmethod
    def _bs(st):
        return BlockState(_ptr(st["tokens"]), _ptr(st["committed"]), _ptr(st["s"]), _ptr(st["round"]),
                          _ptr(st["status"]), _rowstats(st["stats"]))

    def block_init(self, st, stream=None):
        _check(lib().dlm_block_init(self.ctx, C.byref(self._bs(st)), _stream(stream)), self.ctx)

    def round(self, st, tau, mode=COMMIT_THRESHOLD, k=1, stream=None):
        _check(lib().dlm_round(self.ctx, C.byref(self._bs(st)), float(tau), int(mode), int(k), _stream(stream)),
               self.ctx)

    def kv_fill(self, tokens, stream=None):
        _check(lib().dlm_kv_fill(self.ctx, _ptr(tokens), _stream(stream)), self.ctx)

    def kv_flush(self, stream=None):
        _check(lib().dlm_kv_flush(self.ctx, _stream(stream)), self.ctx)

    @property
    def fill_pending(self):
        return bool(lib().dlm_fill_pending(self.ctx))

    def set_fill_mode(self, mode, stream=None):
        _check(lib().dlm_set_fill_mode(self.ctx, int(mode), _stream(stream)), self.ctx)

    def mlp_block(self, layer, h, stream=None):
        """One layer's MLP sub-block on fp32 residual rows h [T][d] (dlm_mlp_block)."""
        import torch
        h = h.contiguous()
        out = torch.empty_like(h)
        _check(lib().dlm_mlp_block(self.ctx, int(layer), _ptr(h), _ptr(out), int(h.shape[0]), _stream(stream)),
               self.ctx)
        return out

    def decode_block(self, tau, mode=COMMIT_THRESHOLD, k=1, tokens_out=None, rounds_out=None, stream=None):
        _check(lib().dlm_decode_block(self.ctx, float(tau), int(mode), int(k), _ptr(tokens_out), _ptr(rounds_out),
                                      _stream(stream)), self.ctx)

    def generate(self, prompt, max_new, tau, mode=COMMIT_THRESHOLD, k=1, stream=None):
        """prompt: host int32 array-like.  Returns (tokens np.int32 [max_new], rounds per block, timing)."""
        import numpy as np
        pr = np.ascontiguousarray(prompt, dtype=np.int32)
        B = self.cfg.block_size
        nblk = (max_new + B - 1) // B
        out = np.zeros(max(max_new, 1), np.int32)
        rpb = np.zeros(max(nblk, 1), np.int32)
        tm = Timing()
        _check(lib().dlm_generate(self.ctx, pr.ctypes.data, len(pr), int(max_new), float(tau), int(mode), int(k),
                                  out.ctypes.data, rpb.ctypes.data, C.byref(tm), _stream(stream)), self.ctx)
        return out[:max_new], rpb[:nblk], tm
