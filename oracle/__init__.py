"""ctypes wrapper of the C++17 CPU oracle (oracle/dlm_oracle.cpp).

TEST INFRASTRUCTURE ONLY: tests/, __graft_entry__.smoke() and bench.py's cpu_baseline /
reference leg are the only callers.  The CUDA library never imports, links or runs
anything from this package, and this package imports nothing from the CUDA library.

All arrays are numpy; weights are bf16 bit patterns (uint16) or NVFP4 triples
(codes uint8 [rows][cols/2], scales uint8 e4m3 [rows][cols/16], fp32 tensor scale).
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dlm_oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")


def build(force: bool = False) -> str:
    """Compile the oracle with g++ (plain -O2, no fast-math: IEEE semantics are part of it)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["g++", "-std=c++17", "-O2", "-fPIC", "-shared", "-pthread",
                               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp])
        os.replace(tmp, _LIB)
    return _LIB


class Mat(C.Structure):
    _fields_ = [("fmt", C.c_int), ("rows", C.c_int), ("cols", C.c_int),
                ("bf16", C.c_void_p), ("codes", C.c_void_p), ("scales", C.c_void_p),
                ("tscale", C.c_float)]


class Cfg(C.Structure):
    _fields_ = [("n_layers", C.c_int), ("d", C.c_int), ("n_q_heads", C.c_int),
                ("n_kv_heads", C.c_int), ("head_dim", C.c_int), ("ffn", C.c_int),
                ("vocab", C.c_int), ("mask_id", C.c_int), ("block_size", C.c_int),
                ("rope_theta", C.c_double), ("rms_eps", C.c_double),
                ("act_round", C.c_int), ("act_fp4", C.c_int), ("kv_fp8", C.c_int)]


class Layer(C.Structure):
    _fields_ = [("attn_norm", C.c_void_p), ("w_qkv", Mat), ("w_o", Mat),
                ("mlp_norm", C.c_void_p), ("w_gate", Mat), ("w_up", Mat), ("w_down", Mat)]


class Model(C.Structure):
    _fields_ = [("embed", Mat), ("w_adapter", Mat), ("final_norm", C.c_void_p),
                ("layers", C.POINTER(Layer))]


class Moe(C.Structure):
    _fields_ = [("n_experts", C.c_int), ("top_k", C.c_int), ("ffn_expert", C.c_int),
                ("w_router", C.c_void_p), ("norm", C.c_void_p), ("gate", Mat), ("up", Mat),
                ("down", Mat)]


class KV(C.Structure):
    _fields_ = [("max_ctx", C.c_int), ("k", C.c_void_p), ("v", C.c_void_p)]


class Stats(C.Structure):
    _fields_ = [("m", C.c_double), ("lse", C.c_double), ("maxprob", C.c_double),
                ("entropy", C.c_double), ("argmax", C.c_int), ("gap2", C.c_double), ("qmargin", C.c_double)]


class Block(C.Structure):
    _fields_ = [("tokens", C.c_void_p), ("committed", C.c_void_p), ("s", C.c_void_p),
                ("round", C.c_int)]


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        L = _lib
        d, i, p, f = C.c_double, C.c_int, C.c_void_p, C.c_float
        L.orc_round_bf16.restype = d
        L.orc_round_bf16.argtypes = [d]
        L.orc_set_threads.argtypes = [i]
        L.orc_hw_threads.restype = i
        L.orc_nvfp4_tensor_scale.restype = f
        L.orc_nvfp4_tensor_scale.argtypes = [p, C.c_long]
        L.orc_nvfp4_quantize.argtypes = [p, i, i, p, p, p]
        L.orc_nvfp4_quantize_row.argtypes = [p, i, f, p, p]
        L.orc_nvfp4_dequant.argtypes = [p, p, f, i, i, p]
        L.orc_e2m1_value.restype = d
        L.orc_e2m1_value.argtypes = [i]
        L.orc_e2m1_encode.restype = i
        L.orc_e2m1_encode.argtypes = [f]
        L.orc_e4m3_round.restype = d
        L.orc_e4m3_round.argtypes = [f]
        L.orc_e4m3_bits.restype = i
        L.orc_e4m3_bits.argtypes = [d]
        L.orc_e4m3_value.restype = d
        L.orc_e4m3_value.argtypes = [i]
        L.orc_linear.argtypes = [p, i, C.POINTER(Mat), p, i]
        L.orc_rmsnorm.argtypes = [p, i, i, p, d, p]
        L.orc_rope.argtypes = [p, i, C.c_long, d]
        L.orc_attention.argtypes = [p, i, i, i, i, p, p, i, i, i, p]
        L.orc_rowstats.argtypes = [p, i, i, i, C.POINTER(Stats)]
        L.orc_kv_quantize_row.restype = C.c_float
        L.orc_kv_quantize_row.argtypes = [p, i, p, p]
        L.orc_lmhead.argtypes = [p, i, C.POINTER(Mat), i, i, p, C.POINTER(Stats), p, p]
        L.orc_moe_mlp.argtypes = [p, i, i, d, C.POINTER(Moe), i, p, p, p, p, p]
        L.orc_commit.restype = i
        L.orc_commit.argtypes = [i, p, p, d, i, i, p, p]
        L.orc_forward.argtypes = [C.POINTER(Model), C.POINTER(Cfg), p, p, i, i, i,
                                  C.POINTER(KV), p]
        L.orc_round.restype = i
        L.orc_round.argtypes = [C.POINTER(Model), C.POINTER(Cfg), C.POINTER(Block),
                                C.POINTER(KV), i, d, i, i, C.POINTER(Stats)]
        L.orc_decode_block.restype = i
        L.orc_decode_block.argtypes = [C.POINTER(Model), C.POINTER(Cfg), C.POINTER(KV), i, d,
                                       i, i, p]
        L.orc_prefill.argtypes = [C.POINTER(Model), C.POINTER(Cfg), C.POINTER(KV), p, i]
        L.orc_generate.restype = i
        L.orc_generate.argtypes = [C.POINTER(Model), C.POINTER(Cfg), C.POINTER(KV), p, i, i,
                                   d, i, i, p, p]
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a


def set_threads(n: int) -> None:
    lib().orc_set_threads(int(n))


def hw_threads() -> int:
    return int(lib().orc_hw_threads())


# ------------------------------------------------------------------ number formats
def round_bf16(x: float) -> float:
    return float(lib().orc_round_bf16(float(x)))


def e2m1_value(code: int) -> float:
    return float(lib().orc_e2m1_value(int(code)))


def e2m1_encode(r: float) -> int:
    return int(lib().orc_e2m1_encode(float(r)))


def e4m3_round(x: float) -> float:
    return float(lib().orc_e4m3_round(float(x)))


def e4m3_bits(v: float) -> int:
    return int(lib().orc_e4m3_bits(float(v)))


def kv_quantize(rows):
    """FP8 KV rows (R13): float [n][hd] -> (codes uint8 [n][hd], scales fp32 [n], values [n][hd])."""
    x = _c(np.atleast_2d(rows), np.float64)
    n, hd = x.shape
    codes = np.zeros((n, hd), np.uint8)
    vals = np.zeros((n, hd), np.float64)
    scales = np.zeros(n, np.float32)
    for r in range(n):
        xr = np.ascontiguousarray(x[r])
        cr = np.zeros(hd, np.uint8)
        vr = np.zeros(hd, np.float64)
        scales[r] = lib().orc_kv_quantize_row(_ptr(xr), hd, _ptr(cr), _ptr(vr))
        codes[r], vals[r] = cr, vr
    return codes, scales, vals


def e4m3_value(b: int) -> float:
    return float(lib().orc_e4m3_value(int(b)))


def nvfp4_quantize(w):
    """w float32 [rows][cols] -> (codes uint8 [rows][cols/2], scales uint8 [rows][cols/16], S)."""
    w = _c(w, np.float32)
    rows, cols = w.shape
    codes = np.zeros((rows, cols // 2), np.uint8)
    scales = np.zeros((rows, cols // 16), np.uint8)
    S = np.zeros(1, np.float32)
    lib().orc_nvfp4_quantize(_ptr(w), rows, cols, _ptr(codes), _ptr(scales), _ptr(S))
    return codes, scales, float(S[0])


def nvfp4_dequant(codes, scales, S, rows, cols):
    out = np.zeros((rows, cols), np.float64)
    lib().orc_nvfp4_dequant(_ptr(_c(codes, np.uint8)), _ptr(_c(scales, np.uint8)), float(S),
                            rows, cols, _ptr(out))
    return out


# ------------------------------------------------------------------ matrices
class Weights:
    """Keeps numpy buffers alive for the ctypes structs that point into them."""

    def __init__(self):
        self._keep = []

    def mat(self, m) -> Mat:
        """m: uint16 bf16-bit array [rows][cols], or a dict(codes=, scales=, tscale=, rows=, cols=)."""
        if isinstance(m, dict):
            codes = _c(m["codes"], np.uint8)
            scales = _c(m["scales"], np.uint8)
            self._keep += [codes, scales]
            return Mat(1, int(m["rows"]), int(m["cols"]), None, _ptr(codes), _ptr(scales),
                       float(m["tscale"]))
        a = _c(m, np.uint16)
        self._keep.append(a)
        return Mat(0, a.shape[0], a.shape[1], _ptr(a), None, None, 0.0)

    def vec(self, v):
        a = _c(v, np.uint16)
        self._keep.append(a)
        return _ptr(a)


def linear(x, W, act_fp4=False):
    """y = x W^T in fp64; x [T][K] float, W bf16 bits [N][K] or NVFP4 dict."""
    x = _c(x, np.float64)
    T = x.shape[0]
    wk = Weights()
    m = wk.mat(W)
    y = np.zeros((T, m.rows), np.float64)
    lib().orc_linear(_ptr(x), T, C.byref(m), _ptr(y), int(act_fp4))
    return y


def rmsnorm(x, g_bits, eps):
    x = _c(x, np.float64)
    rows, n = x.shape
    g = _c(g_bits, np.uint16)
    out = np.zeros_like(x)
    lib().orc_rmsnorm(_ptr(x), rows, n, _ptr(g), float(eps), _ptr(out))
    return out


def rope(x, pos, base):
    x = _c(x, np.float64).copy()
    lib().orc_rope(_ptr(x), x.shape[0], int(pos), float(base))
    return x


def attention(q, kc, vc, pos0, causal=False):
    """q [nq][Hq][hd]; kc, vc [Hkv][max_ctx][hd] -> out [nq][Hq][hd]."""
    q = _c(q, np.float64)
    kc = _c(kc, np.float64)
    vc = _c(vc, np.float64)
    nq, Hq, hd = q.shape
    Hkv, max_ctx, _ = kc.shape
    out = np.zeros_like(q)
    lib().orc_attention(_ptr(q), nq, Hq, Hkv, hd, _ptr(kc), _ptr(vc), max_ctx, int(pos0),
                        int(causal), _ptr(out))
    return out


def _stats_to_dict(st):
    return {k: np.array([getattr(s, k) for s in st])
            for k in ("m", "lse", "maxprob", "entropy", "argmax", "gap2", "qmargin")}


def rowstats(logits, mask_id=-1):
    logits = _c(logits, np.float64)
    B, V = logits.shape
    st = (Stats * B)()
    lib().orc_rowstats(_ptr(logits), B, V, int(mask_id), st)
    return _stats_to_dict(st)


def lmhead(x, E, mask_id=-1, p_given=None, act_fp4=False, want_logits=False):
    """Row stats of x E^T and s = P E (P = softmax of the logits, or p_given)."""
    x = _c(x, np.float64)
    B = x.shape[0]
    wk = Weights()
    m = wk.mat(E)
    st = (Stats * B)()
    s = np.zeros((B, m.cols), np.float64)
    pg = None if p_given is None else _c(p_given, np.float64)
    logits = np.zeros((B, m.rows), np.float64) if want_logits else None
    lib().orc_lmhead(_ptr(x), B, C.byref(m), int(mask_id), int(act_fp4), _ptr(pg), st, _ptr(s),
                     _ptr(logits))
    out = _stats_to_dict(st)
    out["s"] = s
    if want_logits:
        out["logits"] = logits
    return out


def moe_mlp(h_in, moe, eps=1e-6, act_fp4=True):
    """Routed-expert MLP sub-block (R14).  h_in [T][d]; moe: dict(n_experts, top_k,
    ffn_expert, w_router (bf16 bits [E][d]), norm (bf16 bits [d]), gate, up ([E F][d]) and
    down ([d][E F]) as bf16 bits or NVFP4 dicts).  Returns dict(h_out, logits [T][E],
    idx [T][k], w [T][k], qmargin [T])."""
    h = _c(h_in, np.float64)
    T, d = h.shape
    E, k, F = int(moe["n_experts"]), int(moe["top_k"]), int(moe["ffn_expert"])
    wk = Weights()
    m = Moe(E, k, F, wk.vec(moe["w_router"]), wk.vec(moe["norm"]), wk.mat(moe["gate"]),
            wk.mat(moe["up"]), wk.mat(moe["down"]))
    out = np.zeros_like(h)
    logits = np.zeros((T, E), np.float64)
    idx = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float64)
    qm = np.zeros(T, np.float64)
    lib().orc_moe_mlp(_ptr(h), T, d, float(eps), C.byref(m), int(act_fp4), _ptr(out), _ptr(logits),
                      _ptr(idx), _ptr(w), _ptr(qm))
    return {"h_out": out, "logits": logits, "idx": idx, "w": w, "qmargin": qm}


def commit(maxprob, argmax, tau, mode, k, tokens, committed):
    """Applies the commit rule in place on copies; returns (n, tokens, committed)."""
    mp = _c(maxprob, np.float64)
    am = _c(argmax, np.int32)
    tok = _c(tokens, np.int32).copy()
    com = _c(committed, np.uint8).copy()
    n = lib().orc_commit(len(mp), _ptr(mp), _ptr(am), float(tau), int(mode), int(k), _ptr(tok),
                         _ptr(com))
    return int(n), tok, com


# ------------------------------------------------------------------ model level
class OracleModel:
    """Binds a weight dict (see block_diffusion_decoding_denoising_b200.gen) to the oracle."""

    def __init__(self, cfg: dict, weights: dict, act_round=True, max_ctx=None):
        self.cfg_d = dict(cfg)
        self.wk = Weights()
        c = cfg
        nvfp4 = bool(c.get("weight_fmt", 0))
        self.cfg = Cfg(c["n_layers"], c["d"], c["n_q_heads"], c["n_kv_heads"], c["head_dim"],
                       c["ffn"], c["vocab"], c["mask_id"], c["block_size"], float(c["rope_theta"]),
                       float(c["rms_eps"]), int(act_round), int(nvfp4), int(c.get("kv_fmt", 0)))
        layers = (Layer * c["n_layers"])()
        for i, lw in enumerate(weights["layers"]):
            layers[i] = Layer(self.wk.vec(lw["attn_norm"]), self.wk.mat(lw["w_qkv"]),
                              self.wk.mat(lw["w_o"]), self.wk.vec(lw["mlp_norm"]),
                              self.wk.mat(lw["w_gate"]), self.wk.mat(lw["w_up"]),
                              self.wk.mat(lw["w_down"]))
        self._layers = layers
        self.model = Model(self.wk.mat(weights["embed"]), self.wk.mat(weights["w_adapter"]),
                           self.wk.vec(weights["final_norm"]), layers)
        self.max_ctx = int(max_ctx or c["max_ctx"])
        hk = (c["n_layers"], c["n_kv_heads"], self.max_ctx, c["head_dim"])
        self.kc = np.zeros(hk, np.float64)
        self.vc = np.zeros(hk, np.float64)
        self.kv = KV(self.max_ctx, _ptr(self.kc), _ptr(self.vc))

    def prefill(self, prompt):
        pr = _c(prompt, np.int32)
        lib().orc_prefill(C.byref(self.model), C.byref(self.cfg), C.byref(self.kv), _ptr(pr), len(pr))

    def forward(self, tokens, s, pos0, causal=False, want_xf=True):
        tok = _c(tokens, np.int32)
        n = len(tok)
        sa = None if s is None else _c(s, np.float64)
        xf = np.zeros((n, self.cfg.d), np.float64) if want_xf else None
        lib().orc_forward(C.byref(self.model), C.byref(self.cfg), _ptr(tok), _ptr(sa), n, int(pos0),
                          int(causal), C.byref(self.kv), _ptr(xf))
        return xf

    def round(self, tokens, committed, s, rnd, L, tau, mode, k):
        """One round on copies of the given state; returns (n_committed, new_state, stats)."""
        B = self.cfg.block_size
        tok = _c(tokens, np.int32).copy()
        com = _c(committed, np.uint8).copy()
        ss = _c(s, np.float64).copy()
        blk = Block(_ptr(tok), _ptr(com), _ptr(ss), int(rnd))
        st = (Stats * B)()
        n = lib().orc_round(C.byref(self.model), C.byref(self.cfg), C.byref(blk), C.byref(self.kv),
                            int(L), float(tau), int(mode), int(k), st)
        return int(n), dict(tokens=tok, committed=com, s=ss, round=blk.round), _stats_to_dict(st)

    def decode_block(self, L, tau, mode, k):
        B = self.cfg.block_size
        out = np.zeros(B, np.int32)
        r = lib().orc_decode_block(C.byref(self.model), C.byref(self.cfg), C.byref(self.kv), int(L),
                                   float(tau), int(mode), int(k), _ptr(out))
        return int(r), out

    def generate(self, prompt, max_new, tau, mode, k):
        B = self.cfg.block_size
        pr = _c(prompt, np.int32)
        nblk = (max_new + B - 1) // B
        out = np.zeros(max_new, np.int32)
        rpb = np.zeros(nblk, np.int32)
        r = lib().orc_generate(C.byref(self.model), C.byref(self.cfg), C.byref(self.kv), _ptr(pr),
                               len(pr), int(max_new), float(tau), int(mode), int(k), _ptr(out),
                               _ptr(rpb))
        return int(r), out, rpb
