"""ORACLE -- plain, slow CPU definition of the canvas denoising step (fp64).

Test infrastructure only: the tests, the smoke check and the benchmark's CPU-baseline leg may import
it; the product path never does.  The arithmetic lives in ``dg_oracle.c`` (plain C, OpenMP over
rows, fp64); this module only marshals numpy arrays through ctypes and strings the C pieces
together in the order the pages describe the decoder loop ("Composition of DiffusionGemma"
flowchart in the technical-report summary "DiffusionGemma: a diffusion LLM that refines 256-token
blocks in parallel"): prompt -> KV cache; 256-token canvas of noise; denoise step; adaptive-stop
check; commit block to the KV cache; stop at EOS, else a new canvas.

It shares no code with the CUDA path; only the ``synthetic`` input generators serve both.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None

c_int, c_double, c_float, c_void_p, c_uint32, c_uint64 = (
    ctypes.c_int, ctypes.c_double, ctypes.c_float, ctypes.c_void_p, ctypes.c_uint32, ctypes.c_uint64)


def lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.orc_philox4x32_10.argtypes = [c_void_p, c_void_p, c_void_p]
        L.orc_rng_word.argtypes = [c_uint64, c_uint32, c_uint32, c_uint32, c_uint32, c_int]
        L.orc_rng_word.restype = c_uint32
        L.orc_uniform.argtypes = [c_uint32]
        L.orc_uniform.restype = c_double
        L.orc_gumbel.argtypes = [c_uint32]
        L.orc_gumbel.restype = c_double
        L.orc_token_from_word.argtypes = [c_uint32, c_uint32]
        L.orc_token_from_word.restype = ctypes.c_int32
        L.orc_temperature.argtypes = [c_int, c_int, c_float, c_float]
        L.orc_temperature.restype = c_float
        L.orc_e4m3_to_double.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_to_double.restype = c_double
        L.orc_rmsnorm.argtypes = [c_int, c_int, c_void_p, c_void_p, c_double, c_void_p]
        L.orc_rope.argtypes = [c_int, c_int, c_int, c_void_p, c_double, c_void_p]
        L.orc_attention.argtypes = [c_int, c_int, c_int, c_int, c_int, c_void_p, c_void_p, c_void_p,
                                    c_void_p, c_void_p]
        L.orc_router_topk.argtypes = [c_int, c_int, c_int, c_void_p, c_void_p, c_void_p]
        L.orc_router_topk_flip.argtypes = [c_int, c_int, c_int, c_void_p, c_void_p, c_void_p, c_void_p]
        L.orc_moe.argtypes = [c_void_p, c_void_p, c_int, c_int, c_void_p, c_void_p, c_void_p, c_void_p]
        L.orc_layer_forward.argtypes = [c_void_p, c_void_p, c_int, c_void_p, c_void_p, c_int, c_void_p,
                                        c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_void_p]
        L.orc_layer_forward.restype = c_int
        L.orc_layer_forward_flip.argtypes = L.orc_layer_forward.argtypes + [c_void_p]
        L.orc_layer_forward_flip.restype = c_int
        L.orc_forward.argtypes = [c_void_p, c_void_p, c_int, c_void_p, c_void_p, c_int, c_void_p, c_void_p,
                                  c_int, c_int, c_void_p, c_void_p, c_void_p]
        L.orc_forward.restype = c_int
        L.orc_forward_flip.argtypes = L.orc_forward.argtypes + [c_void_p]
        L.orc_forward_flip.restype = c_int
        L.orc_head.argtypes = [c_void_p, c_void_p, c_int, c_void_p, c_void_p]
        L.orc_embed.argtypes = [c_void_p, c_void_p, c_int, c_void_p, c_void_p]
        for name in ("orc_sample_rows_f32", "orc_sample_rows_f64"):
            getattr(L, name).argtypes = [c_int, c_int, c_void_p, c_void_p, c_void_p, c_float, c_uint64, c_int,
                                         c_void_p, c_void_p, c_void_p, c_void_p]
        L.orc_step_rule.argtypes = [c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_double, c_double,
                                    c_double, c_int, c_int, c_int, c_int, c_void_p, c_void_p, c_void_p, c_void_p]
        L.orc_step_rule.restype = c_int
        L.orc_canvas_init.argtypes = [c_int, c_int, c_uint64, c_int, c_void_p, c_void_p]
        _LIB = L
    return _LIB


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(c_void_p)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


# ---------------------------------------------------------------------------------------------
# scalar pieces
# ---------------------------------------------------------------------------------------------

def philox4x32_10(ctr, key) -> np.ndarray:
    c = np.ascontiguousarray(np.asarray(ctr, dtype=np.uint32))
    k = np.ascontiguousarray(np.asarray(key, dtype=np.uint32))
    out = np.zeros(4, dtype=np.uint32)
    lib().orc_philox4x32_10(_p(c), _p(k), _p(out))
    return out


def rng_word(seed, c0, pos, step, tag, word) -> int:
    return int(lib().orc_rng_word(seed, c0, pos, step, tag, word))


def uniform(x: int) -> float:
    return float(lib().orc_uniform(x))


def gumbel(x: int) -> float:
    return float(lib().orc_gumbel(x))


def token_from_word(x: int, vocab: int) -> int:
    return int(lib().orc_token_from_word(x, vocab))


def temperature(s: int, max_steps: int = 48, t_start: float = 0.8, t_end: float = 0.4) -> float:
    return float(lib().orc_temperature(s, max_steps, t_start, t_end))


def e4m3_to_double(q: int) -> float:
    return float(lib().orc_e4m3_to_double(q))


def rmsnorm(x, g, eps=1e-6) -> np.ndarray:
    x = _f64(x)
    n, d = x.shape
    g = np.ascontiguousarray(np.asarray(g, dtype=np.float32))
    out = np.empty_like(x)
    lib().orc_rmsnorm(n, d, _p(x), _p(g), eps, _p(out))
    return out


def rope(x, pos, theta=10000.0) -> np.ndarray:
    """x [n_tok, n_head, dh] -> rotated copy."""
    x = _f64(x).copy()
    n, h, dh = x.shape
    pos = np.ascontiguousarray(np.asarray(pos, dtype=np.int32))
    lib().orc_rope(n, h, dh, _p(pos), theta, _p(x))
    return x


def attention(q, k, v, mask) -> np.ndarray:
    """q [n, Hq, dh], k/v [m, Hkv, dh], mask [n, m] (1 = visible) -> [n, Hq, dh]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    n, hq, dh = q.shape
    m, hkv, _ = k.shape
    mask = np.ascontiguousarray(np.asarray(mask, dtype=np.uint8))
    out = np.empty((n, hq, dh))
    lib().orc_attention(n, m, hq, hkv, dh, _p(q), _p(k), _p(v), _p(mask), _p(out))
    return out


def router_topk(logits, k, flip=None):
    """Top-k selection and gates; flip (optional bool [n]): those tokens take their (k+1)-th expert in
    place of their k-th (the other choice at a near-tie)."""
    logits = _f64(logits)
    n, E = logits.shape
    sel = np.empty((n, k), dtype=np.int32)
    gate = np.empty((n, k))
    if flip is None:
        lib().orc_router_topk(n, E, k, _p(logits), _p(sel), _p(gate))
    else:
        fl = np.ascontiguousarray(np.asarray(flip, dtype=np.uint8))
        lib().orc_router_topk_flip(n, E, k, _p(logits), _p(fl), _p(sel), _p(gate))
    return sel, gate


# ---------------------------------------------------------------------------------------------
# model marshalling
# ---------------------------------------------------------------------------------------------

class _Mat(ctypes.Structure):
    _fields_ = [("bf16", c_void_p), ("e4m3", c_void_p), ("scale", c_void_p), ("rows", c_int), ("cols", c_int)]


class _Cfg(ctypes.Structure):
    _fields_ = [(n, c_int) for n in ("d_model", "n_q", "n_kv", "d_head", "n_exp", "top_k", "d_ff",
                                     "n_layers", "vocab")] + [("rms_eps", c_double), ("rope_theta", c_double)]


class _Layer(ctypes.Structure):
    _fields_ = [("attn_norm", c_void_p), ("w_qkv", _Mat), ("w_o", _Mat), ("ffn_norm", c_void_p),
                ("w_router", _Mat), ("w_gate_up", _Mat), ("w_down", _Mat)]


class _Model(ctypes.Structure):
    _fields_ = [("emb", c_void_p), ("final_norm", c_void_p), ("head", c_void_p), ("layers", ctypes.POINTER(_Layer))]


def _np_weight(t):
    """torch tensor (bf16 / fp32 / uint8) or numpy array -> contiguous numpy array."""
    import torch
    if isinstance(t, torch.Tensor):
        t = t.detach().contiguous().cpu()
        if t.dtype == torch.bfloat16:
            return t.view(torch.int16).numpy().view(np.uint16)
        return t.numpy()
    return np.ascontiguousarray(t)


class Model:
    """Holds numpy views of one model's weights in the layout documented in ``synthetic`` and the
    ctypes structs that point at them.  A layer matrix may be given in bf16 or, for the FP8 form,
    as a dict {"e4m3": uint8 [rows, cols], "scale": fp32 [ceil(rows/128), ceil(cols/128)]}."""

    def __init__(self, cfg, weights: dict, layers=None):
        self.cfg = cfg
        self._keep = []
        self.c_cfg = _Cfg(cfg.d_model, cfg.n_q, cfg.n_kv, cfg.d_head, cfg.n_exp, cfg.top_k, cfg.d_ff,
                          cfg.n_layers, cfg.vocab, cfg.rms_eps, cfg.rope_theta)
        lw = weights["layers"] if layers is None else layers
        self.c_layers = (_Layer * max(len(lw), 1))()
        for i, L in enumerate(lw):
            self.c_layers[i] = self._layer(L)
        self.emb = self._arr(weights["emb"]) if "emb" in weights else None
        self.head = self._arr(weights["head"]) if "head" in weights else None
        self.final_norm = self._arr(weights["final_norm"]) if "final_norm" in weights else None
        self.c_model = _Model(self._ptr(self.emb), self._ptr(self.final_norm), self._ptr(self.head),
                              ctypes.cast(self.c_layers, ctypes.POINTER(_Layer)))

    def _arr(self, t):
        a = _np_weight(t)
        self._keep.append(a)
        return a

    @staticmethod
    def _ptr(a):
        return None if a is None else a.ctypes.data_as(c_void_p).value

    def _mat(self, t, rows, cols):
        if isinstance(t, dict):
            q = self._arr(t["e4m3"]).reshape(rows, cols)
            s = self._arr(t["scale"]).astype(np.float32, copy=False)
            self._keep.append(s)
            assert q.dtype == np.uint8
            return _Mat(None, self._ptr(q), self._ptr(s), rows, cols)
        a = self._arr(t)
        assert a.dtype == np.uint16 and a.size == rows * cols, (a.dtype, a.shape, rows, cols)
        return _Mat(self._ptr(a), None, None, rows, cols)

    def _layer(self, L):
        c = self.cfg
        an = self._arr(L["attn_norm"]).astype(np.float32, copy=False)
        fn = self._arr(L["ffn_norm"]).astype(np.float32, copy=False)
        self._keep += [an, fn]
        return _Layer(self._ptr(an),
                      self._mat(L["w_qkv"], c.qkv_rows, c.d_model),
                      self._mat(L["w_o"], c.d_model, c.n_q * c.d_head),
                      self._ptr(fn),
                      self._mat(L["w_router"], c.n_exp, c.d_model),
                      self._mat(L["w_gate_up"], c.n_exp * 2 * c.d_ff, c.d_model),
                      self._mat(L["w_down"], c.n_exp * c.d_model, c.d_ff))


def layer_forward(model: Model, layer: int, x, pos, P=0, k_cache=None, v_cache=None, causal=False, want_mid=False,
                  flip=None):
    """One decoder layer on rows x [n, d] (fp64, updated copy returned) at positions pos, keys =
    cache[0:P] + the rows.  Returns (x_out, k_new, v_new, router_logits) and, with want_mid, x after
    the attention residual as a fifth item.  flip (optional bool [n]): tokens routed to their
    (k+1)-th expert in place of their k-th."""
    c = model.cfg
    x = _f64(x).copy()
    n = x.shape[0]
    pos = np.ascontiguousarray(np.asarray(pos, dtype=np.int32))
    kc = _f64(k_cache) if P > 0 else np.zeros(1)
    vc = _f64(v_cache) if P > 0 else np.zeros(1)
    kn = np.empty((n, c.n_kv, c.d_head))
    vn = np.empty((n, c.n_kv, c.d_head))
    rl = np.empty((n, c.n_exp))
    mid = np.empty_like(x) if want_mid else None
    fl = None if flip is None else np.ascontiguousarray(np.asarray(flip, dtype=np.uint8))
    rc = lib().orc_layer_forward_flip(ctypes.byref(model.c_cfg), ctypes.byref(model.c_layers[layer]), n, _p(pos),
                                      _p(x), P, _p(kc), _p(vc), int(causal), _p(kn), _p(vn), _p(rl),
                                      None if mid is None else _p(mid), None if fl is None else _p(fl))
    assert rc == 0
    return (x, kn, vn, rl, mid) if want_mid else (x, kn, vn, rl)


def moe(model: Model, layer: int, h, sel, gate):
    h = _f64(h)
    n = h.shape[0]
    sel = np.ascontiguousarray(np.asarray(sel, dtype=np.int32))
    gate = _f64(gate)
    y = np.empty_like(h)
    lib().orc_moe(ctypes.byref(model.c_cfg), ctypes.byref(model.c_layers[layer]), n, sel.shape[1], _p(h), _p(sel),
                  _p(gate), _p(y))
    return y


def forward(model: Model, ids, pos, P, k_caches, v_caches, causal=False, write_cache=False,
            want_hidden=False, want_router=False, want_logits=True, flip=None):
    """Full stack on rows ids at positions pos; caches are per-layer fp64 arrays [ctx, Hkv, dh]
    (rows [0:P) read; with write_cache rows [P:P+n) receive the rows' K/V).  flip (optional bool
    [L, n]): per layer, tokens routed to their (k+1)-th expert in place of their k-th."""
    c = model.cfg
    ids = np.ascontiguousarray(np.asarray(ids, dtype=np.int32))
    pos = np.ascontiguousarray(np.asarray(pos, dtype=np.int32))
    n = ids.shape[0]
    kp = (c_void_p * c.n_layers)(*[a.ctypes.data for a in k_caches])
    vp = (c_void_p * c.n_layers)(*[a.ctypes.data for a in v_caches])
    for a in list(k_caches) + list(v_caches):
        assert a.dtype == np.float64 and a.flags["C_CONTIGUOUS"]
    hid = np.empty((c.n_layers + 1, n, c.d_model)) if want_hidden else None
    rtr = np.empty((c.n_layers, n, c.n_exp)) if want_router else None
    logits = np.empty((n, c.vocab)) if want_logits else None
    fl = None if flip is None else np.ascontiguousarray(np.asarray(flip, dtype=np.uint8).reshape(c.n_layers, n))
    rc = lib().orc_forward_flip(ctypes.byref(model.c_cfg), ctypes.byref(model.c_model), n, _p(ids), _p(pos), P,
                                kp, vp, int(causal), int(write_cache),
                                None if hid is None else _p(hid), None if rtr is None else _p(rtr),
                                None if logits is None else _p(logits), None if fl is None else _p(fl))
    assert rc == 0
    return {"hidden": hid, "router": rtr, "logits": logits}


def embed(model: Model, ids):
    """Embedding rows of ids (bf16 upcast exactly) as fp64 [n, d]."""
    ids = np.ascontiguousarray(np.asarray(ids, dtype=np.int32))
    x = np.empty((ids.shape[0], model.cfg.d_model))
    lib().orc_embed(ctypes.byref(model.c_cfg), model.c_model.emb, ids.shape[0], _p(ids), _p(x))
    return x


def head(model: Model, x):
    x = _f64(x)
    n = x.shape[0]
    out = np.empty((n, model.cfg.vocab))
    lib().orc_head(ctypes.byref(model.c_cfg), ctypes.byref(model.c_model), n, _p(x), _p(out))
    return out


# ---------------------------------------------------------------------------------------------
# sampler
# ---------------------------------------------------------------------------------------------

def sample_rows(logits, skip, pos, T, seed, step):
    """Per-row entropy H, Gumbel-argmax y, top-2 perturbed-score margin and re-randomisation id.
    logits fp32 or fp64 [n, V]."""
    n, V = logits.shape
    if logits.dtype == np.float32:
        fn, lg = lib().orc_sample_rows_f32, np.ascontiguousarray(logits)
    else:
        fn, lg = lib().orc_sample_rows_f64, _f64(logits)
    skip = np.zeros(n, np.uint8) if skip is None else np.ascontiguousarray(np.asarray(skip, dtype=np.uint8))
    pos = np.ascontiguousarray(np.asarray(pos, dtype=np.int32))
    H = np.empty(n)
    y = np.empty(n, np.int32)
    margin = np.empty(n)
    rr = np.empty(n, np.int32)
    fn(n, V, _p(lg), _p(skip), _p(pos), T, seed, step, _p(H), _p(y), _p(margin), _p(rr))
    return {"H": H, "y": y, "margin": margin, "rr": rr}


def step_rule(commit, ids, H, y, rr, s, entropy_bound=0.1, rerand_entropy=None, stop_mean_entropy=0.005,
              max_steps=48, fixed_steps=0, vocab=None, cumulative=False):
    """One step's decisions.  cumulative: the entropy-bound reading that commits the lowest-entropy
    positions while their entropy sum stays within the bound; the result then also holds "cum",
    each uncommitted position's running sum in ascending (H, position) order."""
    n = len(ids)
    if rerand_entropy is None:
        rerand_entropy = 0.5 * np.log(vocab)
    commit = np.ascontiguousarray(np.asarray(commit, dtype=np.uint8))
    ids = np.ascontiguousarray(np.asarray(ids, dtype=np.int32))
    H = _f64(H)
    y = np.ascontiguousarray(np.asarray(y, dtype=np.int32))
    rr = np.ascontiguousarray(np.asarray(rr, dtype=np.int32))
    ids_out = np.empty(n, np.int32)
    commit_out = np.empty(n, np.uint8)
    mean = np.zeros(1)
    cum = np.zeros(n)
    stop = lib().orc_step_rule(n, _p(commit), _p(ids), _p(H), _p(y), _p(rr), entropy_bound, rerand_entropy,
                               stop_mean_entropy, s, max_steps, fixed_steps, int(bool(cumulative)), _p(ids_out),
                               _p(commit_out), _p(mean), _p(cum))
    assert stop >= 0
    out = {"ids": ids_out, "commit": commit_out, "stop": int(stop), "mean_H": float(mean[0])}
    if cumulative:
        out["cum"] = cum
    return out


def canvas_init(n, P, seed, vocab):
    ids = np.empty(n, np.int32)
    commit = np.empty(n, np.uint8)
    lib().orc_canvas_init(n, P, seed, vocab, _p(ids), _p(commit))
    return ids, commit


# ---------------------------------------------------------------------------------------------
# the decoder loop of one sequence
# ---------------------------------------------------------------------------------------------

class SamplerParams:
    def __init__(self, vocab, canvas_len=256, max_steps=48, fixed_steps=0, t_start=0.8, t_end=0.4,
                 entropy_bound=0.1, stop_mean_entropy=0.005, rerand_entropy=None, seed=0, eos_id=-1,
                 commit_rule=0):
        self.canvas_len, self.max_steps, self.fixed_steps = canvas_len, max_steps, fixed_steps
        self.commit_rule = commit_rule
        self.t_start, self.t_end = t_start, t_end
        self.entropy_bound, self.stop_mean_entropy = entropy_bound, stop_mean_entropy
        self.rerand_entropy = 0.5 * np.log(vocab) if rerand_entropy is None else rerand_entropy
        self.seed, self.eos_id = seed, eos_id


class Sequence:
    """One sequence: a per-layer fp64 KV cache, the committed length P and the canvas step index."""

    def __init__(self, model: Model, max_ctx: int, prefix_k=None, prefix_v=None):
        c = model.cfg
        self.model, self.max_ctx = model, max_ctx
        self.k = [np.zeros((max_ctx, c.n_kv, c.d_head)) for _ in range(c.n_layers)]
        self.v = [np.zeros((max_ctx, c.n_kv, c.d_head)) for _ in range(c.n_layers)]
        self.P = 0
        self.step = 0
        if prefix_k is not None:
            P = prefix_k[0].shape[0]
            for l in range(c.n_layers):
                self.k[l][:P] = _f64(_as_float(prefix_k[l]))
                self.v[l][:P] = _f64(_as_float(prefix_v[l]))
            self.P = P

    def prefill(self, ids, want_router=False):
        """Returns the router logits [L][n][E] of the prompt rows when want_router."""
        n = len(ids)
        assert self.P + n <= self.max_ctx
        fw = forward(self.model, ids, np.arange(self.P, self.P + n), self.P, self.k, self.v, causal=True,
                     write_cache=True, want_router=want_router, want_logits=False)
        self.P += n
        return fw["router"]

    def canvas_init(self, prm: SamplerParams):
        self.step = 0
        return canvas_init(prm.canvas_len, self.P, prm.seed, self.model.cfg.vocab)

    def canvas_step(self, prm: SamplerParams, ids, commit, want_hidden=False, want_router=False, flip=None,
                    advance=True):
        """One denoising step.  flip (optional bool [L, n]): the routing alternative for the flagged
        (layer, token) pairs (see forward).  advance=False leaves the step counter as it is (a second
        evaluation of the same step)."""
        n = len(ids)
        pos = np.arange(self.P, self.P + n)
        fw = forward(self.model, ids, pos, self.P, self.k, self.v, causal=False, write_cache=False,
                     want_hidden=want_hidden, want_router=want_router, want_logits=True, flip=flip)
        T = temperature(self.step, prm.max_steps, prm.t_start, prm.t_end)
        smp = sample_rows(fw["logits"], commit, pos, T, prm.seed, self.step)
        rule = step_rule(commit, ids, smp["H"], smp["y"], smp["rr"], self.step, prm.entropy_bound,
                         prm.rerand_entropy, prm.stop_mean_entropy, prm.max_steps, prm.fixed_steps,
                         cumulative=prm.commit_rule == 1)
        out = dict(smp)
        out.update(rule)
        out.update({"T": T, "step": self.step, "logits": fw["logits"], "hidden": fw["hidden"],
                    "router": fw["router"]})
        if advance:
            self.step += 1
        return out

    def block_commit(self, ids, want_router=False):
        """Returns the router logits [L][256][E] of the commit pass when want_router."""
        n = len(ids)
        assert self.P + n <= self.max_ctx
        fw = forward(self.model, ids, np.arange(self.P, self.P + n), self.P, self.k, self.v, causal=False,
                     write_cache=True, want_router=want_router, want_logits=False)
        self.P += n
        return fw["router"]

    def decode(self, prm: SamplerParams, max_blocks: int):
        out = []
        for _ in range(max_blocks):
            ids, commit = self.canvas_init(prm)
            while True:
                r = self.canvas_step(prm, ids, commit)
                ids, commit = r["ids"], r["commit"]
                if r["stop"]:
                    break
            self.block_commit(ids)
            out.extend(int(i) for i in ids)
            if prm.eos_id >= 0 and prm.eos_id in ids:
                out = out[: out.index(prm.eos_id, len(out) - len(ids)) + 1]
                break
        return np.asarray(out, dtype=np.int32)


def _as_float(t):
    import torch
    if isinstance(t, torch.Tensor):
        return t.detach().cpu().to(torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)
