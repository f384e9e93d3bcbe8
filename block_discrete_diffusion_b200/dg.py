"""Python binding of libdg.so (include/dg.h): argument marshalling only.

Every function here has the name of the C entry point it calls and passes device pointers of torch
CUDA tensors straight through.  PyTorch provides device memory and the stream; all computation runs
in the library's kernels.  There is no fallback: if libdg.so is missing or fails to load, every call
raises.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libdg.so")

c_int, c_float, c_void_p, c_size_t, c_uint64 = ctypes.c_int, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_uint64

# the entry points declared in include/dg.h
ENTRY_POINTS = (
    "dg_last_error", "dg_model_create", "dg_model_destroy", "dg_kv_bytes", "dg_workspace_bytes", "dg_seqs_create",
    "dg_seqs_destroy", "dg_seqs_get_state", "dg_load_prefix", "dg_prefill", "dg_canvas_init", "dg_canvas_step",
    "dg_block_commit", "dg_decode", "dg_layer_forward", "dg_sample_workspace_bytes", "dg_sample", "dg_device_error",
    "dg_temperature", "dg_stats_reset", "dg_stats_read", "dg_sample_noalloc", "dg_sample_noalloc_max_rows",
    "dg_block_commit_last_kv", "dg_head_sample_workspace_bytes", "dg_head_sample", "dg_head_sample_error",
)

# dg_kernel_class, in order
KERNEL_CLASSES = ("embed", "rmsnorm", "qkv", "attn", "attn_merge", "oproj", "router", "topk", "bucket", "expert_up",
                  "expert_down", "combine", "head", "sampler", "misc", "dequant")
WDTYPE_BF16, WDTYPE_FP8_BLOCK128 = 0, 1
MATRICES = ("w_qkv", "w_o", "w_router", "w_gate_up", "w_down")

DG_OK, DG_ERR_INVALID_ARG, DG_ERR_CAPACITY, DG_ERR_STATE, DG_ERR_CUDA, DG_ERR_UNSUPPORTED, DG_ERR_DEVICE = range(7)


class DGError(RuntimeError):
    def __init__(self, fn, status, msg):
        super().__init__(f"{fn} -> status {status}: {msg}")
        self.status = status


class dg_model_config(ctypes.Structure):
    _fields_ = [(n, c_int) for n in ("d_model", "n_q", "n_kv", "d_head", "n_exp", "top_k", "d_ff", "n_layers",
                                     "vocab")] + [("rms_eps", c_float), ("rope_theta", c_float), ("wdtype", c_int)]


class dg_layer_weights(ctypes.Structure):
    _fields_ = [(n, c_void_p) for n in ("attn_norm", "w_qkv", "w_o", "ffn_norm", "w_router", "w_gate_up", "w_down",
                                        "s_qkv", "s_o", "s_router", "s_gate_up", "s_down")]


class dg_weights(ctypes.Structure):
    _fields_ = [("emb", c_void_p), ("final_norm", c_void_p), ("head", c_void_p),
                ("layers", ctypes.POINTER(dg_layer_weights))]


class dg_sampler_params(ctypes.Structure):
    _fields_ = [("canvas_len", c_int), ("max_steps", c_int), ("fixed_steps", c_int), ("t_start", c_float),
                ("t_end", c_float), ("entropy_bound", c_float), ("stop_mean_entropy", c_float),
                ("rerand_entropy", c_float), ("seed", c_uint64), ("eos_id", c_int), ("commit_mode", c_int),
                ("commit_rule", c_int)]


def sampler_params(vocab, seed=0, canvas_len=256, max_steps=48, fixed_steps=0, t_start=0.8, t_end=0.4,
                   entropy_bound=0.1, stop_mean_entropy=0.005, rerand_entropy=None, eos_id=-1,
                   commit_mode=0, commit_rule=0) -> dg_sampler_params:
    if rerand_entropy is None:
        rerand_entropy = 0.5 * math.log(vocab)
    return dg_sampler_params(canvas_len, max_steps, fixed_steps, t_start, t_end, entropy_bound, stop_mean_entropy,
                             rerand_entropy, seed, eos_id, commit_mode, commit_rule)


_LIB = None


def lib():
    """Load libdg.so (raises if it is missing: there is no other implementation)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with block_discrete_diffusion_b200.build.build()")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER
        L.dg_last_error.restype = ctypes.c_char_p
        L.dg_model_create.argtypes = [P(dg_model_config), P(dg_weights), P(c_void_p)]
        L.dg_model_destroy.argtypes = [c_void_p]
        L.dg_model_destroy.restype = None
        L.dg_kv_bytes.argtypes = [P(dg_model_config), c_int, c_int]
        L.dg_kv_bytes.restype = c_size_t
        L.dg_workspace_bytes.argtypes = [P(dg_model_config), c_int, c_int]
        L.dg_workspace_bytes.restype = c_size_t
        L.dg_seqs_create.argtypes = [c_void_p, c_int, c_int, c_void_p, c_size_t, c_void_p, c_size_t, c_void_p,
                                     P(c_void_p)]
        L.dg_seqs_destroy.argtypes = [c_void_p]
        L.dg_seqs_destroy.restype = None
        L.dg_seqs_get_state.argtypes = [c_void_p, c_void_p, c_void_p]
        L.dg_load_prefix.argtypes = [c_void_p, c_int, c_int, c_void_p, c_void_p]
        L.dg_prefill.argtypes = [c_void_p, c_void_p, c_void_p]
        L.dg_canvas_init.argtypes = [c_void_p, P(dg_sampler_params), c_void_p, c_void_p]
        L.dg_canvas_step.argtypes = [c_void_p, P(dg_sampler_params), c_void_p, c_void_p, c_void_p, c_void_p,
                                     c_void_p, c_void_p]
        L.dg_block_commit.argtypes = [c_void_p, c_void_p]
        L.dg_block_commit_last_kv.argtypes = [c_void_p]
        L.dg_decode.argtypes = [c_void_p, P(dg_sampler_params), c_int, c_void_p, c_void_p, c_void_p]
        L.dg_layer_forward.argtypes = [c_void_p, c_int, c_int, c_int, c_void_p, c_void_p, c_void_p]
        L.dg_sample_workspace_bytes.argtypes = [c_int, c_int]
        L.dg_sample_workspace_bytes.restype = c_size_t
        L.dg_sample.argtypes = [c_void_p, c_int, c_int, P(dg_sampler_params), c_int, c_void_p, c_void_p, c_void_p,
                                c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]
        L.dg_sample_noalloc.argtypes = [c_void_p, c_int, c_int, P(dg_sampler_params), c_int, c_void_p, c_void_p,
                                        c_void_p, c_void_p, c_void_p, c_void_p]
        L.dg_sample_noalloc_max_rows.argtypes = [c_int]
        L.dg_sample_noalloc_max_rows.restype = c_size_t
        L.dg_head_sample_workspace_bytes.argtypes = [c_int]
        L.dg_head_sample_workspace_bytes.restype = c_size_t
        L.dg_head_sample.argtypes = [c_void_p, c_void_p, c_int, c_int, c_int, P(dg_sampler_params), c_int, c_void_p,
                                     c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]
        L.dg_head_sample_error.argtypes = [c_void_p, c_void_p, P(c_int)]
        L.dg_device_error.argtypes = [c_void_p, P(c_int)]
        L.dg_stats_reset.argtypes = [c_void_p, c_int]
        L.dg_stats_read.argtypes = [c_void_p, c_void_p, c_void_p]
        L.dg_temperature.argtypes = [P(dg_sampler_params), c_int]
        L.dg_temperature.restype = c_float
        _LIB = L
    return _LIB


def _check(fn, status):
    if status != DG_OK:
        raise DGError(fn, status, lib().dg_last_error().decode())


def _ptr(t):
    if t is None:
        return None
    assert isinstance(t, torch.Tensor) and t.is_cuda and t.is_contiguous(), "expected a contiguous CUDA tensor"
    return t.data_ptr()


def _stream_handle(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def make_config(cfg) -> dg_model_config:
    return dg_model_config(cfg.d_model, cfg.n_q, cfg.n_kv, cfg.d_head, cfg.n_exp, cfg.top_k, cfg.d_ff, cfg.n_layers,
                           cfg.vocab, cfg.rms_eps, cfg.rope_theta, getattr(cfg, "wdtype", WDTYPE_BF16))


def _layer_struct(L: dict) -> "dg_layer_weights":
    """A layer dict of device tensors; in the FP8 form each matrix is {"e4m3": uint8, "scale": fp32}."""
    def mat(k):
        t = L[k]
        return (_ptr(t["e4m3"]), _ptr(t["scale"])) if isinstance(t, dict) else (_ptr(t), None)
    (q, sq), (o, so), (r, sr), (gu, sgu), (dn, sdn) = (mat(k) for k in MATRICES)
    return dg_layer_weights(_ptr(L["attn_norm"]), q, o, _ptr(L["ffn_norm"]), r, gu, dn, sq, so, sr, sgu, sdn)


# ---------------------------------------------------------------------------------------------
# thin wrappers, one per entry point
# ---------------------------------------------------------------------------------------------
class Model:
    """dg_model handle; keeps the weight tensors (borrowed by the library) alive."""

    def __init__(self, handle, cfg, weights, c_cfg):
        self.handle, self.cfg, self.weights, self.c_cfg = handle, cfg, weights, c_cfg

    def __del__(self):
        if getattr(self, "handle", None) and _LIB is not None:
            _LIB.dg_model_destroy(self.handle)
            self.handle = None


def dg_model_create(cfg, weights: dict) -> Model:
    c = make_config(cfg)
    layers = (dg_layer_weights * cfg.n_layers)()
    for i, L in enumerate(weights["layers"]):
        layers[i] = _layer_struct(L)
    w = dg_weights(_ptr(weights["emb"]), _ptr(weights["final_norm"]), _ptr(weights["head"]),
                   ctypes.cast(layers, ctypes.POINTER(dg_layer_weights)))
    h = c_void_p()
    _check("dg_model_create", lib().dg_model_create(ctypes.byref(c), ctypes.byref(w), ctypes.byref(h)))
    return Model(h, cfg, weights, c)


def dg_kv_bytes(cfg, n_seq, max_ctx) -> int:
    c = make_config(cfg)
    return int(lib().dg_kv_bytes(ctypes.byref(c), n_seq, max_ctx))


def dg_workspace_bytes(cfg, n_seq, max_ctx) -> int:
    c = make_config(cfg)
    return int(lib().dg_workspace_bytes(ctypes.byref(c), n_seq, max_ctx))


class Seqs:
    """dg_seqs handle; keeps the model, the KV cache and the workspace tensors alive."""

    def __init__(self, handle, model, n_seq, max_ctx, kv, ws, stream):
        self.handle, self.model, self.n_seq, self.max_ctx, self.kv, self.ws, self.stream = (
            handle, model, n_seq, max_ctx, kv, ws, stream)

    def __del__(self):
        if getattr(self, "handle", None) and _LIB is not None:
            _LIB.dg_seqs_destroy(self.handle)
            self.handle = None


def dg_seqs_create(model: Model, n_seq, max_ctx, kv=None, ws=None, stream=None) -> Seqs:
    """kv / ws: caller device buffers (uint8 CUDA tensors); allocated here through torch if None."""
    dev = torch.device("cuda", torch.cuda.current_device())
    if kv is None:
        kv = torch.empty(dg_kv_bytes(model.cfg, n_seq, max_ctx), dtype=torch.uint8, device=dev)
    if ws is None:
        ws = torch.empty(dg_workspace_bytes(model.cfg, n_seq, max_ctx), dtype=torch.uint8, device=dev)
    h = c_void_p()
    _check("dg_seqs_create", lib().dg_seqs_create(model.handle, n_seq, max_ctx, _ptr(kv), kv.numel(), _ptr(ws),
                                                  ws.numel(), _stream_handle(stream), ctypes.byref(h)))
    return Seqs(h, model, n_seq, max_ctx, kv, ws, stream)


def dg_seqs_get_state(seqs: Seqs):
    P = (c_int * seqs.n_seq)()
    step = c_int()
    _check("dg_seqs_get_state", lib().dg_seqs_get_state(seqs.handle, P, ctypes.byref(step)))
    return list(P), step.value


def dg_load_prefix(seqs: Seqs, seq, P, k_layers, v_layers):
    n = len(k_layers)
    ks = (c_void_p * n)(*[_ptr(k) for k in k_layers])
    vs = (c_void_p * n)(*[_ptr(v) for v in v_layers])
    _check("dg_load_prefix", lib().dg_load_prefix(seqs.handle, seq, P, ks, vs))


def dg_prefill(seqs: Seqs, ids: torch.Tensor, lens):
    lens_c = (ctypes.c_int32 * len(lens))(*lens)
    _check("dg_prefill", lib().dg_prefill(seqs.handle, _ptr(ids), lens_c))


def dg_canvas_init(seqs: Seqs, params: dg_sampler_params, ids, commit):
    _check("dg_canvas_init", lib().dg_canvas_init(seqs.handle, ctypes.byref(params), _ptr(ids), _ptr(commit)))


def dg_canvas_step(seqs: Seqs, params, ids, commit, entropy, stop, hidden=None, logits=None):
    _check("dg_canvas_step", lib().dg_canvas_step(seqs.handle, ctypes.byref(params), _ptr(ids), _ptr(commit),
                                                  _ptr(entropy), _ptr(stop), _ptr(hidden), _ptr(logits)))


def dg_block_commit(seqs: Seqs, ids):
    _check("dg_block_commit", lib().dg_block_commit(seqs.handle, _ptr(ids)))


def dg_block_commit_last_kv(seqs: Seqs):
    _check("dg_block_commit_last_kv", lib().dg_block_commit_last_kv(seqs.handle))


def dg_decode(seqs: Seqs, params, max_blocks, out):
    n_out = (ctypes.c_int32 * seqs.n_seq)()
    steps = (ctypes.c_int32 * max_blocks)()
    _check("dg_decode", lib().dg_decode(seqs.handle, ctypes.byref(params), max_blocks, _ptr(out), n_out, steps))
    return list(n_out), list(steps)


def dg_layer_forward(seqs: Seqs, layer, x, x_mid=None, router_logits=None, n_rows=256, causal=False):
    _check("dg_layer_forward", lib().dg_layer_forward(seqs.handle, layer, n_rows, int(bool(causal)), _ptr(x), _ptr(x_mid),
                                                      _ptr(router_logits)))


def dg_sample_workspace_bytes(n_rows, vocab) -> int:
    return int(lib().dg_sample_workspace_bytes(n_rows, vocab))


def dg_sample(logits, n_seq, vocab, params, step, seq_P, ids, commit, entropy, stop, ws, stream=None):
    _check("dg_sample", lib().dg_sample(_ptr(logits), n_seq, vocab, ctypes.byref(params), step, _ptr(seq_P),
                                        _ptr(ids), _ptr(commit), _ptr(entropy), _ptr(stop), _ptr(ws), ws.numel(),
                                        _stream_handle(stream)))


def dg_sample_noalloc(logits, n_seq, vocab, params, step, seq_P, ids, commit, entropy, stop, stream=None):
    """dg_sample with its scratch in the library's static device array (no workspace argument)."""
    _check("dg_sample_noalloc", lib().dg_sample_noalloc(_ptr(logits), n_seq, vocab, ctypes.byref(params), step,
                                                        _ptr(seq_P), _ptr(ids), _ptr(commit), _ptr(entropy),
                                                        _ptr(stop), _stream_handle(stream)))


def dg_sample_noalloc_max_rows(vocab) -> int:
    return int(lib().dg_sample_noalloc_max_rows(vocab))


def dg_head_sample_workspace_bytes(vocab) -> int:
    return int(lib().dg_head_sample_workspace_bytes(vocab))


def dg_head_sample(xn, head, params, step, seq_P, ids, commit, entropy, stop, ws, nv=128, logits=None, stream=None):
    """The fused vocabulary head + sampler on caller inputs (xn bf16 [256, d], head bf16 [V, d])."""
    _check("dg_head_sample", lib().dg_head_sample(_ptr(xn), _ptr(head), xn.shape[1], head.shape[0], nv,
                                                  ctypes.byref(params), step, _ptr(seq_P), _ptr(ids), _ptr(commit),
                                                  _ptr(entropy), _ptr(stop), _ptr(logits), _ptr(ws), ws.numel(),
                                                  _stream_handle(stream)))


def dg_head_sample_error(ws, stream=None) -> int:
    code = c_int()
    st = lib().dg_head_sample_error(_ptr(ws), _stream_handle(stream), ctypes.byref(code))
    if st not in (DG_OK, DG_ERR_DEVICE):
        _check("dg_head_sample_error", st)
    return code.value


def dg_device_error(seqs: Seqs) -> int:
    code = c_int()
    st = lib().dg_device_error(seqs.handle, ctypes.byref(code))
    if st not in (DG_OK, DG_ERR_DEVICE):
        _check("dg_device_error", st)
    return code.value


def dg_temperature(params, step) -> float:
    return float(lib().dg_temperature(ctypes.byref(params), step))


def dg_stats_reset(seqs: Seqs, timing=False):
    _check("dg_stats_reset", lib().dg_stats_reset(seqs.handle, int(bool(timing))))


def dg_stats_read(seqs: Seqs):
    """{class: (launches, device ms)} accumulated since the last reset (synchronises the stream)."""
    n = len(KERNEL_CLASSES)
    launches = (ctypes.c_longlong * n)()
    ms = (ctypes.c_double * n)()
    _check("dg_stats_read", lib().dg_stats_read(seqs.handle, launches, ms))
    return {k: (int(launches[i]), float(ms[i])) for i, k in enumerate(KERNEL_CLASSES)}
