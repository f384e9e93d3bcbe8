"""Seeded synthetic inputs shared by the CUDA path's tests/benchmark and by the oracle's tests.

This module draws random numbers and lays them out; it holds none of the decoder's arithmetic.
Weights are random-init (no trained checkpoint exists here); ids are uniform; logits for the
standalone sampler workload are Gaussian with sparse spikes.

Weight layout (row-major, PyTorch ``Linear`` convention: [out_features, in_features]):
  emb        [V, d]            bf16   embedding table
  head       [V, d]            bf16   untied vocabulary projection
  final_norm [d]               fp32   RMSNorm gain
  per layer:
    attn_norm [d]              fp32
    w_qkv     [(Hq+2Hkv)*dh, d] bf16  Q rows, then K rows, then V rows
    w_o       [d, Hq*dh]        bf16
    ffn_norm  [d]              fp32
    w_router  [E, d]            bf16
    w_gate_up [E, 2F, d]        bf16  per expert: F gate rows, then F up rows
    w_down    [E, d, F]         bf16
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class ModelConfig:
    d_model: int
    n_q: int
    n_kv: int
    d_head: int
    n_exp: int
    top_k: int
    d_ff: int
    n_layers: int
    vocab: int
    rms_eps: float = 1e-6
    rope_theta: float = 10000.0
    wdtype: int = 0   # per-layer matrices: 0 bf16; 1 FP8 e4m3 with one fp32 scale per 128 x 128 tile

    @property
    def qkv_rows(self) -> int:
        return (self.n_q + 2 * self.n_kv) * self.d_head


# Tiny oracle model: 2 layers, d 256, 4 Q / 2 KV heads of dim 64, 8 experts top-2, FFN 512, V 4096.
TINY = ModelConfig(d_model=256, n_q=4, n_kv=2, d_head=64, n_exp=8, top_k=2, d_ff=512, n_layers=2, vocab=4096)
# Full-width decoder layer of the Gemma-4-26B-A4B shape: d 2816, 16 Q / 8 KV heads of dim 128,
# 128 experts top-8 with FFN 704, vocabulary 262144.
FULL = ModelConfig(d_model=2816, n_q=16, n_kv=8, d_head=128, n_exp=128, top_k=8, d_ff=704, n_layers=30,
                   vocab=262144)
ONE_LAYER = dataclasses.replace(FULL, n_layers=1)

CANVAS = 256
MAX_STEPS = 48
T_START, T_END = 0.8, 0.4
ENTROPY_BOUND = 0.1
STOP_MEAN_ENTROPY = 0.005


def default_rerand_entropy(vocab: int) -> float:
    """Threshold above which a non-committing position is re-randomised (a stated default: half of
    the maximum entropy ln V)."""
    return 0.5 * math.log(vocab)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _normal_bf16(shape, std, gen, device) -> torch.Tensor:
    t = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    t.mul_(std)
    return t.to(torch.bfloat16)


FP8_E4M3_MAX = 448.0


def quantize_fp8_block128(w: torch.Tensor) -> dict:
    """FP8 storage form of a random weight matrix [rows, cols] (an expert stack [E, rows, cols] is
    viewed as [E rows, cols]): per 128 x 128 tile the scale s = amax / 448 (1 for an all-zero
    tile) and the bytes q = w / s cast to e4m3 (torch's round-to-nearest-even cast, clamped to
    +-448).  The stored weight is q * s.  Returns {"e4m3": uint8 [same shape], "scale": fp32
    [ceil(rows/128), ceil(cols/128)]}."""
    shape = w.shape
    w2 = w.reshape(-1, shape[-1]).float()
    R, C = w2.shape
    tr, tc = -(-R // 128), -(-C // 128)
    pad = torch.zeros((tr * 128, tc * 128), dtype=torch.float32, device=w.device)
    pad[:R, :C] = w2
    del w2
    tiles = pad.view(tr, 128, tc, 128)
    amax = tiles.abs().amax(dim=(1, 3))
    scale = torch.where(amax > 0, amax / FP8_E4M3_MAX, torch.ones_like(amax))
    tiles.div_(scale[:, None, :, None]).clamp_(-FP8_E4M3_MAX, FP8_E4M3_MAX)
    q = pad.to(torch.float8_e4m3fn)
    del pad, tiles
    q = q[:R, :C].contiguous().view(torch.uint8).reshape(shape)
    return {"e4m3": q, "scale": scale.contiguous()}


def _matrix(shape, std, gen, device, wdtype):
    if wdtype == 0:
        return _normal_bf16(shape, std, gen, device)
    t = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    t.mul_(std)
    return quantize_fp8_block128(t)


def make_layer_weights(cfg: ModelConfig, gen: torch.Generator, device="cpu", w_std=0.02,
                       router_std=None, out_std=None) -> dict:
    """One layer.  ``out_std`` is the std of the two residual-branch output matrices (w_o, w_down);
    it defaults to w_std.  With cfg.wdtype == 1 the five matrices come in the FP8 form of
    quantize_fp8_block128 (same random draws, no bf16 rounding before the quantisation)."""
    d, E, F = cfg.d_model, cfg.n_exp, cfg.d_ff
    if router_std is None:
        router_std = w_std
    if out_std is None:
        out_std = w_std
    wd = cfg.wdtype
    return {
        "attn_norm": torch.ones(d, dtype=torch.float32, device=device),
        "w_qkv": _matrix((cfg.qkv_rows, d), w_std, gen, device, wd),
        "w_o": _matrix((d, cfg.n_q * cfg.d_head), out_std, gen, device, wd),
        "ffn_norm": torch.ones(d, dtype=torch.float32, device=device),
        "w_router": _matrix((E, d), router_std, gen, device, wd),
        "w_gate_up": _matrix((E, 2 * F, d), w_std, gen, device, wd),
        "w_down": _matrix((E, d, F), out_std, gen, device, wd),
    }


def dequantize_fp8_block128(m: dict) -> torch.Tensor:
    """fp64 weights q * s of the FP8 form (for building test inputs only)."""
    q = m["e4m3"]
    shape = q.shape
    v = q.reshape(-1, shape[-1]).view(torch.float8_e4m3fn).double()
    s = m["scale"].double().repeat_interleave(128, 0).repeat_interleave(128, 1)[:v.shape[0], :v.shape[1]]
    return (v * s).reshape(shape)


GAIN_SEED_OFFSET = 7919


def draw_gains(w: dict, d: int, seed: int, gain_std: float, device="cpu") -> dict:
    """Replace every RMSNorm gain of a weight set (each layer's attn_norm and ffn_norm, then
    final_norm) by an independent draw 1 + N(0, gain_std^2) in fp32, from a generator of its own
    (seed + GAIN_SEED_OFFSET) so that the matrices drawn before stay the same."""
    gen = _gen(seed + GAIN_SEED_OFFSET, device)

    def one():
        return torch.randn(d, generator=gen, device=device, dtype=torch.float32).mul_(gain_std).add_(1.0)

    for L in w["layers"]:
        L["attn_norm"] = one()
        L["ffn_norm"] = one()
    if "final_norm" in w:
        w["final_norm"] = one()
    return w


def make_model_weights(cfg: ModelConfig, seed: int, device="cpu", w_std=0.02, router_std=None,
                       head_scale=1.0, emb_std=None, out_std=None, gain_std=0.0, emb_split=None,
                       copy_head=0.0) -> dict:
    """Random-init weights N(0, w_std^2) rounded to bf16 (round-to-nearest-even).  Norm gains are 1,
    or with gain_std > 0 independent draws 1 + N(0, gain_std^2) (see draw_gains).
    ``head_scale`` multiplies the LM head's std (a larger head gives confident rows that commit);
    ``emb_std`` / ``out_std`` override the embedding std and the residual-output std.
    ``emb_split`` = (k, loud_std, quiet_std, loud_frac): a fraction loud_frac of the tokens ("loud")
    get embedding rows N(0, loud_std^2) in the first k channels and 0 elsewhere, the others
    ("quiet") N(0, quiet_std^2) in the remaining channels and 0 in the first k; ``copy_head`` = s adds
    s * emb to the head, so each position scores its own token: a loud token's row is confident, a
    quiet token's row sees only small logits (the two kinds live in orthogonal channels).  Both are
    applied after every other draw, so the other weights do not change."""
    gen = _gen(seed, device)
    w = {
        "emb": _normal_bf16((cfg.vocab, cfg.d_model), w_std if emb_std is None else emb_std, gen, device),
        "layers": [make_layer_weights(cfg, gen, device, w_std, router_std, out_std) for _ in range(cfg.n_layers)],
        "final_norm": torch.ones(cfg.d_model, dtype=torch.float32, device=device),
    }
    w["head"] = _normal_bf16((cfg.vocab, cfg.d_model), w_std * head_scale, gen, device)
    if emb_split is not None:
        k, loud_std, quiet_std, loud_frac = emb_split
        loud = torch.rand(cfg.vocab, generator=gen, device=device) < loud_frac
        e = torch.randn((cfg.vocab, cfg.d_model), generator=gen, device=device)
        e[:, :k].mul_(loud_std).mul_(loud[:, None])
        e[:, k:].mul_(quiet_std).mul_(~loud[:, None])
        w["emb"] = e.to(torch.bfloat16)
    if copy_head:
        w["head"] = (w["head"].float() + copy_head * w["emb"].float()).to(torch.bfloat16)
    if gain_std > 0:
        draw_gains(w, cfg.d_model, seed, gain_std, device)
    return w


def full_stack_init(cfg: ModelConfig) -> dict:
    """Keyword arguments of make_model_weights for the full-depth benchmark model: router logits of
    unit-RMS inputs ~ N(0, 1) (router std d^-1/2), unit-variance embeddings, and residual-branch
    output matrices scaled by 1/sqrt(2L) (the scaled init of deep pre-norm transformers).  With all
    matrices at N(0, 0.02^2) the random residual stream of the 30-layer model collapses onto one
    direction after the first layer (cross-token cosine ~0.97) and the router sends the whole canvas
    to ~12 of the 128 experts; a trained MoE routes a 256-token canvas to nearly all of them, which
    sets the weight traffic this workload has to model."""
    return {"router_std": cfg.d_model ** -0.5, "emb_std": 1.0, "out_std": 0.02 / math.sqrt(2 * cfg.n_layers)}


def make_ids(n: int, vocab: int, seed: int, device="cpu") -> torch.Tensor:
    return torch.randint(0, vocab, (n,), generator=_gen(seed, device), device=device, dtype=torch.int32)


def make_hidden(n: int, d: int, seed: int, device="cpu") -> torch.Tensor:
    """N(0,1) hidden states, rounded to bf16-representable values, held as fp32."""
    t = torch.randn((n, d), generator=_gen(seed, device), device=device, dtype=torch.float32)
    return t.to(torch.bfloat16).to(torch.float32)


def make_prefix_kv(n_layers: int, P: int, n_kv: int, dh: int, seed: int, device="cpu"):
    """Synthetic committed-prefix cache: K (taken as already rotated) and V ~ N(0,1) in bf16,
    one [P, n_kv, dh] pair per layer."""
    gen = _gen(seed, device)
    ks, vs = [], []
    for _ in range(n_layers):
        ks.append(torch.randn((P, n_kv, dh), generator=gen, device=device).to(torch.bfloat16))
        vs.append(torch.randn((P, n_kv, dh), generator=gen, device=device).to(torch.bfloat16))
    return ks, vs


def make_sampler_logits(rows: int, vocab: int, seed: int, std=3.0, spike=12.0, spike_every=10,
                        device="cpu"):
    """fp32 logits ~ N(0, std^2); rows r with r % spike_every == 0 get +spike at one uniformly
    chosen column.  Returns (logits, spike_columns)."""
    gen = _gen(seed, device)
    logits = torch.randn((rows, vocab), generator=gen, device=device, dtype=torch.float32).mul_(std)
    spike_rows = torch.arange(0, rows, spike_every, device=device)
    cols = torch.randint(0, vocab, (spike_rows.numel(),), generator=gen, device=device)
    if spike:
        logits[spike_rows, cols] += spike
    return logits, cols


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """The raw bf16 bit patterns of a CPU bf16 tensor, as a uint16 numpy array (no copy)."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)
