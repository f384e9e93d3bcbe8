"""Pins of the oracle against facts outside itself: the pages' constants, closed forms, library
routines (cuRAND's host Philox, torch's scaled-dot-product attention), brute force and invariants.

CPU only.  Each test names what it pins and why a plausible mistake would fail it.
"""
import ctypes
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_constants():
    out = {}
    with open(os.path.join(GOLDEN, "sampler_constants.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            name, value = line.split("|")[0].split()
            out[name] = float(value)
    return out


# ------------------------------------------------------------------------------------------------
# constants and schedule (the pages' numbers)
# ------------------------------------------------------------------------------------------------

def test_page_constants_match_defaults():
    g = _golden_constants()
    assert g["canvas_length"] == synthetic.CANVAS
    assert g["max_steps"] == synthetic.MAX_STEPS
    assert g["t_start"] == synthetic.T_START and g["t_end"] == synthetic.T_END
    assert g["entropy_bound"] == synthetic.ENTROPY_BOUND
    assert g["stop_mean_entropy"] == synthetic.STOP_MEAN_ENTROPY
    p = oracle.SamplerParams(vocab=4096)
    assert (p.canvas_len, p.max_steps, p.entropy_bound, p.stop_mean_entropy) == (256, 48, 0.1, 0.005)


def test_temperature_schedule_linear_0p8_to_0p4_over_48():
    g = _golden_constants()
    S = int(g["max_steps"])
    T = [oracle.temperature(s, S, g["t_start"], g["t_end"]) for s in range(S)]
    assert T[0] == np.float32(0.8) and T[-1] == np.float32(0.4)
    assert abs(T[12] - 0.6978723) < 1e-7
    d = np.diff(np.asarray(T, dtype=np.float64))
    assert np.all(d < 0)
    np.testing.assert_allclose(d, -0.4 / 47, atol=1e-7)    # linear: constant decrement up to fp32 rounding


# ------------------------------------------------------------------------------------------------
# Philox4x32-10 vs an independent implementation (cuRAND's host generator)
# ------------------------------------------------------------------------------------------------

def _curand_words(seed, n):
    try:
        lib = ctypes.CDLL("libcurand.so")
    except OSError:
        path = "/usr/local/cuda/lib64/libcurand.so"
        if not os.path.exists(path):
            pytest.skip("libcurand not available")
        lib = ctypes.CDLL(path)
    gen = ctypes.c_void_p()
    CURAND_RNG_PSEUDO_PHILOX4_32_10 = 161
    assert lib.curandCreateGeneratorHost(ctypes.byref(gen), CURAND_RNG_PSEUDO_PHILOX4_32_10) == 0
    assert lib.curandSetPseudoRandomGeneratorSeed(gen, ctypes.c_ulonglong(seed)) == 0
    buf = (ctypes.c_uint32 * n)()
    assert lib.curandGenerate(gen, buf, n) == 0
    lib.curandDestroyGenerator(gen)
    return np.frombuffer(buf, dtype=np.uint32).copy()


@pytest.mark.parametrize("seed", [0, 7, 0x123456789ABCDEF0, 2**64 - 1])
def test_philox_matches_curand_host_generator(seed):
    """cuRAND's host Philox4x32-10 emits, for block j, the 4 words of counter (0, 0, j, 0) under
    key (seed low, seed high).  Any slip in a multiplier, the Weyl bump, the round wiring or the
    round count changes every word."""
    blocks = 2048
    w = _curand_words(seed, 4 * blocks)
    key = [seed & 0xFFFFFFFF, seed >> 32]
    for j in list(range(64)) + list(range(64, blocks, 97)):
        np.testing.assert_array_equal(oracle.philox4x32_10([0, 0, j, 0], key), w[4 * j: 4 * j + 4])


def test_rng_word_uses_counter_and_key_layout():
    seed = 0xDEADBEEF01234567
    key = [seed & 0xFFFFFFFF, seed >> 32]
    for (c0, pos, step, tag, word) in [(0, 0, 0, 0, 0), (5, 17, 3, 1, 2), (123, 4000, 47, 2, 3)]:
        ref = oracle.philox4x32_10([c0, pos, step, tag], key)[word]
        assert oracle.rng_word(seed, c0, pos, step, tag, word) == ref


def test_uniform_gumbel_token_closed_forms():
    assert oracle.uniform(0) == 2.0 ** -24
    assert oracle.uniform(0xFFFFFFFF) == 1 - 2.0 ** -24
    assert oracle.uniform(1 << 31) == 0.5 + 2.0 ** -24
    # the Gumbel range follows from the uniform's range
    assert abs(oracle.gumbel(0) - (-math.log(-math.log(2.0 ** -24)))) < 1e-12
    assert abs(oracle.gumbel(0xFFFFFFFF) - 16.635532333438686) < 1e-6
    for V in (4096, 262144):
        assert oracle.token_from_word(0, V) == 0
        assert oracle.token_from_word(0xFFFFFFFF, V) == V - 1
        sh = 32 - int(math.log2(V))
        for x in (1, 12345, 0x80000000, 0xDEADBEEF):
            assert oracle.token_from_word(x, V) == x >> sh   # power-of-two V: the top bits


def test_philox_words_are_balanced():
    """Bit balance and counter-neighbour independence of the stream (statistical sanity)."""
    seed = 99
    words = np.array([oracle.rng_word(seed, i, 3, 0, 0, w) for i in range(2000) for w in range(4)], dtype=np.uint64)
    bits = ((words[:, None] >> np.arange(32, dtype=np.uint64)) & 1).astype(np.float64)
    assert np.all(np.abs(bits.mean(0) - 0.5) < 0.05)
    u = (2 * (words >> 9) + 1) / 2.0 ** 24
    assert abs(np.corrcoef(u[:-1], u[1:])[0, 1]) < 0.05


# ------------------------------------------------------------------------------------------------
# entropy, temperature and Gumbel-max sampling
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("V", [4096, 262144])
def test_entropy_of_uniform_logits_is_lnV(V):
    r = oracle.sample_rows(np.full((1, V), 1.25, dtype=np.float32), None, [0], 0.8, 0, 0)
    assert abs(r["H"][0] - math.log(V)) < 1e-9


def test_entropy_of_one_hot_is_zero():
    l = np.zeros((1, 4096))
    l[0, 77] = 200.0
    r = oracle.sample_rows(l, None, [0], 0.8, 1, 0)
    assert abs(r["H"][0]) < 1e-12 and r["y"][0] == 77


@pytest.mark.parametrize("delta,T", [(0.0, 1.0), (1.0, 1.0), (2.0, 0.5), (-3.0, 0.8)])
def test_entropy_two_point_binary_closed_form(delta, T):
    l = np.array([[0.0, delta]])
    r = oracle.sample_rows(l, None, [0], T, 3, 0)
    T = float(np.float32(T))              # the sampler takes its temperature as fp32
    p = 1.0 / (1.0 + math.exp(-delta / T))
    H = -(p * math.log(p) + (1 - p) * math.log(1 - p))
    assert abs(r["H"][0] - H) < 1e-12


def test_entropy_invariances_shift_and_temperature():
    rng = np.random.default_rng(0)
    l = rng.normal(0, 3, (1, 4096))
    a = oracle.sample_rows(l, None, [0], 0.8, 0, 0)["H"][0]
    b = oracle.sample_rows(l + 11.0, None, [0], 0.8, 0, 0)["H"][0]
    c = oracle.sample_rows(l / float(np.float32(0.8)), None, [0], 1.0, 0, 0)["H"][0]
    assert abs(a - b) < 1e-9 and abs(a - c) < 1e-9


@pytest.mark.parametrize("T", [1.0, 0.5])
def test_gumbel_max_frequencies_follow_softmax(T):
    """argmax(z + Gumbel) over 10^6 positions at V = 8 has the softmax(l/T) law (chi-square, 7 dof)."""
    z = np.array([0.0, 0.5, 1.0, -1.0, 2.0, 0.3, -0.7, 1.5])
    n = 1_000_000
    logits = np.ascontiguousarray(np.broadcast_to(z, (n, 8)))
    r = oracle.sample_rows(logits, None, np.arange(n), T, 2024, 5)
    counts = np.bincount(r["y"], minlength=8)
    p = np.exp(z / T - (z / T).max())
    p /= p.sum()
    chi2 = float(((counts - n * p) ** 2 / (n * p)).sum())
    assert chi2 < 30.0, (chi2, counts, n * p)       # p-value ~1e-4 at 7 dof


def test_rerandomisation_ids_are_uniform():
    n, V = 200_000, 16
    r = oracle.sample_rows(np.zeros((n, V)), None, np.arange(n), 1.0, 11, 2)
    counts = np.bincount(r["rr"], minlength=V)
    chi2 = float(((counts - n / V) ** 2 / (n / V)).sum())
    assert chi2 < 45.0


def test_canvas_init_is_uniform_and_deterministic():
    ids, commit = oracle.canvas_init(256, 128, 0, 4096)
    ids2, _ = oracle.canvas_init(256, 128, 0, 4096)
    np.testing.assert_array_equal(ids, ids2)
    assert commit.sum() == 0 and ids.min() >= 0 and ids.max() < 4096
    big, _ = oracle.canvas_init(100_000, 0, 5, 64)
    counts = np.bincount(big, minlength=64)
    assert float(((counts - 100_000 / 64) ** 2 / (100_000 / 64)).sum()) < 120.0
    # the word used is tag 2, step 0, counter word 0 at the absolute position
    assert ids[3] == oracle.token_from_word(oracle.rng_word(0, 0, 131, 0, 2, 0), 4096)


# ------------------------------------------------------------------------------------------------
# step rule (commit / re-randomise / stop)
# ------------------------------------------------------------------------------------------------

def test_step_rule_cases():
    V = 100
    commit = np.array([1, 0, 0, 0, 0], np.uint8)
    ids = np.array([9, 1, 2, 3, 4], np.int32)
    H = np.array([0.0, 0.05, 0.1, 1.0, 4.0])
    y = np.array([-1, 11, 12, 13, 14], np.int32)
    rr = np.array([-1, 21, 22, 23, 24], np.int32)
    r = oracle.step_rule(commit, ids, H, y, rr, s=0, rerand_entropy=2.0, vocab=V)
    np.testing.assert_array_equal(r["ids"], [9, 11, 12, 13, 24])     # keep / commit / commit (<=) / y / rr
    np.testing.assert_array_equal(r["commit"], [1, 1, 1, 0, 0])
    assert r["stop"] == 0 and abs(r["mean_H"] - 5.15 / 5) < 1e-12
    # last step of the budget: everything commits with y
    r = oracle.step_rule(commit, ids, H, y, rr, s=47, rerand_entropy=2.0, vocab=V)
    assert r["stop"] == 1
    np.testing.assert_array_equal(r["ids"], [9, 11, 12, 13, 14])
    np.testing.assert_array_equal(r["commit"], [1, 1, 1, 1, 1])
    # adaptive stop on the canvas-mean entropy
    H2 = np.array([0.0, 0.2, 0.0, 0.0, 0.0])
    r = oracle.step_rule(commit, ids, H2, y, rr, s=3, stop_mean_entropy=0.05, vocab=V)
    assert r["stop"] == 1 and r["commit"].all()
    # fixed steps: no adaptive stop, stop exactly at s+1 == fixed
    r = oracle.step_rule(commit, ids, H2, y, rr, s=3, stop_mean_entropy=0.05, fixed_steps=12, vocab=V)
    assert r["stop"] == 0
    r = oracle.step_rule(commit, ids, H, y, rr, s=11, fixed_steps=12, vocab=V)
    assert r["stop"] == 1 and r["commit"].all()
    # all committed -> stop
    r = oracle.step_rule(commit, ids, np.zeros(5), y, rr, s=0, vocab=V)
    assert r["stop"] == 1


# ------------------------------------------------------------------------------------------------
# model pieces
# ------------------------------------------------------------------------------------------------

def test_rmsnorm_closed_forms():
    d = 64
    g = np.linspace(0.5, 2.0, d).astype(np.float32)
    for c in (0.3, -2.0, 10.0):
        out = oracle.rmsnorm(np.full((1, d), c), g, eps=1e-6)
        np.testing.assert_allclose(out[0], c / math.sqrt(c * c + 1e-6) * g.astype(np.float64), rtol=1e-14)
    x = np.random.default_rng(1).normal(size=(3, d))
    out = oracle.rmsnorm(x, np.ones(d, np.float32), eps=0.0)
    np.testing.assert_allclose(np.sqrt((out ** 2).mean(1)), 1.0, rtol=1e-12)
    np.testing.assert_allclose(oracle.rmsnorm(x * 7.0, np.ones(d, np.float32), eps=0.0), out, rtol=1e-12)


def test_rope_closed_forms():
    rng = np.random.default_rng(2)
    x = rng.normal(size=(5, 3, 8))
    np.testing.assert_array_equal(oracle.rope(x, np.zeros(5), 10000.0), x)         # position 0 = identity
    # dh = 2: a plain rotation by `pos` radians (theta^0 = 1)
    v = rng.normal(size=(4, 1, 2))
    pos = np.array([1, 2, 5, 100])
    out = oracle.rope(v, pos, 10000.0)
    c, s = np.cos(pos), np.sin(pos)
    np.testing.assert_allclose(out[:, 0, 0], v[:, 0, 0] * c - v[:, 0, 1] * s, rtol=1e-12)
    np.testing.assert_allclose(out[:, 0, 1], v[:, 0, 1] * c + v[:, 0, 0] * s, rtol=1e-12)
    # half-split pairing: pair (i, i + dh/2) keeps its norm
    r = oracle.rope(x, np.arange(5) * 37, 10000.0)
    np.testing.assert_allclose(r[..., :4] ** 2 + r[..., 4:] ** 2, x[..., :4] ** 2 + x[..., 4:] ** 2, rtol=1e-12)
    # relative position: <R(m) q, R(n) k> depends on m - n only
    q, k = rng.normal(size=(1, 1, 8)), rng.normal(size=(1, 1, 8))
    a = (oracle.rope(q, [9], 10000.0) * oracle.rope(k, [4], 10000.0)).sum()
    b = (oracle.rope(q, [1009], 10000.0) * oracle.rope(k, [1004], 10000.0)).sum()
    assert abs(a - b) < 1e-10


def _sdpa_ref(q, k, v, mask):
    """torch's scaled-dot-product attention (fp64, CPU), with K/V heads repeated for GQA."""
    rep = q.shape[1] // k.shape[1]
    Q = torch.from_numpy(q).transpose(0, 1)
    K = torch.from_numpy(k).repeat_interleave(rep, dim=1).transpose(0, 1)
    V = torch.from_numpy(v).repeat_interleave(rep, dim=1).transpose(0, 1)
    o = F.scaled_dot_product_attention(Q, K, V, attn_mask=torch.from_numpy(mask.astype(bool)))
    return o.transpose(0, 1).numpy()


@pytest.mark.parametrize("P", [0, 1, 17, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("hq,hkv", [(4, 2), (4, 4), (8, 1)])
def test_attention_matches_torch_sdpa_with_block_mask(P, causal, hq, hkv):
    rng = np.random.default_rng(P * 7 + hq + hkv)
    n, dh = 19, 16
    q = rng.normal(size=(n, hq, dh))
    k = rng.normal(size=(P + n, hkv, dh))
    v = rng.normal(size=(P + n, hkv, dh))
    mask = np.ones((n, P + n), np.uint8)
    if causal:
        mask[:, P:] = np.tril(np.ones((n, n), np.uint8))
    np.testing.assert_allclose(oracle.attention(q, k, v, mask), _sdpa_ref(q, k, v, mask), rtol=1e-10, atol=1e-12)


def test_attention_single_visible_key_returns_its_value():
    rng = np.random.default_rng(3)
    q, k, v = rng.normal(size=(3, 2, 8)), rng.normal(size=(5, 1, 8)), rng.normal(size=(5, 1, 8))
    mask = np.zeros((3, 5), np.uint8)
    mask[0, 2] = mask[1, 4] = mask[2, 0] = 1
    out = oracle.attention(q, k, v, mask)
    for i, j in [(0, 2), (1, 4), (2, 0)]:
        np.testing.assert_allclose(out[i, 0], v[j, 0], rtol=1e-14)
        np.testing.assert_allclose(out[i, 1], v[j, 0], rtol=1e-14)


def test_router_topk_order_ties_and_gates():
    l = np.array([[0.1, 3.0, -1.0, 3.0, 2.0, 0.0, 5.0, 1.0]])
    sel, gate = oracle.router_topk(l, 3)
    np.testing.assert_array_equal(sel[0], [6, 1, 3])           # tie 3.0: lower id first
    e = np.exp(np.array([5.0, 3.0, 3.0]) - 5.0)
    np.testing.assert_allclose(gate[0], e / e.sum(), rtol=1e-14)
    perm = np.random.default_rng(4).permutation(16).astype(np.float64)
    sel, gate = oracle.router_topk(perm[None], 16)
    np.testing.assert_array_equal(sel[0], np.argsort(-perm))
    np.testing.assert_allclose(gate[0], np.exp(perm[sel[0]] - 15) / np.exp(perm - 15).sum(), rtol=1e-12)


def _tiny_model(seed=0, **kw):
    cfg = synthetic.TINY
    w = synthetic.make_model_weights(cfg, seed, **kw)
    return cfg, w, oracle.Model(cfg, w)


def _dense_moe_torch(L, cfg, h, gates_full):
    """Dense mixture: every expert evaluated with torch matmuls, weighted by a [n, E] gate matrix that
    is zero outside each token's selection."""
    H = torch.from_numpy(h)
    Wgu = L["w_gate_up"].to(torch.float64)
    Wd = L["w_down"].to(torch.float64)
    out = torch.zeros_like(H)
    for e in range(cfg.n_exp):
        g = H @ Wgu[e, : cfg.d_ff].T
        u = H @ Wgu[e, cfg.d_ff:].T
        out += torch.from_numpy(gates_full[:, e: e + 1]) * ((F.silu(g) * u) @ Wd[e].T)
    return out.numpy()


def test_moe_sparse_selection_equals_dense_masked_mixture():
    cfg, w, M = _tiny_model(5)
    rng = np.random.default_rng(5)
    h = rng.normal(size=(6, cfg.d_model))
    logits = rng.normal(size=(6, cfg.n_exp))
    sel, gate = oracle.router_topk(logits, cfg.top_k)
    gf = np.zeros((6, cfg.n_exp))
    for t in range(6):
        gf[t, sel[t]] = gate[t]
    y = oracle.moe(M, 0, h, sel, gate)
    np.testing.assert_allclose(y, _dense_moe_torch(w["layers"][0], cfg, h, gf), rtol=1e-9, atol=1e-12)
    # k = E: the plain softmax mixture over all experts
    sel, gate = oracle.router_topk(logits, cfg.n_exp)
    p = np.exp(logits - logits.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    np.testing.assert_allclose(oracle.moe(M, 0, h, sel, gate), _dense_moe_torch(w["layers"][0], cfg, h, p),
                               rtol=1e-9, atol=1e-12)


# ------------------------------------------------------------------------------------------------
# layer / model invariants
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("gain_std", [0.0, 0.1])
def test_layer_forward_composition_matches_pieces(gain_std):
    """The layer equals its pieces strung together: norm -> QKV -> RoPE -> masked attention -> O ->
    residual -> norm -> router -> top-k -> experts -> residual (each piece pinned above).  With
    gain_std > 0 the attention and MoE norms have distinct random gains, so a layer that applied one
    in place of the other, or left a gain out, would not match."""
    cfg, w, M = _tiny_model(6, gain_std=gain_std)
    L = w["layers"][0]
    if gain_std:
        assert not torch.equal(L["attn_norm"], L["ffn_norm"])
    rng = np.random.default_rng(6)
    n, P = 9, 5
    x = rng.normal(size=(n, cfg.d_model))
    kc = rng.normal(size=(P, cfg.n_kv, cfg.d_head))
    vc = rng.normal(size=(P, cfg.n_kv, cfg.d_head))
    pos = np.arange(P, P + n)
    out, kn, vn, rl = oracle.layer_forward(M, 0, x, pos, P, kc, vc, causal=False)

    f64 = lambda t: t.to(torch.float64).numpy()
    h = oracle.rmsnorm(x, L["attn_norm"].numpy())
    qkv = h @ f64(L["w_qkv"]).T
    nq, nkv, dh = cfg.n_q, cfg.n_kv, cfg.d_head
    q = oracle.rope(qkv[:, : nq * dh].reshape(n, nq, dh), pos)
    k = oracle.rope(qkv[:, nq * dh: (nq + nkv) * dh].reshape(n, nkv, dh), pos)
    v = qkv[:, (nq + nkv) * dh:].reshape(n, nkv, dh)
    att = oracle.attention(q, np.concatenate([kc, k]), np.concatenate([vc, v]), np.ones((n, P + n), np.uint8))
    x1 = x + att.reshape(n, -1) @ f64(L["w_o"]).T
    h2 = oracle.rmsnorm(x1, L["ffn_norm"].numpy())
    r = h2 @ f64(L["w_router"]).T
    sel, gate = oracle.router_topk(r, cfg.top_k)
    x2 = x1 + oracle.moe(M, 0, h2, sel, gate)
    np.testing.assert_allclose(out, x2, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(kn, k, rtol=1e-12)
    np.testing.assert_allclose(vn, v, rtol=1e-12)
    np.testing.assert_allclose(rl, r, rtol=1e-10, atol=1e-14)


def test_routing_flip_takes_the_next_expert():
    """The tests' routing alternative: a flagged token takes its (k+1)-th expert in place of its k-th,
    gates renormalised over the new selection; unflagged tokens keep the model's routing.  Pinned
    against hand-picked logits and against the layer built from its pieces with that selection."""
    l = np.array([[0.1, 3.0, -1.0, 2.5, 2.0, 0.0, 5.0, 1.0], [0.0, 1.0, 2.0, 3.0, 4.0, 5.0, 6.0, 7.0]])
    sel, gate = oracle.router_topk(l, 3, flip=[1, 0])
    np.testing.assert_array_equal(sel, [[6, 1, 4], [7, 6, 5]])
    e = np.exp(np.array([5.0, 3.0, 2.0]) - 5.0)
    np.testing.assert_allclose(gate[0], e / e.sum(), rtol=1e-14)
    s0, g0 = oracle.router_topk(l, 3)
    np.testing.assert_array_equal(s0[1], sel[1])
    np.testing.assert_array_equal(g0[1], gate[1])
    # a layer with flagged tokens equals its pieces with the flipped selection
    cfg, w, M = _tiny_model(14, gain_std=0.1)
    L = w["layers"][0]
    rng = np.random.default_rng(14)
    n = 6
    x = rng.normal(size=(n, cfg.d_model))
    pos = np.arange(n)
    flip = np.array([1, 0, 0, 1, 1, 0], np.uint8)
    out, _, _, r, mid = oracle.layer_forward(M, 0, x, pos, want_mid=True, flip=flip)
    h2 = oracle.rmsnorm(mid, L["ffn_norm"].numpy())
    sel, gate = oracle.router_topk(r, cfg.top_k, flip=flip)
    np.testing.assert_allclose(out, mid + oracle.moe(M, 0, h2, sel, gate), rtol=1e-12, atol=1e-13)
    plain = oracle.layer_forward(M, 0, x, pos)[0]
    np.testing.assert_array_equal(out[flip == 0], plain[flip == 0])   # no attention after the MoE
    assert np.abs(out[flip == 1] - plain[flip == 1]).max() > 1e-4


def test_head_is_final_norm_then_vocabulary_projection():
    """The vocabulary head is the final RMSNorm (with its own gain) followed by x W_head^T, built here
    from the pinned RMSNorm and a torch matmul; a head that skipped the norm or used another gain
    would not match."""
    cfg, w, M = _tiny_model(12, gain_std=0.1)
    rng = np.random.default_rng(12)
    x = rng.normal(size=(5, cfg.d_model)) * 3.0
    want = oracle.rmsnorm(x, w["final_norm"].numpy()) @ w["head"].to(torch.float64).numpy().T
    np.testing.assert_allclose(oracle.head(M, x), want, rtol=1e-10, atol=1e-12)
    plain = oracle.rmsnorm(x, np.ones(cfg.d_model, np.float32)) @ w["head"].to(torch.float64).numpy().T
    assert np.abs(oracle.head(M, x) - plain).max() > 1e-3


def test_forward_chains_layers_in_order_with_their_own_gains():
    """The full forward is embedding -> layer 0 -> layer 1 -> head, each layer with its own weights and
    gains (distinct random gains per layer): hidden[l + 1] = layer_forward(l, hidden[l]) and the
    logits are the head of the last hidden state."""
    cfg, w, M = _tiny_model(13, gain_std=0.1)
    ids = synthetic.make_ids(20, cfg.vocab, 13).numpy()
    P = 7
    rng = np.random.default_rng(13)
    kc = [rng.normal(size=(64, cfg.n_kv, cfg.d_head)) for _ in range(cfg.n_layers)]
    vc = [rng.normal(size=(64, cfg.n_kv, cfg.d_head)) for _ in range(cfg.n_layers)]
    pos = np.arange(P, P + 20)
    fw = oracle.forward(M, ids, pos, P, kc, vc, want_hidden=True)
    x = fw["hidden"][0]
    np.testing.assert_array_equal(x, w["emb"][torch.from_numpy(ids).long()].to(torch.float64).numpy())
    for l in range(cfg.n_layers):
        x = oracle.layer_forward(M, l, x, pos, P, kc[l][:P], vc[l][:P])[0]
        np.testing.assert_allclose(fw["hidden"][l + 1], x, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(fw["logits"], oracle.head(M, x), rtol=1e-12, atol=1e-13)


def test_canvas_layer_is_permutation_equivariant():
    """Bidirectional canvas attention has no mask inside the canvas: permuting the rows together with
    their positions permutes the outputs.  An accidental causal mask breaks this."""
    cfg, w, M = _tiny_model(7)
    rng = np.random.default_rng(7)
    n, P = 12, 6
    x = rng.normal(size=(n, cfg.d_model))
    kc, vc = rng.normal(size=(P, cfg.n_kv, cfg.d_head)), rng.normal(size=(P, cfg.n_kv, cfg.d_head))
    pos = np.arange(P, P + n)
    perm = rng.permutation(n)
    a = oracle.layer_forward(M, 0, x, pos, P, kc, vc)[0]
    b = oracle.layer_forward(M, 0, x[perm], pos[perm], P, kc, vc)[0]
    np.testing.assert_allclose(b, a[perm], rtol=1e-9, atol=1e-12)


def test_causal_prefill_rows_ignore_later_rows():
    cfg, w, M = _tiny_model(8)
    rng = np.random.default_rng(8)
    x = rng.normal(size=(10, cfg.d_model))
    a = oracle.layer_forward(M, 1, x, np.arange(10), causal=True)[0]
    b = oracle.layer_forward(M, 1, x[:6], np.arange(6), causal=True)[0]
    np.testing.assert_allclose(a[:6], b, rtol=1e-10, atol=1e-12)
    c = oracle.layer_forward(M, 1, x, np.arange(10), causal=False)[0]
    assert np.abs(c[:6] - b).max() > 1e-6          # the canvas mask does see later rows


def test_canvas_steps_leave_prefix_cache_untouched_and_commit_writes_block_kv():
    cfg, w, M = _tiny_model(9)
    seq = oracle.Sequence(M, max_ctx=128 + 2 * 256)
    prompt = synthetic.make_ids(128, cfg.vocab, 0).numpy()
    seq.prefill(prompt)
    before = [k.copy() for k in seq.k] + [v.copy() for v in seq.v]
    prm = oracle.SamplerParams(cfg.vocab, max_steps=48, fixed_steps=2, seed=0)
    ids, commit = seq.canvas_init(prm)
    for _ in range(2):
        r = seq.canvas_step(prm, ids, commit)
        ids, commit = r["ids"], r["commit"]
    after = [k for k in seq.k] + [v for v in seq.v]
    for a, b in zip(before, after):
        np.testing.assert_array_equal(a, b)
    assert r["stop"] == 1 and commit.all()
    # block commit: cache rows [P, P+256) are the per-layer K/V of a canvas forward on the final ids
    P = seq.P
    kc = [k.copy() for k in seq.k]
    vc = [v.copy() for v in seq.v]
    seq.block_commit(ids)
    assert seq.P == P + 256
    x = np.empty((256, cfg.d_model))
    oracle.lib().orc_embed(ctypes.byref(M.c_cfg), M.emb.ctypes.data_as(ctypes.c_void_p), 256,
                           np.ascontiguousarray(ids).ctypes.data_as(ctypes.c_void_p),
                           x.ctypes.data_as(ctypes.c_void_p))
    pos = np.arange(P, P + 256)
    for l in range(cfg.n_layers):
        x, kn, vn, _ = oracle.layer_forward(M, l, x, pos, P, kc[l][:P], vc[l][:P])
        np.testing.assert_allclose(seq.k[l][P:P + 256], kn, rtol=1e-12)
        np.testing.assert_allclose(seq.v[l][P:P + 256], vn, rtol=1e-12)
        np.testing.assert_array_equal(seq.k[l][:P], kc[l][:P])


def test_decode_invariants_with_confident_head():
    """With a sharpened head, positions commit over the steps: committed ids never change, the count
    of committed positions never drops, and the block ends with all 256 committed."""
    cfg, w, M = _tiny_model(0, head_scale=50.0)
    seq = oracle.Sequence(M, max_ctx=128 + 256)
    seq.prefill(synthetic.make_ids(128, cfg.vocab, 0).numpy())
    prm = oracle.SamplerParams(cfg.vocab, seed=0)
    ids, commit = seq.canvas_init(prm)
    n_prev = 0
    for s in range(48):
        r = seq.canvas_step(prm, ids, commit)
        was = commit.astype(bool)
        np.testing.assert_array_equal(r["ids"][was], ids[was])
        assert np.all(r["H"][was] == 0.0)
        assert r["commit"].sum() >= n_prev
        n_prev = int(r["commit"].sum())
        ids, commit = r["ids"], r["commit"]
        if r["stop"]:
            break
    assert r["stop"] == 1 and commit.all()
    assert 0 < s < 47            # some positions commit early and the block stops before the budget


# ------------------------------------------------------------------------------------------------
# FP8 weight form (e4m3 bytes with one fp32 scale per 128 x 128 tile)
# ------------------------------------------------------------------------------------------------

def test_e4m3_decode_matches_torch_float8_e4m3fn():
    """Every one of the 256 codes decodes as torch's float8_e4m3fn (an independent implementation
    of the OCP E4M3 format: subnormals, the 448 maximum, the two NaN codes, signed zero)."""
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3_to_double(int(q)) for q in range(256)])
    nan = np.isnan(ref)
    assert nan.sum() == 2 and np.array_equal(nan, np.isnan(got))
    np.testing.assert_array_equal(got[~nan], ref[~nan])
    np.testing.assert_array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))
    assert oracle.e4m3_to_double(0x7E) == 448.0 and oracle.e4m3_to_double(0x01) == 2.0 ** -9


def _fp8_pow2_layer(cfg, seed):
    """A layer in the FP8 form whose tile scales are distinct powers of two (so q * s is exactly a
    bf16 value) together with the same layer as bf16 tensors holding q * s."""
    rng = np.random.default_rng(seed)
    shapes = {"w_qkv": (cfg.qkv_rows, cfg.d_model), "w_o": (cfg.d_model, cfg.n_q * cfg.d_head),
              "w_router": (cfg.n_exp, cfg.d_model), "w_gate_up": (cfg.n_exp, 2 * cfg.d_ff, cfg.d_model),
              "w_down": (cfg.n_exp, cfg.d_model, cfg.d_ff)}
    fp8 = {"attn_norm": torch.ones(cfg.d_model), "ffn_norm": torch.ones(cfg.d_model)}
    bf = dict(fp8)
    for k, shp in shapes.items():
        codes = rng.integers(0, 256, size=shp).astype(np.uint8)
        codes[(codes & 0x7F) == 0x7F] = 0x38          # no NaN codes (0x38 = 1.0)
        R, C = int(np.prod(shp[:-1])), shp[-1]
        tr, tc = -(-R // 128), -(-C // 128)
        expo = -(4 + (np.arange(tr)[:, None] * 3 + np.arange(tc)[None, :] * 5) % 7)
        scale = np.ldexp(1.0, expo).astype(np.float32)
        q = torch.from_numpy(codes)
        fp8[k] = {"e4m3": q, "scale": torch.from_numpy(scale)}
        s_full = torch.from_numpy(scale).double().repeat_interleave(128, 0).repeat_interleave(128, 1)[:R, :C]
        w = q.view(torch.float8_e4m3fn).double().reshape(R, C) * s_full
        wb = w.to(torch.bfloat16)
        assert torch.equal(wb.double(), w)              # exactly representable
        bf[k] = wb.reshape(shp)
    return fp8, bf


def test_fp8_layer_equals_bf16_layer_holding_q_times_s():
    """The oracle's FP8 matrices are q * s with the scale of tile [r / 128][c / 128]: a layer in the
    FP8 form equals, bit for bit, the layer given as bf16 weights q * s (distinct per-tile scales
    catch a transposed or shifted tile index, in every matrix including the expert stacks)."""
    cfg = synthetic.TINY
    fp8, bf = _fp8_pow2_layer(cfg, 11)
    M8 = oracle.Model(cfg, {"layers": [fp8]}, layers=[fp8])
    Mb = oracle.Model(cfg, {"layers": [bf]}, layers=[bf])
    rng = np.random.default_rng(12)
    n, P = 10, 7
    x = rng.normal(size=(n, cfg.d_model))
    kc, vc = rng.normal(size=(P, cfg.n_kv, cfg.d_head)), rng.normal(size=(P, cfg.n_kv, cfg.d_head))
    pos = np.arange(P, P + n)
    a = oracle.layer_forward(M8, 0, x, pos, P, kc, vc)
    b = oracle.layer_forward(Mb, 0, x, pos, P, kc, vc)
    for u, v in zip(a, b):
        np.testing.assert_array_equal(u, v)


def test_cumulative_entropy_bound_commits_the_lowest_entropy_prefix():
    """The cumulative reading of the entropy bound: uncommitted positions in ascending (H, position)
    order commit while the running entropy sum stays within the bound.  Hand-built case: with bound
    0.1 the per-position rule commits every H <= 0.1, the cumulative one only the prefix 0.015, 0.02,
    0.03, 0.03 (equal entropies by position) -> sums 0.015, 0.035, 0.065, 0.095; the next (0.04)
    would exceed."""
    V = 4096
    H = np.array([0.04, 0.03, 0.5, 0.02, 0.03, 0.015, 3.0, 0.09])
    commit = np.array([0, 0, 0, 0, 0, 0, 0, 1], np.uint8)          # position 7 already committed
    ids = np.arange(8, dtype=np.int32) + 100
    y = np.arange(8, dtype=np.int32) + 200
    rr = np.arange(8, dtype=np.int32) + 300
    per = oracle.step_rule(commit, ids, H, y, rr, s=0, rerand_entropy=1.0, vocab=V)
    np.testing.assert_array_equal(per["commit"], [1, 1, 0, 1, 1, 1, 0, 1])
    cu = oracle.step_rule(commit, ids, H, y, rr, s=0, rerand_entropy=1.0, vocab=V, cumulative=True)
    np.testing.assert_array_equal(cu["commit"], [0, 1, 0, 1, 1, 1, 0, 1])
    np.testing.assert_array_equal(cu["ids"], [200, 201, 202, 203, 204, 205, 306, 107])   # 6 re-randomised
    np.testing.assert_allclose(cu["cum"][[5, 3, 1, 4, 0]], [0.015, 0.035, 0.065, 0.095, 0.135], rtol=1e-12)
    assert cu["cum"][7] == 0.0
    # a bound below every entropy commits nothing; a huge bound commits every uncommitted position
    assert oracle.step_rule(commit, ids, H, y, rr, s=0, entropy_bound=0.01, rerand_entropy=1.0, vocab=V,
                            cumulative=True)["commit"].sum() == 1
    assert oracle.step_rule(commit, ids, H, y, rr, s=0, entropy_bound=10.0, rerand_entropy=1.0, vocab=V,
                            cumulative=True)["commit"].all()
