"""CUDA path (libdg.so through the C ABI) vs the oracle, element by element, on seeded inputs.

Marked gpu: they need an sm_100a device.  Shapes: the tiny model (several tiles plus ragged tails),
the full-width single layer, and the full-size sampler workload; full-size cases compare sampled
rows the oracle computes one by one plus properties that hold at any size.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synthetic
from dg_testutil import (ENTROPY_TOL, HIDDEN_TOL, MARGIN, ROUTER_TIE_REL_E2E, derived_tolerances, judge_step, kv_views,
                         rel_err, router_tie_tokens, to_device)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dg(cuda_ok):
    from block_discrete_diffusion_b200 import build, dg as dgmod
    build.build()
    return dgmod


def _oracle_sample(logits_cpu, commit, ids, pos, prm, step, vocab):
    T = oracle.temperature(step, prm.max_steps, prm.t_start, prm.t_end)
    smp = oracle.sample_rows(logits_cpu, commit, pos, T, prm.seed, step)
    rule = oracle.step_rule(commit, ids, smp["H"], smp["y"], smp["rr"], step, prm.entropy_bound, prm.rerand_entropy,
                            prm.stop_mean_entropy, prm.max_steps, prm.fixed_steps)
    out = dict(smp)
    out.update(rule)
    return out


# ------------------------------------------------------------------------------------------------
# sampler alone
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("vocab,spike,step,rows_checked,std", [
    (4096, 12.0, 0, None, 3.0),
    (4096, 40.0, 47, None, 3.0),
    (5120, 12.0, 5, None, 3.0),        # 1280 float4 groups: a full batch of 1024 and a ragged one
    (4096, 12.0, 30, None, 1000.0),    # tempered logits beyond the screen's range: accurate draws only
    (262144, 12.0, 12, None, 3.0),     # the full-size sampler workload, every row
    (262144, 40.0, 0, 48, 3.0),        # spike +40 rows commit; sampled rows
    (262144, 12.0, 47, 48, 3.0),
])
def test_sampler_matches_oracle(dg, vocab, spike, step, rows_checked, std):
    n_seq, canvas = 1, 256
    logits, _ = synthetic.make_sampler_logits(canvas, vocab, seed=7, std=std, spike=spike)
    prm_o = oracle.SamplerParams(vocab, seed=7)
    prm = dg.sampler_params(vocab, seed=7)
    rng = np.random.default_rng(step)
    commit0 = (rng.random(canvas) < 0.2).astype(np.uint8)      # some positions already committed
    ids0 = rng.integers(0, vocab, canvas).astype(np.int32)
    d_logits = logits.cuda()
    ids = torch.from_numpy(ids0).cuda()
    commit = torch.from_numpy(commit0).cuda()
    H = torch.empty(canvas, device="cuda")
    stop = torch.empty(n_seq, dtype=torch.int32, device="cuda")
    ws = torch.empty(dg.dg_sample_workspace_bytes(canvas, vocab), dtype=torch.uint8, device="cuda")
    dg.dg_sample(d_logits, n_seq, vocab, prm, step, None, ids, commit, H, stop, ws)
    torch.cuda.synchronize()
    g = {"ids": ids.cpu().numpy(), "commit": commit.cpu().numpy(), "H": H.cpu().numpy(), "stop": int(stop.item())}
    lg = logits.numpy()
    rows = np.arange(canvas) if rows_checked is None else np.unique(
        np.concatenate([np.arange(0, canvas, 10)[: rows_checked // 2], rng.choice(canvas, rows_checked // 2)]))
    if rows_checked is None:
        o = _oracle_sample(lg, commit0, ids0, np.arange(canvas), prm_o, step, vocab)
        fails, judged = judge_step(g, o, prm_o, commit0)
        assert not fails, fails[:10]
        assert judged > canvas // 2
    else:
        # per-row decisions on a sample of rows (the stop flag needs every row and is checked above)
        sub = np.ascontiguousarray(lg[rows])
        T = oracle.temperature(step)
        smp = oracle.sample_rows(sub, commit0[rows], rows, T, 7, step)
        assert np.abs(g["H"][rows] - smp["H"]).max() <= ENTROPY_TOL
        for k, r in enumerate(rows):
            if commit0[r]:
                assert g["ids"][r] == ids0[r] and g["commit"][r] == 1
                continue
            Hk = smp["H"][k]
            if abs(Hk - 0.1) <= 1e-3 or abs(Hk - prm_o.rerand_entropy) <= 1e-3:
                continue
            if Hk <= 0.1:
                assert g["commit"][r] == 1 and (smp["margin"][k] <= 1e-2 or g["ids"][r] == smp["y"][k])
            elif not g["stop"]:
                assert g["commit"][r] == 0
                if Hk > prm_o.rerand_entropy:
                    assert g["ids"][r] == smp["rr"][k]
                elif smp["margin"][k] > 1e-2:
                    assert g["ids"][r] == smp["y"][k]
    if spike == 40.0:
        spiked = np.arange(0, canvas, 10)
        assert g["commit"][spiked].all()       # near-one-hot rows commit


def test_sampler_cumulative_commit_rule_matches_oracle(dg):
    """commit_rule 1: the lowest-entropy uncommitted positions commit while their entropy sum stays
    within the bound.  Every third row gets a spike of height 11-14 above N(0,1) logits, so the
    spiked rows have entropies between ~0.002 and ~0.1 and the running sum crosses the bound part
    of the way through them."""
    vocab, canvas, step = 4096, 256, 0
    rng = np.random.default_rng(21)
    lg = rng.normal(size=(canvas, vocab)).astype(np.float32)
    for r in range(0, canvas, 3):
        lg[r, rng.integers(vocab)] += rng.uniform(11.0, 14.0)
    commit0 = (rng.random(canvas) < 0.1).astype(np.uint8)
    ids0 = rng.integers(0, vocab, canvas).astype(np.int32)
    prm_o = oracle.SamplerParams(vocab, seed=3, commit_rule=1)
    prm = dg.sampler_params(vocab, seed=3, commit_rule=1)
    ids = torch.from_numpy(ids0).cuda()
    commit = torch.from_numpy(commit0).cuda()
    H = torch.empty(canvas, device="cuda")
    stop = torch.empty(1, dtype=torch.int32, device="cuda")
    ws = torch.empty(dg.dg_sample_workspace_bytes(canvas, vocab), dtype=torch.uint8, device="cuda")
    dg.dg_sample(torch.from_numpy(lg).cuda(), 1, vocab, prm, step, None, ids, commit, H, stop, ws)
    torch.cuda.synchronize()
    g = {"ids": ids.cpu().numpy(), "commit": commit.cpu().numpy(), "H": H.cpu().numpy(), "stop": int(stop.item())}
    T = oracle.temperature(step)
    smp = oracle.sample_rows(lg, commit0, np.arange(canvas), T, 3, step)
    o = dict(smp)
    o.update(oracle.step_rule(commit0, ids0, smp["H"], smp["y"], smp["rr"], step, vocab=vocab, cumulative=True))
    fails, judged = judge_step(g, o, prm_o, commit0)
    assert not fails, fails[:10]
    new_commits = int(o["commit"].sum() - commit0.sum())
    per_position = int(((smp["H"] <= 0.1) & (commit0 == 0)).sum())
    assert 0 < new_commits < per_position            # the cumulative rule cut in, but not at zero
    assert judged > canvas // 2


def test_sampler_is_deterministic(dg):
    vocab, canvas = 262144, 256
    logits, _ = synthetic.make_sampler_logits(canvas, vocab, seed=3)
    d_logits = logits.cuda()
    prm = dg.sampler_params(vocab, seed=3)
    ws = torch.empty(dg.dg_sample_workspace_bytes(canvas, vocab), dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(2):
        ids = torch.zeros(canvas, dtype=torch.int32, device="cuda")
        commit = torch.zeros(canvas, dtype=torch.uint8, device="cuda")
        H = torch.empty(canvas, device="cuda")
        stop = torch.empty(1, dtype=torch.int32, device="cuda")
        dg.dg_sample(d_logits, 1, vocab, prm, 5, None, ids, commit, H, stop, ws)
        outs.append((ids.cpu(), commit.cpu(), H.cpu()))
    for a, b in zip(outs[0], outs[1]):
        assert torch.equal(a, b)


# ------------------------------------------------------------------------------------------------
# one decoder layer (attention block + MoE block)
# ------------------------------------------------------------------------------------------------

GAIN_STD = 0.1   # RMSNorm gains 1 + N(0, 0.1^2), distinct per norm and layer


def _layer_case(dg, cfg, P, seed, router_std=None):
    w = synthetic.make_model_weights(cfg, seed, router_std=router_std, gain_std=GAIN_STD)
    wd = to_device(w)
    model = dg.dg_model_create(cfg, wd)
    max_ctx = ((P + 256 + 255) // 256) * 256
    seqs = dg.dg_seqs_create(model, 1, max_ctx)
    ks, vs = synthetic.make_prefix_kv(cfg.n_layers, P, cfg.n_kv, cfg.d_head, seed + 1)
    if P > 0:
        dg.dg_load_prefix(seqs, 0, P, [k.cuda() for k in ks], [v.cuda() for v in vs])
    x = synthetic.make_hidden(256, cfg.d_model, seed + 2)
    return w, model, seqs, ks, vs, x


@pytest.mark.parametrize("cfg_name,P,n_rows,causal,route", [
    ("tiny", 0, 256, False, "folded"), ("tiny", 128, 256, False, "folded"), ("tiny", 300, 256, False, "folded"),
    ("tiny", 0, 44, True, "folded"), ("tiny", 256, 128, True, "folded"), ("tiny", 200, 56, True, "folded"),
    ("tiny", 384, 256, True, "folded"), ("tiny", 128, 256, False, "separate"), ("tiny", 200, 56, True, "separate"),
    ("tiny", 300, 256, False, "cluster_merge"),
    ("one_layer", 4096, 256, False, "folded"), ("one_layer", 2048, 200, True, "folded"),
    ("one_layer", 4096, 256, False, "separate"), ("one_layer", 4096, 256, False, "cluster_merge"),
    ("one_layer", 2048, 256, False, "topk_gather"), ("tiny", 128, 256, False, "topk_gather"),
])
def test_layer_matches_oracle(dg, monkeypatch, cfg_name, P, n_rows, causal, route):
    """One layer (attention block, then MoE block) on canvas rows (bidirectional) or on a prefill
    chunk (causal, ragged row counts), against a committed prefix of P positions.  route "folded":
    the FFN RMSNorm and the router folded into the O-projection epilogue (the default for up to 1024
    rows) and the attention's key splits merged by a launch of their own (the defaults); "separate":
    DG_ROUTE_FUSED=0, an RMSNorm launch and a router GEMM; "cluster_merge": DG_ATTN_CLUSTER_MERGE=1,
    the key splits merged inside the attention launch over a thread-block cluster; "topk_gather":
    DG_TOPK_GATHER=1, the routed rows bucketed and gathered inside the top-k launch (by default a
    gather launch of their own)."""
    monkeypatch.setenv("DG_ROUTE_FUSED", "0" if route == "separate" else "1")
    monkeypatch.setenv("DG_ATTN_CLUSTER_MERGE", "1" if route == "cluster_merge" else "0")
    monkeypatch.setenv("DG_TOPK_GATHER", "1" if route == "topk_gather" else "0")
    if cfg_name == "tiny":
        cfg, router_std = synthetic.TINY, None
    else:
        import dataclasses
        cfg = dataclasses.replace(synthetic.ONE_LAYER, vocab=1024)   # the layer does not read the vocabulary
        router_std = cfg.d_model ** -0.5                            # router logits ~ N(0, 1)
    w, model, seqs, ks, vs, x = _layer_case(dg, cfg, P, 11, router_std)
    xd = x.cuda()
    mid = torch.zeros_like(xd)
    rl = torch.zeros(256, cfg.n_exp, device="cuda")
    dg.dg_layer_forward(seqs, 0, xd, mid, rl, n_rows=n_rows, causal=causal)
    torch.cuda.synchronize()
    assert dg.dg_device_error(seqs) == 0
    n = n_rows
    M = oracle.Model(cfg, w)
    kc = ks[0].double().numpy() if P else None
    vc = vs[0].double().numpy() if P else None
    xo, kn, vn, rlo, mido = oracle.layer_forward(M, 0, x[:n].double().numpy(), np.arange(P, P + n), P, kc, vc,
                                                 causal=causal, want_mid=True)
    e_mid = rel_err(mid.cpu().numpy()[:n], mido)
    assert e_mid <= HIDDEN_TOL, f"attention block rel err {e_mid}"
    e_rl = rel_err(rl.cpu().numpy()[:n], rlo)
    assert e_rl <= HIDDEN_TOL, f"router logits rel err {e_rl}"
    keep = ~router_tie_tokens(rlo, cfg.top_k)
    e_out = rel_err(xd.cpu().numpy()[:n][keep], xo[keep])
    assert e_out <= HIDDEN_TOL, f"layer output rel err {e_out} ({keep.sum()} tokens judged)"
    # rows beyond n_rows are not touched
    if n < 256:
        assert torch.equal(xd[n:].cpu(), x[n:])
    # the rows' K/V went to cache rows [P, P+n); the prefix rows are unchanged
    K, Vt = kv_views(seqs.kv, cfg, 1, seqs.max_ctx)
    Kg = K[0, 0, :, P:P + n].permute(1, 0, 2).float().cpu().numpy()
    Vg = Vt[0, 0, :, :, P:P + n].permute(2, 0, 1).float().cpu().numpy()
    assert rel_err(Kg, kn) <= HIDDEN_TOL and rel_err(Vg, vn) <= HIDDEN_TOL
    if P:
        assert torch.equal(K[0, 0, :, :P].permute(1, 0, 2).cpu(), ks[0])
        assert torch.equal(Vt[0, 0, :, :, :P].permute(2, 0, 1).cpu(), vs[0])


# ------------------------------------------------------------------------------------------------
# full tiny model: prefill, canvas steps (resynchronised to the oracle), block commit, decode
# ------------------------------------------------------------------------------------------------

# Head variants of the tiny model: "x1" the stated init (logits ~N(0, 0.32^2): nothing commits before
# the step budget); "x50" the head's std x50 (confident rows commit; large logits, judged with the
# derived tolerances); "copy" the stated head plus emb / 16, over embeddings where 10% of the tokens
# ("loud", std 1.2) live in the first 128 channels and the rest ("quiet", std 0.1) in the others:
# a loud token's row scores its own token ~17 above the rest and commits (entropy ~1e-4), a quiet
# token's row sees logits as small as the stated head's (entropy ~8, re-randomised) -- the commit
# branch with the base tolerances.
HEADS = {"x1": {}, "x50": {"head_scale": 50.0},
         "copy": {"emb_split": (128, 1.2, 0.1, 0.1), "copy_head": 1.0 / 16}}


def _tiny_model_pair(dg, head="x1", seed=0, top_k=None, router="unit"):
    """router "stated": every matrix N(0, 0.02^2) as the tiny configuration states (router logits
    ~N(0, 0.32^2), many near-ties); "unit": router std d^-1/2 (logits ~N(0, 1)) when top_k < E."""
    import dataclasses
    if isinstance(head, float):
        head = "x1" if head == 1.0 else "x50"
    cfg = synthetic.TINY if top_k is None else dataclasses.replace(synthetic.TINY, top_k=top_k)
    router_std = cfg.d_model ** -0.5 if (cfg.top_k < cfg.n_exp and router == "unit") else None
    w = synthetic.make_model_weights(cfg, seed, router_std=router_std, gain_std=GAIN_STD, **HEADS[head])
    model = dg.dg_model_create(cfg, to_device(w))
    return cfg, w, model, oracle.Model(cfg, w)


def _cache_rows(seqs, cfg, max_ctx, l, a, b):
    K, Vt = kv_views(seqs.kv, cfg, 1, max_ctx)
    kg = K[l, 0, :, a:b].permute(1, 0, 2).float().cpu().numpy()
    vg = Vt[l, 0, :, :, a:b].permute(2, 0, 1).float().cpu().numpy()
    return kg, vg


# Router near-ties.  A token whose k-th and (k+1)-th router logits are within 1e-2 is a legitimate
# near-tie: the GPU may route it either way.  In the last layer the choice only moves that token's own
# output, and the token is left out of the comparison.  In an earlier layer it also moves every other
# row a little (its K/V in the next layer), so instead of leaving the step unjudged the tie is resolved
# the way the GPU resolved it: the token's output of that layer is compared with the oracle's output
# under each of the two routings (the MoE is per token, so the other tokens' choices do not enter);
# it must match exactly one of them, and the oracle step is then recomputed with the GPU's choices.
# Every other row -- and the early-tie token itself -- is judged against that recomputed step with
# the base tolerances.
def _resolve_early_ties(oseq, prm_o, oids, ocommit, r, hg, cfg):
    """The oracle step with every router near-tie before the last layer routed as the GPU routed it.
    Returns (step result, number of resolved tokens, number routed to the (k+1)-th expert)."""
    ties = np.stack([router_tie_tokens(r_l, cfg.top_k, rel=ROUTER_TIE_REL_E2E) for r_l in r["router"]])
    flip = np.zeros((cfg.n_layers, 256), bool)
    cur = r
    resolved = 0
    for l in range(cfg.n_layers - 1):
        if not ties[l].any():
            continue
        alt_flip = flip.copy()
        alt_flip[l] |= ties[l]
        alt = oseq.canvas_step(prm_o, oids, ocommit, want_hidden=True, want_router=True, flip=alt_flip,
                               advance=False)
        for t in np.nonzero(ties[l])[0]:
            d_keep = np.abs(hg[l + 1][t] - cur["hidden"][l + 1][t]).max()
            d_flip = np.abs(hg[l + 1][t] - alt["hidden"][l + 1][t]).max()
            gap = np.abs(alt["hidden"][l + 1][t] - cur["hidden"][l + 1][t]).max()
            assert min(d_keep, d_flip) <= 0.25 * gap, ("near-tie token routed neither way", l, t, d_keep, d_flip)
            flip[l, t] = d_flip < d_keep
            resolved += 1
        if flip[l].any():
            cur = oseq.canvas_step(prm_o, oids, ocommit, want_hidden=True, want_router=True, flip=flip,
                                   advance=False)
    return cur, resolved, int(flip.sum())


def _diagnose(hg, r, l, keep, cfg):
    """The worst rows of a failed hidden-state comparison with their router gaps per layer."""
    err = np.abs(hg[l] - r["hidden"][l]).max(1) / max(np.abs(r["hidden"][l][keep]).max(), 1e-30)
    err[~keep] = 0
    out = []
    for t in np.argsort(-err)[:4]:
        gaps = []
        for ll in range(cfg.n_layers):
            srt = -np.sort(-r["router"][ll][t])
            gaps.append(round(float(srt[cfg.top_k - 1] - srt[cfg.top_k]), 4) if cfg.top_k < cfg.n_exp else None)
        out.append(f"row {t} err {err[t]:.3g} router gaps {gaps}")
    return "; ".join(out)


@pytest.mark.parametrize("top_k,head,router,prompt_len,n_steps,head_impl", [
    (8, "x1", "unit", 128, 4, "pair"), (8, "x1", "unit", 300, 3, "pair"), (8, "x50", "unit", 128, 48, "pair"),
    (8, "x50", "unit", 300, 6, "pair"), (8, "copy", "unit", 128, 48, "pair"),
    (2, "x1", "stated", 128, 48, "pair"),   # the tiny configuration as stated: top-2, head x1, 48-step adaptive run
    (2, "x1", "unit", 128, 12, "pair"), (2, "x50", "unit", 300, 48, "pair"), (2, "copy", "stated", 128, 48, "pair"),
    (8, "x50", "unit", 128, 6, "unfused"), (8, "copy", "unit", 300, 6, "nv128"),
])
def test_canvas_steps_match_oracle(dg, monkeypatch, top_k, head, router, prompt_len, n_steps, head_impl):
    """head_impl: the vocabulary head + sampler of the step as the fused CTA-pair kernel (the default),
    the fused single-CTA kernel with 128 vocabulary rows per tile (DG_HEAD_SAMPLER=128), or the head GEMM
    followed by the sampler kernels (DG_HEAD_SAMPLER=0)."""
    monkeypatch.setenv("DG_HEAD_SAMPLER", {"pair": "2", "nv128": "128", "unfused": "0"}[head_impl])
    cfg, w, model, M = _tiny_model_pair(dg, head, top_k=top_k, router=router)
    max_ctx = 1024
    seqs = dg.dg_seqs_create(model, 1, max_ctx)
    prompt = synthetic.make_ids(prompt_len, cfg.vocab, 0)
    dg.dg_prefill(seqs, prompt.cuda(), [prompt_len])
    oseq = oracle.Sequence(M, max_ctx)
    tie = router_tie_tokens(oseq.prefill(prompt.numpy(), want_router=True), cfg.top_k, rel=ROUTER_TIE_REL_E2E)
    for l in range(cfg.n_layers):
        kg, vg = _cache_rows(seqs, cfg, max_ctx, l, 0, prompt_len)
        assert rel_err(kg[~tie], oseq.k[l][:prompt_len][~tie]) <= HIDDEN_TOL, f"prefill K layer {l}"
        assert rel_err(vg[~tie], oseq.v[l][:prompt_len][~tie]) <= HIDDEN_TOL, f"prefill V layer {l}"

    prm = dg.sampler_params(cfg.vocab, seed=0)
    prm_o = oracle.SamplerParams(cfg.vocab, seed=0)
    ids = torch.empty(256, dtype=torch.int32, device="cuda")
    commit = torch.empty(256, dtype=torch.uint8, device="cuda")
    dg.dg_canvas_init(seqs, prm, ids, commit)
    oids, ocommit = oseq.canvas_init(prm_o)
    np.testing.assert_array_equal(ids.cpu().numpy(), oids)          # Philox stream, bit-exact
    assert commit.sum().item() == 0

    H = torch.empty(256, device="cuda")
    stop = torch.empty(1, dtype=torch.int32, device="cuda")
    hidden = torch.empty(cfg.n_layers + 1, 256, cfg.d_model, device="cuda")
    logits = torch.empty(256, cfg.vocab, device="cuda")
    prefix_before = seqs.kv.clone()
    total_judged, steps_judged, commits_seen, resolved_total = 0, 0, 0, 0
    log = []
    for s in range(n_steps):
        # resynchronise: the GPU starts each step from the oracle's state
        ids.copy_(torch.from_numpy(oids))
        commit.copy_(torch.from_numpy(ocommit))
        dg.dg_canvas_step(seqs, prm, ids, commit, H, stop, hidden, logits)
        torch.cuda.synchronize()
        hg = hidden.cpu().numpy()
        r = oseq.canvas_step(prm_o, oids, ocommit, want_hidden=True, want_router=True, advance=False)
        r, resolved, flipped = _resolve_early_ties(oseq, prm_o, oids, ocommit, r, hg, cfg)
        oseq.step += 1
        resolved_total += resolved
        last_tie = router_tie_tokens(r["router"][-1], cfg.top_k, rel=ROUTER_TIE_REL_E2E)   # judged nowhere
        keep = ~last_tie
        for l in range(cfg.n_layers + 1):
            e = rel_err(hg[l][keep], r["hidden"][l][keep])
            assert e <= HIDDEN_TOL, f"step {s} hidden {l} rel err {e}: " + _diagnose(hg, r, l, keep, cfg)
        lg = logits.cpu().numpy()
        el = rel_err(lg[keep], r["logits"][keep])
        assert el <= HIDDEN_TOL, f"step {s} logits rel err {el}"
        g = {"ids": ids.cpu().numpy(), "commit": commit.cpu().numpy(), "H": H.cpu().numpy(), "stop": int(stop.item())}
        mt, ht = derived_tolerances(r["logits"], r["T"], cfg.n_layers) if head == "x50" else (None, None)
        fails, judged = judge_step(g, r, prm_o, ocommit, exclude=last_tie, margin_tol=mt, h_tol=ht)
        assert not fails, (s, fails[:10])
        total_judged += judged
        steps_judged += 1
        new_commits = int(r["commit"].sum() - ocommit.sum())
        commits_seen += new_commits
        log.append((s, new_commits, judged, resolved, flipped, int(last_tie.sum())))
        oids, ocommit = r["ids"], r["commit"]
        if r["stop"]:
            break
    print(f"[{top_k=} {head=} {router=} P={prompt_len}] per step (step, commits, ids judged, early near-ties resolved, "
          f"of them routed to the (k+1)-th expert, last-layer near-ties) {log}")
    assert steps_judged > 0 and total_judged > 0, (steps_judged, total_judged, log)
    if top_k < cfg.n_exp and router == "stated":
        assert resolved_total > 0, log          # early near-ties are frequent here: they were resolved and judged
    if head != "x1":
        assert commits_seen > 0
    # the committed prefix [0, P) is untouched by canvas steps
    P = prompt_len
    K, Vt = kv_views(seqs.kv, cfg, 1, max_ctx)
    Kb, Vb = kv_views(prefix_before, cfg, 1, max_ctx)
    assert torch.equal(K[:, :, :, :P], Kb[:, :, :, :P]) and torch.equal(Vt[..., :P], Vb[..., :P])
    # block commit of the final ids: cache rows [P, P+256) hold the K/V of a canvas forward
    ids.copy_(torch.from_numpy(oids))
    dg.dg_block_commit(seqs, ids)
    tie = router_tie_tokens(oseq.block_commit(oids, want_router=True), cfg.top_k, rel=ROUTER_TIE_REL_E2E)
    torch.cuda.synchronize()
    Pn, _ = dg.dg_seqs_get_state(seqs)
    assert Pn[0] == P + 256 == oseq.P
    for l in range(cfg.n_layers):
        kg, vg = _cache_rows(seqs, cfg, max_ctx, l, P, P + 256)
        assert rel_err(kg[~tie], oseq.k[l][P:P + 256][~tie]) <= HIDDEN_TOL
        assert rel_err(vg[~tie], oseq.v[l][P:P + 256][~tie]) <= HIDDEN_TOL
    assert dg.dg_device_error(seqs) == 0


def test_canvas_step_without_prompt_and_determinism(dg):
    cfg, w, model, M = _tiny_model_pair(dg, 50.0, seed=4, top_k=8)
    seqs = dg.dg_seqs_create(model, 1, 512)
    prm = dg.sampler_params(cfg.vocab, seed=9, fixed_steps=2)
    outs = []
    for rep in range(2):
        ids = torch.empty(256, dtype=torch.int32, device="cuda")
        commit = torch.empty(256, dtype=torch.uint8, device="cuda")
        H = torch.empty(256, device="cuda")
        stop = torch.empty(1, dtype=torch.int32, device="cuda")
        dg.dg_canvas_init(seqs, prm, ids, commit)
        for s in range(2):
            dg.dg_canvas_step(seqs, prm, ids, commit, H, stop)
        outs.append((ids.cpu(), commit.cpu(), H.cpu(), stop.cpu()))
        with pytest.raises(dg.DGError) as ei:                    # budget used: state error, no launch
            dg.dg_canvas_step(seqs, prm, ids, commit, H, stop)
        assert ei.value.status == dg.DG_ERR_STATE
    for a, b in zip(outs[0], outs[1]):
        assert torch.equal(a, b)                                 # bit-identical reruns
    assert outs[0][3].item() == 1 and outs[0][1].all()           # fixed budget reached: all committed


def test_decode_equals_the_step_sequence(dg):
    """dg_decode is the loop init -> steps until stop -> commit, per block: its output is
    bit-identical to driving the same calls one by one (each of which is checked against the oracle
    above), and its bookkeeping (counts, P, EOS cut) follows the loop's rules."""
    cfg, w, model, M = _tiny_model_pair(dg, 50.0, seed=1, top_k=8)
    max_ctx = 1024
    prompt = synthetic.make_ids(128, cfg.vocab, 1).cuda()
    prm = dg.sampler_params(cfg.vocab, seed=5)                    # adaptive stop
    s1 = dg.dg_seqs_create(model, 1, max_ctx)
    dg.dg_prefill(s1, prompt, [128])
    out = torch.full((1, 3 * 256), -1, dtype=torch.int32, device="cuda")
    n_out, steps = dg.dg_decode(s1, prm, 3, out)
    assert n_out == [768] and all(1 <= k <= 48 for k in steps)
    assert dg.dg_seqs_get_state(s1)[0] == [128 + 768]
    s2 = dg.dg_seqs_create(model, 1, max_ctx)
    dg.dg_prefill(s2, prompt, [128])
    ids = torch.empty(256, dtype=torch.int32, device="cuda")
    commit = torch.empty(256, dtype=torch.uint8, device="cuda")
    H = torch.empty(256, device="cuda")
    stop = torch.empty(1, dtype=torch.int32, device="cuda")
    manual = []
    for b in range(3):
        dg.dg_canvas_init(s2, prm, ids, commit)
        k = 0
        while True:
            dg.dg_canvas_step(s2, prm, ids, commit, H, stop)
            k += 1
            if stop.item():
                break
        assert k == steps[b]
        assert commit.cpu().bool().all()
        dg.dg_block_commit(s2, ids)
        manual.append(ids.cpu().clone())
    assert torch.equal(out.cpu()[0], torch.cat(manual))
    # EOS: the first EOS of a block ends the sequence; output cut after it
    eos = int(manual[1][17])
    first = int(torch.nonzero(torch.cat(manual) == eos)[0])
    s3 = dg.dg_seqs_create(model, 1, max_ctx)
    dg.dg_prefill(s3, prompt, [128])
    out3 = torch.full((1, 3 * 256), -1, dtype=torch.int32, device="cuda")
    n3, steps3 = dg.dg_decode(s3, dg.sampler_params(cfg.vocab, seed=5, eos_id=eos), 3, out3)
    assert n3 == [first + 1]
    assert len([x for x in steps3 if x]) == first // 256 + 1


def _oracle_block_with_safety(oseq, prm_o):
    """One block of the oracle's decode loop (init, steps until stop).  Returns (ids, steps, unsafe):
    unsafe counts the decisions of the block that the judging rules leave open (an id taken from the
    Gumbel-argmax with a top-2 margin <= 1e-2, an entropy within 1e-3 of the commit or re-randomise
    threshold, a canvas-mean entropy within 1e-3 of the stop threshold)."""
    ids, commit = oseq.canvas_init(prm_o)
    unsafe, steps = 0, 0
    while True:
        r = oseq.canvas_step(prm_o, ids, commit)
        steps += 1
        unc = commit == 0
        takes_y = unc & ((r["commit"] == 1) | (r["H"] <= prm_o.rerand_entropy) | bool(r["stop"]))
        bad = takes_y & (r["margin"] <= MARGIN)
        bad |= unc & (np.abs(r["H"] - prm_o.entropy_bound) <= 1e-3)
        bad |= unc & (np.abs(r["H"] - prm_o.rerand_entropy) <= 1e-3)
        unsafe += int(bad.sum()) + int(abs(r["mean_H"] - prm_o.stop_mean_entropy) <= 1e-3)
        ids, commit = r["ids"], r["commit"]
        if r["stop"]:
            return ids, steps, unsafe


def test_decode_matches_oracle_decode(dg):
    """dg_decode (one call, two blocks, adaptive stop) against the oracle's decode loop on the same
    model, prompt and seed.  A block whose every decision the judging rules fix (no near-tie) must
    come out bit for bit equal, with the same step count; a block with an open decision may differ,
    and the oracle then commits the GPU's ids so that the next block starts from the same tokens.
    The copy head makes rows commit over several steps (every block here is decided in full).  Then
    an EOS id from the output: dg_decode must cut exactly where oracle.Sequence.decode cuts."""
    cfg, w, model, M = _tiny_model_pair(dg, "copy", seed=0, top_k=8)
    max_ctx = 768
    prompt = synthetic.make_ids(128, cfg.vocab, 1)
    prm = dg.sampler_params(cfg.vocab, seed=1)
    prm_o = oracle.SamplerParams(cfg.vocab, seed=1)
    seqs = dg.dg_seqs_create(model, 1, max_ctx)
    dg.dg_prefill(seqs, prompt.cuda(), [128])
    out = torch.full((1, 2 * 256), -1, dtype=torch.int32, device="cuda")
    n_out, steps = dg.dg_decode(seqs, prm, 2, out)
    assert n_out == [512]
    assert dg.dg_device_error(seqs) == 0
    gout = out.cpu().numpy()[0]
    oseq = oracle.Sequence(M, max_ctx)
    oseq.prefill(prompt.numpy())
    decided = 0
    for b in range(2):
        oids, osteps, unsafe = _oracle_block_with_safety(oseq, prm_o)
        g = gout[256 * b: 256 * (b + 1)]
        if unsafe == 0:
            decided += 1
            assert steps[b] == osteps, (b, steps[b], osteps)
            np.testing.assert_array_equal(g, oids)
        oseq.block_commit(g)                                  # resynchronise on the GPU's tokens
    assert decided == 2, decided
    # EOS: the first EOS of a block ends the sequence, output cut after it -- where the oracle's decode
    # loop (same computations up to that block) cuts
    eos = int(gout[256 + 17])
    first = int(np.nonzero(gout == eos)[0][0])
    prm_e = dg.sampler_params(cfg.vocab, seed=1, eos_id=eos)
    s2 = dg.dg_seqs_create(model, 1, max_ctx)
    dg.dg_prefill(s2, prompt.cuda(), [128])
    out2 = torch.full((1, 2 * 256), -1, dtype=torch.int32, device="cuda")
    n2, steps2 = dg.dg_decode(s2, prm_e, 2, out2)
    assert n2 == [first + 1]
    np.testing.assert_array_equal(out2.cpu().numpy()[0][: first + 1], gout[: first + 1])
    assert steps2[: first // 256 + 1] == steps[: first // 256 + 1]


@pytest.mark.parametrize("n_seq,commit_mode,fixed", [(1, 0, 0), (2, 0, 0), (1, 1, 5)])
def test_decode_loop_on_the_device_equals_the_host_loop(dg, monkeypatch, n_seq, commit_mode, fixed):
    """dg_decode's device-resident block loop (a CUDA graph whose while-node repeats the step body
    until the stop flags end it; step index and temperature on the device) gives the same tokens and
    step counts as the host loop that reads the stop flags after every step (DG_DECODE_GRAPH=0)."""
    cfg, w, model, M = _tiny_model_pair(dg, "copy", seed=3, top_k=8)
    prompt = synthetic.make_ids(128 * n_seq, cfg.vocab, 3).cuda()
    prm = dg.sampler_params(cfg.vocab, seed=3, commit_mode=commit_mode, fixed_steps=fixed)
    outs = []
    for graph in ("1", "0"):
        monkeypatch.setenv("DG_DECODE_GRAPH", graph)
        seqs = dg.dg_seqs_create(model, n_seq, 1024)
        dg.dg_prefill(seqs, prompt, [128] * n_seq)
        out = torch.full((n_seq, 3 * 256), -1, dtype=torch.int32, device="cuda")
        n_out, steps = dg.dg_decode(seqs, prm, 3, out)
        assert dg.dg_device_error(seqs) == 0
        outs.append((out.cpu(), n_out, steps, dg.dg_seqs_get_state(seqs)[0], seqs.kv.clone()))
    assert torch.equal(outs[0][0], outs[1][0])
    assert outs[0][1] == outs[1][1] == [768] * n_seq
    assert outs[0][2] == outs[1][2] and all(1 <= k <= 48 for k in outs[0][2]), (outs[0][2], outs[1][2])
    if fixed:
        assert outs[0][2] == [fixed] * 3
    assert outs[0][3] == outs[1][3]
    assert torch.equal(outs[0][4], outs[1][4])                      # the caches hold the same K/V


def test_commit_keeping_the_last_steps_kv(dg):
    """dg_block_commit_last_kv: the cache rows of the block keep the K/V of the ids the last step
    read (the oracle's commit pass over those ids), the prefix is untouched, P advances; dg_decode
    with commit_mode 1 equals the same calls made one by one; a commit before any step is a state
    error."""
    cfg, w, model, M = _tiny_model_pair(dg, 50.0, seed=2, top_k=8)
    max_ctx = 1024
    prompt = synthetic.make_ids(128, cfg.vocab, 2)
    prm = dg.sampler_params(cfg.vocab, seed=6, fixed_steps=3)
    seqs = dg.dg_seqs_create(model, 1, max_ctx)
    dg.dg_prefill(seqs, prompt.cuda(), [128])
    ids = torch.empty(256, dtype=torch.int32, device="cuda")
    commit = torch.empty(256, dtype=torch.uint8, device="cuda")
    H = torch.empty(256, device="cuda")
    stop = torch.empty(1, dtype=torch.int32, device="cuda")
    dg.dg_canvas_init(seqs, prm, ids, commit)
    with pytest.raises(dg.DGError) as ei:
        dg.dg_block_commit_last_kv(seqs)
    assert ei.value.status == dg.DG_ERR_STATE
    for _ in range(3):
        last_in = ids.cpu().clone()
        dg.dg_canvas_step(seqs, prm, ids, commit, H, stop)
    before = seqs.kv.clone()
    dg.dg_block_commit_last_kv(seqs)
    torch.cuda.synchronize()
    assert dg.dg_seqs_get_state(seqs)[0] == [128 + 256]
    assert torch.equal(seqs.kv, before)                        # nothing recomputed or moved
    oseq = oracle.Sequence(M, max_ctx)
    oseq.prefill(prompt.numpy())
    oseq.block_commit(last_in.numpy())
    for l in range(cfg.n_layers):
        kg, vg = _cache_rows(seqs, cfg, max_ctx, l, 128, 384)
        assert rel_err(kg, oseq.k[l][128:384]) <= HIDDEN_TOL and rel_err(vg, oseq.v[l][128:384]) <= HIDDEN_TOL
        kp, vp = _cache_rows(seqs, cfg, max_ctx, l, 0, 128)
        assert rel_err(kp, oseq.k[l][:128]) <= HIDDEN_TOL
    # dg_decode with commit_mode 1 is the loop with this commit
    prm1 = dg.sampler_params(cfg.vocab, seed=6, fixed_steps=3, commit_mode=1)
    s1 = dg.dg_seqs_create(model, 1, max_ctx)
    dg.dg_prefill(s1, prompt.cuda(), [128])
    out = torch.full((1, 2 * 256), -1, dtype=torch.int32, device="cuda")
    n_out, steps = dg.dg_decode(s1, prm1, 2, out)
    assert n_out == [512] and steps == [3, 3]
    s2 = dg.dg_seqs_create(model, 1, max_ctx)
    dg.dg_prefill(s2, prompt.cuda(), [128])
    manual = []
    for b in range(2):
        dg.dg_canvas_init(s2, prm1, ids, commit)
        for _ in range(3):
            dg.dg_canvas_step(s2, prm1, ids, commit, H, stop)
        dg.dg_block_commit_last_kv(s2)
        manual.append(ids.cpu().clone())
    assert torch.equal(out.cpu()[0], torch.cat(manual))
    assert torch.equal(s1.kv, s2.kv)
    assert dg.dg_device_error(s1) == 0 and dg.dg_device_error(s2) == 0


def test_capacity_and_argument_errors(dg):
    cfg, w, model, M = _tiny_model_pair(dg)
    seqs = dg.dg_seqs_create(model, 1, 256)
    prm = dg.sampler_params(cfg.vocab)
    ids = torch.zeros(256, dtype=torch.int32, device="cuda")
    with pytest.raises(dg.DGError) as ei:
        dg.dg_prefill(seqs, ids, [10])            # 10 + 256 > 256
    assert ei.value.status == dg.DG_ERR_CAPACITY
    commit = torch.zeros(256, dtype=torch.uint8, device="cuda")
    dg.dg_canvas_init(seqs, prm, ids, commit)
    dg.dg_block_commit(seqs, ids)
    with pytest.raises(dg.DGError) as ei:
        dg.dg_block_commit(seqs, ids)             # cache full
    assert ei.value.status == dg.DG_ERR_CAPACITY
    bad = dg.sampler_params(cfg.vocab, canvas_len=128)
    seqs2 = dg.dg_seqs_create(model, 1, 512)
    with pytest.raises(dg.DGError) as ei:
        dg.dg_canvas_init(seqs2, bad, ids, commit)
    assert ei.value.status == dg.DG_ERR_UNSUPPORTED
    # an out-of-range id is recorded as a device-side error, not a fault
    ids_bad = torch.full((256,), cfg.vocab + 5, dtype=torch.int32, device="cuda")
    dg.dg_canvas_init(seqs2, prm, ids, commit)
    H = torch.empty(256, device="cuda")
    stop = torch.empty(1, dtype=torch.int32, device="cuda")
    dg.dg_canvas_step(seqs2, prm, ids_bad, commit, H, stop)
    assert dg.dg_device_error(seqs2) != 0
    assert dg.dg_device_error(seqs2) == 0         # the record is cleared by reading it


def test_block_replays_bit_identically_from_a_cuda_graph(dg):
    """The library issues only stream-ordered work on the sequence set's stream (no host reads,
    allocations or synchronisation inside a step), so a whole block -- canvas init and its fixed
    steps -- can be captured into a CUDA graph (the programmatic dependent launches become
    programmatic edges) and replayed with the same results as the direct calls."""
    cfg, w, model, M = _tiny_model_pair(dg, 50.0, seed=4, top_k=2)
    s = torch.cuda.Stream()
    seqs = dg.dg_seqs_create(model, 1, 512, stream=s)
    prm = dg.sampler_params(cfg.vocab, seed=11, fixed_steps=6)
    prompt = synthetic.make_ids(128, cfg.vocab, seed=5, device="cuda")
    ids = torch.empty(256, dtype=torch.int32, device="cuda")
    commit = torch.empty(256, dtype=torch.uint8, device="cuda")
    H = torch.empty(256, device="cuda")
    stop = torch.empty(1, dtype=torch.int32, device="cuda")

    def block():
        dg.dg_canvas_init(seqs, prm, ids, commit)
        for _ in range(6):
            dg.dg_canvas_step(seqs, prm, ids, commit, H, stop)

    with torch.cuda.stream(s):
        dg.dg_prefill(seqs, prompt, [128])
        block()
    torch.cuda.synchronize()
    direct = (ids.clone(), commit.clone(), H.clone(), stop.clone())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        block()
    for t in (ids, commit, H, stop):
        t.zero_()
    torch.cuda.synchronize()
    for _ in range(2):
        with torch.cuda.stream(s):
            g.replay()
        torch.cuda.synchronize()
        for a, b in zip((ids, commit, H, stop), direct):
            assert torch.equal(a, b)
    assert dg.dg_device_error(seqs) == 0
    del g
