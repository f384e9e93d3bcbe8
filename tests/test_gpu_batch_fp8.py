"""Several sequences in one call, and the FP8 block-scaled weight form, against the oracle.

Every sequence of a batch is independent: sequence i has its own prompt, its own committed length
and the sampler stream of seed + i, so each one is compared with its own oracle sequence.  With FP8
weights (e4m3 bytes, one fp32 scale per 128 x 128 tile) the oracle multiplies with the exact q * s
and the hidden-state tolerance is 6e-2.  Marked gpu.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import synthetic
from dg_testutil import (HIDDEN_TOL, HIDDEN_TOL_FP8, derived_tolerances, judge_step, kv_views, rel_err,
                         router_tie_tokens, to_device)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dg(cuda_ok):
    from block_discrete_diffusion_b200 import build, dg as dgmod
    build.build()
    return dgmod


def _tiny(wdtype, head_scale=50.0, seed=0):
    cfg = dataclasses.replace(synthetic.TINY, top_k=8, wdtype=wdtype)    # top_k = E: no routing decision
    w = synthetic.make_model_weights(cfg, seed, head_scale=head_scale)
    return cfg, w


@pytest.mark.parametrize("wdtype,head_scale", [(0, 50.0), (1, 50.0), (1, 1.0)])
def test_batched_sequences_match_their_oracles(dg, wdtype, head_scale):
    """Three sequences (prompts of 128, 300 and 0 tokens) prefilled, initialised and stepped in one
    batch; each sequence's hidden states, logits and sampler decisions match its own oracle run
    (resynchronised every step), then one block commit per sequence.  Head x50: rows commit, ids and
    entropies judged with the derived large-logit tolerances; head x1: the base tolerances."""
    cfg, w = _tiny(wdtype, head_scale)
    tol = HIDDEN_TOL if wdtype == 0 else HIDDEN_TOL_FP8
    model = dg.dg_model_create(cfg, to_device(w))
    M = oracle.Model(cfg, w)
    lens = [128, 300, 0]
    n = len(lens)
    max_ctx = 1024
    seqs = dg.dg_seqs_create(model, n, max_ctx)
    prompts = [synthetic.make_ids(L, cfg.vocab, 10 + i) for i, L in enumerate(lens)]
    dg.dg_prefill(seqs, torch.cat(prompts).cuda(), lens)
    oseqs = [oracle.Sequence(M, max_ctx) for _ in range(n)]
    for i in range(n):
        if lens[i]:
            oseqs[i].prefill(prompts[i].numpy())
    K, Vt = kv_views(seqs.kv, cfg, n, max_ctx)
    for i in range(n):
        for l in range(cfg.n_layers):
            if lens[i]:
                kg = K[l, i, :, :lens[i]].permute(1, 0, 2).float().cpu().numpy()
                assert rel_err(kg, oseqs[i].k[l][:lens[i]]) <= tol, (i, l)
    Pn, _ = dg.dg_seqs_get_state(seqs)
    assert list(Pn) == lens

    seed = 5
    prm = dg.sampler_params(cfg.vocab, seed=seed)
    prm_o = [oracle.SamplerParams(cfg.vocab, seed=seed + i) for i in range(n)]
    ids = torch.empty(n, 256, dtype=torch.int32, device="cuda")
    commit = torch.empty(n, 256, dtype=torch.uint8, device="cuda")
    dg.dg_canvas_init(seqs, prm, ids, commit)
    st = [oseqs[i].canvas_init(prm_o[i]) for i in range(n)]
    for i in range(n):
        np.testing.assert_array_equal(ids[i].cpu().numpy(), st[i][0])    # stream of seed + i, bit-exact

    H = torch.empty(n, 256, device="cuda")
    stop = torch.empty(n, dtype=torch.int32, device="cuda")
    hidden = torch.empty(cfg.n_layers + 1, n * 256, cfg.d_model, device="cuda")
    logits = torch.empty(n * 256, cfg.vocab, device="cuda")
    stopped = [False] * n
    judged = 0
    for s in range(8):
        for i in range(n):
            ids[i].copy_(torch.from_numpy(st[i][0]))
            commit[i].copy_(torch.from_numpy(st[i][1]))
        dg.dg_canvas_step(seqs, prm, ids, commit, H, stop, hidden, logits)
        torch.cuda.synchronize()
        hg, lg = hidden.cpu().numpy(), logits.cpu().numpy()
        for i in range(n):
            r = oseqs[i].canvas_step(prm_o[i], st[i][0], st[i][1], want_hidden=True)
            rows = slice(256 * i, 256 * (i + 1))
            if not stopped[i]:
                for l in range(cfg.n_layers + 1):
                    e = rel_err(hg[l][rows], r["hidden"][l])
                    assert e <= tol, f"step {s} seq {i} hidden {l} rel err {e}"
                assert rel_err(lg[rows], r["logits"]) <= tol, (s, i)
                if head_scale == 1.0:
                    mt, ht = None, None
                else:
                    mt, ht = derived_tolerances(r["logits"], r["T"], cfg.n_layers, fp8=wdtype == 1)
                g = {"ids": ids[i].cpu().numpy(), "commit": commit[i].cpu().numpy(), "H": H[i].cpu().numpy(),
                     "stop": int(stop[i].item())}
                fails, j = judge_step(g, r, prm_o[i], st[i][1], margin_tol=mt, h_tol=ht)
                assert not fails, (s, i, fails[:8])
                judged += j
            else:                                                   # a stopped canvas stays as it is
                assert (commit[i].cpu().numpy() == 1).all()
                np.testing.assert_array_equal(ids[i].cpu().numpy(), st[i][0])
            st[i] = (r["ids"], r["commit"])
            stopped[i] = stopped[i] or bool(r["stop"])
        if all(stopped):
            break
    assert judged > 0

    final = torch.from_numpy(np.stack([st[i][0] for i in range(n)])).cuda()
    dg.dg_block_commit(seqs, final)
    for i in range(n):
        oseqs[i].block_commit(st[i][0])
    torch.cuda.synchronize()
    Pn, _ = dg.dg_seqs_get_state(seqs)
    assert [p for p in Pn] == [L + 256 for L in lens]
    K, Vt = kv_views(seqs.kv, cfg, n, max_ctx)
    for i in range(n):
        P = lens[i]
        for l in range(cfg.n_layers):
            kg = K[l, i, :, P:P + 256].permute(1, 0, 2).float().cpu().numpy()
            vg = Vt[l, i, :, :, P:P + 256].permute(2, 0, 1).float().cpu().numpy()
            assert rel_err(kg, oseqs[i].k[l][P:P + 256]) <= tol and rel_err(vg, oseqs[i].v[l][P:P + 256]) <= tol
    assert dg.dg_device_error(seqs) == 0


def _layer_sequences(dg, cfg, n_seq, prefix_lens, seed, check):
    """One full-width FP8 layer on n_seq canvases with prefixes of the given lengths; the
    sequences in `check` are compared with the oracle."""
    w = synthetic.make_model_weights(cfg, seed, device="cuda", router_std=cfg.d_model ** -0.5)
    model = dg.dg_model_create(cfg, w)
    max_ctx = ((max(prefix_lens) + 256 + 255) // 256) * 256
    seqs = dg.dg_seqs_create(model, n_seq, max_ctx)
    kept = {}
    for i, P in enumerate(prefix_lens):
        if P:
            ks, vs = synthetic.make_prefix_kv(1, P, cfg.n_kv, cfg.d_head, seed + 100 + i, device="cuda")
            dg.dg_load_prefix(seqs, i, P, ks, vs)
            if i in check:
                kept[i] = (ks[0].double().cpu().numpy(), vs[0].double().cpu().numpy())
            del ks, vs
    x = synthetic.make_hidden(n_seq * 256, cfg.d_model, seed + 1, device="cuda")
    xd = x.clone()
    mid = torch.zeros_like(xd)
    rl = torch.zeros(n_seq * 256, cfg.n_exp, device="cuda")
    dg.dg_layer_forward(seqs, 0, xd, mid, rl)
    torch.cuda.synchronize()
    assert dg.dg_device_error(seqs) == 0
    wc = {"layers": [{k: ({a: b.cpu() for a, b in v.items()} if isinstance(v, dict) else v.cpu())
                      for k, v in w["layers"][0].items()}]}
    M = oracle.Model(cfg, wc, layers=wc["layers"])
    for i in check:
        P = prefix_lens[i]
        rows = slice(256 * i, 256 * (i + 1))
        kc, vc = kept.get(i, (None, None))
        xo, kn, vn, rlo, mido = oracle.layer_forward(M, 0, x[rows].double().cpu().numpy(), np.arange(P, P + 256), P,
                                                     kc, vc, want_mid=True)
        assert rel_err(mid[rows].cpu().numpy(), mido) <= HIDDEN_TOL_FP8, ("attention block", i)
        assert rel_err(rl[rows].cpu().numpy(), rlo) <= HIDDEN_TOL_FP8, ("router logits", i)
        keep = ~router_tie_tokens(rlo, cfg.top_k)
        e = rel_err(xd[rows].cpu().numpy()[keep], xo[keep])
        assert e <= HIDDEN_TOL_FP8, ("layer output", i, e, int(keep.sum()))
        K, Vt = kv_views(seqs.kv, cfg, n_seq, max_ctx)
        kg = K[0, i, :, P:P + 256].permute(1, 0, 2).float().cpu().numpy()
        assert rel_err(kg, kn) <= HIDDEN_TOL_FP8
    return seqs


def test_fp8_full_width_layer_four_sequences(dg):
    """The full-width layer (d 2816, 128 experts top-8) with FP8 weights on four canvases whose
    prefixes differ (4096, 1000, 0 and 2048 positions)."""
    cfg = dataclasses.replace(synthetic.ONE_LAYER, vocab=1024, wdtype=1)
    _layer_sequences(dg, cfg, 4, [4096, 1000, 0, 2048], 21, check=[0, 1, 2, 3])


def test_fp8_layer_32_sequences_of_32k_prefix(dg):
    """The largest batch shape: 32 canvases, each behind a 32768-position prefix (FP8 weights, one
    full-width layer); the first and the last sequence are compared with the oracle."""
    cfg = dataclasses.replace(synthetic.ONE_LAYER, vocab=1024, wdtype=1)
    _layer_sequences(dg, cfg, 32, [32768] * 32, 31, check=[0, 31])
