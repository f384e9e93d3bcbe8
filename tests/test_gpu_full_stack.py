"""The 30-layer benchmark model (d 2816, 128 experts top-8, vocabulary 262144, bf16, residual-scaled
random init, random RMSNorm gains) against the oracle, through one whole dg_canvas_step.

The step runs on the GPU behind a 2048-token prompt that dg_prefill put into the cache (the
benchmark's configuration), with the residual stream of every layer and the logits copied out.  Then
each piece is judged from the GPU's own input to it, so that a router near-tie in one layer cannot
carry into the next:
  - every layer: the oracle's layer on the GPU's hidden state before it (and on the GPU's prompt
    cache) against the GPU's hidden state after it -- this is the fused path of the step, where the
    previous kernel applies the next norm's gain -- and against dg_layer_forward on the same input
    (the unfused path); the canvas K/V of the layer as well;
  - the 262144-wide vocabulary head on sampled rows: the oracle's final RMSNorm + head on the GPU's
    last hidden state against the GPU's logits;
  - the sampler on the GPU's logits: the oracle's entropies, Gumbel-argmax and step rule on the same
    fp32 logits, judged with the base tolerances.
Tokens with a router near-tie in a layer are excluded from that layer's comparison.  Marked gpu.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import synthetic
from dg_testutil import HIDDEN_TOL, judge_step, kv_views, rel_err, router_tie_tokens

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dg(cuda_ok):
    from block_discrete_diffusion_b200 import build, dg as dgmod
    build.build()
    return dgmod


def _host(t):
    return {k: v.cpu() for k, v in t.items()} if isinstance(t, dict) else t.cpu()


def test_full_stack_canvas_step_matches_oracle(dg):
    cfg = synthetic.FULL
    P = 2048
    w = synthetic.make_model_weights(cfg, 2, device="cuda", gain_std=0.1, **synthetic.full_stack_init(cfg))
    model = dg.dg_model_create(cfg, w)
    max_ctx = P + 256
    seqs = dg.dg_seqs_create(model, 1, max_ctx)
    prompt = synthetic.make_ids(P, cfg.vocab, 2)
    dg.dg_prefill(seqs, prompt.cuda(), [P])
    # re-randomisation off (threshold above ln V): every row's id is the Gumbel-argmax of its logits
    prm = dg.sampler_params(cfg.vocab, seed=2, fixed_steps=12, rerand_entropy=1e9)
    ids = torch.empty(256, dtype=torch.int32, device="cuda")
    commit = torch.empty(256, dtype=torch.uint8, device="cuda")
    H = torch.empty(256, device="cuda")
    stop = torch.empty(1, dtype=torch.int32, device="cuda")
    hidden = torch.empty(cfg.n_layers + 1, 256, cfg.d_model, device="cuda")
    logits = torch.empty(256, cfg.vocab, device="cuda")
    dg.dg_canvas_init(seqs, prm, ids, commit)
    ids0 = ids.cpu().numpy().copy()
    dg.dg_canvas_step(seqs, prm, ids, commit, H, stop, hidden, logits)
    torch.cuda.synchronize()
    assert dg.dg_device_error(seqs) == 0
    np.testing.assert_array_equal(ids0, oracle.canvas_init(256, P, 2, cfg.vocab)[0])   # Philox, bit-exact

    hg = hidden.cpu().numpy().astype(np.float64)
    Me = oracle.Model(cfg, {"emb": w["emb"].cpu()}, layers=[])
    np.testing.assert_allclose(hg[0], oracle.embed(Me, ids0), rtol=0, atol=0)   # the embedding rows, exact
    del Me
    K, Vt = kv_views(seqs.kv, cfg, 1, max_ctx)
    pos = np.arange(P, P + 256)
    c1 = dataclasses.replace(cfg, n_layers=1)
    judged_min = 256
    for l in range(cfg.n_layers):
        L = {k: _host(v) for k, v in w["layers"][l].items()}
        M = oracle.Model(c1, {"layers": [L]}, layers=[L])
        kc = K[l, 0, :, :P].permute(1, 0, 2).double().cpu().numpy()
        vc = Vt[l, 0, :, :, :P].permute(2, 0, 1).double().cpu().numpy()
        xo, kn, vn, rlo, mido = oracle.layer_forward(M, 0, hg[l], pos, P, kc, vc, want_mid=True)
        keep = ~router_tie_tokens(rlo, cfg.top_k)
        # fused path of the step: layer l's output and its canvas K/V
        e_step = rel_err(hg[l + 1][keep], xo[keep])
        kg = K[l, 0, :, P:P + 256].permute(1, 0, 2).float().cpu().numpy()
        vg = Vt[l, 0, :, :, P:P + 256].permute(2, 0, 1).float().cpu().numpy()
        assert e_step <= HIDDEN_TOL, ("canvas step, layer", l, e_step, int(keep.sum()))
        assert rel_err(kg, kn) <= HIDDEN_TOL and rel_err(vg, vn) <= HIDDEN_TOL, ("canvas step K/V", l)
        # unfused path: dg_layer_forward from the same input
        xd = hidden[l].clone()
        mid = torch.zeros_like(xd)
        rl = torch.zeros(256, cfg.n_exp, device="cuda")
        dg.dg_layer_forward(seqs, l, xd, mid, rl)
        torch.cuda.synchronize()
        assert rel_err(mid.cpu().numpy(), mido) <= HIDDEN_TOL, ("layer forward, attention block", l)
        assert rel_err(rl.cpu().numpy(), rlo) <= HIDDEN_TOL, ("layer forward, router logits", l)
        e_lf = rel_err(xd.cpu().numpy()[keep], xo[keep])
        assert e_lf <= HIDDEN_TOL, ("layer forward, output", l, e_lf)
        judged_min = min(judged_min, int(keep.sum()))
    assert judged_min >= 128

    # vocabulary head on sampled rows (final RMSNorm with its gain, then the 262144-wide projection)
    rows = np.array([0, 37, 101, 128, 200, 255])
    Mh = oracle.Model(cfg, {"layers": [], "head": w["head"].cpu(), "final_norm": w["final_norm"].cpu()}, layers=[])
    lo = oracle.head(Mh, hg[cfg.n_layers][rows])
    lg = logits.cpu().numpy()
    e_head = rel_err(lg[rows], lo)
    assert e_head <= HIDDEN_TOL, ("head logits", e_head)

    # sampler on the GPU's logits: same fp32 inputs, base tolerances
    prm_o = oracle.SamplerParams(cfg.vocab, seed=2, fixed_steps=12, rerand_entropy=1e9)
    T = oracle.temperature(0)
    smp = oracle.sample_rows(lg, np.zeros(256, np.uint8), pos, T, 2, 0)
    rule = oracle.step_rule(np.zeros(256, np.uint8), ids0, smp["H"], smp["y"], smp["rr"], 0, prm_o.entropy_bound,
                            prm_o.rerand_entropy, prm_o.stop_mean_entropy, prm_o.max_steps, prm_o.fixed_steps)
    orc = dict(smp)
    orc.update(rule)
    orc["step"] = 0
    orc["logits"] = lg
    g = {"ids": ids.cpu().numpy(), "commit": commit.cpu().numpy(), "H": H.cpu().numpy(), "stop": int(stop.item())}
    fails, judged = judge_step(g, orc, prm_o, np.zeros(256, np.uint8))
    assert not fails, fails[:10]
    assert judged >= 240, judged
    print(f"full stack: {judged_min}+ tokens judged per layer, head rel err {e_head:.2e}, {judged} ids judged")
