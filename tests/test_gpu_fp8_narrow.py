"""The FP8 form with e4m3 activations on the tiny model end to end (one sequence: prefill, canvas
steps resynchronised to the oracle, block commit), through the expert GEMMs that multiply e4m3 by
e4m3 with per-slice scale promotion.  The tiny model routes hundreds of tokens to each of its 8
experts, which would select the wide-chunk path; DG_EXPERT_WIDE=0 (read once per process, so this
file runs in a child process) keeps the 32-token chunks of the batch-1 path.  Hidden states within
6e-2 (the FP8 tolerance: weights q * s exactly in the oracle, activations quantized per 128 channels
and 64 features on the GPU only); the sampler on the GPU's logits with the base tolerances.  Marked gpu.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import dataclasses, sys
import numpy as np, torch
sys.path.insert(0, ROOT); sys.path.insert(0, ROOT + "/tests")
import oracle, synthetic
from block_discrete_diffusion_b200 import build, dg
from dg_testutil import HIDDEN_TOL_FP8, judge_step, kv_views, rel_err, router_tie_tokens, to_device
build.build()
cfg = dataclasses.replace(synthetic.TINY, top_k=8, wdtype=1)
w = synthetic.make_model_weights(cfg, 5, gain_std=0.1)
model = dg.dg_model_create(cfg, to_device(w))
M = oracle.Model(cfg, w)
seqs = dg.dg_seqs_create(model, 1, 1024)
prompt = synthetic.make_ids(200, cfg.vocab, 5)
dg.dg_prefill(seqs, prompt.cuda(), [200])
oseq = oracle.Sequence(M, 1024)
oseq.prefill(prompt.numpy())
K, Vt = kv_views(seqs.kv, cfg, 1, 1024)
for l in range(cfg.n_layers):
    kg = K[l, 0, :, :200].permute(1, 0, 2).float().cpu().numpy()
    assert rel_err(kg, oseq.k[l][:200]) <= HIDDEN_TOL_FP8, ("prefill K", l)
prm = dg.sampler_params(cfg.vocab, seed=5, fixed_steps=3)
prm_o = oracle.SamplerParams(cfg.vocab, seed=5, fixed_steps=3)
ids = torch.empty(256, dtype=torch.int32, device="cuda"); commit = torch.empty(256, dtype=torch.uint8, device="cuda")
H = torch.empty(256, device="cuda"); stop = torch.empty(1, dtype=torch.int32, device="cuda")
hidden = torch.empty(cfg.n_layers + 1, 256, cfg.d_model, device="cuda"); logits = torch.empty(256, cfg.vocab, device="cuda")
dg.dg_canvas_init(seqs, prm, ids, commit)
oids, ocommit = oseq.canvas_init(prm_o)
worst = 0.0
for s in range(3):
    ids.copy_(torch.from_numpy(oids)); commit.copy_(torch.from_numpy(ocommit))
    dg.dg_canvas_step(seqs, prm, ids, commit, H, stop, hidden, logits)
    torch.cuda.synchronize()
    r = oseq.canvas_step(prm_o, oids, ocommit, want_hidden=True)
    hg = hidden.cpu().numpy()
    for l in range(cfg.n_layers + 1):
        e = rel_err(hg[l], r["hidden"][l])
        worst = max(worst, e)
        assert e <= HIDDEN_TOL_FP8, ("hidden", s, l, e)
    lg = logits.cpu().numpy()
    assert rel_err(lg, r["logits"]) <= HIDDEN_TOL_FP8, ("logits", s)
    # the sampler's decisions on the GPU's own logits, base tolerances
    pos = np.arange(oseq.P, oseq.P + 256)
    smp = oracle.sample_rows(lg, ocommit, pos, r["T"], prm_o.seed, s)
    rule = oracle.step_rule(ocommit, oids, smp["H"], smp["y"], smp["rr"], s, prm_o.entropy_bound, prm_o.rerand_entropy,
                            prm_o.stop_mean_entropy, prm_o.max_steps, prm_o.fixed_steps)
    orc = dict(smp); orc.update(rule); orc["step"] = s; orc["logits"] = lg
    g = {"ids": ids.cpu().numpy(), "commit": commit.cpu().numpy(), "H": H.cpu().numpy(), "stop": int(stop.item())}
    fails, judged = judge_step(g, orc, prm_o, ocommit)
    assert not fails, (s, fails[:5])
    oids, ocommit = r["ids"], r["commit"]
ids.copy_(torch.from_numpy(oids))
dg.dg_block_commit(seqs, ids)
oseq.block_commit(oids)
torch.cuda.synchronize()
for l in range(cfg.n_layers):
    kg = K[l, 0, :, 200:456].permute(1, 0, 2).float().cpu().numpy()
    assert rel_err(kg, oseq.k[l][200:456]) <= HIDDEN_TOL_FP8, ("commit K", l)
assert dg.dg_device_error(seqs) == 0
st = dg.dg_stats_read(seqs)
print("fp8 narrow ok, worst hidden rel err", worst, "expert launches", st["expert_up"][0], st["expert_down"][0])
'''


def test_fp8_e4m3_activations_tiny_end_to_end(cuda_ok):
    env = dict(os.environ, DG_EXPERT_WIDE="0")
    r = subprocess.run([sys.executable, "-c", "ROOT = %r\n" % ROOT + CHILD], env=env, capture_output=True, text=True,
                       timeout=600)
    print(r.stdout[-2000:])
    assert r.returncode == 0, r.stderr[-4000:]
    assert "fp8 narrow ok" in r.stdout
