"""The fused vocabulary head + sampler (dg_head_sample, the head and sampler of a one-canvas step)
against the oracle, through the C ABI.

Inputs are built so that the logits l = xn head^T have the sampler workload's shape: xn ~ N(0, 1)
rounded to bf16, head rows N(0, (3 / sqrt(d))^2) so that l ~ N(0, 3^2), and every tenth row gets a
spike of +12 or +40 at its own column (that head row moved by spike / d * xn_row).  The oracle
computes the logits exactly (fp64 products of the same bf16 values) and runs its sampler on them;
ids, commit bits and the random stream are judged bit for bit where the oracle's margins leave the
decision fixed, entropies within 1e-3.  Marked gpu.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from dg_testutil import judge_step, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dg(cuda_ok):
    from block_discrete_diffusion_b200 import build, dg as dgmod
    build.build()
    return dgmod


def _inputs(d, vocab, spike, seed):
    g = torch.Generator().manual_seed(seed)
    xn = torch.randn(256, d, generator=g).to(torch.bfloat16)
    head = torch.randn(vocab, d, generator=g).mul_(3.0 / d ** 0.5)
    rows = torch.arange(0, 256, 10)
    cols = torch.randperm(vocab, generator=g)[: rows.numel()]
    head[cols] += (spike / d) * xn[rows].float()
    return xn, head.to(torch.bfloat16), rows.numpy(), cols.numpy()


@pytest.mark.parametrize("d,vocab,nv,spike,step", [
    (2816, 262144, 128, 40.0, 0),     # full size; the +40 rows commit
    (2816, 262144, 256, 12.0, 12),
    (2816, 262144, 128, 12.0, 47),
    (2816, 262144, 2, 40.0, 0),       # CTA pairs (M = 256 over two SMs)
    (2816, 262144, 2, 12.0, 47),
    (256, 4096, 256, 40.0, 5),        # 16 tiles of 256: fewer items than SMs
    (256, 4096, 2, 12.0, 5),          # 16 pair tiles
])
def test_fused_head_sampler_matches_oracle(dg, d, vocab, nv, spike, step):
    seed = 7
    xn, head, srows, scols = _inputs(d, vocab, spike, seed)
    prm = dg.sampler_params(vocab, seed=seed)
    prm_o = oracle.SamplerParams(vocab, seed=seed)
    rng = np.random.default_rng(step)
    commit0 = (rng.random(256) < 0.2).astype(np.uint8)
    ids0 = rng.integers(0, vocab, 256).astype(np.int32)
    P = 1000
    ids = torch.from_numpy(ids0).cuda()
    commit = torch.from_numpy(commit0).cuda()
    H = torch.empty(256, device="cuda")
    stop = torch.empty(1, dtype=torch.int32, device="cuda")
    seq_P = torch.tensor([P], dtype=torch.int32, device="cuda")
    logits = torch.empty(256, vocab, device="cuda")
    ws = torch.empty(dg.dg_head_sample_workspace_bytes(vocab), dtype=torch.uint8, device="cuda")
    dg.dg_head_sample(xn.cuda(), head.cuda(), prm, step, seq_P, ids, commit, H, stop, ws, nv=nv, logits=logits)
    assert dg.dg_head_sample_error(ws) == 0

    l64 = xn.double().numpy() @ head.double().numpy().T          # exact products of the bf16 inputs
    assert rel_err(logits.cpu().numpy(), l64) <= 1e-5
    pos = np.arange(P, P + 256)
    T = oracle.temperature(step)
    smp = oracle.sample_rows(l64, commit0, pos, T, seed, step)
    rule = oracle.step_rule(commit0, ids0, smp["H"], smp["y"], smp["rr"], step, prm_o.entropy_bound,
                            prm_o.rerand_entropy, prm_o.stop_mean_entropy, prm_o.max_steps, prm_o.fixed_steps)
    orc = dict(smp)
    orc.update(rule)
    orc["step"] = step
    orc["logits"] = l64
    g = {"ids": ids.cpu().numpy(), "commit": commit.cpu().numpy(), "H": H.cpu().numpy(), "stop": int(stop.item())}
    fails, judged = judge_step(g, orc, prm_o, commit0)
    assert not fails, fails[:10]
    assert judged >= 150, judged
    if spike == 40.0:
        newly = rule["commit"].astype(bool) & ~commit0.astype(bool)
        assert newly[srows].any()                                  # spiked rows commit on their spike
        assert (g["ids"][srows][newly[srows]] == scols[newly[srows]]).all()
