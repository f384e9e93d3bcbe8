"""Helpers shared by the GPU parity tests: moving synthetic weights to the device, reading the KV
cache layout of include/dg.h, and the judging rules for comparing the CUDA path with the oracle.

Judging rules (tolerances of the spec):
  - hidden states: max|gpu - oracle| / max|oracle| <= 2e-2 per (layer, tensor) for bf16 weights,
    excluding tokens whose router k-th vs (k+1)-th logit margin is below 1e-2 in some layer;
  - entropies: |gpu - oracle| <= 1e-3 absolute;
  - sampled ids are bit-exact wherever the oracle's top-2 perturbed-score margin exceeds 1e-2;
    re-randomised ids (integer Philox arithmetic) are always bit-exact;
  - a commit bit is judged where |H - entropy_bound| > 1e-3 (and |H - rerand_entropy| > 1e-3 for the
    re-randomise branch); the stop flag where |mean H - stop_mean_entropy| > 1e-3.
"""
import numpy as np
import torch

HIDDEN_TOL = 2e-2
ENTROPY_TOL = 1e-3
MARGIN = 1e-2
DECISION_BAND = 1e-3


def to_device(w: dict, device="cuda") -> dict:
    out = {k: v.to(device) for k, v in w.items() if k != "layers"}
    out["layers"] = [{k: v.to(device) for k, v in L.items()} for L in w["layers"]]
    return out


def rel_err(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-30))


def kv_views(kv: torch.Tensor, cfg, n_seq, max_ctx):
    """(K [L, n_seq, n_kv, max_ctx, dh], Vt [L, n_seq, n_kv, dh, max_ctx]) bf16 views of the cache."""
    n = cfg.n_layers * n_seq * cfg.n_kv * max_ctx * cfg.d_head
    flat = kv.view(torch.bfloat16)
    K = flat[:n].view(cfg.n_layers, n_seq, cfg.n_kv, max_ctx, cfg.d_head)
    Vt = flat[n: 2 * n].view(cfg.n_layers, n_seq, cfg.n_kv, cfg.d_head, max_ctx)
    return K, Vt


def router_tie_tokens(router_logits, top_k, margin=MARGIN):
    """Tokens whose k-th and (k+1)-th router logits are closer than `margin` (any layer)."""
    r = np.asarray(router_logits)
    if r.ndim == 2:
        r = r[None]
    bad = np.zeros(r.shape[1], bool)
    if r.shape[2] <= top_k:
        return bad
    s = -np.sort(-r, axis=2)
    bad |= ((s[:, :, top_k - 1] - s[:, :, top_k]) < margin).any(0)
    return bad


def judge_step(gpu, orc, prm, commit_before):
    """Compare one sampler step.  gpu/orc: dicts with ids, commit, H (numpy), stop; orc also y, margin,
    rr, mean_H.  Returns a list of failure strings (empty = pass) and the number of judged ids."""
    fails = []
    was = commit_before.astype(bool)
    H_o, H_g = orc["H"], gpu["H"]
    dH = np.abs(H_g - H_o)
    if dH.max() > ENTROPY_TOL:
        i = int(dH.argmax())
        fails.append(f"entropy row {i}: gpu {H_g[i]} oracle {H_o[i]}")
    near_bound = np.abs(H_o - prm.entropy_bound) <= DECISION_BAND
    near_rr = np.abs(H_o - prm.rerand_entropy) <= DECISION_BAND
    stop_judged = abs(orc["mean_H"] - prm.stop_mean_entropy) > DECISION_BAND or prm.fixed_steps > 0
    if stop_judged and int(gpu["stop"]) != int(orc["stop"]):
        fails.append(f"stop flag gpu {gpu['stop']} oracle {orc['stop']} (mean H {orc['mean_H']})")
    judged = 0
    for i in range(len(H_o)):
        if was[i]:
            if gpu["ids"][i] != orc["ids"][i] or not gpu["commit"][i]:
                fails.append(f"committed row {i} changed")
            continue
        if near_bound[i] or not stop_judged:
            continue
        if gpu["commit"][i] != orc["commit"][i]:
            fails.append(f"commit row {i}: gpu {gpu['commit'][i]} oracle {orc['commit'][i]} H {H_o[i]}")
            continue
        took_rr = (not orc["commit"][i]) and H_o[i] > prm.rerand_entropy and not orc["stop"]
        if near_rr[i] and not orc["commit"][i] and not orc["stop"]:
            continue
        if took_rr:
            judged += 1
            if gpu["ids"][i] != orc["rr"][i]:
                fails.append(f"re-randomised id row {i}: gpu {gpu['ids'][i]} oracle {orc['rr'][i]}")
        elif orc["margin"][i] > MARGIN:
            judged += 1
            if gpu["ids"][i] != orc["y"][i]:
                fails.append(f"sampled id row {i}: gpu {gpu['ids'][i]} oracle {orc['y'][i]} margin {orc['margin'][i]}")
    return fails, judged
