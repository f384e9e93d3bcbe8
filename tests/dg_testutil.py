"""Helpers shared by the GPU parity tests: moving synthetic weights to the device, reading the KV
cache layout of include/dg.h, and the judging rules for comparing the CUDA path with the oracle.

Judging rules.
  Base tolerances (used as stated wherever the compared quantities come from identical inputs, and
  for end-to-end steps whose logits are small):
    - hidden states: max|gpu - oracle| / max|oracle| <= 2e-2 per (layer, tensor);
    - entropies: |gpu - oracle| <= 1e-3 absolute;
    - sampled ids bit-exact wherever the oracle's top-2 perturbed-score margin exceeds 1e-2;
      re-randomised ids (integer Philox arithmetic) always bit-exact;
    - a commit bit is judged where |H - entropy_bound| > 1e-3 (likewise for the re-randomise
      threshold); the stop flag where |mean H - stop_mean_entropy| > 1e-3.
  Router near-ties: a token whose k-th and (k+1)-th router logits (oracle) are closer than 1e-2 in
  any layer may pick a different expert on the GPU (its inputs carry bf16 rounding); such tokens are
  excluded from every comparison of that step.
  Large logits: the tempered scores z = l/T of an end-to-end step carry the bf16 rounding of the
  step's sequential GEMM inputs.  Each rounding adds a relative error of rms 2^-9/sqrt(3) to its
  products; with 2L+1 sequential roundings the rms relative error of z is about
  sigma_z = sqrt(2L+1) * 2^-9 / sqrt(3) (FP8 weights add 5L roundings, see c_z).  A test judges
  thousands of decisions, so the bounds sit at 6 sigma: c_z = 6 sigma_z (1.5e-2 for L = 2).  Where
  c_z * std(z_row) exceeds the base margin, ids are judged where the oracle margin -- a difference of
  two scores, whose error is sqrt(2) times that of one -- exceeds sqrt(2) c_z std(z_row), and
  entropies within c_z * (std(z) std_p(z) + Var_p(z)) (the first-order change of the entropy under a
  perturbation of that size: random part std(dz) std_p(z), scale part Var_p(z) c_z).  These derived
  bounds are only used by the tests that say so (the head x50 cases).
"""
import math

import numpy as np
import torch

HIDDEN_TOL = 2e-2
HIDDEN_TOL_FP8 = 6e-2      # hidden states with FP8 block-scaled weights
ENTROPY_TOL = 1e-3
MARGIN = 1e-2
DECISION_BAND = 1e-3


def _dev(v, device):
    return {k: t.to(device) for k, t in v.items()} if isinstance(v, dict) else v.to(device)


def to_device(w: dict, device="cuda") -> dict:
    """Weights to the device; FP8 matrices ({"e4m3", "scale"}) move as pairs."""
    out = {k: v.to(device) for k, v in w.items() if k != "layers"}
    out["layers"] = [{k: _dev(v, device) for k, v in L.items()} for L in w["layers"]]
    return out


def rel_err(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    if a.size == 0:
        return 0.0
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-30))


def kv_views(kv: torch.Tensor, cfg, n_seq, max_ctx):
    """(K [L, n_seq, n_kv, max_ctx, dh], Vt [L, n_seq, n_kv, dh, max_ctx]) bf16 views of the cache."""
    n = cfg.n_layers * n_seq * cfg.n_kv * max_ctx * cfg.d_head
    flat = kv.view(torch.bfloat16)
    K = flat[:n].view(cfg.n_layers, n_seq, cfg.n_kv, max_ctx, cfg.d_head)
    Vt = flat[n: 2 * n].view(cfg.n_layers, n_seq, cfg.n_kv, cfg.d_head, max_ctx)
    return K, Vt


# Router near-ties in end-to-end steps.  A token's router logits in an end-to-end step carry, besides
# the bf16 rounding of the layer's normed input, the hidden-state error carried from the layers before,
# so the gap between its k-th and (k+1)-th logits is known only to a fraction of a percent of the
# logits' spread: on unit-spread logits the GPU routed tokens the other way at gaps of 1.1e-2 to
# 1.9e-2 (a few among ~1e5 decisions).  End-to-end comparisons therefore treat gaps below 5% of the
# layer's router-logit standard deviation, and never below the base 1e-2, as near-ties.
ROUTER_TIE_REL_E2E = 0.05


def router_tie_tokens(router_logits, top_k, margin=MARGIN, rel=0.0):
    """Tokens whose k-th and (k+1)-th router logits are closer than max(margin, rel * std of that
    layer's router logits) in any layer."""
    r = np.asarray(router_logits)
    if r.ndim == 2:
        r = r[None]
    bad = np.zeros(r.shape[1], bool)
    if r.shape[2] <= top_k:
        return bad
    s = -np.sort(-r, axis=2)
    tol = np.maximum(margin, rel * r.reshape(r.shape[0], -1).std(axis=1))[:, None]
    bad |= ((s[:, :, top_k - 1] - s[:, :, top_k]) < tol).any(0)
    return bad


def c_z(n_layers, fp8=False):
    """6-sigma relative error of the tempered scores after n_r sequential bf16 roundings:
    n_r = 2L+1 activation roundings; with FP8 weights each of the five per-layer matrices is also
    rounded once (the kernels multiply bf16(q*s), the oracle q*s), 5L more roundings of the same
    size, independent of the others."""
    n_r = 2 * n_layers + 1 + (5 * n_layers if fp8 else 0)
    return 6.0 * math.sqrt(n_r) * 2.0 ** -9 / math.sqrt(3.0)


def derived_tolerances(logits, T, n_layers, fp8=False):
    """Per-row (margin, entropy) judging tolerances for end-to-end steps at large logits (see the
    module docstring); never below the base 1e-2 / 1e-3."""
    z = np.asarray(logits, np.float64) / T
    cz = c_z(n_layers, fp8)
    std_z = z.std(axis=1)
    zs = z - z.max(axis=1, keepdims=True)
    p = np.exp(zs)
    p /= p.sum(axis=1, keepdims=True)
    mean_p = (p * z).sum(axis=1, keepdims=True)
    var_p = (p * (z - mean_p) ** 2).sum(axis=1)
    margin = np.maximum(MARGIN, math.sqrt(2.0) * cz * std_z)
    htol = np.maximum(ENTROPY_TOL, cz * (std_z * np.sqrt(var_p) + var_p))
    return margin, htol


def prm_vocab(orc):
    """Vocabulary size of a step's logits (the re-randomisation ids lie below it)."""
    lg = orc.get("logits")
    return lg.shape[1] if lg is not None else 262144


def judge_step(gpu, orc, prm, commit_before, exclude=None, margin_tol=None, h_tol=None):
    """Compare one sampler step.  gpu/orc: dicts with ids, commit, H (numpy), stop; orc also y, margin,
    rr, mean_H.  exclude: rows not judged (router near-ties).  margin_tol / h_tol: per-row tolerances
    (default: the base tolerances).  Returns (failures, number of ids judged)."""
    n = len(orc["H"])
    exclude = np.zeros(n, bool) if exclude is None else np.asarray(exclude, bool)
    margin_tol = np.full(n, MARGIN) if margin_tol is None else np.asarray(margin_tol)
    h_tol = np.full(n, ENTROPY_TOL) if h_tol is None else np.asarray(h_tol)
    fails = []
    was = commit_before.astype(bool)
    H_o, H_g = orc["H"], gpu["H"]
    dH = np.abs(H_g - H_o)
    bad = np.where((dH > h_tol) & ~exclude)[0]
    for i in bad[:5]:
        fails.append(f"entropy row {i}: gpu {H_g[i]} oracle {H_o[i]} tol {h_tol[i]}")
    band = np.maximum(DECISION_BAND, h_tol)
    # per-position rule: H against the bound; cumulative rule: the running entropy sum ("cum")
    near_bound = np.abs((orc["cum"] if "cum" in orc else H_o) - prm.entropy_bound) <= band
    near_rr = np.abs(H_o - prm.rerand_entropy) <= band
    # The stop flag is judged when no admissible difference can move it: a fixed budget, or a canvas
    # mean far from the threshold even if every excluded row's entropy moved by its whole range
    # (ln V each), and -- when excluded rows exist -- an uncommitted judged row that keeps the
    # "all committed" test false (or the budget reached).
    mean_band = max(DECISION_BAND, float(np.mean(h_tol))) + exclude.sum() * math.log(prm_vocab(orc)) / n
    budget_end = orc.get("step", -1) + 1 >= prm.max_steps
    open_row = bool((~exclude & ~orc["commit"].astype(bool)).any())
    stop_judged = prm.fixed_steps > 0 or budget_end or (
        abs(orc["mean_H"] - prm.stop_mean_entropy) > mean_band and (not exclude.any() or open_row))
    if stop_judged and int(gpu["stop"]) != int(orc["stop"]):
        fails.append(f"stop flag gpu {gpu['stop']} oracle {orc['stop']} (mean H {orc['mean_H']})")
    # a row that commits in this step, or takes its Gumbel-argmax y without committing (entropy below
    # the re-randomisation threshold), ends with id y whether the block stops or not: its id (and, if it
    # commits, its commit bit) is judged even when the stop flag is not
    crit = orc["cum"] if "cum" in orc else H_o
    commits_anyway = crit <= prm.entropy_bound
    judged = 0
    for i in range(n):
        if was[i]:
            if gpu["ids"][i] != orc["ids"][i] or not gpu["commit"][i]:
                fails.append(f"committed row {i} changed")
            continue
        if exclude[i] or near_bound[i]:
            continue
        if not stop_judged:
            if near_rr[i] or not (commits_anyway[i] or H_o[i] <= prm.rerand_entropy):
                continue                      # re-randomised unless the block stops: open
            if commits_anyway[i] and not gpu["commit"][i]:
                fails.append(f"commit row {i}: gpu 0 oracle 1 H {H_o[i]}")
                continue
            if orc["margin"][i] > margin_tol[i]:
                judged += 1
                if gpu["ids"][i] != orc["y"][i]:
                    fails.append(f"sampled id row {i}: gpu {gpu['ids'][i]} oracle {orc['y'][i]} "
                                 f"margin {orc['margin'][i]} tol {margin_tol[i]}")
            continue
        if gpu["commit"][i] != orc["commit"][i]:
            fails.append(f"commit row {i}: gpu {gpu['commit'][i]} oracle {orc['commit'][i]} H {H_o[i]}")
            continue
        if near_rr[i] and not orc["commit"][i] and not orc["stop"]:
            continue
        took_rr = (not orc["commit"][i]) and H_o[i] > prm.rerand_entropy and not orc["stop"]
        if took_rr:
            judged += 1
            if gpu["ids"][i] != orc["rr"][i]:
                fails.append(f"re-randomised id row {i}: gpu {gpu['ids'][i]} oracle {orc['rr'][i]}")
        elif orc["margin"][i] > margin_tol[i]:
            judged += 1
            if gpu["ids"][i] != orc["y"][i]:
                fails.append(f"sampled id row {i}: gpu {gpu['ids'][i]} oracle {orc['y'][i]} "
                             f"margin {orc['margin'][i]} tol {margin_tol[i]}")
    return fails, judged
