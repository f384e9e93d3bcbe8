"""The C ABI library without a GPU: it builds, loads, exports every entry point include/dg.h
declares, and its host-side logic (sizes, argument checks, temperature schedule) is right.
No compute call is made here."""
import ctypes
import math
import os
import re

import pytest

import oracle
import synthetic

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def dg():
    from block_discrete_diffusion_b200 import build, dg as dgmod
    build.build()
    return dgmod


def _declared_entry_points():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", f)).read()
            txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
            names |= set(re.findall(r"\b(dg_[a-z0-9_]+)\s*\(", txt))
    return names


def test_library_exports_every_declared_entry_point(dg):
    declared = _declared_entry_points()
    assert "dg_canvas_step" in declared and "dg_prefill" in declared and "dg_decode" in declared
    L = ctypes.CDLL(dg.LIB_PATH)
    for name in sorted(declared):
        assert hasattr(L, name), f"{name} declared in include/ but not exported"
    assert declared == set(dg.ENTRY_POINTS), declared ^ set(dg.ENTRY_POINTS)


def test_kv_and_workspace_sizes(dg):
    for cfg in (synthetic.TINY, synthetic.FULL):
        kv = dg.dg_kv_bytes(cfg, 2, 4096)
        assert kv == 2 * cfg.n_layers * 2 * cfg.n_kv * 4096 * cfg.d_head * 2
        ws = dg.dg_workspace_bytes(cfg, 2, 4096)
        # the workspace holds at least the fp32 logits of both canvases and the expert buffers
        R, A = 2 * 256, 2 * 256 * cfg.top_k
        assert ws >= 4 * R * cfg.vocab + 4 * A * cfg.d_model + 2 * A * cfg.d_model
        assert dg.dg_kv_bytes(cfg, 1, 1000) == 0           # max_ctx must be a multiple of 256
        assert dg.dg_workspace_bytes(cfg, 0, 4096) == 0
    assert dg.dg_sample_workspace_bytes(256, 262144) >= 4 * 8 * 256 * 8


@pytest.mark.parametrize("field,value", [("d_head", 96), ("d_model", 200), ("n_q", 5), ("top_k", 0),
                                         ("vocab", 1000), ("n_exp", 300), ("d_ff", 100)])
def test_model_create_rejects_unsupported_shapes_on_the_host(dg, field, value):
    import dataclasses
    cfg = dataclasses.replace(synthetic.TINY, **{field: value})
    c = dg.make_config(cfg)
    w = dg.dg_weights()
    h = ctypes.c_void_p()
    st = dg.lib().dg_model_create(ctypes.byref(c), ctypes.byref(w), ctypes.byref(h))
    assert st == dg.DG_ERR_INVALID_ARG
    assert dg.lib().dg_last_error().decode()


def test_null_weights_rejected(dg):
    c = dg.make_config(synthetic.TINY)
    w = dg.dg_weights()
    h = ctypes.c_void_p()
    assert dg.lib().dg_model_create(ctypes.byref(c), ctypes.byref(w), ctypes.byref(h)) == dg.DG_ERR_INVALID_ARG
    assert dg.lib().dg_model_create(ctypes.byref(c), None, ctypes.byref(h)) == dg.DG_ERR_INVALID_ARG


def test_temperature_schedule_matches_oracle(dg):
    prm = dg.sampler_params(4096)
    for s in range(48):
        assert dg.dg_temperature(prm, s) == oracle.temperature(s)
    assert math.isclose(dg.dg_temperature(prm, 0), 0.8, rel_tol=1e-7)


def test_sampler_params_defaults(dg):
    p = dg.sampler_params(262144, seed=7)
    assert (p.canvas_len, p.max_steps, p.fixed_steps) == (256, 48, 0)
    assert math.isclose(p.t_start, 0.8, rel_tol=1e-7) and math.isclose(p.t_end, 0.4, rel_tol=1e-7)
    assert math.isclose(p.entropy_bound, 0.1, rel_tol=1e-7)
    assert math.isclose(p.stop_mean_entropy, 0.005, rel_tol=1e-6)
    assert math.isclose(p.rerand_entropy, 0.5 * math.log(262144), rel_tol=1e-6)
    assert ctypes.sizeof(dg.dg_sampler_params) == 56


def test_product_path_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "block_discrete_diffusion_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in txt and "from oracle" not in txt and "dg_oracle" not in txt, f


@pytest.mark.parametrize("case,expected", [
    ("null_logits", "DG_ERR_INVALID_ARG"), ("vocab_not_multiple_of_1024", "DG_ERR_INVALID_ARG"),
    ("canvas_128", "DG_ERR_UNSUPPORTED"), ("negative_step", "DG_ERR_INVALID_ARG"),
    ("workspace_too_small", "DG_ERR_CAPACITY"), ("no_rows", "DG_ERR_INVALID_ARG"),
    ("step_past_schedule", "DG_ERR_INVALID_ARG"), ("fixed_steps_past_schedule", "DG_ERR_INVALID_ARG"),
    ("zero_temperature", "DG_ERR_INVALID_ARG"),
])
def test_sampler_argument_checks_happen_on_the_host(dg, case, expected):
    """dg_sample rejects bad arguments before it touches the device (fake, never dereferenced
    pointers stand in for device buffers)."""
    vocab, n_seq, step = 4096, 1, 0
    prm = dg.sampler_params(vocab, seed=1)
    fake = ctypes.c_void_p(4096)
    logits = fake
    ws_bytes = dg.dg_sample_workspace_bytes(256, vocab)
    if case == "null_logits":
        logits = None
    elif case == "vocab_not_multiple_of_1024":
        vocab = 4000
    elif case == "canvas_128":
        prm.canvas_len = 128
    elif case == "negative_step":
        step = -1
    elif case == "workspace_too_small":
        ws_bytes -= 1
    elif case == "no_rows":
        n_seq = 0
    elif case == "step_past_schedule":
        step = prm.max_steps                      # the schedule has steps 0 .. max_steps - 1
    elif case == "fixed_steps_past_schedule":
        prm.fixed_steps = prm.max_steps + 1
    elif case == "zero_temperature":
        prm.t_end = 0.0
    st = dg.lib().dg_sample(logits, n_seq, vocab, ctypes.byref(prm), step, None, fake, fake, fake, fake, fake,
                            ws_bytes, None)
    assert st == getattr(dg, expected)
    assert dg.lib().dg_last_error().decode()


def test_binding_structs_match_the_header_layout(dg, tmp_path):
    """Every ctypes structure of the binding has the size and field offsets the C compiler gives the
    structure of include/dg.h (a small C program built with the host compiler prints them)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no host C compiler")
    structs = [dg.dg_model_config, dg.dg_layer_weights, dg.dg_weights, dg.dg_sampler_params]
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "dg.h"', "int main(void) {"]
    for S in structs:
        lines.append(f'  printf("{S.__name__} size %zu\\n", sizeof({S.__name__}));')
        for name, _ in S._fields_:
            lines.append(f'  printf("{S.__name__} {name} %zu\\n", offsetof({S.__name__}, {name}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run([cc, "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = {}
    for line in subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.splitlines():
        s, f, v = line.split()
        got[(s, f)] = int(v)
    for S in structs:
        assert got[(S.__name__, "size")] == ctypes.sizeof(S), S.__name__
        for name, _ in S._fields_:
            assert got[(S.__name__, name)] == getattr(S, name).offset, (S.__name__, name)


@pytest.mark.parametrize("case", ["step_past_schedule", "fixed_steps_past_schedule", "bad_vocab", "huge_n_seq"])
def test_noalloc_argument_checks_happen_on_the_host(dg, case):
    """dg_sample_noalloc checks its arguments like dg_sample, and compares its capacity without an
    integer overflow for any canvas count; its limit query answers 0 for vocabularies it rejects."""
    vocab, n_seq, step = 262144, 1, 0
    prm = dg.sampler_params(vocab, seed=1)
    fake = ctypes.c_void_p(4096)
    expected = dg.DG_ERR_INVALID_ARG
    if case == "step_past_schedule":
        step = prm.max_steps
    elif case == "fixed_steps_past_schedule":
        prm.fixed_steps = prm.max_steps + 1
    elif case == "bad_vocab":
        vocab = 99000
        assert dg.dg_sample_noalloc_max_rows(vocab) == 0
    elif case == "huge_n_seq":
        n_seq = 2 ** 31 - 1                          # n_seq * 256 would overflow an int
        expected = dg.DG_ERR_CAPACITY
    st = dg.lib().dg_sample_noalloc(fake, n_seq, vocab, ctypes.byref(prm), step, None, fake, fake, fake, fake, None)
    assert st == expected, (st, dg.lib().dg_last_error().decode())
    assert dg.dg_sample_noalloc_max_rows(99328) == 32768 // 2      # 99328 = 97 * 1024: two chunks
