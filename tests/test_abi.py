"""The C-ABI library builds, loads and exports every declared symbol (no GPU needed)."""
import ctypes
import os
import re

import pytest

import gpt_step_b200 as gs
from gpt_step_b200 import build, workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not h.endswith(".h"):
            continue
        src = open(os.path.join(ROOT, "include", h)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names += re.findall(r"^[A-Za-z_][\w \*]*?\b(gpt2\w*)\s*\(", src, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return gs.lib()


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 30
    raw = ctypes.CDLL(gs.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), n
        assert n in gs._SIGNATURES, f"binding lacks {n}"


def test_param_count_through_the_library(lib):
    cfg = gs.Config.make(**workloads.model_args("gpt2_124m"))
    assert gs.num_params(cfg) == 124_439_808          # numbat §4.1
    assert gs.num_params(cfg, padded=True) == 124_439_808 + 47 * 768


def test_arena_sizes(lib):
    for name in workloads.WORKLOADS:
        cfg = gs.Config.make(**workloads.model_args(name))
        n = gs.arena_bytes(cfg)
        assert n > gs.num_params(cfg, padded=True) * 18, name
        assert n < 40 * 2 ** 30, name     # fits easily in 180 GB
    bad = gs.Config.make(n_layer=2, n_head=3, n_embd=144, seq_len=64, vocab_real=100)
    assert gs.arena_bytes(bad) == 0      # head size 48 is not supported


def test_status_strings(lib):
    for st in range(7):
        assert len(lib.gpt2_status_string(st)) > 0


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(gs, "LIB_PATH", str(tmp_path / "nope.so"))
    monkeypatch.setattr(gs, "_lib_handle", None)
    with pytest.raises(RuntimeError, match="no fallback"):
        gs.lib()


def test_noalloc_layernorm_bwd_rejects_oversized_calls_before_touching_the_gpu(lib):
    cap = lib.gpt2op_layernorm_bwd_noalloc_max_bytes()
    assert cap == 296 * 2 * 1024 * 4
    dummy = ctypes.c_void_p(16)   # never dereferenced: the size check comes first
    st = lib.gpt2op_layernorm_bwd_noalloc(dummy, dummy, dummy, dummy, dummy, None, dummy, dummy, dummy,
                                          100000, 1536, None)
    assert st == 1                # GPT2_ERR_ARG


def test_head_and_masked_ce_reject_bad_arguments_before_touching_the_gpu(lib):
    """Argument errors of the newer entry points come back as GPT2_ERR_ARG from
    host-side checks alone (dummy pointers are never dereferenced)."""
    assert lib.gpt2op_lm_head_ce_workspace(19456, 50304) == 19456 * 2 * 197 * 8
    assert lib.gpt2op_lm_head_ce_workspace(0, 50304) == 0
    d = ctypes.c_void_p(16)
    f = ctypes.c_float(1.0)
    # null input, V > Vp, missing workspace, short workspace
    assert lib.gpt2op_lm_head_ce(None, d, d, d, d, 256, 64, 100, 128, f, 1, d, 1 << 20, d, None) == 1
    assert lib.gpt2op_lm_head_ce(d, d, d, d, d, 256, 64, 129, 128, f, 1, d, 1 << 20, d, None) == 1
    assert lib.gpt2op_lm_head_ce(d, d, d, d, d, 256, 64, 100, 128, f, 1, None, 1 << 20, d, None) == 1
    assert lib.gpt2op_lm_head_ce(d, d, d, d, d, 256, 64, 100, 128, f, 1, d, 256 * 8 - 8, d, None) == 1
    # the masked CE needs an ignore index (INT_MIN means none)
    assert lib.gpt2op_softmax_ce_masked(d, d, d, 4, 100, 128, -2 ** 31, f, d, None) == 1
    ptr, n = ctypes.c_void_p(), ctypes.c_int64()
    assert lib.gpt2_state_device_ptr(None, 1, ctypes.byref(ptr), ctypes.byref(n)) == 1


def test_schedule_matches_the_oracle_on_the_cpu(lib):
    """The library's warmup + cosine schedule (the one gpt2_clip_adamw applies)
    against the oracle's lr_at, across warmup, the cosine branch and past its end."""
    from oracle import gpt2 as G
    for name in ("gpt2_124m", "small", "tiny"):
        args = workloads.model_args(name)
        cfg, ocfg = gs.Config.make(**args), G.Config(**args)
        S, W = args["total_steps"], args["warmup_steps"]
        steps = sorted({0, 1, W // 2, max(W - 1, 0), W, W + 1, (W + S) // 2, S - 1, S, S + 100, 3 * S})
        for s in steps:
            # the C config holds max_lr as a float (6e-4 -> 6.0000002e-4): agreement to that rounding
            assert gs.schedule_lr(cfg, s) == pytest.approx(G.lr_at(ocfg, s), rel=1e-7, abs=1e-18), (name, s)
    c124 = gs.Config.make(**workloads.model_args("gpt2_124m"))
    assert gs.schedule_lr(c124, 699) == pytest.approx(6e-4, rel=1e-7)
    assert gs.schedule_lr(c124, 9782) == pytest.approx(3e-4, rel=1e-4)
    assert lib.gpt2_schedule_lr(None, 0) == -1.0


def test_grouped_backward_and_wait_selftest_reject_bad_arguments(lib):
    d = ctypes.c_void_p(16)
    # M below one pair tile, N or K not multiples of 256, colsum without GELU'
    assert lib.gpt2op_linear_bwd(d, d, d, None, d, d, None, 128, 768, 768, None, d, None) == 1
    assert lib.gpt2op_linear_bwd(d, d, d, None, d, d, None, 1024, 640, 768, None, d, None) == 1
    assert lib.gpt2op_linear_bwd(d, d, d, None, d, d, None, 1024, 768, 704, None, d, None) == 1
    assert lib.gpt2op_linear_bwd(d, d, d, None, d, d, d, 1024, 768, 768, None, d, None) == 1
    assert lib.gpt2op_wait_selftest(10, d, None) == 1            # limit below 1 ms
    assert lib.gpt2op_wait_selftest(10 ** 10, d, None) == 1      # above 5 s
    assert lib.gpt2op_wait_selftest(10 ** 7, None, None) == 1
