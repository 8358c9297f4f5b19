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
