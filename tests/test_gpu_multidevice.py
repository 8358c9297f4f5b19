"""The one-time set-up of the kernels (dynamic shared-memory opt-ins, occupancy
queries, the no-alloc scratch address) is made per device: the same calls on a
second GPU of the process give the first GPU's results. Skips unless at least
two devices are visible.
"""
import numpy as np
import pytest

import gpt_step_b200 as gs

from gpu_util import bf16, err_word, f32, host, rel_l2, require_gpu, torch

pytestmark = pytest.mark.gpu


def _run_on(dev):
    """LayerNorm forward and the no-alloc backward, a pair GEMM, attention forward
    and backward on device `dev`; every input from the same seeds."""
    with torch.cuda.device(dev):
        rng = np.random.default_rng(7)
        rows, C, H = 1024, 768, 12
        x = bf16(rng.standard_normal((rows, C)))
        w, b = f32(1.0 + 0.1 * rng.standard_normal(C)), f32(0.1 * rng.standard_normal(C))
        y = torch.empty(rows, C, dtype=torch.bfloat16, device="cuda")
        mean, rstd = torch.empty(rows, device="cuda"), torch.empty(rows, device="cuda")
        gs.layernorm_fwd(x, w, b, y, mean, rstd)
        dy = bf16(rng.standard_normal((rows, C)))
        dx = torch.empty_like(dy)
        dw, db = torch.zeros(C, device="cuda"), torch.zeros(C, device="cuda")
        gs.layernorm_bwd_noalloc(dy, x, mean, rstd, w, None, dx, dw, db)
        wq = bf16(0.05 * rng.standard_normal((3 * C, C)))
        qkv = torch.empty(rows, 3 * C, dtype=torch.bfloat16, device="cuda")
        err = err_word()
        gs.linear_fwd(y, wq, None, None, qkv, err)
        B, T = 1, rows
        qkv3 = qkv.view(B, T, 3 * C)
        out = torch.empty(B, T, C, dtype=torch.bfloat16, device="cuda")
        lse = torch.empty(B, H, T, device="cuda")
        gs.attention_fwd(qkv3, out, lse, H, err)
        dout = bf16(rng.standard_normal((B, T, C)))
        dqkv = torch.empty_like(qkv3)
        ws = torch.empty(gs.attention_bwd_workspace(B, T, H, C // H), dtype=torch.uint8, device="cuda")
        gs.attention_bwd(qkv3, out, dout, lse, dqkv, H, ws, err)
        torch.cuda.synchronize()
        assert int(err.sum()) == 0
        return [host(t) for t in (y, dx, dw, db, qkv, out, dqkv)]


def test_kernels_on_a_second_device_match_the_first():
    require_gpu()
    if torch.cuda.device_count() < 2:
        pytest.skip("needs two visible devices")
    first = _run_on(0)
    second = _run_on(1)
    for a, b in zip(first, second):
        assert rel_l2(b, a) < 2e-3   # fp32 atomics may add in another order
