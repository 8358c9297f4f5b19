"""The LayerNorm backward entry point that allocates nothing.

Some callers cannot call cudaMalloc (for instance a plugin whose host
application owns all device memory, or a thread that must not block on the
device synchronisation an allocation may trigger). For them the library offers
gpt2op_layernorm_bwd_noalloc, whose partial sums live in a fixed device array
inside the library instead of a caller-provided workspace. This test calls it
twice in a row through the C ABI, on different shapes so that the second call
runs over the first call's leftovers, and checks each result against the
workspace-taking gpt2op_layernorm_bwd with the LayerNorm tolerances used
elsewhere in the tests. It sits in a file of its own that pytest collects last.
"""
import numpy as np
import pytest

import gpt_step_b200 as gs

from gpu_util import bf16, f32, host, rel_l2, require_gpu, torch

pytestmark = pytest.mark.gpu

BF16_TOL = 6e-3


def _inputs(rows, C, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, C)) * 1.5 + 0.3
    w, b = 1.0 + 0.1 * rng.standard_normal(C), 0.1 * rng.standard_normal(C)
    y = torch.empty(rows, C, dtype=torch.bfloat16, device="cuda")
    mean, rstd = torch.empty(rows, device="cuda"), torch.empty(rows, device="cuda")
    xd, wd = bf16(x), f32(w)
    gs.layernorm_fwd(xd, wd, f32(b), y, mean, rstd)
    dy = bf16(rng.standard_normal((rows, C)))
    dres = bf16(rng.standard_normal((rows, C)))
    dw0, db0 = rng.standard_normal(C), rng.standard_normal(C)
    return xd, wd, mean, rstd, dy, dres, dw0, db0


@pytest.mark.parametrize("first", [True, False])
def test_noalloc_layernorm_bwd_matches_workspace_version(first):
    require_gpu()
    cases = [(1000, 768, True), (333, 384, False)]
    if not first:
        cases = cases[::-1]
    for rows, C, with_resid in cases:            # two calls in a row
        xd, wd, mean, rstd, dy, dres, dw0, db0 = _inputs(rows, C, rows + C)
        resid = dres if with_resid else None
        # existing entry point with a caller-provided workspace
        dx_ref = torch.empty_like(dy)
        dw_ref, db_ref = f32(dw0), f32(db0)
        ws = torch.empty(gs.layernorm_bwd_workspace(rows, C), dtype=torch.uint8, device="cuda")
        gs.layernorm_bwd(dy, xd, mean, rstd, wd, resid, dx_ref, dw_ref, db_ref, ws)
        # the entry point that allocates nothing
        dx = torch.empty_like(dy)
        dw, db = f32(dw0), f32(db0)
        gs.layernorm_bwd_noalloc(dy, xd, mean, rstd, wd, resid, dx, dw, db)
        torch.cuda.synchronize()
        assert rel_l2(host(dx), host(dx_ref)) < BF16_TOL
        assert rel_l2(host(dw), host(dw_ref)) < 1e-5
        assert rel_l2(host(db), host(db_ref)) < 1e-5
