"""moe_permute_noalloc: the permutation for callers that cannot give the
library scratch memory (a host framework that owns all device memory and
offers no allocator, or a fixed device-memory budget with no allocation at
run time).  It must give exactly what moe_permute gives with a caller
workspace, call after call, although its built-in scratch keeps whatever the
previous call left in it.  Collected last so a failure here comes after
every other test has run."""
import numpy as np
import pytest
import torch

import fine_grained_moe_gate_b200 as moe
from fine_grained_moe_gate_b200.inputs import CONFIGS, make_layer, make_tokens

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _routing(cfg):
    sh = moe.shape_of(cfg)
    p = make_layer(cfg.scaled(I=128, Is=128, S=0), DEV)
    x = make_tokens(cfg, DEV)
    idx = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device=DEV)
    w = torch.empty((cfg.T, cfg.k), dtype=torch.float32, device=DEV)
    counts = torch.empty(cfg.E, dtype=torch.int32, device=DEV)
    moe.moe_route(x, p["w_gate"], p["bias"], sh, idx, w, counts)
    return sh, x, idx, counts


def _outputs(cfg, x):
    T, k, d, E = cfg.T, cfg.k, cfg.d, cfg.E
    return (torch.full((T * k, d), -1, dtype=x.dtype, device=DEV), torch.full((E + 1,), -7, dtype=torch.int32, device=DEV),
            torch.full((T * k,), -7, dtype=torch.int32, device=DEV), torch.full((T * k,), -7, dtype=torch.int32, device=DEV))


def test_permute_noalloc_matches_permute_on_consecutive_calls():
    v3 = CONFIGS["v3_prefill"]
    # two calls in a row; the second is smaller, so the built-in scratch
    # still holds counters from the first call beyond what it needs
    cases = [v3.scaled(T=1000, d=256, E=256, k=8), v3.scaled(T=300, d=128, E=64, k=6, dtype="f32")]
    for cfg in cases:
        sh, x, idx, counts = _routing(cfg)
        ref = _outputs(cfg, x)
        ws = torch.empty(max(moe.moe_permute_workspace_size(sh), 256), dtype=torch.uint8, device=DEV)
        moe.moe_permute(x, idx, counts, sh, *ref, ws)
        got = _outputs(cfg, x)
        moe.moe_permute_noalloc(x, idx, counts, sh, *got)
        torch.cuda.synchronize()
        assert moe.moe_get_last_error() == 0
        bits = torch.int16 if x.dtype == torch.bfloat16 else torch.int32
        assert torch.equal(got[0].view(bits), ref[0].view(bits)), "x_perm differs"
        for a, b, name in zip(got[1:], ref[1:], ("offsets", "perm_tok", "inv_row")):
            assert torch.equal(a, b), f"{name} differs"
        assert int(got[1][-1]) == cfg.T * cfg.k


def test_permute_noalloc_largest_accepted_problem():
    """ceil(T/128) * E = 256 * 256 = 65536 counters: exactly the built-in
    scratch's capacity, so the size check's edge is exercised; the result is
    still bit-identical to moe_permute with a caller workspace, twice."""
    cfg = CONFIGS["v3_prefill"].scaled(T=32768, d=64, E=256, k=2)
    sh, x, idx, counts = _routing(cfg)
    ref = _outputs(cfg, x)
    ws = torch.empty(max(moe.moe_permute_workspace_size(sh), 256), dtype=torch.uint8, device=DEV)
    moe.moe_permute(x, idx, counts, sh, *ref, ws)
    for _ in range(2):
        got = _outputs(cfg, x)
        moe.moe_permute_noalloc(x, idx, counts, sh, *got)
        torch.cuda.synchronize()
        assert moe.moe_get_last_error() == 0
        assert torch.equal(got[0].view(torch.int16), ref[0].view(torch.int16)), "x_perm differs"
        for a, b, name in zip(got[1:], ref[1:], ("offsets", "perm_tok", "inv_row")):
            assert torch.equal(a, b), f"{name} differs"


def test_permute_noalloc_rejects_problems_beyond_its_scratch():
    cfg = CONFIGS["v3_prefill"].scaled(T=32768 + 128, d=64, E=256, k=2)   # needs 65792 counters > 65536
    sh = moe.shape_of(cfg)
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_permute_noalloc(0x10000, 0x10000, 0x10000, sh, 0x10000, 0x10000, 0x10000, 0x10000)
    assert ei.value.status == 2   # MOE_ERR_UNSUPPORTED, nothing launched
