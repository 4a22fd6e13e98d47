"""moe_route_static, the routing entry point that allocates nothing.

Some callers can't call cudaMalloc (code inside an allocator or pool callback, serving loops
that forbid allocation after start-up, embedders whose device memory another allocator has
reserved).  moe_route_static keeps its scratch in a fixed array inside the library instead of
a caller workspace.  These tests call it through the C ABI and compare it with moe_route, the
workspace-based entry point, on two calls in a row (the second call finds the first call's
leftovers in the shared array).  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import moe_synth
import mixture_experts_ffn_13_b200 as moe


def _static(L, logits, k, out):
    T, E = logits.shape
    p = lambda t: t.data_ptr()
    return L.moe_route_static(T, E, k, p(logits), p(out["topk_idx"]), p(out["topk_w"]), p(out["counts"]),
                              p(out["offsets"]), p(out["perm_tok"]), torch.cuda.current_stream().cuda_stream)


def _outs(T, E, k):
    return dict(topk_idx=torch.full((T, k), -7, dtype=torch.int32, device="cuda"),
                topk_w=torch.full((T, k), -7.0, dtype=torch.float32, device="cuda"),
                counts=torch.full((E,), -7, dtype=torch.int32, device="cuda"),
                offsets=torch.full((E + 1,), -7, dtype=torch.int32, device="cuda"),
                perm_tok=torch.full((max(T * k, 1),), -7, dtype=torch.int32, device="cuda"))


def test_rejects_sizes_beyond_the_static_scratch():
    L = moe.load_library()
    # T*k + ceil(T/256)*E + 2*(E+1) > 2^19: rejected before any device work (no GPU needed)
    assert L.moe_route_static(40000, 64, 16, None, None, None, None, None, None, None) == -2
    assert L.moe_route_static(10, 8, 9, None, None, None, None, None, None, None) == -1
    assert L.moe_route_static(10, 2048, 2, None, None, None, None, None, None, None) == -2


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["decode", "prefill", "skewed"])
def test_matches_workspace_route_twice(name):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L = moe.load_library()
    cfg = moe_synth.CONFIGS[name]
    T, E, k = cfg["T"], cfg["E"], cfg["k"]
    small = moe_synth.make_layer(dict(cfg, H=128, I=128, Is=0, wfmt="fp8"), device="cuda")
    logits = small["logits"]
    plan = moe.Plan(T, 128, E, 128, k)
    ws = plan.new_workspace()
    ref = moe.moe_route(plan, logits, ws)
    # a different batch first, so the second call meets stale scratch contents
    other = torch.randn((T, E), device="cuda", generator=torch.Generator(device="cuda").manual_seed(1))
    for call, lg in enumerate((other, logits, logits)):
        out = _outs(T, E, k)
        assert _static(L, lg, k, out) == 0
        torch.cuda.synchronize()
        if call == 0:
            continue
        for key in ("topk_idx", "counts", "offsets"):
            assert torch.equal(out[key], ref[key]), key
        assert torch.equal(out["perm_tok"][:T * k], ref["perm_tok"][:T * k])
        assert np.allclose(out["topk_w"].cpu().numpy(), ref["topk_w"].cpu().numpy(), rtol=2e-6, atol=1e-7)
