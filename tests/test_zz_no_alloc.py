"""moe_route_static, the routing entry point that allocates nothing.

Some callers can't call cudaMalloc (code inside an allocator or pool callback, serving loops
that forbid allocation after start-up, embedders whose device memory another allocator has
reserved).  moe_route_static keeps its scratch in a fixed array inside the library instead of
a caller workspace.  These tests call it through the C ABI and check it:
  * against the oracle's routing and permutation (bit-exact indices, counts, offsets and rows),
    including one expert group per token, E = 1024 and batches up to 4096 tokens, where it
    runs the histogram -> scan -> scatter permutation;
  * against moe_route, the workspace-based entry point, on two calls in a row (the second
    call finds the first call's leftovers in the shared array);
  * on an empty batch (counts and offsets zeroed) and on the capacity limit.
This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

import moe_synth
import oracle
import mixture_experts_ffn_13_b200 as moe


def _static(L, logits, k, out, stream=None):
    T, E = logits.shape
    p = lambda t: t.data_ptr()
    s = (stream or torch.cuda.current_stream()).cuda_stream
    return L.moe_route_static(T, E, k, p(logits), p(out["topk_idx"]), p(out["topk_w"]), p(out["counts"]),
                              p(out["offsets"]), p(out["perm_tok"]), s)


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
    # E <= 1024 and k <= 32 (both supported) but 16384*32 + 64*1024 + 2050 > 2^19: the size check
    assert L.moe_route_static(16384, 1024, 32, None, None, None, None, None, None, None) == -2
    assert L.moe_route_static(10, 8, 9, None, None, None, None, None, None, None) == -1   # k > E
    assert L.moe_route_static(10, 2048, 2, None, None, None, None, None, None, None) == -2  # E > 1024


def _check_against_oracle(out, logits, k):
    L_ = logits.cpu().numpy()
    T, E = L_.shape
    idx, w = oracle.route(L_, k)
    counts, offsets, perm, _ = oracle.permute(idx, E)
    assert np.array_equal(out["topk_idx"].cpu().numpy(), idx)
    assert np.array_equal(out["counts"].cpu().numpy(), counts)
    assert np.array_equal(out["offsets"].cpu().numpy(), offsets)
    assert np.array_equal(out["perm_tok"].cpu().numpy()[:T * k], perm)
    assert np.allclose(out["topk_w"].cpu().numpy(), w, rtol=2e-6, atol=1e-7)


@pytest.mark.gpu
@pytest.mark.parametrize("T,E,k", [(1, 8, 2), (1, 1024, 32), (513, 512, 10), (513, 8, 8), (4096, 1024, 8),
                                   (4096, 512, 10), (300, 1024, 1)])
def test_matches_oracle(T, E, k):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L = moe.load_library()
    g = torch.Generator(device="cuda").manual_seed(T * 31 + E + k)
    logits = torch.randn((T, E), generator=g, device="cuda")
    # a stale previous call first: nothing may depend on the array's old contents
    other = torch.randn((T, E), generator=g, device="cuda")
    assert _static(L, other, k, _outs(T, E, k)) == 0
    out = _outs(T, E, k)
    assert _static(L, logits, k, out) == 0
    torch.cuda.synchronize()
    _check_against_oracle(out, logits, k)


@pytest.mark.gpu
def test_empty_batch_zeroes_counts_and_offsets():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L = moe.load_library()
    E, k = 64, 4
    out = _outs(0, E, k)
    logits = torch.empty((0, E), dtype=torch.float32, device="cuda")
    assert _static(L, logits, k, out) == 0
    torch.cuda.synchronize()
    assert torch.all(out["counts"] == 0) and torch.all(out["offsets"] == 0)


@pytest.mark.gpu
def test_side_stream_and_binding():
    """Calls on a non-default stream of the current device, and through the Python binding
    (which makes the logits' device current and takes its current stream)."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L = moe.load_library()
    T, E, k = 64, 16, 2
    logits = torch.randn((T, E), device="cuda")
    side = torch.cuda.Stream()
    out = _outs(T, E, k)
    assert _static(L, logits, k, out, stream=side) == 0
    side.synchronize()
    _check_against_oracle(out, logits, k)
    # the binding enters the logits' device and uses its current stream
    r = moe.moe_route_static(logits, k)
    torch.cuda.synchronize()
    _check_against_oracle(r, logits, k)


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
    _check_against_oracle(out, logits, k)
