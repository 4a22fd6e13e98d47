"""Router logits on the tensor cores (moe_router_logits) against the fp64 oracle.

logits = x . W_router^T with bf16 inputs: every product is exact and the GPU sums them in fp32,
so a logit may differ from the exact sum by at most a few units of fp32 rounding per addition
times sum_i |x_i w_i|.  Routing is compared with the exact top-k on every token whose top-k
boundary margin is wider than the logit errors actually seen on that token (elsewhere either
selection is a correct rounding of the exact logits), and the layer output on such tokens.
"""
import numpy as np
import pytest
import torch

import moe_synth
import oracle
import mixture_experts_ffn_13_b200 as moe
from test_gpu_parity import check_out

pytestmark = pytest.mark.gpu


def _rel(H):
    """Bound on |fp32 sum - exact| / sum|x_i w_i| for H products summed in 16-term blocks,
    each addition rounding (or truncating) once: (H/16 + 16) units of 2^-23, doubled."""
    return (H / 16 + 16) * 2.0 ** -22


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    moe.load_library()


def _bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _clear_tokens(got, want, k):
    """Tokens whose exact k-th and (k+1)-th logits are further apart than twice the largest
    logit error seen on that token; returns (mask, exact top-k index sets sorted)."""
    T, E = want.shape
    order = np.argsort(-want, axis=1, kind="stable")
    rows = np.arange(T)
    if k == E:
        return np.ones(T, bool), np.sort(order[:, :k], 1)
    margin = want[rows, order[:, k - 1]] - want[rows, order[:, k]]
    delta = np.abs(got - want).max(axis=1)
    clear = margin > 2 * delta + 1e-6 * np.abs(want[rows, order[:, k - 1]])
    return clear, np.sort(order[:, :k], 1)


CASES = {
    "tiny": moe_synth.CONFIGS["tiny"],
    "decode": moe_synth.CONFIGS["decode"],
    "int4": moe_synth.CONFIGS["int4"],
    # ragged token tile, two expert tiles with the second partial, H of 12 K slices
    # (small batches like this one and the three above take the cluster split-K form)
    "ragged": dict(T=300, H=768, E=200, I=128, k=6, Is=0, wfmt="fp8", seed=60, bias=None),
    # enough token tiles that every SM gets whole tiles: the one-CTA-per-tile form, again with
    # a partial second expert tile
    "persistent": dict(T=4096, H=256, E=200, I=128, k=6, Is=0, wfmt="fp8", seed=61, bias=None),
}


@pytest.mark.parametrize("name", list(CASES))
def test_router_logits_and_routing(name):
    cfg = dict(CASES[name], I=128, Is=0)
    T, H, E, k = cfg["T"], cfg["H"], cfg["E"], cfg["k"]
    x = moe_synth.make_layer(cfg, device="cuda")["x"]
    w = moe_synth.make_router(cfg, device="cuda")
    plan = moe.Plan(T, H, E, 128, k, 0, cfg["wfmt"])
    lg = moe.moe_router_logits(plan, x, w)
    torch.cuda.synchronize()
    assert moe.moe_get_status(plan) == 0
    want, bound = oracle.router_logits(_bits(x), _bits(w))
    got = lg.cpu().numpy().astype(np.float64)
    err = np.abs(got - want)
    assert np.all(err <= _rel(H) * bound), f"worst relative error {np.max(err / bound):.3e}"
    # routing the GPU's logits selects the exact top-k wherever the margin allows only that
    r = moe.moe_route(plan, lg, plan.new_workspace())
    torch.cuda.synchronize()
    clear, exact_sets = _clear_tokens(got, want, k)
    assert clear.mean() > 0.99
    gi = np.sort(r["topk_idx"].cpu().numpy(), 1)
    assert np.array_equal(gi[clear], exact_sets[clear])


def test_router_logits_rejects_bad_arguments():
    plan = moe.Plan(16, 512, 8, 256, 2, 0, "fp8")
    x = torch.zeros((17, 512), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((8, 512), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoEError) as ei:  # T above the plan's T_max
        moe.moe_router_logits(plan, x, w)
    assert ei.value.code == -1
    lg = moe.moe_router_logits(plan, x[:0], w)  # T = 0 is a no-op
    assert lg.shape == (0, 8)


def test_router_then_layer_decode():
    cfg = moe_synth.CONFIGS["decode"]
    layer = moe_synth.make_layer("decode", device="cuda")
    w = moe_synth.make_router(cfg, device="cuda")
    m = moe.MoELayer(layer)
    lg = moe.moe_router_logits(m.plan, layer["x"], w)
    out = m(layer["x"], lg)
    torch.cuda.synchronize()
    assert moe.moe_get_status(m.plan) == 0
    exact, _ = oracle.router_logits(_bits(layer["x"]), _bits(w))
    clear, _ = _clear_tokens(lg.cpu().numpy().astype(np.float64), exact, cfg["k"])
    sel = np.nonzero(clear)[0][::51][:10].astype(np.int32)
    L = moe_synth.to_numpy(layer)
    L["logits"] = exact.astype(np.float32)  # the oracle routes on the exact logits
    want, _, amb = oracle.layer(L, sel, ambiguity=True)
    check_out(out[torch.from_numpy(sel).long().cuda()], want, "router + layer", amb)


@pytest.mark.parametrize("name", ["tiny", "decode", "int4", "ragged", "persistent", "e1024", "fallback"])
def test_router_topk_selects_what_route_selects(name):
    """moe_router_topk: logits within the fp32 bound of the exact sums, and the selection (and
    its weights) identical to the oracle's top-k of those same fp32 logits."""
    cfg = dict(EXTRA[name]) if name in EXTRA else dict(CASES[name], I=128, Is=0)
    T, H, E, k = cfg["T"], cfg["H"], cfg["E"], cfg["k"]
    x = moe_synth.make_layer(dict(cfg, I=128, Is=0), device="cuda")["x"]
    w = moe_synth.make_router(cfg, device="cuda")
    plan = moe.Plan(T, H, E, 128, k, 0, cfg["wfmt"])
    r = moe.moe_router_topk(plan, x, w)
    torch.cuda.synchronize()
    assert moe.moe_get_status(plan) == 0
    want, bound = oracle.router_logits(_bits(x), _bits(w))
    got = r["logits"].cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - want) <= _rel(H) * bound)
    idx, wts = oracle.route(r["logits"].cpu().numpy(), k)
    assert np.array_equal(r["topk_idx"].cpu().numpy(), idx)
    assert np.allclose(r["topk_w"].cpu().numpy(), wts, rtol=2e-6, atol=1e-7)


EXTRA = {
    # the largest expert count (32 logits per lane in the warp top-k)
    "e1024": dict(T=96, H=512, E=1024, I=128, k=8, Is=0, wfmt="fp8", seed=62, bias=None),
    # a prefill-sized batch of a small layer (one-CTA-per-tile router GEMM)
    "fallback": dict(T=8192, H=256, E=200, I=128, k=6, Is=0, wfmt="fp8", seed=63, bias=None),
}


@pytest.mark.parametrize("name", ["decode", "int4", "tiny"])
def test_forward_x_equals_router_then_forward(name):
    """moe_forward_x (hidden states + router weights) is bit-identical to moe_router_logits
    followed by moe_forward on those logits, and matches the oracle on clear tokens."""
    cfg = moe_synth.CONFIGS[name]
    layer = moe_synth.make_layer(name, device="cuda")
    w = moe_synth.make_router(cfg, device="cuda")
    m = moe.MoELayer(layer)
    got = moe.moe_forward_x(m.plan, layer["x"], w, m.weights, m.workspace)
    torch.cuda.synchronize()
    assert moe.moe_get_status(m.plan) == 0
    assert moe.moe_launch_count(m.plan) >= 7
    lg = moe.moe_router_logits(m.plan, layer["x"], w)
    ref = m(layer["x"], lg)
    torch.cuda.synchronize()
    assert torch.equal(got, ref)
    exact, _ = oracle.router_logits(_bits(layer["x"]), _bits(w))
    clear, _ = _clear_tokens(lg.cpu().numpy().astype(np.float64), exact, cfg["k"])
    sel = np.nonzero(clear)[0][::37][:8].astype(np.int32)
    L = moe_synth.to_numpy(layer)
    L["logits"] = exact.astype(np.float32)
    want, _, amb = oracle.layer(L, sel, ambiguity=True)
    check_out(got[torch.from_numpy(sel).long().cuda()], want, "forward_x", amb)


def test_forward_x_argument_errors_launch_nothing():
    cfg = dict(T=16, H=512, E=8, I=256, k=2, Is=0, seed=64, bias=None, wfmt="fp8")
    layer = moe_synth.make_layer(cfg, device="cuda")
    m = moe.MoELayer(layer)
    w = moe_synth.make_router(cfg, device="cuda")
    with pytest.raises(moe.MoEError) as ei:  # workspace one byte short
        moe.moe_forward_x(m.plan, layer["x"], w, m.weights, m.workspace[: m.plan.workspace_bytes - 1])
    assert ei.value.code == -3 and moe.moe_launch_count(m.plan) == 0
    bad = dict(m.weights)
    bad["w_down"] = None
    with pytest.raises((moe.MoEError, TypeError, AttributeError)):
        moe.moe_forward_x(m.plan, layer["x"], w, bad, m.workspace)
