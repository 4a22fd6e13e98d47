"""The seeded synthetic inputs are a pure function of the configuration: the same seed gives
the same bytes (every parity test and the oracle depend on it), a different seed does not."""
import torch

import moe_synth


def _same(a, b):
    keys = [k for k, v in a.items() if isinstance(v, torch.Tensor)]
    assert keys == [k for k, v in b.items() if isinstance(v, torch.Tensor)]
    return all(torch.equal(a[k], b[k]) for k in keys)


def test_layer_and_router_are_reproducible():
    cfg = dict(T=20, H=512, E=6, I=128, k=2, Is=128, seed=3, bias="zipf", wfmt="fp8")
    assert _same(moe_synth.make_layer(cfg), moe_synth.make_layer(cfg))
    assert torch.equal(moe_synth.make_router(cfg), moe_synth.make_router(cfg))
    assert not _same(moe_synth.make_layer(cfg), moe_synth.make_layer(dict(cfg, seed=4)))


def test_int4_layer_is_reproducible():
    cfg = dict(T=8, H=256, E=3, I=128, k=2, Is=0, seed=5, bias=None, wfmt="int4")
    assert _same(moe_synth.make_layer(cfg), moe_synth.make_layer(cfg))


def test_mxfp4_layer_is_reproducible():
    cfg = dict(T=8, H=256, E=3, I=128, k=2, Is=128, seed=5, bias=None, wfmt="mxfp4")
    assert _same(moe_synth.make_layer(cfg), moe_synth.make_layer(cfg))
    assert not _same(moe_synth.make_layer(cfg), moe_synth.make_layer(dict(cfg, seed=6)))
