"""Pins of the oracle's NVFP4 expert weights.

The NVIDIA co-design commentary (section on reading vendor guidance) describes NVFP4 as a
4-bit format that keeps near-8-bit accuracy through two levels of scale factors.  Here: E2M1
elements (as in MXFP4), one E4M3 scale per 16 elements, and one fp32 scale per weight matrix;
the weight is e2m1 * e4m3(s) * t.
"""
import math

import numpy as np
import pytest
import torch

import moe_synth
from test_oracle_layer import _bits, _t_route
from test_oracle_mxfp4 import E2M1


def _t_deq_nvfp4(packed: np.ndarray, scales: np.ndarray, t: np.ndarray) -> torch.Tensor:
    """Dequantised [E, N, K] weights from the E2M1 value table, torch's E4M3 cast and t."""
    p = torch.from_numpy(packed.astype(np.int64))
    nib = torch.stack([p & 0xF, (p >> 4) & 0xF], -1).reshape(*packed.shape[:-1], packed.shape[-1] * 2)
    v = torch.tensor(E2M1, dtype=torch.float64)[nib]
    s = torch.from_numpy(np.ascontiguousarray(scales)).view(torch.float8_e4m3fn).to(torch.float64)
    tt = torch.from_numpy(np.asarray(t, np.float32)).double().reshape(-1, 1, 1)
    return v * s.repeat_interleave(16, dim=-1) * tt


def _t_dense_masked_nvfp4(L: dict) -> torch.Tensor:
    d = L["dims"]
    T, H, E, k, Is = (d[n] for n in ("T", "H", "E", "k", "Is"))
    x = torch.from_numpy(L["x"].view(np.int16)).view(torch.bfloat16).double()
    idx, p = _t_route(L["logits"], k)
    M = torch.zeros(T, E, dtype=torch.float64)
    M.scatter_(1, idx, p)
    silu = torch.nn.functional.silu

    def ffn(Wg, Wu, Wd):
        h = (silu(x @ Wg.T) * (x @ Wu.T)).to(torch.bfloat16).double()
        return h @ Wd.T

    W = [_t_deq_nvfp4(L[f"w_{n}"], L[f"s_{n}"], L[f"t_{n}"]) for n in ("gate", "up", "down")]
    out = torch.zeros(T, H, dtype=torch.float64)
    for e in range(E):
        out += M[:, e:e + 1] * ffn(W[0][e], W[1][e], W[2][e])
    if Is > 0:
        S = [_t_deq_nvfp4(L[f"ws_{n}"], L[f"ss_{n}"], L[f"ts_{n}"])[0] for n in ("gate", "up", "down")]
        out += ffn(*S)
    return out


@pytest.mark.parametrize("cfg", [
    dict(T=5, H=256, E=4, I=128, k=2, Is=128, wfmt="nvfp4", seed=31, bias=None),
    dict(T=4, H=384, E=3, I=256, k=3, Is=0, wfmt="nvfp4", seed=32, bias="normal"),
], ids=["shared", "k=E"])
def test_nvfp4_layer_equals_dense_masked_bruteforce(orc, cfg):
    L = moe_synth.to_numpy(moe_synth.make_layer(cfg))
    out, _ = orc.layer(L)
    want = _t_dense_masked_nvfp4(L).numpy()
    assert np.allclose(out, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


def test_nvfp4_equals_mxfp4_on_power_of_two_scales(orc):
    """E4M3 block scales that are powers of two, equal over each 32-element block, with t = 1,
    describe the same weights as MXFP4 with those exponents: the layers agree to the last bit."""
    rng = np.random.default_rng(7)
    T, H, E, I, k = 6, 256, 3, 128, 2

    def both(N, K):
        nib = rng.integers(0, 16, size=(E, N, K)).astype(np.uint8)
        packed = (nib[..., 0::2] | (nib[..., 1::2] << 4)).astype(np.uint8)
        x = rng.integers(-6, 3, size=(E, N, K // 32))             # 2^x: a normal E4M3 value
        mx = (x + 127).astype(np.uint8)
        nv = np.repeat(((x + 7) << 3).astype(np.uint8), 2, axis=-1)  # E4M3 code of 2^x, per 16
        return (packed, mx), (packed, nv)

    g, u, d = both(I, H), both(I, H), both(H, I)
    x = _bits(rng.standard_normal((T, H)))
    logits = rng.standard_normal((T, E)).astype(np.float32)
    ones = np.ones(E, np.float32)
    outs = []
    for f, j in (("mxfp4", 0), ("nvfp4", 1)):
        L = dict(dims=dict(T=T, H=H, E=E, I=I, k=k, Is=0, wfmt=f), x=x, logits=logits,
                 w_gate=g[j][0], s_gate=g[j][1], w_up=u[j][0], s_up=u[j][1], w_down=d[j][0], s_down=d[j][1])
        if f == "nvfp4":
            L.update(t_gate=ones, t_up=ones, t_down=ones)
        outs.append(orc.layer(L)[0])
    assert np.array_equal(outs[0], outs[1]) and np.abs(outs[0]).max() > 0


def test_tensor_scales_apply_to_their_own_matrices(orc):
    """Doubling t_down doubles every output exactly (y is linear in W_down); doubling t_up
    doubles h before its bf16 rounding, which commutes with a power of two, so the output
    doubles exactly too; doubling t_gate does not (silu is not linear)."""
    cfg = dict(T=4, H=256, E=3, I=128, k=2, Is=128, wfmt="nvfp4", seed=33, bias=None)
    L = moe_synth.to_numpy(moe_synth.make_layer(cfg))
    base, _ = orc.layer(L)
    for name in ("t_down", "t_up"):
        L2 = dict(L)
        L2[name] = L[name] * 2
        L2["ts" + name[1:]] = L["ts" + name[1:]] * 2
        out, _ = orc.layer(L2)
        assert np.array_equal(out, 2 * base), name
    L3 = dict(L)
    L3["t_gate"], L3["ts_gate"] = L["t_gate"] * 2, L["ts_gate"] * 2
    out, _ = orc.layer(L3)
    assert not np.allclose(out, 2 * base, rtol=1e-3) and not np.allclose(out, base, rtol=1e-3)


def test_nvfp4_one_hot_reads_single_weights(orc):
    """Nibble 0x7 is +6 and 0xD is -3; block 1 (K 16..31) of row 0 has scale 1.5 (E4M3 0x3C),
    block 0 has 0.25 (0x28); the gate's tensor scale is 0.5."""
    H, I = 128, 128
    wg = np.zeros((1, I, H // 2), np.uint8)
    wg[0, 0, 0] = 0xD7   # k=0 -> +6, k=1 -> -3 (block 0)
    wg[0, 0, 8] = 0x07   # k=16 -> +6 (block 1)
    sg = np.full((1, I, H // 16), 0x38, np.uint8)  # 1.0
    sg[0, 0, 0], sg[0, 0, 1] = 0x28, 0x3C
    wu = np.full((1, I, H // 2), 0x22, np.uint8)   # every up weight 1.0
    su = np.full((1, I, H // 16), 0x38, np.uint8)
    wd = np.zeros((1, H, I // 2), np.uint8)
    wd[0, 3, 0] = 0x02   # Y[3] = h[0] * 1
    sd = np.full((1, H, I // 16), 0x38, np.uint8)
    one = np.ones(1, np.float32)
    x = np.zeros((3, H), np.float32)
    x[0, 0], x[1, 1], x[2, 16] = 1.0, 1.0, 1.0
    L = dict(dims=dict(T=3, H=H, E=1, I=I, k=1, Is=0, wfmt="nvfp4"), x=_bits(x),
             logits=np.zeros((3, 1), np.float32), w_gate=wg, s_gate=sg, w_up=wu, s_up=su, w_down=wd,
             s_down=sd, t_gate=np.full(1, 0.5, np.float32), t_up=one, t_down=one)
    out, _ = orc.layer(L)
    silu = lambda z: z / (1 + math.exp(-z))
    b = lambda v: float((np.uint32(orc.double_to_bf16(v)) << 16).view(np.float32))
    assert out[0, 3] == b(silu(6 * 0.25 * 0.5))
    assert out[1, 3] == b(silu(-3 * 0.25 * 0.5))
    assert out[2, 3] == b(silu(6 * 1.5 * 0.5))
    assert np.count_nonzero(out) == 3


def test_nvfp4_needs_its_tensor_scales(orc):
    cfg = dict(T=2, H=128, E=2, I=128, k=1, Is=0, wfmt="nvfp4", seed=34, bias=None)
    L = moe_synth.to_numpy(moe_synth.make_layer(cfg))
    del L["t_up"]
    with pytest.raises(ValueError):
        orc.layer(L)


def test_quantiser_error_within_half_a_step():
    """Every dequantised weight is the nearest E2M1 multiple of s * t (saturating at 6 s t);
    the tensor scale puts the largest block scale near the top of E4M3's range."""
    g = torch.Generator().manual_seed(10)
    w = torch.randn((2, 32, 512), generator=g) / 20
    packed, sc, t = moe_synth._quant_nvfp4(w)
    deq = _t_deq_nvfp4(packed.numpy(), sc.numpy(), t.numpy()).numpy()
    assert np.allclose(t.numpy(), w.abs().reshape(2, -1).amax(1).numpy() / (448 * 6), rtol=1e-7)
    step_scale = np.repeat(sc.view(torch.float8_e4m3fn).double().numpy(), 16, axis=-1) * t.double().numpy()[:, None, None]
    wd = w.double().numpy()
    a = np.abs(wd) / step_scale
    spacing = np.where(a < 2, 0.5, np.where(a < 4, 1.0, 2.0))
    err = np.abs(wd - deq) / step_scale
    assert np.all((err <= spacing / 2 + 1e-6) | ((a > 6) & (np.abs(deq) / step_scale == 6)))
    assert sc.view(torch.float8_e4m3fn).float().max() >= 256  # the tensor's largest block
