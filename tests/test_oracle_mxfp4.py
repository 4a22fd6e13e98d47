"""Pins of the oracle's MXFP4 expert weights (OCP Microscaling FP4).

The chip-design page, section on numeric formats, lists MXFP4 among the formats NVIDIA's
tensor units take and gives its cost as 4.25 bits per number: four-bit E2M1 elements plus one
8-bit power-of-two (E8M0) scale shared by 32 of them.  E2M1 has a sign, two exponent bits
(bias 1) and one mantissa bit; its eight magnitudes are 0, 0.5, 1, 1.5, 2, 3, 4 and 6.  E8M0
is a bare biased exponent: code c means 2^(c - 127), and 255 is NaN.
"""
import math

import numpy as np
import pytest
import torch

import moe_synth
from test_oracle_layer import _bits, _t_route

# the format's value table, written out (not derived from its bit fields)
E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0]


def test_e2m1_decode_table(orc):
    for nib, v in enumerate(E2M1):
        got = orc.e2m1_decode(nib)
        assert got == v and math.copysign(1.0, got) == math.copysign(1.0, v), nib


def test_e8m0_decode_matches_torch(orc):
    codes = torch.arange(255, dtype=torch.uint8)
    want = codes.view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    got = np.array([orc.e8m0_decode(c) for c in range(255)])
    assert np.array_equal(got, want)
    assert orc.e8m0_decode(127) == 1.0 and orc.e8m0_decode(0) == 2.0 ** -127
    assert math.isnan(orc.e8m0_decode(255))


def test_storage_is_4_25_bits_per_weight():
    """The page's figure: 4 bits per element plus an 8-bit scale per 32 elements."""
    cfg = dict(T=2, H=256, E=3, I=128, k=1, Is=128, seed=1, bias=None, wfmt="mxfp4")
    L = moe_synth.make_layer(cfg)
    n = 3 * (3 * 256 * 128) + 3 * 256 * 128
    assert moe_synth.weight_bytes(L) * 8 == pytest.approx(4.25 * n, rel=0, abs=0)


# --------------------------------------------------------------------------------------
# the weights that an MXFP4 layer reads
# --------------------------------------------------------------------------------------

def _t_deq_mxfp4(packed: np.ndarray, scales: np.ndarray) -> torch.Tensor:
    """Dequantised weights from the value table and torch's E8M0 conversion."""
    p = torch.from_numpy(packed.astype(np.int64))
    nib = torch.stack([p & 0xF, (p >> 4) & 0xF], -1).reshape(*packed.shape[:-1], packed.shape[-1] * 2)
    v = torch.tensor(E2M1, dtype=torch.float64)[nib]
    s = torch.from_numpy(np.ascontiguousarray(scales)).view(torch.float8_e8m0fnu).to(torch.float64)
    return v * s.repeat_interleave(32, dim=-1)


def _t_dense_masked_mxfp4(L: dict) -> torch.Tensor:
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

    W = [_t_deq_mxfp4(L[a], L[b]) for a, b in (("w_gate", "s_gate"), ("w_up", "s_up"), ("w_down", "s_down"))]
    out = torch.zeros(T, H, dtype=torch.float64)
    for e in range(E):
        out += M[:, e:e + 1] * ffn(W[0][e], W[1][e], W[2][e])
    if Is > 0:
        S = [_t_deq_mxfp4(L[a], L[b])[0] for a, b in
             (("ws_gate", "ss_gate"), ("ws_up", "ss_up"), ("ws_down", "ss_down"))]
        out += ffn(*S)
    return out


@pytest.mark.parametrize("cfg", [
    dict(T=5, H=256, E=4, I=128, k=2, Is=128, wfmt="mxfp4", seed=21, bias=None),
    dict(T=4, H=384, E=3, I=256, k=3, Is=0, wfmt="mxfp4", seed=22, bias="normal"),
], ids=["shared", "k=E"])
def test_mxfp4_layer_equals_dense_masked_bruteforce(orc, cfg):
    L = moe_synth.to_numpy(moe_synth.make_layer(cfg))
    out, _ = orc.layer(L)
    want = _t_dense_masked_mxfp4(L).numpy()
    assert np.allclose(out, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


def test_mxfp4_one_hot_reads_single_weights(orc):
    """Nibble 0x9 is -0.5 and 0xF is -6 (the high nibble is the odd K index); 0x7 is +6.
    Block 0 of row 0 has scale code 128 (x2), block 1 code 125 (x1/4)."""
    H, I = 128, 128
    wg = np.zeros((1, I, H // 2), np.uint8)
    wg[0, 0, 0] = 0xF9   # k=0 -> -0.5, k=1 -> -6
    wg[0, 0, 16] = 0x07  # k=32 -> +6 (block 1), k=33 -> 0
    wu = np.full((1, I, H // 2), 0x22, np.uint8)  # every up weight 1.0
    sg = np.full((1, I, H // 32), 127, np.uint8)
    sg[0, 0, 0], sg[0, 0, 1] = 128, 125
    wd = np.zeros((1, H, I // 2), np.uint8)
    wd[0, 3, 0] = 0x02   # Y[3] = h[0] * 1
    L = dict(dims=dict(T=3, H=H, E=1, I=I, k=1, Is=0, wfmt="mxfp4"), logits=np.zeros((3, 1), np.float32),
             w_gate=wg, w_up=wu, w_down=wd, s_gate=sg, s_up=np.full((1, I, H // 32), 127, np.uint8),
             s_down=np.full((1, H, I // 32), 127, np.uint8))
    x = np.zeros((3, H), np.float32)
    x[0, 0], x[1, 1], x[2, 32] = 1.0, 1.0, 1.0
    L["x"] = _bits(x)
    out, _ = orc.layer(L)
    silu = lambda z: z / (1 + math.exp(-z))
    b = lambda v: float((np.uint32(orc.double_to_bf16(v)) << 16).view(np.float32))
    assert out[0, 3] == b(silu(-1.0) * 1.0)    # -0.5 * 2
    assert out[1, 3] == b(silu(-12.0) * 1.0)   # -6 * 2
    assert out[2, 3] == b(silu(1.5) * 1.0)     # 6 / 4
    assert np.count_nonzero(out) == 3


def test_mxfp4_equals_int4_on_shared_weights(orc):
    """Weights in {0, +-1, +-2, +-3, +-4, +-6} * 2^x with x constant over each 128-element
    group are exact in both 4-bit formats: the two layers must agree to the last bit."""
    rng = np.random.default_rng(3)
    T, H, E, I, k = 6, 256, 3, 128, 2
    vals = np.array([0, 1, 2, 3, 4, 6])
    e2m1_code = {0: 0, 1: 2, 2: 4, 3: 5, 4: 6, 6: 7}

    def both(N, K):
        v = rng.choice(vals, size=(E, N, K)) * rng.choice([-1, 1], size=(E, N, K))
        xg = rng.integers(-9, -3, size=(E, N, K // 128))  # one exponent per 128-group
        i4 = (v & 0xF).astype(np.uint8)
        mx = np.vectorize(lambda a: e2m1_code[abs(int(a))] | (8 if a < 0 else 0))(v).astype(np.uint8)
        pack = lambda n: (n[..., 0::2] | (n[..., 1::2] << 4)).astype(np.uint8)
        s_i4 = torch.from_numpy(np.ldexp(1.0, xg).astype(np.float32)).to(torch.bfloat16)
        s_i4 = s_i4.view(torch.int16).numpy().view(np.uint16)
        s_mx = np.repeat(xg + 127, 4, axis=-1).astype(np.uint8)
        return (pack(i4), s_i4), (pack(mx), s_mx)

    g, u, d = both(I, H), both(I, H), both(H, I)
    x = _bits(rng.standard_normal((T, H)))
    logits = rng.standard_normal((T, E)).astype(np.float32)
    outs = []
    for f, j in (("int4", 0), ("mxfp4", 1)):
        L = dict(dims=dict(T=T, H=H, E=E, I=I, k=k, Is=0, wfmt=f), x=x, logits=logits,
                 w_gate=g[j][0], s_gate=g[j][1], w_up=u[j][0], s_up=u[j][1], w_down=d[j][0], s_down=d[j][1])
        outs.append(orc.layer(L)[0])
    assert np.array_equal(outs[0], outs[1]) and np.abs(outs[0]).max() > 0


# --------------------------------------------------------------------------------------
# the input generator's MXFP4 quantiser
# --------------------------------------------------------------------------------------

def test_quantiser_returns_representable_weights_unchanged(orc):
    """W = e2m1 * 2^x with a magnitude of 4 or 6 in every block (so that the block's largest
    power of two is 2^(x+2)) quantises back to the same codes and exponents."""
    rng = np.random.default_rng(4)
    R, K = 64, 256
    nib = rng.integers(0, 16, size=(R, K))
    nib[nib == 8] = 0  # -0 comes back as +0
    nib[:, ::32] = rng.choice([6, 7, 14, 15], size=(R, K // 32))
    x = rng.integers(-20, 4, size=(R, K // 32))
    w = np.array([[E2M1[c] for c in row] for row in nib]) * np.ldexp(1.0, np.repeat(x, 32, axis=1))
    packed, sc = moe_synth._quant_mxfp4(torch.from_numpy(w.astype(np.float32)))
    assert np.array_equal(sc.numpy(), (x + 127).astype(np.uint8))
    back = packed.numpy()
    assert np.array_equal(back & 0xF, nib[:, 0::2]) and np.array_equal(back >> 4, nib[:, 1::2])


def test_quantiser_error_within_half_a_step(orc):
    """Every dequantised weight is the nearest E2M1 multiple of its block scale, saturating
    at 6 * 2^x: the error is at most half the local spacing, or the saturation gap."""
    g = torch.Generator().manual_seed(9)
    w = torch.randn((32, 512), generator=g) / 20
    packed, sc = moe_synth._quant_mxfp4(w)
    deq = _t_deq_mxfp4(packed.numpy()[None], sc.numpy()[None])[0].numpy()
    wd = w.double().numpy()
    scale = np.repeat(np.ldexp(1.0, sc.numpy().astype(np.int64) - 127), 32, axis=1)
    a = np.abs(wd) / scale
    spacing = np.where(a < 2, 0.5, np.where(a < 4, 1.0, 2.0))
    err = np.abs(wd - deq) / scale
    assert np.all((err <= spacing / 2 + 1e-12) | ((a > 6) & (np.abs(deq) / scale == 6)))
