"""Pins of the oracle's whole layer: hand-worked cases, a dense SwiGLU special case, and a
brute-force dense-masked evaluation written independently in torch fp64.

Layer (TPU7x MoE page: sections on sparsity and on the grouped GEMM v2 kernel; Flash-Next
page, section ① expert FFN): out[t] = sum_j p_hat[t,j] * FFN_{e_j}(x_t) + FFN_shared(x_t),
FFN(x) = (silu(x Wg^T) * (x Wu^T)) Wd^T with FP8 512-sub-channel or int4 128-group weights.
"""
import math

import numpy as np
import pytest
import torch

import moe_synth


def _bits(x) -> np.ndarray:
    return torch.as_tensor(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _f32(v):
    return float(np.float32(v))


# --------------------------------------------------------------------------------------
# hand-worked 2-expert / 2-token case
# --------------------------------------------------------------------------------------

def _code(orc, v):
    return int(orc.e4m3_encode(np.float32(v))[0])


def test_hand_worked_two_experts_two_tokens(orc):
    """H = 512 (one block, amax 448 so the activation scale is exactly 1), I = 1, k = 2."""
    T, E, H, I = 2, 2, 512, 1
    x = np.zeros((T, H), np.float32)
    x[0, 0], x[1, 0] = 1.0, 2.0
    x[:, 511] = 448.0  # block amax -> s_x = 1; its weights are zero below
    wg = np.zeros((E, I, H), np.uint8)
    wu = np.zeros((E, I, H), np.uint8)
    wd = np.zeros((E, H, I), np.uint8)
    wg[0, 0, 0], wu[0, 0, 0] = _code(orc, 1.0), _code(orc, 0.5)
    wg[1, 0, 0], wu[1, 0, 0] = _code(orc, -1.0), _code(orc, 1.0)
    wd[0, 0, 0], wd[0, 1, 0] = _code(orc, 1.0), _code(orc, -2.0)
    wd[1, 0, 0], wd[1, 2, 0] = _code(orc, 0.25), _code(orc, 3.0)
    ones = lambda *s: np.ones(s, np.float32)
    ln3 = np.float32(math.log(3.0))
    logits = np.array([[0.0, ln3], [1.0, 1.0]], np.float32)
    layer = dict(dims=dict(T=T, H=H, E=E, I=I, k=2, Is=0, wfmt="fp8"), x=_bits(x), logits=logits,
                 w_gate=wg, w_up=wu, w_down=wd, s_gate=ones(E, I, 1), s_up=ones(E, I, 1),
                 s_down=ones(E, H, 1))
    out, outb = orc.layer(layer)

    def qh(h):  # one-element block: s = |h32|/448 (fp32), code = +-448 -> h~ = +-448 * s
        h32 = np.float32(h)
        s = np.float32(abs(h32)) / np.float32(448.0)
        return math.copysign(448.0 * float(s), float(h32))

    sig = lambda z: 1.0 / (1.0 + math.exp(-z))
    # token 0: x0 = 1.  expert 0: G = 1, U = 0.5; expert 1: G = -1, U = 1
    h00 = qh(1.0 * sig(1.0) * 0.5)
    h01 = qh(-1.0 * sig(-1.0) * 1.0)
    p1 = 1.0 / (1.0 + math.exp(-float(ln3)))  # expert 1 has the larger logit
    p0 = 1.0 - p1
    # token 1: x0 = 2.  expert 0: G = 2, U = 1; expert 1: G = -2, U = 2; equal logits
    h10 = qh(2.0 * sig(2.0) * 1.0)
    h11 = qh(-2.0 * sig(-2.0) * 2.0)
    want = np.zeros((T, H))
    want[0, 0] = p0 * h00 * 1.0 + p1 * h01 * 0.25
    want[0, 1] = p0 * h00 * -2.0
    want[0, 2] = p1 * h01 * 3.0
    want[1, 0] = 0.5 * h10 + 0.5 * h11 * 0.25
    want[1, 1] = 0.5 * h10 * -2.0
    want[1, 2] = 0.5 * h11 * 3.0
    assert np.allclose(out, want, rtol=1e-14, atol=1e-300)
    assert np.array_equal(outb, np.array([[orc.double_to_bf16(v) for v in row] for row in want], np.uint16))


# --------------------------------------------------------------------------------------
# independent torch fp64 compositions
# --------------------------------------------------------------------------------------

def _t_quant(x32: torch.Tensor) -> torch.Tensor:
    """Dequantised FP8 rows: per 512-block s = amax/448 (fp32), q = float8 cast of x/s."""
    R, K = x32.shape
    nb = (K + 511) // 512
    xp = torch.nn.functional.pad(x32, (0, nb * 512 - K)).reshape(R, nb, 512)
    amax = xp.abs().amax(-1, keepdim=True)
    s = torch.where(amax == 0, torch.ones_like(amax), amax / 448.0)
    q = (xp / s).to(torch.float8_e4m3fn).to(torch.float64)
    return (q * s.double()).reshape(R, nb * 512)[:, :K]


def _t_deq_fp8(codes: np.ndarray, scales: np.ndarray) -> torch.Tensor:
    q = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64)
    K = q.shape[-1]
    s = torch.from_numpy(scales).double().repeat_interleave(512, dim=-1)[..., :K]
    return q * s


def _t_deq_int4(packed: np.ndarray, scales_bits: np.ndarray) -> torch.Tensor:
    p = torch.from_numpy(packed.astype(np.int32))
    lo, hi = p & 0xF, (p >> 4) & 0xF
    q = torch.stack([lo, hi], -1).reshape(*packed.shape[:-1], packed.shape[-1] * 2)
    q = torch.where(q >= 8, q - 16, q).double()
    s = torch.from_numpy(scales_bits.view(np.int16)).view(torch.bfloat16).double()
    return q * s.repeat_interleave(128, dim=-1)


def _t_route(logits: np.ndarray, k: int):
    L = torch.from_numpy(logits)
    _, order = torch.sort(-L, dim=1, stable=True)  # ties keep the lower index first
    idx = order[:, :k]
    lv = torch.gather(L, 1, idx).double()
    p = torch.softmax(lv, dim=1)
    return idx, p


def _t_dense_masked(L: dict) -> torch.Tensor:
    """Every expert on every token, masked by a [T,E] matrix of p_hat (0 off the top-k)."""
    d = L["dims"]
    T, H, E, I, k, Is = (d[n] for n in ("T", "H", "E", "I", "k", "Is"))
    x = torch.from_numpy(L["x"].view(np.int16)).view(torch.bfloat16).float()
    idx, p = _t_route(L["logits"], k)
    M = torch.zeros(T, E, dtype=torch.float64)
    M.scatter_(1, idx, p)
    silu = torch.nn.functional.silu
    if d["wfmt"] == "fp8":
        xa = _t_quant(x)
        Wg, Wu, Wd = (_t_deq_fp8(L[a], L[b]) for a, b in
                      (("w_gate", "s_gate"), ("w_up", "s_up"), ("w_down", "s_down")))

        def ffn(Wg_, Wu_, Wd_):
            h = silu(xa @ Wg_.T) * (xa @ Wu_.T)
            return _t_quant(h.float()) @ Wd_.T
    else:
        xa = x.double()
        Wg, Wu, Wd = (_t_deq_int4(L[a], L[b]) for a, b in
                      (("w_gate", "s_gate"), ("w_up", "s_up"), ("w_down", "s_down")))

        def ffn(Wg_, Wu_, Wd_):
            h = (silu(xa @ Wg_.T) * (xa @ Wu_.T)).to(torch.bfloat16).double()
            return h @ Wd_.T
    out = torch.zeros(T, H, dtype=torch.float64)
    for e in range(E):
        out += M[:, e:e + 1] * ffn(Wg[e], Wu[e], Wd[e])
    if Is > 0:
        if d["wfmt"] == "fp8":
            S = [_t_deq_fp8(L[a], L[b])[0] for a, b in
                 (("ws_gate", "ss_gate"), ("ws_up", "ss_up"), ("ws_down", "ss_down"))]
        else:
            S = [_t_deq_int4(L[a], L[b])[0] for a, b in
                 (("ws_gate", "ss_gate"), ("ws_up", "ss_up"), ("ws_down", "ss_down"))]
        out += ffn(*S)
    return out


SMALL = [
    dict(T=6, H=512, E=4, I=128, k=2, Is=0, wfmt="fp8", seed=11, bias=None),
    dict(T=5, H=1024, E=6, I=256, k=3, Is=128, wfmt="fp8", seed=12, bias="normal"),
    dict(T=4, H=768, E=5, I=640, k=2, Is=384, wfmt="fp8", seed=13, bias="zipf"),  # partial blocks
    dict(T=5, H=256, E=4, I=128, k=2, Is=128, wfmt="int4", seed=14, bias=None),
]


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: f"{c['wfmt']}-T{c['T']}-H{c['H']}-I{c['I']}-Is{c['Is']}")
def test_layer_equals_dense_masked_bruteforce(orc, cfg):
    L = moe_synth.to_numpy(moe_synth.make_layer(cfg))
    out, _ = orc.layer(L)
    want = _t_dense_masked(L).numpy()
    scale = np.abs(want).max()
    assert np.allclose(out, want, rtol=1e-12, atol=1e-12 * scale)


def test_single_expert_reduces_to_dense_swiglu(orc):
    """E = 1, k = 1, no shared expert: the layer is one dense SwiGLU FFN (p_hat = 1)."""
    cfg = dict(T=7, H=1024, E=1, I=384, k=1, Is=0, wfmt="fp8", seed=15, bias=None)
    L = moe_synth.to_numpy(moe_synth.make_layer(cfg))
    out, _ = orc.layer(L)
    x = torch.from_numpy(L["x"].view(np.int16)).view(torch.bfloat16).float()
    xa = _t_quant(x)
    Wg = _t_deq_fp8(L["w_gate"], L["s_gate"])[0]
    Wu = _t_deq_fp8(L["w_up"], L["s_up"])[0]
    Wd = _t_deq_fp8(L["w_down"], L["s_down"])[0]
    F = torch.nn.functional
    h = F.silu(F.linear(xa, Wg)) * F.linear(xa, Wu)
    want = F.linear(_t_quant(h.float()), Wd).numpy()
    assert np.allclose(out, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


def test_int4_all_ones_weights(orc):
    """q = 1, s = 1 everywhere -> W = ones: G = U = sum(x) for every row, Y = I * h."""
    T, H, I = 3, 256, 128
    rng = np.random.default_rng(0)
    x = rng.standard_normal((T, H)).astype(np.float32)
    xb = _bits(x)
    one = np.uint16(0x3F80)
    L = dict(dims=dict(T=T, H=H, E=1, I=I, k=1, Is=0, wfmt="int4"), x=xb,
             logits=np.zeros((T, 1), np.float32),
             w_gate=np.full((1, I, H // 2), 0x11, np.uint8), w_up=np.full((1, I, H // 2), 0x11, np.uint8),
             w_down=np.full((1, H, I // 2), 0x11, np.uint8),
             s_gate=np.full((1, I, H // 128), one), s_up=np.full((1, I, H // 128), one),
             s_down=np.full((1, H, I // 128), one))
    out, _ = orc.layer(L)
    xd = (xb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    for t in range(T):
        S = xd[t].sum()
        h = S / (1 + math.exp(-S)) * S
        # h is rounded to bf16 once (its rounding is pinned in the format tests)
        hb = (np.uint32(orc.double_to_bf16(h)) << 16).view(np.float32)
        assert np.allclose(out[t], I * float(hb), rtol=1e-15)


def test_int4_negative_nibbles(orc):
    """Nibble 0x9 is -7, 0xF is -1, 0x7 is +7: a one-hot input reads single weights back."""
    H, I = 128, 128
    wg = np.zeros((1, I, H // 2), np.uint8)
    wg[0, 0, 0] = 0xF9  # k=0 -> -7, k=1 -> -1
    wg[0, 1, 0] = 0x07  # k=0 -> +7, k=1 -> 0
    wu = np.zeros((1, I, H // 2), np.uint8)
    wu[0, :, 0] = 0x11
    wd = np.zeros((1, H, I // 2), np.uint8)
    wd[0, 5, 0] = 0x01  # Y[5] = h[0]
    wd[0, 6, 0] = 0x10  # Y[6] = h[1]
    s = lambda *shape: np.full(shape, np.uint16(0x3F80))
    x = np.zeros((2, H), np.float32)
    x[0, 0] = 1.0  # picks column k = 0
    x[1, 1] = 1.0  # picks column k = 1
    L = dict(dims=dict(T=2, H=H, E=1, I=I, k=1, Is=0, wfmt="int4"), x=_bits(x),
             logits=np.zeros((2, 1), np.float32), w_gate=wg, w_up=wu, w_down=wd,
             s_gate=s(1, I, 1), s_up=s(1, I, 1), s_down=s(1, H, 1))
    out, _ = orc.layer(L)
    silu = lambda z: z / (1 + math.exp(-z))
    b = lambda v: float((np.uint32(orc.double_to_bf16(v)) << 16).view(np.float32))
    assert out[0, 5] == b(silu(-7.0) * 1.0) and out[0, 6] == b(silu(7.0) * 1.0)
    assert out[1, 5] == b(silu(-1.0) * 1.0) and out[1, 6] == 0.0


def test_token_subset_equals_full_rows(orc):
    L = moe_synth.to_numpy(moe_synth.make_layer(SMALL[1]))
    full, fullb = orc.layer(L)
    sel = np.array([4, 0, 2], np.int32)
    part, partb = orc.layer(L, sel, nthreads=2)
    assert np.array_equal(part, full[sel]) and np.array_equal(partb, fullb[sel])


def test_shared_expert_adds_with_weight_one(orc):
    cfg = dict(SMALL[1])
    L = moe_synth.to_numpy(moe_synth.make_layer(cfg))
    with_shared, _ = orc.layer(L)
    L0 = dict(L)
    L0["dims"] = dict(L["dims"], Is=0)
    routed, _ = orc.layer(L0)
    Ls = dict(L)
    Ls["dims"] = dict(L["dims"], E=1, k=1, I=L["dims"]["Is"], Is=0)
    Ls["w_gate"], Ls["w_up"], Ls["w_down"] = L["ws_gate"], L["ws_up"], L["ws_down"]
    Ls["s_gate"], Ls["s_up"], Ls["s_down"] = L["ss_gate"], L["ss_up"], L["ss_down"]
    Ls["logits"] = np.zeros((cfg["T"], 1), np.float32)
    shared, _ = orc.layer(Ls)
    assert np.allclose(with_shared, routed + shared, rtol=1e-14, atol=1e-14)


def test_h_on_a_rounding_midpoint_reports_the_envelope(orc):
    """G = 64 (silu(64) = 64 in fp64), U = (7, 2.625): h = (448, 168) exactly, so s_h = 1 and
    h[1] = 168 is the midpoint between the e4m3 values 160 and 176.  Round-to-nearest-even
    takes 160; 176 is an equally valid outcome for an fp32 h one ulp higher, so the envelope
    of output n is 16 * |Wd[n, 1]|, and zero in every output that h[1] does not reach."""
    H, I = 512, 2
    x = np.zeros((1, H), np.float32)
    x[0, 0], x[0, 1], x[0, 511] = 1.0, 1.0, 448.0
    wg = np.zeros((1, I, H), np.uint8)
    wu = np.zeros((1, I, H), np.uint8)
    wg[0, :, 0] = _code(orc, 64.0)
    wu[0, 0, 0] = _code(orc, 7.0)
    wu[0, 1, 0], wu[0, 1, 1] = _code(orc, 2.5), _code(orc, 0.125)
    rng = np.random.default_rng(5)
    wd = np.zeros((1, H, I), np.uint8)
    wd[0, :, 0] = rng.integers(0x10, 0x30, H)
    wd[0, :200, 1] = rng.integers(0x10, 0x30, 200) | (rng.integers(0, 2, 200) << 7).astype(np.uint8)
    ones = lambda *s: np.ones(s, np.float32)
    L = dict(dims=dict(T=1, H=H, E=1, I=I, k=1, Is=0, wfmt="fp8"), x=_bits(x),
             logits=np.zeros((1, 1), np.float32), w_gate=wg, w_up=wu, w_down=wd,
             s_gate=ones(1, I, 1), s_up=ones(1, I, 1), s_down=ones(1, H, 1))
    out, _, amb = orc.layer(L, ambiguity=True)
    dec = lambda c: np.array([orc.e4m3_decode(int(v)) for v in c])
    d0, d1 = dec(wd[0, :, 0]), dec(wd[0, :, 1])
    assert np.array_equal(out[0], 448.0 * d0 + 160.0 * d1)
    assert np.array_equal(amb[0], 16.0 * np.abs(d1))
    assert np.all(amb[0, 200:] == 0) and np.all(amb[0, :200] > 0)


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: f"{c['wfmt']}-T{c['T']}-H{c['H']}-I{c['I']}-Is{c['Is']}")
def test_envelope_does_not_change_the_layer_and_stays_small(orc, cfg):
    """Asking for the envelope leaves the outputs unchanged, and on random layers the envelope
    is a small part of the tolerance for a typical output: only the few h values whose window
    reaches a rounding boundary contribute, each by one step of the coarse format."""
    L = moe_synth.to_numpy(moe_synth.make_layer(cfg))
    out, outb, amb = orc.layer(L, ambiguity=True)
    out2, _ = orc.layer(L)
    assert np.array_equal(out, out2)
    assert np.all(amb >= 0)
    assert np.median(amb / (2e-3 + 1e-2 * np.abs(out))) < 0.05
