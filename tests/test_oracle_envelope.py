"""Pins of the oracle's envelope of equally valid outputs (reading R10a).

The layer holds h = silu(G) * U in fp32 and rounds it to a coarser format: e4m3 codes per
512-block for FP8 layers (reading R10), bf16 for the 4-bit layers (reading R11).  Where the exact
h lies within the rounding budget of an fp32 evaluation of G and U from a rounding boundary of
that format, both neighbours are valid results, and the oracle reports, per output, the largest
move the alternatives allow through the down projection.  These cases put h exactly on a
boundary (bf16 for int4, MXFP4 and NVFP4; e4m3 with and without cancellation in G), so the
envelope has a closed form: one step of the coarse format times |W_down| (times the NVFP4 down
matrix's tensor scale), in the outputs that element reaches and nowhere else.
"""
import numpy as np
import pytest
import torch


def _bits(x) -> np.ndarray:
    return torch.as_tensor(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _bf16(v) -> np.uint16:
    return _bits([v])[0]


# E2M1 codes of the magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 (format definition: S.EE.M, bias 1)
_E2M1 = {0.0: 0, 0.5: 1, 1.0: 2, 1.5: 3, 2.0: 4, 3.0: 5, 4.0: 6, 6.0: 7}


def _pack(nibbles: np.ndarray) -> np.ndarray:
    """[N, K] nibbles (0..15) -> [N, K/2] bytes, the even K index in the low nibble."""
    n = nibbles.astype(np.uint8)
    return (n[:, 0::2] | (n[:, 1::2] << 4)).astype(np.uint8)


def _e4m3_byte(v: float) -> int:
    return int(torch.tensor([v]).to(torch.float8_e4m3fn).view(torch.uint8)[0])


class W4:
    """One 4-bit [N, K] weight matrix built element by element with exact values."""

    def __init__(self, fmt, N, K):
        self.fmt, self.N, self.K = fmt, N, K
        self.nib = np.zeros((N, K), np.uint8)
        blk = {"int4": 128, "mxfp4": 32, "nvfp4": 16}[fmt]
        self.blk = blk
        if fmt == "int4":
            self.s = np.full((N, K // blk), _bf16(1.0), np.uint16)
        elif fmt == "mxfp4":
            self.s = np.full((N, K // blk), 127, np.uint8)
        else:
            self.s = np.full((N, K // blk), _e4m3_byte(1.0), np.uint8)

    def set(self, n, i, mag, scale, neg=False):
        """W[n, i] = (+-mag) * scale, with `scale` the block scale of (n, i // blk)."""
        b = i // self.blk
        if self.fmt == "int4":
            q = int(mag) * (-1 if neg else 1)
            self.nib[n, i] = q & 0xF
            self.s[n, b] = _bf16(scale)
        else:
            self.nib[n, i] = _E2M1[mag] | (8 if neg else 0)
            if self.fmt == "mxfp4":
                self.s[n, b] = 127 + int(np.log2(scale))
            else:
                self.s[n, b] = _e4m3_byte(scale)

    def value(self, n, i):
        b = i // self.blk
        nb = int(self.nib[n, i])
        if self.fmt == "int4":
            q = nb - 16 if nb >= 8 else nb
            sc = float(torch.tensor([int(self.s[n, b])], dtype=torch.int16).view(torch.bfloat16).float()[0])
            return q * sc
        mag = {v: k for k, v in _E2M1.items()}[nb & 7] * (-1 if nb & 8 else 1)
        if self.fmt == "mxfp4":
            return mag * 2.0 ** (int(self.s[n, b]) - 127)
        return mag * float(torch.tensor([int(self.s[n, b])], dtype=torch.uint8).view(torch.float8_e4m3fn).float()[0])

    def arrays(self):
        return _pack(self.nib)[None], self.s[None]


@pytest.mark.parametrize("fmt", ["int4", "mxfp4", "nvfp4"])
def test_bf16_h_on_a_rounding_midpoint(orc, fmt):
    """G = 64 (silu(64) = 64 in fp64) and U = 2^-6 + 2^-14, so h = 1 + 2^-8 exactly: the midpoint
    of the bf16 values 1 and 1 + 2^-7.  Round-to-nearest-even takes 1; 1 + 2^-7 is equally valid,
    so the envelope of output n is 2^-7 * |W_down[n, 0]| (times t_down for NVFP4).  The other
    features have U = 0 from no terms at all (h = 0 exactly, no alternative) and add nothing."""
    H, I = 256, 128
    x = np.zeros((1, H), np.float32)
    second = {"int4": 128, "mxfp4": 32, "nvfp4": 16}[fmt]  # first index of another scale block
    x[0, 0] = x[0, second] = 1.0
    t_up, t_down = (2.0 ** -5, 2.0) if fmt == "nvfp4" else (1.0, 1.0)
    wg, wu, wd = W4(fmt, I, H), W4(fmt, I, H), W4(fmt, H, I)
    for n in (0, 1):
        wg.set(n, 0, 4.0 if fmt != "int4" else 1, 16.0 if fmt != "int4" else 64.0)  # G = 64
    # U[0] = 2^-6 + 2^-14 (after the up matrix's tensor scale for NVFP4)
    wu.set(0, 0, 1.0 if fmt != "int4" else 1, 2.0 ** -6 / t_up)
    wu.set(0, second, 1.0 if fmt != "int4" else 1, 2.0 ** -14 / t_up)
    rng = np.random.default_rng(3)
    reach = 200
    for n in range(reach):
        mag = [1.0, 2.0, 3.0, 6.0][rng.integers(4)] if fmt != "int4" else int(rng.integers(1, 8))
        wd.set(n, 0, mag, 0.125, neg=bool(rng.integers(2)))
    (pg, sg), (pu, su), (pd, sd) = wg.arrays(), wu.arrays(), wd.arrays()
    L = dict(dims=dict(T=1, H=H, E=1, I=I, k=1, Is=0, wfmt=fmt), x=_bits(x),
             logits=np.zeros((1, 1), np.float32), w_gate=pg, w_up=pu, w_down=pd, s_gate=sg, s_up=su, s_down=sd)
    if fmt == "nvfp4":
        L.update(t_gate=np.ones(1, np.float32), t_up=np.full(1, t_up, np.float32),
                 t_down=np.full(1, t_down, np.float32))
    out, _, amb = orc.layer(L, ambiguity=True)
    wd0 = np.array([wd.value(n, 0) for n in range(H)])
    # h rounds to 1.0 (ties to even): out = 1.0 * W_down[:, 0] * t_down exactly
    assert np.array_equal(out[0], wd0 * t_down)
    assert np.array_equal(amb[0], 2.0 ** -7 * np.abs(wd0) * t_down)
    assert np.all(amb[0, reach:] == 0) and np.all(amb[0, :reach] > 0)


def test_bf16_envelope_is_zero_off_the_midpoint(orc):
    """The same int4 layer with U = 2^-6 + 2^-13 (h = 1 + 2^-7, a bf16 value, far from every
    rounding midpoint) has no alternative and an all-zero envelope."""
    H, I = 256, 128
    x = np.zeros((1, H), np.float32)
    x[0, 0] = x[0, 128] = 1.0
    wg, wu, wd = W4("int4", I, H), W4("int4", I, H), W4("int4", H, I)
    wg.set(0, 0, 1, 64.0)
    wu.set(0, 0, 1, 2.0 ** -6)
    wu.set(0, 128, 1, 2.0 ** -13)
    for n in range(H):
        wd.set(n, 0, 3, 0.125)
    (pg, sg), (pu, su), (pd, sd) = wg.arrays(), wu.arrays(), wd.arrays()
    L = dict(dims=dict(T=1, H=H, E=1, I=I, k=1, Is=0, wfmt="int4"), x=_bits(x),
             logits=np.zeros((1, 1), np.float32), w_gate=pg, w_up=pu, w_down=pd, s_gate=sg, s_up=su, s_down=sd)
    out, _, amb = orc.layer(L, ambiguity=True)
    assert np.array_equal(out[0], np.full(H, (1.0 + 2.0 ** -7) * 0.375))
    assert np.all(amb == 0)


def _fp8_code(orc, v):
    return int(orc.e4m3_encode(np.float32(v))[0])


def _fp8_midpoint_layer(orc, cancel: float, rel: float):
    """FP8 layer with two features.  Feature 0: G = 64, U = 7, h = 448 (the block amax, so the
    h scale is 1).  Feature 1: G = 64 (+ cancel*448 - cancel*448, leaving G unchanged but not the
    sum of the magnitudes of its products) and U = 2.625 * (1 + rel), so
    h = 168 (1 + rel): just above the midpoint 168 of the e4m3 values 160 and 176.  The down
    weights of feature 1 are 0.5."""
    H, I = 512, 2
    x = np.zeros((1, H), np.float32)
    x[0, 0] = x[0, 1] = 1.0
    x[0, 32] = x[0, 64] = 448.0
    x[0, 511] = 448.0  # block amax 448: activation scale 1
    wg = np.zeros((1, I, H), np.uint8)
    wu = np.zeros((1, I, H), np.uint8)
    wg[0, :, 0] = _fp8_code(orc, 64.0)
    wu[0, 0, 0] = _fp8_code(orc, 7.0)
    if cancel:
        wg[0, 1, 32] = _fp8_code(orc, cancel)
        wg[0, 1, 64] = _fp8_code(orc, -cancel)
    wu[0, 1, 0], wu[0, 1, 1] = _fp8_code(orc, 2.5), _fp8_code(orc, 0.125)
    wd = np.zeros((1, H, I), np.uint8)
    wd[0, :, 1] = _fp8_code(orc, 0.5)
    su = np.ones((1, I, 1), np.float32)
    su[0, 1, 0] = np.float32(1.0 + rel)
    ones = lambda *s: np.ones(s, np.float32)
    return dict(dims=dict(T=1, H=H, E=1, I=I, k=1, Is=0, wfmt="fp8"), x=_bits(x),
                logits=np.zeros((1, 1), np.float32), w_gate=wg, w_up=wu, w_down=wd,
                s_gate=ones(1, I, 1), s_up=su, s_down=ones(1, H, 1))


def test_fp8_window_follows_the_sum_of_magnitudes(orc):
    """The window of equally valid h values scales with the sum of |products| of G's dot
    product, not with G itself.  With h = 168 (1 + 2^-12), i.e. 0.04 above the midpoint 168:
    without cancellation in G the window is far narrower than that and the code 176 is the only
    valid one (zero envelope); with +-448*448 cancelling inside G (G unchanged) the window covers
    the midpoint and 160 is valid too, so each output moves by up to 16 * 0.5 = 8."""
    rel = 2.0 ** -12
    out0, _, amb0 = orc.layer(_fp8_midpoint_layer(orc, 0.0, rel), ambiguity=True)
    out1, _, amb1 = orc.layer(_fp8_midpoint_layer(orc, 448.0, rel), ambiguity=True)
    assert np.array_equal(out0, out1)           # the cancelling terms leave G and the layer alone
    assert np.all(out0 == 176.0 * 0.5)  # h = 168.04 rounds to 176; feature 0 has no down weights
    assert np.all(amb0 == 0)
    assert np.all(amb1 == 8.0)
