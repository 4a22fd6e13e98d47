"""Seeded synthetic inputs for the routed MoE FFN layer.

This module only draws random numbers and stores them in the layer's input formats; it holds
none of the layer's own arithmetic (routing, permutation, activation quantisation, the expert
contractions, the combine).  Both the CUDA path's tests/benchmark and the CPU oracle consume
the same bytes produced here.

Recipe (every tensor has its own seeded torch generator on the chosen device):
  * x       ~ N(0, 1), rounded to bf16 (RNE) -- the hidden states;
  * logits  ~ N(0, 1) fp32, plus a per-expert bias for two workloads:
      - "normal": bias_e ~ N(0, 0.5) (0.5 read as the variance);
      - "zipf":   bias_e = -1.2 * ln(rank_e), rank a seeded permutation of 1..E
                  (the log of a Zipf(s = 1.2) probability up to a constant), so a few
                  experts take most tokens;
  * weights W ~ N(0, 1/fan_in) fp32 (fan_in = H for gate/up, I for down), stored quantised:
      - FP8: one fp32 scale per (row, 512-element K block), s = amax/448 (1 when amax = 0),
             codes = e4m3(W/s) by torch's float8_e4m3fn conversion (round to nearest even);
      - int4: one bf16 scale per (row, 128-element K group), s = bf16(amax/7) (1 when 0),
             q = clamp(round_half_even(W/s), -7, 7), two's-complement nibbles, the even K
             index in the low nibble;
      - MXFP4: one E8M0 byte per (row, 32-element K block) holding the exponent
             x = floor(log2(amax)) - 2 (the largest E2M1 power of two is 2^2; 0 when
             amax = 0), stored as x + 127; each element is W / 2^x rounded to the nearest
             E2M1 value (ties to the even code, magnitudes above 6 saturate to 6), the
             even K index in the low nibble;
      - NVFP4: one fp32 tensor scale per expert matrix, t = amax / (448 * 6) (1 when 0);
             one E4M3 byte per (row, 16-element K block), s = e4m3(amax_block / (6 t))
             (torch's cast, round to nearest even, at least 2^-9; 1 for an all-zero block);
             each element is W / (s t) rounded to the nearest E2M1 value as for MXFP4.
Shapes follow the pages' models: a Qwen3.5-397B-shaped layer (512 experts x 1024, top-10,
one shared expert of 1024, hidden 4096) at decode and prefill sizes; a DeepSeek-R1-shaped
layer (hidden 7168, 256 experts x 2048, top-8, shared 2048) with skewed routing; a 4-bit
128-expert layer (int4, and the same shape with MXFP4 weights); and a tiny layer for the oracle.
"""
from __future__ import annotations

import math

import numpy as np
import torch

CONFIGS = {
    "tiny": dict(T=16, H=512, E=8, I=256, k=2, Is=0, wfmt="fp8", seed=0, bias=None,
                 workload="tiny MoE layer T=16 H=512 E=8 I=256 top-2, FP8 e4m3 sc512"),
    "decode": dict(T=512, H=4096, E=512, I=1024, k=10, Is=1024, wfmt="fp8", seed=1, bias=None,
                   workload="Qwen3.5-397B-shaped MoE decode step T=512 H=4096 E=512 I=1024 "
                            "top-10 + shared 1024, FP8 e4m3 sc512"),
    "prefill": dict(T=8192, H=4096, E=512, I=1024, k=10, Is=1024, wfmt="fp8", seed=2,
                    bias="normal",
                    workload="Qwen3.5-397B-shaped MoE prefill T=8192 H=4096 E=512 I=1024 "
                             "top-10 + shared 1024, FP8 e4m3 sc512, biased logits"),
    "skewed": dict(T=4096, H=7168, E=256, I=2048, k=8, Is=2048, wfmt="fp8", seed=3, bias="zipf",
                   workload="DeepSeek-R1-shaped MoE T=4096 H=7168 E=256 I=2048 top-8 + shared "
                            "2048, FP8 e4m3 sc512, Zipf-skewed routing"),
    "int4": dict(T=1024, H=4096, E=128, I=1536, k=8, Is=0, wfmt="int4", seed=4, bias=None,
                 workload="4-bit-weight MoE T=1024 H=4096 E=128 I=1536 top-8, int4 g128 bf16"),
    "mxfp4": dict(T=1024, H=4096, E=128, I=1536, k=8, Is=0, wfmt="mxfp4", seed=8, bias=None,
                  workload="MXFP4-weight MoE T=1024 H=4096 E=128 I=1536 top-8, e2m1 + E8M0/32, bf16"),
    "nvfp4": dict(T=1024, H=4096, E=128, I=1536, k=8, Is=0, wfmt="nvfp4", seed=10, bias=None,
                  workload="NVFP4-weight MoE T=1024 H=4096 E=128 I=1536 top-8, e2m1 + E4M3/16 + fp32 "
                           "tensor scale, bf16"),
}

# Smaller layers with the same per-expert shapes, for profiler captures (weights still far
# larger than the 126 MB L2, a few GB on the device at most).
PROFILE_CONFIGS = {
    "profile-decode": dict(T=64, H=4096, E=64, I=1024, k=10, Is=1024, wfmt="fp8", seed=5, bias=None,
                           workload="decode-shaped MoE T=64 H=4096 E=64 I=1024 top-10 + shared 1024, FP8"),
    "profile-prefill": dict(T=1024, H=4096, E=64, I=1024, k=10, Is=1024, wfmt="fp8", seed=6, bias="normal",
                            workload="prefill-shaped MoE T=1024 H=4096 E=64 I=1024 top-10 + shared 1024, FP8"),
    "profile-int4": dict(T=128, H=4096, E=16, I=1536, k=8, Is=0, wfmt="int4", seed=7, bias=None,
                         workload="4-bit MoE T=128 H=4096 E=16 I=1536 top-8, int4 g128"),
    "profile-mxfp4": dict(T=128, H=4096, E=16, I=1536, k=8, Is=0, wfmt="mxfp4", seed=9, bias=None,
                          workload="MXFP4 MoE T=128 H=4096 E=16 I=1536 top-8, e2m1 + E8M0/32"),
    "profile-nvfp4": dict(T=128, H=4096, E=16, I=1536, k=8, Is=0, wfmt="nvfp4", seed=11, bias=None,
                          workload="NVFP4 MoE T=128 H=4096 E=16 I=1536 top-8, e2m1 + E4M3/16 + tensor scale"),
    # 16 tokens: the single-kernel small-batch path
    "profile-small": dict(T=16, H=4096, E=64, I=1024, k=10, Is=1024, wfmt="fp8", seed=12, bias=None,
                          workload="decode-shaped MoE T=16 H=4096 E=64 I=1024 top-10 + shared 1024, FP8"),
}

# tensor ids for the per-tensor generators
_TID = {"x": 1, "logits": 2, "bias": 3, "rank": 4, "w_gate": 5, "w_up": 6, "w_down": 7,
        "ws_gate": 8, "ws_up": 9, "ws_down": 10, "w_router": 11}


def _gen(seed: int, tid: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1_000_003 + tid * 7919 + 17)
    return g


def _quant_fp8(w: torch.Tensor):
    """W [..., N, K] fp32 -> (codes uint8 [..., N, K], scales fp32 [..., N, ceil(K/512)])."""
    K = w.shape[-1]
    nb = (K + 511) // 512
    pad = nb * 512 - K
    wp = torch.nn.functional.pad(w, (0, pad)) if pad else w
    blk = wp.reshape(*w.shape[:-1], nb, 512)
    amax = blk.abs().amax(dim=-1)
    s = torch.where(amax == 0, torch.ones_like(amax), amax / 448.0)
    q = (blk / s.unsqueeze(-1)).clamp(-448.0, 448.0).to(torch.float8_e4m3fn)
    q = q.reshape(*w.shape[:-1], nb * 512)[..., :K].contiguous().view(torch.uint8)
    return q, s.contiguous()


def _quant_int4(w: torch.Tensor):
    """W [..., N, K] fp32 -> (packed uint8 [..., N, K/2], scales bf16 [..., N, K/128])."""
    K = w.shape[-1]
    assert K % 128 == 0
    blk = w.reshape(*w.shape[:-1], K // 128, 128)
    amax = blk.abs().amax(dim=-1)
    s = (amax / 7.0).to(torch.bfloat16)
    s = torch.where(s == 0, torch.ones_like(s), s)
    q = torch.round(blk / s.float().unsqueeze(-1)).clamp(-7, 7).to(torch.int16)
    q = q.reshape(*w.shape[:-1], K) & 0xF
    packed = (q[..., 0::2] | (q[..., 1::2] << 4)).to(torch.uint8)
    return packed.contiguous(), s.contiguous()


# E2M1 magnitude code of 2 * |value| for the representable magnitudes 0, 0.5, ..., 6
_E2M1_CODE_OF_2V = {0: 0, 1: 1, 2: 2, 3: 3, 4: 4, 6: 5, 8: 6, 12: 7}


def _e2m1_packed(v: torch.Tensor, shape):
    """Values v (already divided by their scales) -> nearest E2M1 nibbles (ties to the even
    code, magnitudes above 6 saturate), packed two per byte with the even K index low."""
    a = v.abs()
    step = torch.where(a < 2, 0.5, torch.where(a < 4, 1.0, 2.0))
    q2 = (torch.round(a / step) * step).clamp(max=6.0) * 2  # 2|q| in {0, 1, 2, 3, 4, 6, 8, 12}
    lut = torch.zeros(13, dtype=torch.int16, device=v.device)
    for k2, c in _E2M1_CODE_OF_2V.items():
        lut[k2] = c
    mag = lut[q2.long()]
    nib = torch.where((v < 0) & (mag > 0), mag | 8, mag).reshape(shape)
    return (nib[..., 0::2] | (nib[..., 1::2] << 4)).to(torch.uint8).contiguous()


def _quant_mxfp4(w: torch.Tensor):
    """W [..., N, K] fp32 -> (packed uint8 [..., N, K/2], E8M0 scales uint8 [..., N, K/32])."""
    K = w.shape[-1]
    assert K % 32 == 0
    blk = w.reshape(*w.shape[:-1], K // 32, 32).float()
    amax = blk.abs().amax(dim=-1)
    _, e = torch.frexp(amax)  # amax = m * 2^e, m in [0.5, 1): floor(log2(amax)) = e - 1
    xexp = torch.where(amax == 0, torch.zeros_like(e), e - 1 - 2).clamp(-127, 127)
    # dividing by a power of two and the rounding steps are exact in fp32
    v = blk / torch.pow(2.0, xexp.float()).unsqueeze(-1)
    return _e2m1_packed(v, w.shape), (xexp + 127).to(torch.uint8).contiguous()


def _quant_nvfp4(w: torch.Tensor):
    """W [E, N, K] fp32 -> (packed uint8 [E, N, K/2], E4M3 scales uint8 [E, N, K/16],
    tensor scales fp32 [E])."""
    E, N, K = w.shape
    assert K % 16 == 0
    amax_t = w.abs().reshape(E, -1).amax(dim=1)
    t = torch.where(amax_t == 0, torch.ones_like(amax_t), amax_t / (448.0 * 6.0))
    blk = w.reshape(E, N, K // 16, 16).float()
    amax = blk.abs().amax(dim=-1)
    target = (amax / (6.0 * t.view(E, 1, 1))).clamp(min=2.0 ** -9, max=448.0)
    s = target.to(torch.float8_e4m3fn).float()
    s = torch.where(amax == 0, torch.ones_like(s), s)
    v = blk / (s * t.view(E, 1, 1)).unsqueeze(-1)
    codes = s.to(torch.float8_e4m3fn).view(torch.uint8).contiguous()
    return _e2m1_packed(v, w.shape), codes, t.contiguous()


_QUANT = {"fp8": _quant_fp8, "int4": _quant_int4, "mxfp4": _quant_mxfp4, "nvfp4": _quant_nvfp4}


def _weights(seed, tid, shape, fan_in, wfmt, device, chunk_elems=1 << 28):
    """Draw W ~ N(0, 1/fan_in) of `shape` [E, N, K] in expert chunks and quantise."""
    E, N, K = shape
    g = _gen(seed, tid, device)
    per = max(1, chunk_elems // (N * K))
    parts = []
    for e0 in range(0, E, per):
        e1 = min(E, e0 + per)
        w = torch.randn((e1 - e0, N, K), generator=g, device=device, dtype=torch.float32)
        w.mul_(1.0 / math.sqrt(fan_in))
        parts.append(_QUANT[wfmt](w))
        del w
    # (codes, scales) or, for NVFP4, (codes, scales, tensor scales)
    return tuple(torch.cat([p[i] for p in parts], 0) for i in range(len(parts[0])))


def make_layer(name_or_cfg, device="cpu", **overrides) -> dict:
    """Build one synthetic layer.  Returns a dict of torch tensors on `device` plus "dims"."""
    if isinstance(name_or_cfg, str):
        cfg = dict(CONFIGS[name_or_cfg] if name_or_cfg in CONFIGS else PROFILE_CONFIGS[name_or_cfg])
    else:
        cfg = dict(name_or_cfg)
    cfg.update(overrides)
    T, H, E, I, k, Is = (cfg[n] for n in ("T", "H", "E", "I", "k", "Is"))
    seed, wfmt = cfg["seed"], cfg["wfmt"]
    out = {"dims": dict(T=T, H=H, E=E, I=I, k=k, Is=Is, wfmt=wfmt), "cfg": cfg}
    x = torch.randn((T, H), generator=_gen(seed, _TID["x"], device), device=device)
    out["x"] = x.to(torch.bfloat16)
    logits = torch.randn((T, E), generator=_gen(seed, _TID["logits"], device), device=device)
    if cfg.get("bias") == "normal":
        b = torch.randn((E,), generator=_gen(seed, _TID["bias"], device), device=device)
        logits = logits + b * math.sqrt(0.5)
    elif cfg.get("bias") == "zipf":
        rank = torch.randperm(E, generator=_gen(seed, _TID["rank"], device), device=device) + 1
        logits = logits + (-1.2) * torch.log(rank.to(torch.float32))
    out["logits"] = logits.contiguous()
    mats = [("gate", (E, I, H), H, ""), ("up", (E, I, H), H, ""), ("down", (E, H, I), I, "")]
    if Is > 0:
        mats += [("gate", (1, Is, H), H, "s"), ("up", (1, Is, H), H, "s"), ("down", (1, H, Is), Is, "s")]
    for proj, shape, fan_in, sh in mats:
        res = _weights(seed, _TID[f"w{sh}_{proj}"], shape, fan_in, wfmt, device)
        out[f"w{sh}_{proj}"], out[f"s{sh}_{proj}"] = res[0], res[1]
        if len(res) > 2:
            out[f"t{sh}_{proj}"] = res[2]
    return out


def make_router(name_or_cfg, device="cpu", **overrides) -> torch.Tensor:
    """Router weights W_router [E, H] ~ N(0, 1/H), bf16 (so x . W_router^T ~ N(0, 1))."""
    if isinstance(name_or_cfg, str):
        cfg = dict(CONFIGS[name_or_cfg] if name_or_cfg in CONFIGS else PROFILE_CONFIGS[name_or_cfg])
    else:
        cfg = dict(name_or_cfg)
    cfg.update(overrides)
    g = _gen(cfg["seed"], _TID["w_router"], device)
    w = torch.randn((cfg["E"], cfg["H"]), generator=g, device=device) / math.sqrt(cfg["H"])
    return w.to(torch.bfloat16)


def to_numpy(layer: dict) -> dict:
    """Host copies with bf16 tensors as uint16 bit patterns (the oracle's input format)."""
    res = {"dims": dict(layer["dims"])}
    for key, v in layer.items():
        if not isinstance(v, torch.Tensor):
            continue
        v = v.detach().cpu().contiguous()
        if v.dtype == torch.bfloat16:
            v = v.view(torch.int16).numpy().view(np.uint16)
        else:
            v = v.numpy()
        res[key] = v
    return res


def weight_bytes(layer: dict) -> int:
    return sum(v.numel() * v.element_size() for key, v in layer.items()
               if isinstance(v, torch.Tensor) and key[:2] in ("w_", "s_", "ws", "ss", "t_", "ts"))
