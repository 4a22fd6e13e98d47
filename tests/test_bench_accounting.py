"""bench.py's roofline accounting, pinned on the CPU: the algorithmic bytes of each GEMM equal
the bytes of the weight and scale tensors of the experts that received tokens (counted from
the tensors moe_synth builds), and the FLOPs equal 2*M*N*K summed over the GEMMs."""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
import moe_synth  # noqa: E402


def _tensor_bytes(t):
    return t.numel() * t.element_size()


@pytest.mark.parametrize("wfmt", ["fp8", "int4", "mxfp4", "nvfp4"])
@pytest.mark.parametrize("Is", [0, 256])
def test_gemm_bytes_are_the_touched_experts_tensors(wfmt, Is):
    cfg = dict(T=24, H=1024, E=8, I=384, k=2, Is=Is, seed=70, bias=None, wfmt=wfmt)
    layer = moe_synth.make_layer(cfg)
    counts = np.array([3, 0, 5, 0, 0, 1, 2, 1])  # experts 1, 3, 4 untouched
    alg = bench.algorithmic(cfg, counts)
    touched = np.nonzero(counts)[0]
    has = lambda n: n in layer  # NVFP4 adds the per-matrix tensor scales t_*, ts_*
    gu = sum(_tensor_bytes(layer[n][e]) for n in ("w_gate", "w_up", "s_gate", "s_up", "t_gate", "t_up")
             if has(n) for e in touched)
    dn = sum(_tensor_bytes(layer[n][e]) for n in ("w_down", "s_down", "t_down") if has(n) for e in touched)
    if Is:
        gu += sum(_tensor_bytes(layer[n]) for n in ("ws_gate", "ws_up", "ss_gate", "ss_up", "ts_gate", "ts_up")
                  if has(n))
        dn += sum(_tensor_bytes(layer[n]) for n in ("ws_down", "ss_down", "ts_down") if has(n))
    assert alg["touched"] == len(touched)
    assert alg["gemm_gateup"] == gu
    assert alg["gemm_down"] == dn


def test_flops_are_two_mnk_per_gemm():
    cfg = dict(T=24, H=1024, E=8, I=384, k=2, Is=256, seed=70, bias=None, wfmt="fp8")
    alg = bench.algorithmic(cfg, np.ones(8, int))
    T, H, I, k, Is = 24, 1024, 384, 2, 256
    gateup = 2 * (T * k) * (2 * I) * H + 2 * T * (2 * Is) * H
    down = 2 * (T * k) * H * I + 2 * T * H * Is
    assert alg["flops_gemm_gateup"] == gateup
    assert alg["flops_gemm_down"] == down
    assert alg["flops"] == gateup + down


def test_traffic_figure_is_tied_to_the_kernel_source():
    """The stored DRAM-traffic ratio names the hash of the kernel source it was measured on;
    bench.py reports it only while that source is unchanged."""
    tr = bench.TRAFFIC["decode"]
    assert 1.0 <= tr["ratio"] < 1.1
    assert len(tr["src_sha"]) == 16
    sha = bench.src_sha(os.path.join(ROOT, "mixture_experts_ffn_13_b200", "csrc", "gemm_fp8.cu"))
    assert isinstance(sha, str) and len(sha) == 16
