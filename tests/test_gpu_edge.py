"""Edge cases of the CUDA path through the C ABI: degenerate routing shapes, the largest
supported E and k, argument errors that need a device plan, and the bounded device wait."""
import ctypes

import numpy as np
import pytest
import torch

import moe_synth
import oracle
import mixture_experts_ffn_13_b200 as moe
from test_gpu_parity import check_out, check_route

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    moe.load_library()


def _layer_parity(cfg):
    layer = moe_synth.make_layer(cfg, device="cuda")
    m = moe.MoELayer(layer)
    out = m(layer["x"], layer["logits"])
    assert moe.moe_get_status(m.plan) == 0
    want, _, amb = oracle.layer(moe_synth.to_numpy(layer), ambiguity=True)
    check_out(out, want, str(cfg), amb)
    check_route(m.plan, m.workspace, layer["logits"], cfg["k"])
    return m, layer


@pytest.mark.parametrize("cfg", [
    dict(T=50, H=512, E=8, I=256, k=8, Is=128, seed=51, bias=None, wfmt="fp8"),     # k = E: every expert
    dict(T=40, H=512, E=1, I=384, k=1, Is=0, seed=52, bias=None, wfmt="fp8"),       # one expert: a dense FFN
    dict(T=33, H=256, E=64, I=128, k=32, Is=0, seed=53, bias=None, wfmt="fp8"),     # the largest k
    dict(T=64, H=256, E=1024, I=128, k=4, Is=128, seed=54, bias="zipf", wfmt="fp8"),  # the largest E
    dict(T=24, H=256, E=4, I=128, k=4, Is=0, seed=55, bias=None, wfmt="int4"),      # k = E, 4-bit
    dict(T=9, H=256, E=1, I=256, k=1, Is=128, seed=56, bias=None, wfmt="int4"),     # one 4-bit expert + shared
    dict(T=24, H=256, E=4, I=128, k=4, Is=0, seed=59, bias=None, wfmt="mxfp4"),     # k = E, MXFP4
    dict(T=9, H=128, E=1, I=256, k=1, Is=128, seed=60, bias=None, wfmt="mxfp4"),    # one MXFP4 expert + shared
    dict(T=24, H=256, E=4, I=128, k=4, Is=0, seed=61, bias=None, wfmt="nvfp4"),     # k = E, NVFP4
    dict(T=9, H=128, E=1, I=256, k=1, Is=128, seed=62, bias=None, wfmt="nvfp4"),    # one NVFP4 expert + shared
], ids=lambda c: f"{c['wfmt']}-T{c['T']}-E{c['E']}-k{c['k']}-Is{c['Is']}")
def test_degenerate_and_extreme_shapes(cfg):
    _layer_parity(cfg)


def test_identical_logits_everywhere():
    """Every token ties on every expert: the k lowest indices win, weights are uniform."""
    cfg = dict(T=70, H=512, E=16, I=128, k=4, Is=0, seed=57, bias=None, wfmt="fp8")
    layer = moe_synth.make_layer(cfg, device="cuda")
    layer["logits"] = torch.zeros_like(layer["logits"])
    m = moe.MoELayer(layer)
    r = m.route(layer["logits"])
    torch.cuda.synchronize()
    assert np.array_equal(r["topk_idx"].cpu().numpy(), np.tile(np.arange(4, dtype=np.int32), (70, 1)))
    assert np.allclose(r["topk_w"].cpu().numpy(), 0.25)
    out = m(layer["x"], layer["logits"])
    want, _, amb = oracle.layer(moe_synth.to_numpy(layer), ambiguity=True)
    check_out(out, want, "ties", amb)


def test_argument_errors_need_no_device_work():
    cfg = dict(T=16, H=512, E=8, I=256, k=2, Is=0, seed=58, bias=None, wfmt="fp8")
    layer = moe_synth.make_layer(cfg, device="cuda")
    m = moe.MoELayer(layer)
    with pytest.raises(moe.MoEError) as ei:  # workspace one byte short
        moe.moe_forward(m.plan, layer["x"], layer["logits"], m.weights, m.workspace[: m.plan.workspace_bytes - 1])
    assert ei.value.code == -3
    with pytest.raises(moe.MoEError) as ei:  # T above the plan's T_max
        big = torch.zeros((17, 512), dtype=torch.bfloat16, device="cuda")
        moe.moe_forward(m.plan, big, torch.zeros((17, 8), device="cuda"), m.weights, m.workspace)
    assert ei.value.code == -1
    L = moe.load_library()
    W = moe._weights_struct(m.weights)
    out = torch.empty((16, 512), dtype=torch.bfloat16, device="cuda")
    x_off = layer["x"].view(-1)[1:].data_ptr()  # 2 bytes past a 16-byte boundary
    rc = L.moe_forward(m.plan.handle, 16, x_off, layer["logits"].data_ptr(), ctypes.byref(W), out.data_ptr(),
                       m.workspace.data_ptr(), m.workspace.numel(), None)
    assert rc == -1
    W.w_down = None
    rc = L.moe_forward(m.plan.handle, 16, layer["x"].data_ptr(), layer["logits"].data_ptr(), ctypes.byref(W),
                       out.data_ptr(), m.workspace.data_ptr(), m.workspace.numel(), None)
    assert rc == -1
    # the plan is still good after rejected calls
    good = m(layer["x"], layer["logits"])
    want, _, amb = oracle.layer(moe_synth.to_numpy(layer), ambiguity=True)
    check_out(good, want, "after errors", amb)


def test_bounded_wait_gives_up_and_reports():
    """A wait on a barrier nothing arrives at ends after its limit with MOE_ERR_DEVICE_TIMEOUT;
    the context stays usable."""
    L = moe.load_library()
    L.moe_test_bounded_wait.argtypes = [ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p]
    L.moe_test_bounded_wait.restype = ctypes.c_int
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    assert L.moe_test_bounded_wait(status.data_ptr(), 10_000, stream) == 0
    torch.cuda.synchronize()
    assert int(status[0]) == -5
    assert L.moe_test_bounded_wait(None, 10, stream) == -1
    assert L.moe_test_bounded_wait(status.data_ptr(), 0, stream) == -1
    # the device still runs the layer correctly afterwards
    _layer_parity(dict(T=16, H=512, E=8, I=256, k=2, Is=0, seed=0, bias=None, wfmt="fp8"))


def test_checked_mode_reports_non_finite_logits():
    """Checked mode: a NaN or infinite router logit is reported as MOE_ERR_BOUNDS through the
    status word (for moe_route and moe_forward); unchecked, nothing is reported; finite logits
    pass; the plan keeps working afterwards."""
    cfg = dict(T=40, H=512, E=16, I=128, k=4, Is=128, seed=65, bias=None, wfmt="fp8")
    layer = moe_synth.make_layer(cfg, device="cuda")
    m = moe.MoELayer(layer)
    bad = layer["logits"].clone()
    bad[7, 3] = float("nan")
    bad[20, 0] = float("inf")
    bad[31, :] = float("nan")                        # a whole row: selection still stays in range
    m(layer["x"], bad)                               # unchecked: no device check
    assert moe.moe_get_status(m.plan) == 0
    moe.moe_set_checked(m.plan, True)
    m(layer["x"], layer["logits"])                   # checked, finite logits: passes
    assert moe.moe_get_status(m.plan) == 0
    m(layer["x"], bad)
    assert moe.moe_get_status(m.plan) == -6          # MOE_ERR_BOUNDS, then the word is cleared
    m.route(bad)
    assert moe.moe_get_status(m.plan) == -6
    out = m(layer["x"], layer["logits"])             # still correct afterwards
    assert moe.moe_get_status(m.plan) == 0
    want, _, amb = oracle.layer(moe_synth.to_numpy(layer), ambiguity=True)
    check_out(out, want, "checked mode", amb)
    moe.moe_set_checked(m.plan, False)


def test_nvfp4_without_tensor_scales_is_rejected():
    """NVFP4 reads one fp32 tensor scale per weight matrix: a missing one is an argument error
    that launches nothing."""
    cfg = dict(T=8, H=256, E=4, I=128, k=2, Is=128, seed=63, bias=None, wfmt="nvfp4")
    layer = moe_synth.make_layer(cfg, device="cuda")
    m = moe.MoELayer(layer)
    for name in ("t_down", "ts_up"):
        w = dict(m.weights)
        del w[name]
        with pytest.raises(moe.MoEError) as ei:
            moe.moe_forward(m.plan, layer["x"], layer["logits"], w, m.workspace)
        assert ei.value.code == -1 and moe.moe_launch_count(m.plan) == 0
