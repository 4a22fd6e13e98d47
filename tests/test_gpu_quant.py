"""Step A2 and the h quantiser, bit for bit against the oracle.

Page "把 397B MoE 榨進 TPU7x：Google 拿到 4.7 倍加速", section "Kernel 手術台": the expert FFN runs
on FP8 with 512-element sub-channel quantisation.  Per (row, 512-block): s = amax / 448 in fp32
(1 for an all-zero block) and q = e4m3(x / s), round to nearest even with saturation (readings
R5, R6, R13).  Both sides make every rounding decision in fp32 with IEEE division, so the codes
and scales must agree exactly: a one-code error here would otherwise hide inside the layer's
output tolerance.  The kernels run through the test entry points of the C ABI on caller
buffers (the same launchers moe_forward uses).
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import mixture_experts_ffn_13_b200 as moe

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = moe.load_library()
    P, I32 = ctypes.c_void_p, ctypes.c_int32
    lib.moe_test_quant_x.argtypes = [I32, I32, I32, P, P, P, P, P]
    lib.moe_test_quant_x.restype = ctypes.c_int
    lib.moe_test_quant_rows.argtypes = [I32, I32, P, P, P, P]
    lib.moe_test_quant_rows.restype = ctypes.c_int
    return lib


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _special_rows(rng, R, K, dtype):
    """Random rows plus the cases the rule singles out: an all-zero row and an all-zero block,
    a block whose amax is 448 (s = 1) holding exact e4m3 midpoints (ties to even), values that
    land in the e4m3 subnormal range after scaling, very large and very small magnitudes."""
    x = rng.standard_normal((R, K)).astype(np.float32)
    x[1] = 0.0
    x[2, :min(512, K)] = 0.0
    blk = x[3, :min(512, K)]
    blk[:] = 0.0
    blk[0] = 448.0
    mids = np.array([17.0, 19.0, 9.5, 0.5625, 0.0029296875, 1.0 + 1.0 / 16, 208.0, 232.0, -17.0, -0.5625])
    blk[1:1 + mids.size] = mids
    x[4] *= 1e-4
    x[4, 7] = 3.0  # one large value: the rest scale into e4m3 subnormals
    x[5] *= 1e30
    x[6] *= 1e-30
    x[7, ::2] = -x[7, ::2] * 7.0
    if dtype == "bf16":
        t = torch.from_numpy(x).to(torch.bfloat16)
        return t.view(torch.int16).numpy().view(np.uint16), t
    return x, torch.from_numpy(x)


@pytest.mark.parametrize("H", [640, 4096, 7168])
def test_quant_x_bit_exact(L, H):
    T, k = 37, 3
    rng = np.random.default_rng(H)
    bits, xt = _special_rows(rng, T, H, "bf16")
    R = T * k + 5
    pos = rng.permutation(R)[: T * k].astype(np.int32).reshape(T, k)
    nb = (H + 511) // 512
    xq = torch.full((R, H), 0xEE, dtype=torch.uint8, device="cuda")
    sx = torch.full((R, nb), -3.0, dtype=torch.float32, device="cuda")
    xd = xt.cuda()
    posd = torch.from_numpy(pos).cuda()
    assert L.moe_test_quant_x(T, H, k, xd.data_ptr(), posd.data_ptr(), xq.data_ptr(), sx.data_ptr(), _stream()) == 0
    torch.cuda.synchronize()
    want_q, want_s = oracle.quant_rows_bf16(bits)
    got_q, got_s = xq.cpu().numpy(), sx.cpu().numpy()
    for j in range(k):
        assert np.array_equal(got_q[pos[:, j]], want_q), f"codes, slot {j}"
        assert np.array_equal(got_s[pos[:, j]].view(np.uint32), want_s.view(np.uint32)), f"scales, slot {j}"
    # rows no pos entry names are untouched
    free = np.setdiff1d(np.arange(R), pos.reshape(-1))
    assert np.all(got_q[free] == 0xEE) and np.all(got_s[free] == -3.0)


@pytest.mark.parametrize("K", [640, 1024, 2048])
def test_quant_h_rows_bit_exact(L, K):
    R = 50
    rng = np.random.default_rng(K + 1)
    x, _ = _special_rows(rng, R, K, "f32")
    # h values: silu(G) * U has a long tail on one side; mix in some such rows
    g = rng.standard_normal((8, K)).astype(np.float32)
    x[20:28] = (g / (1 + np.exp(-g)) * rng.standard_normal((8, K))).astype(np.float32)
    nb = (K + 511) // 512
    hd = torch.from_numpy(x).cuda()
    q = torch.empty((R, K), dtype=torch.uint8, device="cuda")
    s = torch.empty((R, nb), dtype=torch.float32, device="cuda")
    assert L.moe_test_quant_rows(R, K, hd.data_ptr(), q.data_ptr(), s.data_ptr(), _stream()) == 0
    torch.cuda.synchronize()
    want_q, want_s = oracle.quant_rows_f32(x)
    assert np.array_equal(q.cpu().numpy(), want_q)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), want_s.view(np.uint32))


def test_quantiser_argument_errors(L):
    st = _stream()
    assert L.moe_test_quant_x(4, 520, 1, None, None, None, None, st) == -1   # H not a multiple of 16
    assert L.moe_test_quant_x(4, 512, 0, None, None, None, None, st) == -1   # k < 1
    assert L.moe_test_quant_x(4, 512, 1, None, None, None, None, st) == -1   # NULL buffers
    assert L.moe_test_quant_x(0, 512, 1, None, None, None, None, st) == 0    # nothing to do
    assert L.moe_test_quant_rows(4, 8, None, None, None, st) == -1
    assert L.moe_test_quant_rows(0, 512, None, None, None, st) == 0
