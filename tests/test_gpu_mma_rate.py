"""Tensor-core issue-rate microbenchmark (one GPU, through the C ABI's test entry point).

The 4-bit grouped GEMMs issue kind::f16 MMAs with the A operand in tensor memory at N <= 96,
and clock traces of them showed ~800 cycles to issue a stage's four MMAs against ~200 cycles
of tensor work.  This isolates that cost from everything around it (TMA, dequantisation,
barrier waits): one CTA issues N back-to-back MMAs on operands already on chip, in each form the
kernels use or could use -- kind::f16 with A and B in shared memory, kind::f16 with A in tensor
memory, kind::f8f6f4, and both over a CTA pair (cta_group::2, M = 256) -- with and without a
commit every 4 MMAs (one pipeline stage).  The ideal is one MMA per 2*M*N*K / 8192 cycles per
SM (the bf16 rate; FP8 does twice the K in the same time).  It prints the table and checks
only that every run completed.
"""
import ctypes

import numpy as np
import pytest
import torch

import mixture_experts_ffn_13_b200 as moe

pytestmark = pytest.mark.gpu

FORMS = {0: "f16 SS", 1: "f16 TS", 2: "f8 SS", 3: "f16 pair", 4: "f8 pair"}


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = moe.load_library()
    lib.moe_test_mma_rate.argtypes = [ctypes.c_int32] * 5 + [ctypes.c_void_p] * 3
    lib.moe_test_mma_rate.restype = ctypes.c_int
    return lib


def test_mma_issue_rate_table(L):
    cyc = torch.zeros(2, dtype=torch.int64, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    count = 2048
    rows = []
    for form, name in FORMS.items():
        for N in (32, 64, 96, 128, 192, 256):
            for every in (0, 4):
                for _ in range(2):  # the first launch warms the instruction cache
                    assert L.moe_test_mma_rate(form, N, count, every, 0, cyc.data_ptr(), status.data_ptr(), st) == 0
                torch.cuda.synchronize()
                c = cyc.cpu().numpy()
                assert int(status.item()) == 0 and c[1] > 0, (name, N, every)
                ideal = N / 2.0  # cycles per MMA of M = 128 (per SM for the pair forms)
                rows.append((name, N, every, c[0] / count, c[1] / count, ideal))
    print("\nform      N  commit/4  issue cyc/MMA  done cyc/MMA  ideal cyc/MMA  tensor busy")
    for name, N, every, iss, done, ideal in rows:
        print(f"{name:8s} {N:4d} {every:6d} {iss:14.1f} {done:13.1f} {ideal:13.1f} {ideal / done:11.2f}")


def test_mma_rate_argument_errors(L):
    cyc = torch.zeros(2, dtype=torch.int64, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    assert L.moe_test_mma_rate(0, 24, 8, 0, 0, cyc.data_ptr(), status.data_ptr(), st) == -1   # N % 16
    assert L.moe_test_mma_rate(3, 16, 8, 0, 0, cyc.data_ptr(), status.data_ptr(), st) == -1   # pair N < 32
    assert L.moe_test_mma_rate(9, 64, 8, 0, 0, cyc.data_ptr(), status.data_ptr(), st) == -1   # form
    assert L.moe_test_mma_rate(0, 64, 0, 0, 0, cyc.data_ptr(), status.data_ptr(), st) == -1   # count
    assert L.moe_test_mma_rate(0, 64, 8, 0, 8, cyc.data_ptr(), status.data_ptr(), st) == -1   # flags > 7
    assert L.moe_test_mma_rate(0, 64, 8, 0, 5, cyc.data_ptr(), status.data_ptr(), st) == -1   # two issuers + alternation
    assert L.moe_test_mma_rate(3, 64, 8, 0, 4, cyc.data_ptr(), status.data_ptr(), st) == -1   # two issuers on a pair form
    assert L.moe_test_mma_rate(1, 256, 8, 4, 1, cyc.data_ptr(), status.data_ptr(), st) == -1  # TS A overlap


def test_commit_cost_table(L):
    """What a commit costs the issuing thread: 2048 MMAs of the FP8 prefill tile shape (M = 128,
    N = 192, K = 32) and the bf16 4-bit shape (N = 96), committing every 1 .. 64 MMAs, with one
    accumulator or two alternating ones, one barrier or two alternating ones, or (flags 4) two
    issuing threads in different warps with an accumulator each."""
    cyc = torch.zeros(2, dtype=torch.int64, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    count = 2048
    print("\nform      N  commit/  flags  issue cyc/MMA  done cyc/MMA")
    for form, N in ((2, 192), (0, 96), (1, 96), (4, 192)):
        for every in (1, 2, 4, 8, 16, 64):
            for flags in ((0, 1, 2, 3) if form == 4 else (0, 1, 2, 3, 4)):
                for _ in range(2):
                    assert L.moe_test_mma_rate(form, N, count, every, flags, cyc.data_ptr(), status.data_ptr(), st) == 0
                torch.cuda.synchronize()
                c = cyc.cpu().numpy()
                assert int(status.item()) == 0 and c[1] > 0
                print(f"{FORMS[form]:8s} {N:4d} {every:6d} {flags:6d} {c[0] / count:14.1f} {c[1] / count:13.1f}")
