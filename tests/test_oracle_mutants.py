"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of moe_oracle.c (a swapped nibble order, a wrong
exponent bias, SiLU read as the sigmoid, a scale applied to the wrong matrix, a dropped
rounding, a reordered sort key, ...), compiles the copy with the oracle's own flags, and runs
the pins against it: at least one pin must fail.  The planted text must occur in the oracle
exactly as written, so a later edit of the oracle that moves it makes this test fail loudly
rather than pass vacuously.
"""
import shutil
import subprocess

import pytest

import oracle
import test_oracle_envelope as ENV
import test_oracle_formats as F
import test_oracle_layer as LY
import test_oracle_mxfp4 as MX
import test_oracle_nvfp4 as NV
import test_oracle_quant as Q
import test_oracle_route as R

# the pins, cheapest first (the first failure ends a case)
PINS = [
    (F.test_e4m3_decode_known_values, {}),
    (F.test_e4m3_roundtrip_all_finite_codes, {}),
    (MX.test_e2m1_decode_table, {}),
    (MX.test_e8m0_decode_matches_torch, {}),
    (R.test_route_ties_lower_index_wins, {}),
    (R.test_route_two_experts_closed_form, {}),
    (R.test_route_k_equals_E_is_full_softmax, {}),
    (R.test_permute_matches_lexsort, {}),
    (R.test_router_logits_against_exact_sums, {}),
    (Q.test_identity_when_block_amax_is_448, {}),
    (Q.test_matches_torch_composition, {}),
    (LY.test_hand_worked_two_experts_two_tokens, {}),
    (LY.test_int4_all_ones_weights, {}),
    (LY.test_int4_negative_nibbles, {}),
    (MX.test_mxfp4_one_hot_reads_single_weights, {}),
    (NV.test_nvfp4_one_hot_reads_single_weights, {}),
    (NV.test_tensor_scales_apply_to_their_own_matrices, {}),
    (LY.test_shared_expert_adds_with_weight_one, {}),
    (LY.test_h_on_a_rounding_midpoint_reports_the_envelope, {}),
    (ENV.test_fp8_window_follows_the_sum_of_magnitudes, {}),
    (ENV.test_bf16_h_on_a_rounding_midpoint, {"fmt": "int4"}),
    (ENV.test_bf16_h_on_a_rounding_midpoint, {"fmt": "mxfp4"}),
    (ENV.test_bf16_h_on_a_rounding_midpoint, {"fmt": "nvfp4"}),
    (LY.test_layer_equals_dense_masked_bruteforce, {"cfg": LY.SMALL[1]}),
    (LY.test_layer_equals_dense_masked_bruteforce, {"cfg": LY.SMALL[3]}),
]

# (what the mistake is, text in moe_oracle.c, replacement, occurrences)
MUTANTS = [
    ("e4m3 subnormals one binade low", "v = ldexp((double)m / 8.0, -6);", "v = ldexp((double)m / 8.0, -7);", 1),
    ("e2m1 exponent bias 2", "ldexp(1.0 + 0.5 * (double)m, e - 1);", "ldexp(1.0 + 0.5 * (double)m, e - 2);", 1),
    ("E8M0 bias 126", "return ldexp(1.0, (int)c - 127);", "return ldexp(1.0, (int)c - 126);", 1),
    ("top-k ties to the higher index", "return (a->e < b->e) ? -1 : (a->e > b->e);",
     "return (a->e > b->e) ? -1 : (a->e < b->e);", 1),
    ("permutation keyed by token first",
     "    if (a->e != b->e) return (a->e < b->e) ? -1 : 1;\n    if (a->t != b->t) return (a->t < b->t) ? -1 : 1;",
     "    if (a->t != b->t) return (a->t < b->t) ? -1 : 1;\n    if (a->e != b->e) return (a->e < b->e) ? -1 : 1;", 1),
    ("router logits drop the last product",
     "            for (int i = 0; i < H; ++i) {\n                double p = orc_bf16_to_double",
     "            for (int i = 0; i < H - 1; ++i) {\n                double p = orc_bf16_to_double", 1),
    ("activation scale amax/447", "volatile float sc = amax / 448.0f;", "volatile float sc = amax / 447.0f;", 1),
    ("FP8 promotion with block 0's activation scale", "acc += (double)sx[kb] * (double)sw[(size_t)n * nb + kb] * part;",
     "acc += (double)sx[0] * (double)sw[(size_t)n * nb + kb] * part;", 1),
    ("SiLU read as the sigmoid", "return z * (1.0 / (1.0 + exp(-z)));", "return (1.0 / (1.0 + exp(-z)));", 1),
    ("int4 odd K index in the low nibble", "int v = (i & 1) ? (b >> 4) : (b & 0xF);",
     "int v = (i & 1) ? (b & 0xF) : (b >> 4);", 1),
    ("4-bit h not rounded to bf16", "h[n] = orc_bf16_to_double(orc_double_to_bf16(hx[n]));", "h[n] = hx[n];", 1),
    ("NVFP4 gate takes the up tensor scale", "nv ? (double)w->t_gate[e] : 1.0, w->w_up",
     "nv ? (double)w->t_up[e] : 1.0, w->w_up", 1),
    ("NVFP4 block scales per 32", "orc_dec_tab[sc[(size_t)n * (K / 16) + i / 16]]",
     "orc_dec_tab[sc[(size_t)n * (K / 16) + i / 32]]", 1),
    ("combine ignores the routing weights", "for (int n = 0; n < H; ++n) out[n] += p[j] * y[n];",
     "for (int n = 0; n < H; ++n) out[n] += y[n] / k;", 2),
    ("bf16 envelope without the down matrix's tensor scale",
     "env[n] += D * fabs(orc_w4(wfmt, I, wd, sd, n, i) * td);", "env[n] += D * fabs(orc_w4(wfmt, I, wd, sd, n, i));",
     1),
    ("bf16 envelope measured from the exact h", "double b = orc_bf16_to_double(orc_double_to_bf16(hx[i]));",
     "double b = hx[i];", 1),
    ("bf16 alternatives ignore the window above h",
     "double hi = orc_bf16_to_double(orc_double_to_bf16(hx[i] + dh[i]));", "double hi = b;", 1),
    ("FP8 window from the block sums instead of the sum of |products|",
     "mag += fabs((double)sx[kb] * (double)sw[(size_t)n * nb + kb]) * apart;",
     "mag += fabs((double)sx[kb] * (double)sw[(size_t)n * nb + kb] * part);", 1),
    ("FP8 envelope one code step too wide", "D *= s;", "D *= 2.0 * s;", 1),
    ("shared expert weighted like a routed one", "            for (int n = 0; n < H; ++n) out[n] += y[n];\n",
     "            for (int n = 0; n < H; ++n) out[n] += p[0] * y[n];\n", 2),
]


@pytest.fixture(scope="module")
def gcc():
    g = shutil.which("gcc")
    if g is None:
        pytest.skip("gcc not found")
    return g


def _first_failing_pin():
    for fn, kw in PINS:
        try:
            fn(oracle, **kw)
        except Exception:  # an assertion, or the oracle refusing its own output
            return fn.__name__
    return None


@pytest.mark.parametrize("what,old,new,count", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_fails_a_pin(tmp_path, monkeypatch, gcc, what, old, new, count):
    with open(oracle._SRC) as f:
        src = f.read()
    assert src.count(old) == count, f"the oracle no longer contains the text of '{what}'"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.run([gcc, "-O2", "-fno-fast-math", "-ffp-contract=off", "-fPIC", "-shared", "-o", str(lib),
                    str(path), "-lm", "-lpthread"], check=True)
    monkeypatch.setattr(oracle, "_lib", oracle.load(str(lib)))
    assert _first_failing_pin() is not None, f"no pin catches: {what}"


def test_unmodified_copy_passes_every_pin(tmp_path, monkeypatch, gcc):
    """The control: the same build of the oracle as written fails no pin, so a failure above
    is the planted mistake's doing."""
    lib = tmp_path / "libcopy.so"
    subprocess.run([gcc, "-O2", "-fno-fast-math", "-ffp-contract=off", "-fPIC", "-shared", "-o", str(lib),
                    oracle._SRC, "-lm", "-lpthread"], check=True)
    monkeypatch.setattr(oracle, "_lib", oracle.load(str(lib)))
    assert _first_failing_pin() is None
