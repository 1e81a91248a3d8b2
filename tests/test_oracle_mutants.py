"""The oracle's pins must catch plausible mistakes (CPU only).

Each case copies the oracle's C source to a temporary directory, plants one
mistake in the copy (a window off by one, a wrong sign, a wrong head index, a
transposed operand, a reversed tie-break, ...), builds it, and checks that at
least one pin of tests/test_oracle_pins.py fails against it.  The oracle in
the repository is never modified.
"""
import contextlib
import ctypes
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins
from tests import test_oracle_threshold as tpins
from tests import test_oracle_decode as dpins
from tests import test_oracle_backward as bpins

SRC = os.path.join(os.path.dirname(oracle.__file__), "logo_oracle.c")

MUTANTS = {
    "window_off_by_one": ("int64_t j_lo = i - p->W + 1;", "int64_t j_lo = i - p->W;"),
    "merge_sign": ("out[r + c] = loc[c] + (sel ? gs * glo[c] : 0.0);",
                   "out[r + c] = loc[c] - (sel ? gs * glo[c] : 0.0);"),
    "gqa_head_map": ("int hk = h / G;", "int hk = h % p->Hkv;"),
    "scores_read_v": ("const uint16_t *kr = kh + (j_lo + t) * (int64_t)d;",
                      "const uint16_t *kr = vh + (j_lo + t) * (int64_t)d;"),
    "tie_break_upper": ("return (a->idx < b->idx) ? -1 : (a->idx > b->idx ? 1 : 0);",
                        "return (a->idx > b->idx) ? -1 : (a->idx < b->idx ? 1 : 0);"),
    "nan_on_top": ("if (a_nan != b_nan) return a_nan ? 1 : -1;",
                   "if (a_nan != b_nan) return a_nan ? -1 : 1;"),
    "sigmoid_sign": ("return 1.0 / (1.0 + exp(-x));", "return 1.0 / (1.0 + exp(x));"),
    "budget_floor": ("double kk = (fabs(x - r) <= tol) ? r : ceil(x);",
                     "double kk = (fabs(x - r) <= tol) ? r : floor(x);"),
    "budget_no_snap": ("double kk = (fabs(x - r) <= tol) ? r : ceil(x);", "double kk = ceil(x);"),
    "scale_one_over_d": ("return scale > 0.0 ? scale : 1.0 / sqrt((double)d);",
                         "return scale > 0.0 ? scale : 1.0 / (double)d;"),
    "denominator_dropped_term": ("den += w;", "den += (t == 0) ? 0.0 : w;"),
    "global_not_full_prefix": ("attend_row(qr, kh, vh, 0, i, p->d, p->scale, scratch, glo);",
                               "attend_row(qr, kh, vh, i > 0 ? 1 : 0, i, p->d, p->scale, scratch, glo);"),
    "threshold_ge": ("if (g[i] > tau) out[n++] = (int32_t)i;", "if (g[i] >= tau) out[n++] = (int32_t)i;"),
    "target_kth_not_next": ("float q = items[k].g;", "float q = items[k > 0 ? k - 1 : 0].g;"),
    "update_drops_tau": ("volatile float out = tau + step;", "volatile float out = step;"),
    "update_sign": ("volatile float diff = q - tau;", "volatile float diff = tau - q;"),
    "decode_selection_ge": ("int sel = (g[b] > tau) ? 1 : 0; /* false for NaN on either side */",
                            "int sel = (g[b] >= tau) ? 1 : 0;"),
    "decode_cache_last": ("int64_t t = (int64_t)cache_len[b] - 1;", "int64_t t = (int64_t)cache_len[b] - 2;"),
    "bwd_drop_D": ("double ds = pj * (dp - D);", "double ds = pj * dp;"),
    "bwd_gate_no_derivative": ("dg[b * L + s0 + i] = sg * (1.0 - sg) * e;", "dg[b * L + s0 + i] = sg * e;"),
    "bwd_global_upstream_ungated": (
        "row_grad(qr, kh, vh, er, a, 0, i, d, pr.scale, p, o, dqr, dkp, dvp, -1);",
        "row_grad(qr, kh, vh, er, 1.0, 0, i, d, pr.scale, p, o, dqr, dkp, dvp, -1);"),
    "bwd_dk_unscaled": ("if (dkr) dkr[c] += scale * ds * bf16_bits_to_double(q[c]);",
                        "if (dkr) dkr[c] += ds * bf16_bits_to_double(q[c]);"),
    "bwd_dv_drops_gate_factor": ("if (dvr) dvr[c] += pj * a * bf16_bits_to_double(dout[c]);",
                                 "if (dvr) dvr[c] += pj * bf16_bits_to_double(dout[c]);"),
    "bwd_dq_reads_v": ("dq[c] += scale * ds * bf16_bits_to_double(kr[c]);",
                       "dq[c] += scale * ds * bf16_bits_to_double(vr[c]);"),
    "bwd_local_drops_self_key": (
        "row_grad(qr, kh, vh, er, 1.0, j_lo, i, d, pr.scale, p, o, dqr, dkp, dvp, -1);",
        "row_grad(qr, kh, vh, er, 1.0, j_lo, i > j_lo ? i - 1 : i, d, pr.scale, p, o, dqr, dkp, dvp, -1);"),
    "bwd_gqa_first_head_only": (
        "for (int h = hk * G; h < (hk + 1) * G; ++h) {\n                    for (int64_t i = 0; i < len; ++i) {\n"
        "                        const uint16_t *qr = row_ptr(q, b, Hq, h, L, s0 + i, d);\n"
        "                        const uint16_t *er",
        "for (int h = hk * G; h < hk * G + 1; ++h) {\n                    for (int64_t i = 0; i < len; ++i) {\n"
        "                        const uint16_t *qr = row_ptr(q, b, Hq, h, L, s0 + i, d);\n"
        "                        const uint16_t *er"),
}

PINS = [
    pins.test_num_selected_golden,
    pins.test_select_golden,
    lambda: [pins.test_select_bruteforce_ties_nan_inf(s) for s in range(4)],
    lambda: [pins.test_oracle_vs_dense_masks(s) for s in pins.SHAPES],
    pins.test_oracle_vs_dense_masks_varlen,
    pins.test_oracle_vs_sdpa,
    pins.test_closed_form_uniform_weights,
    pins.test_closed_form_weights_one_e_e2,
    pins.test_ratio_one_full_window_is_gated_causal,
    tpins.test_threshold_golden,
    lambda: [tpins.test_threshold_select_and_target_bruteforce(s) for s in range(3)],
    tpins.test_target_leaves_exactly_k_above_distinct_logits,
    tpins.test_threshold_update_fp32_arithmetic,
    lambda: [dpins.test_decode_vs_dense_masks(s) for s in range(2)],
    dpins.test_decode_matches_prefill_rows,
    dpins.test_decode_closed_forms,
    lambda: [bpins.test_backward_matches_finite_differences(c) for c in bpins.FD_CASES],
    lambda: [bpins.test_backward_vs_sdpa_autograd(*c) for c in ((0, 16, 0.2), (3, 1, 1.0))],
    bpins.test_backward_invariants,
]


@contextlib.contextmanager
def swapped_oracle(so_path):
    saved = oracle._lib
    oracle._lib = None
    real_so = oracle._SO
    real_src = oracle._SRC
    try:
        oracle._SO = so_path
        oracle._SRC = so_path  # mtime check passes: no rebuild
        oracle._load()
        yield
    finally:
        oracle._lib = saved
        oracle._SO = real_so
        oracle._SRC = real_src


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor not found exactly once: {old}"
    mutated = tmp_path / "mutant.c"
    mutated.write_text(src.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O1", "-fPIC", "-std=gnu11", "-shared", "-o", str(so), str(mutated), "-lm"],
                   check=True)
    caught = []
    with swapped_oracle(str(so)):
        for pin in PINS:
            try:
                pin()
            except AssertionError:
                caught.append(getattr(pin, "__name__", "pin"))
    assert caught, f"no pin caught the planted mistake {name}"


def test_unmutated_copy_passes_every_pin(tmp_path):
    so = tmp_path / "libcopy.so"
    subprocess.run(["gcc", "-O1", "-fPIC", "-std=gnu11", "-shared", "-o", str(so), SRC, "-lm"],
                   check=True)
    with swapped_oracle(str(so)):
        for pin in PINS:
            pin()
