"""Plant plausible mistakes in the oracle's C source and check that the pins catch each one.

Every mutant below is a copy of oracle/sdm_oracle.c with one planted error, built
into a temporary library on the CPU.  At least one pin in tests/oracle_pins.py
must fail for each, which shows the pins are strong enough to expose that class
of mistake in the real oracle.
"""
import os

import pytest

import oracle
from tests import oracle_pins

MUTANTS = {
    "error_sign_flipped": [
        ("e[c] = v[(size_t)t * dv + c] - p[c];", "e[c] = p[c] - v[(size_t)t * dv + c];"),
        ("e[c] = v[(size_t)t * dv + c] - p;", "e[c] = p - v[(size_t)t * dv + c];"),
    ],
    "decay_dropped": [
        ("M[q] *= alpha[t];", "M[q] *= 1.0;"),
        ("L += log(alpha[t]);", "L += 0.0;"),
        ("for (int c = 0; c < dv; ++c) M[(size_t)ws[i] * dv + c] *= alpha[t];",
         "for (int c = 0; c < dv; ++c) M[(size_t)ws[i] * dv + c] *= 1.0;"),
    ],
    "backward_prediction_term_dropped": [
        ("dww[(size_t)t * W + i] -= dot(de, Mt + (size_t)i * dv, dv);", "(void)0;"),
    ],
    "backward_decay_not_propagated": [
        ("for (size_t q = 0; q < ND; ++q) dM[q] *= alpha[t];", "(void)0;"),
    ],
    "backward_error_gradient_sign": [
        ("for (int c = 0; c < dv; ++c) dM[(size_t)ws[i] * dv + c] -= wt[i] * de[c];",
         "for (int c = 0; c < dv; ++c) dM[(size_t)ws[i] * dv + c] += wt[i] * de[c];"),
    ],
    "score_backward_softmax_centre_dropped": [
        ("for (int q = 0; q < top; ++q) ds[q] = w[q] * (dw[(size_t)r * top + q] - s);",
         "for (int q = 0; q < top; ++q) ds[q] = w[q] * dw[(size_t)r * top + q];"),
    ],
    "score_backward_halves_crossed": [
        ("dsk[(size_t)i * hd + d] += ds[q] * xr[d];", "dsk[(size_t)i * hd + d] += ds[q] * xr[hd + d];"),
    ],
    "touched_decay_hits_every_slot": [
        ("for (int c = 0; c < dv; ++c) M[(size_t)ws[i] * dv + c] *= alpha[t];",
         "if (i == 0) for (size_t q = 0; q < (size_t)N * dv; ++q) M[q] *= alpha[t];"),
    ],
    "touched_decay_after_prediction": [
        ("        /* (i') decay the write slots */\n"
         "        for (int i = 0; i < W; ++i)\n"
         "            for (int c = 0; c < dv; ++c) M[(size_t)ws[i] * dv + c] *= alpha[t];\n"
         "        /* (ii) prediction */\n"
         "        for (int c = 0; c < dv; ++c) p[c] = 0.0;\n"
         "        for (int i = 0; i < W; ++i)\n"
         "            for (int c = 0; c < dv; ++c) p[c] += ww[(size_t)t * W + i] * M[(size_t)ws[i] * dv + c];\n",
         "        /* (ii) prediction */\n"
         "        for (int c = 0; c < dv; ++c) p[c] = 0.0;\n"
         "        for (int i = 0; i < W; ++i)\n"
         "            for (int c = 0; c < dv; ++c) p[c] += ww[(size_t)t * W + i] * M[(size_t)ws[i] * dv + c];\n"
         "        for (int i = 0; i < W; ++i)\n"
         "            for (int c = 0; c < dv; ++c) M[(size_t)ws[i] * dv + c] *= alpha[t];\n"),
    ],
    "beta_ignored": [
        ("M[(size_t)ws[i] * dv + c] += beta[t] *", "M[(size_t)ws[i] * dv + c] += 1.0 *"),
        ("seen[(size_t)i * dv + c] + beta[t] *", "seen[(size_t)i * dv + c] + 1.0 *"),
    ],
    "halves_swapped": [
        ("s1[i] = dot(x, c1 + (size_t)i * hd, hd);", "s1[i] = dot(x + hd, c1 + (size_t)i * hd, hd);"),
        ("s2[j] = dot(x + hd, c2 + (size_t)j * hd, hd);", "s2[j] = dot(x, c2 + (size_t)j * hd, hd);"),
    ],
    "slot_numbering_transposed": [
        ("cand[i * n + j].id = i * n + j;", "cand[i * n + j].id = j * n + i;"),
        ("cand[a * k_half + b].id = i * n + j;", "cand[a * k_half + b].id = j * n + i;"),
    ],
    "tie_order_reversed": [
        ("if (a->id < b->id) return -1;\n    if (a->id > b->id) return 1;",
         "if (a->id < b->id) return 1;\n    if (a->id > b->id) return -1;"),
    ],
    "softmax_unnormalised": [
        ("for (int i = 0; i < m; ++i) w[i] /= z;", "for (int i = 0; i < m; ++i) w[i] /= 1.0;"),
    ],
    "first_weight_everywhere": [
        ("p[c] += ww[(size_t)t * W + i] *", "p[c] += ww[(size_t)t * W] *"),
        ("p += ww[(size_t)t * W + i] *", "p += ww[(size_t)t * W] *"),
    ],
    "lazy_stamp_not_updated": [
        ("stamp[ws[i]] = L;", "(void)0;"),
    ],
    "pk_shortlist_short_by_one": [
        ("for (int a = 0; a < k_half; ++a)\n            for (int b = 0; b < k_half; ++b) {",
         "for (int a = 0; a < k_half; ++a)\n            for (int b = 0; b < k_half - (a == 0); ++b) {"),
    ],
    "entropy_in_bits": [
        ("if (wr[k] > 0.0) H -= wr[k] * log(wr[k]);", "if (wr[k] > 0.0) H -= wr[k] * log2(wr[k]);"),
    ],
    "quantile_index_rounded_up": [
        ("quant[q] = e[(size_t)floor(probs[q] * (rows - 1))];",
         "quant[q] = e[(size_t)ceil(probs[q] * (rows - 1))];"),
    ],
    "rms_without_mean": [
        ("const double r = 1.0 / sqrt(ms / dv + eps);", "const double r = 1.0 / sqrt(ms + eps);"),
    ],
    "gate_sigmoid_only": [
        ("const double sw = z / (1.0 + exp(-z));", "const double sw = 1.0 / (1.0 + exp(-z));"),
    ],
    "wo_not_transposed": [
        ("acc += a[k] * Wo_t[(size_t)n * K + k];", "acc += a[k] * Wo_t[(size_t)k * dm + n];"),
    ],
    "decay_gate_without_exp_scale": [
        ("alpha[(size_t)ri * H + h] = exp(-exp(A_log[h]) * softplus_d(a + dt_bias[h]));",
         "alpha[(size_t)ri * H + h] = exp(-A_log[h] * softplus_d(a + dt_bias[h]));"),
    ],
    "q_k_swapped": [
        ("q[((size_t)ri * H + h) * dk + c] = ph[c];", "q[((size_t)ri * H + h) * dk + c] = ph[dk + c];"),
    ],
    "backward_end_gradient_ignored": [
        ("if (dM_end) memcpy(dM, dM_end, sizeof(double) * ND);", "(void)dM_end;"),
    ],
    "read_weights_from_write": [
        ("o += rw[(size_t)t * R + j] * M[(size_t)rs[j] * dv + c];",
         "o += rw[(size_t)t * R + j] * M[(size_t)ws[j % W] * dv + c];"),
        ("o += rw[(size_t)t * R + j] * Mraw[(size_t)rs[j] * dv + c] * exp(L - stamp[rs[j]]);",
         "o += rw[(size_t)t * R + j] * Mraw[(size_t)ws[j % W] * dv + c] * exp(L - stamp[ws[j % W]]);"),
    ],
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    with open(oracle.SRC) as f:
        src = f.read()
    for old, new in MUTANTS[name]:
        assert old in src, f"mutation site not found for {name}: {old!r}"
        src = src.replace(old, new)
    path = tmp_path / f"mut_{name}.c"
    path.write_text(src)
    lib = oracle.build(force=True, src=str(path), out=str(tmp_path / f"libmut_{name}.so"))
    o = oracle.Oracle(lib)
    failed = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(o)
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"no pin caught mutant {name}"
