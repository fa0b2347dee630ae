"""Planted mistakes in the oracle must trip the pins.

Each mutation below is a plausible slip (a dropped term, a wrong sign or
index, a mean for a sum, a transposed pairing).  It is applied to a copy of
``oracle/tri_oracle.c`` in a temporary directory, built on the CPU, swapped in
for the real oracle, and the pins of ``test_oracle_pins.py`` are run against
it: at least one must fail.  The real oracle is never modified.
"""
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "tri_oracle.c")

# (name, [(old, new), ...]) - every `old` must occur in the source.
MUTATIONS = [
    ("norm term dropped",
     [(" + ((ldbl)mnorm[g * F + f] - qn[g * F + f]) * kn;", ";")]),
    ("mean over offsets instead of sum",
     [("sg += qn[g * F + f] * kn * trig", "sg += qn[g * F + f] * kn * trig / n_off")]),
    ("offset subtracted",
     [("(p_now + offsets[e] - pos[j])", "(p_now - offsets[e] - pos[j])")]),
    ("frequency exponent -f/d",
     [("-2.0L * (ldbl)f / (ldbl)d", "-1.0L * (ldbl)f / (ldbl)d")]),
    ("de-rotation by +angle",
     [("*re = xr * c + xi * s;", "*re = xr * c - xi * s;"),
      ("*im = xi * c - xr * s;", "*im = xi * c + xr * s;")]),
    ("interleaved pairing where rotate-half is asked",
     [("        *ire = f;\n        *iim = f + d / 2;", "        *ire = 2 * f;\n        *iim = 2 * f + 1;")]),
    ("interleaved pair with real and imaginary swapped",
     [("        *ire = 2 * f;\n        *iim = 2 * f + 1;", "        *ire = 2 * f + 1;\n        *iim = 2 * f;")]),
    ("phase sign flipped",
     [("ldbl phi = qa[g * F + f] - atan2l(ki, kr);", "ldbl phi = atan2l(ki, kr) - qa[g * F + f];")]),
    ("distance uses slot sign reversed",
     [("cosl(w[f] * (ldbl)(p_now + offsets[e] - pos[j]) + phi)",
       "cosl(w[f] * (ldbl)(pos[j] - p_now - offsets[e]) + phi)")]),
    ("GQA sum instead of mean",
     [("out[j] = (double)(total / (ldbl)G);", "out[j] = (double)total;")]),
    ("calibration norm of the mean",
     [("mnorm[f] = (double)(sn / (ldbl)nq);", "mnorm[f] = (double)hypotl(sr / (ldbl)nq, si / (ldbl)nq);")]),
    ("calibration drops the imaginary half",
     [("ldbl xr = q[t * d + ire], xi = q[t * d + iim];", "ldbl xr = q[t * d + ire], xi = 0.0L * q[t * d + iim];")]),
    ("online decay favours older batches",
     [("powl((ldbl)decay, (ldbl)(n_updates - 1 - update_of[t]))", "powl((ldbl)decay, (ldbl)update_of[t])")]),
    ("online weights not normalised",
     [("centre[2 * f] = (double)(sr / sw);", "centre[2 * f] = (double)(sr / (ldbl)nq);")]),
    ("drift without the norm term",
     [("dd += fabsl((ldbl)mnorm[f] - ref_mnorm[f]);", "dd += 0.0L;")]),
    ("concentration inverted",
     [("conc[f] = mnorm[f] > 0.0 ? (double)(a / (ldbl)mnorm[f]) : 0.0;",
       "conc[f] = a > 0.0L ? (double)((ldbl)mnorm[f] / a) : 0.0;")]),
    ("attention scale dropped",
     [("s[j] = (ldbl)scale * a;", "s[j] = a;")]),
    ("attention normalised by the row length",
     [("out[t] = (double)(acc[t] / den);", "out[t] = (double)(acc[t] / (ldbl)n);")]),
    ("tie-break keeps the older slot",
     [("if (a->i != b->i) return a->i > b->i ? -1 : 1;", "if (a->i != b->i) return a->i < b->i ? -1 : 1;")]),
    ("window not protected",
     [("for (int64_t j = M; j < n; j++) keep[j] = 1;", "for (int64_t j = M; j < n; j++) keep[j] = 0;")]),
    ("budget excludes the window",
     [("const int64_t M = n - W, K = B - W;", "const int64_t M = n - W, K = B;")]),
    ("gather off by one",
     [("memcpy(dst + t * width, src + idx[t] * width, (size_t)width);",
       "memcpy(dst + t * width, src + (idx[t] > 0 ? idx[t] - 1 : 0) * width, (size_t)width);")]),
    # slips confined to one form of the score (the collapsed form is the one the
    # kernels are compared with), to the single series term, and to the diagnostics
    ("collapsed: sine term added",
     [("ldbl trig = cosl(x) * sr[f] - sinl(x) * si[f];", "ldbl trig = cosl(x) * sr[f] + sinl(x) * si[f];")]),
    ("collapsed: offset phasor sum of cosines only",
     [("si[f] += sinl(w[f] * (ldbl)offsets[e]);", "si[f] += cosl(w[f] * (ldbl)offsets[e]);")]),
    ("collapsed: key phase added",
     [("(ldbl)(p_now - pos[j]) + qa[g * F + f] - atan2l(ki, kr);",
       "(ldbl)(p_now - pos[j]) + qa[g * F + f] + atan2l(ki, kr);")]),
    ("absorbed: key not conjugated",
     [("s += br * kr + bi * ki + cf[f] * hypotl(kr, ki);", "s += br * kr - bi * ki + cf[f] * hypotl(kr, ki);")]),
    ("absorbed: rotation to p_now backwards",
     [("ar[f] = tr * ec - ti * es;\n            ai[f] = tr * es + ti * ec;",
       "ar[f] = tr * ec + ti * es;\n            ai[f] = ti * ec - tr * es;")]),
    ("absorbed: norm coefficient summed over the group",
     [("cf[f] = c / (ldbl)G;", "cf[f] = c;")]),
    ("absorbed: pre-RoPE distance reversed",
     [("ldbl a = w[f] * (ldbl)(p_now - pos[j]), ec", "ldbl a = w[f] * (ldbl)(pos[j] - p_now), ec")]),
    ("series term: key phase added",
     [("ldbl phi = atan2l(qi, qr) - atan2l(ki, kr);", "ldbl phi = atan2l(qi, qr) + atan2l(ki, kr);")]),
    ("key centres: cached keys left rotated",
     [("key_pair(d, il, keys + j * d, f, post_rope, w, pos[j], &kr, &ki);",
       "key_pair(d, il, keys + j * d, f, 0, w, pos[j], &kr, &ki);")]),
    ("key centres: mean norm as the norm of the mean",
     [("mnorm[f] = n ? (double)(sn / (ldbl)n) : 0.0;", "mnorm[f] = n ? (double)(hypotl(sr, si) / (ldbl)n) : 0.0;")]),
    ("key centres: imaginary part from the real dimension",
     [("si += ki;", "si += kr;")]),
    ("stats: centre magnitudes squared",
     [("sc += a;", "sc += a * a;")]),
    ("stats: drift relative to the current norms",
     [("rm += ref_mnorm[f];", "rm += mnorm[f];")]),
    ("online: magnitudes not weighted",
     [("sn += w * hypotl(xr, xi);", "sn += hypotl(xr, xi);")]),
    ("attention: lse without the maximum",
     [("*lse = (double)(m + logl(den));", "*lse = (double)logl(den);")]),
    ("attention: weights applied to the keys",
     [("acc[t] += p * (ldbl)values[j * d + t];", "acc[t] += p * (ldbl)keys[j * d + t];")]),
    ("select: NaN ranks first",
     [("if (an != bn) return an ? 1 : -1;", "if (an != bn) return an ? -1 : 1;")]),
]

PIN_FUNCS = [
    lambda: pins.test_omega_is_theta_power(),
    lambda: pins.test_trig_series_equals_rope_dot_at_every_distance(0),
    lambda: pins.test_trig_series_equals_rope_dot_other_layouts(64, True),
    lambda: pins.test_golden_closed_forms(),
    lambda: pins.test_identical_queries_give_attention_logit_sum(True),
    lambda: pins.test_identical_queries_give_attention_logit_sum(False),
    lambda: pins.test_zero_centre_gives_norm_sum(True),
    lambda: pins.test_two_queries_trig_and_norm_parts(),
    lambda: pins.test_calib_single_query(),
    lambda: pins.test_calib_matches_numpy_and_triangle_inequality(),
    lambda: pins.test_select_brute_force_tiny_rows(),
    lambda: pins.test_select_matches_lexsort_and_invariants(),
    lambda: pins.test_select_all_equal_keeps_most_recent(),
    lambda: pins.test_gather_matches_fancy_indexing(),
    lambda: pins.test_calib_online_equals_weighted_mean(),
    lambda: pins.test_key_centres_undo_rope(False),
    lambda: pins.test_calib_stats_closed_forms(),
    lambda: pins.test_attention_matches_torch_sdpa_and_closed_forms(),
    lambda: pins.test_trig_series_negative_distance(),
    lambda: pins.test_identical_queries_logit_sum_other_layouts(True, 64, True),
    lambda: pins.test_identical_queries_logit_sum_other_layouts(False, 256, False),
    lambda: pins.test_key_centres_undo_rope(True),
    lambda: pins.test_select_nan_ranks_last_and_bad_args(),
    lambda: pins.test_calib_interleaved_pairs(),
]


def _failing_pins():
    failed = 0
    for fn in PIN_FUNCS:
        try:
            fn()
        except (AssertionError, ValueError, IndexError):
            failed += 1
    return failed


@pytest.mark.parametrize("name,edits", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(tmp_path, name, edits):
    src = open(SRC).read()
    for old, new in edits:
        assert old in src, f"mutation anchor not found: {old!r}"
        src = src.replace(old, new)
    mpath = tmp_path / "mut.c"
    mpath.write_text(src)
    so = tmp_path / "libmut.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", str(so),
                    str(mpath), "-lm"], check=True)
    saved = oracle.lib()
    oracle._lib = oracle.load(str(so))
    try:
        assert _failing_pins() >= 1, f"no pin caught: {name}"
    finally:
        oracle._lib = saved


def test_unmutated_oracle_passes_every_pin():
    assert _failing_pins() == 0
