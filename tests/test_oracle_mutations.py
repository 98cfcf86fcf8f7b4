"""Planted mistakes in the oracle must be caught by its pins.

Each case copies the oracle's C source, plants one plausible mistake (a
dropped term, a wrong sign, index or operand), compiles the copy into a
temporary shared object and runs every pin against it: at least one pin has
to fail. This checks that the pins constrain every step of the oracle, not
just that the oracle passes them. CPU only; nothing here touches a GPU.
"""
import os

import pytest

import oracle
import oracle_pins
from oracle import build as obuild

# (name, [(old, new, which occurrence)]) -- each `old` must exist in the source.
MUTATIONS = [
    ("eps_outside_root", [("return 1.0 / sqrt(ms + eps);",
                           "return 1.0 / (sqrt(ms) + eps);", 0)]),
    ("sum_not_mean", [("ms /= (double)D;", "ms /= 1.0;", 0)]),
    ("mean_over_pair_count", [("ms /= (double)D;", "ms /= (double)(D / 2);", 0)]),
    ("gamma_dropped", [("n[d] = x[d] * r * gamma[d];", "n[d] = x[d] * r;", 0)]),
    ("gamma_after_rotation",
     [("n[d] = x[d] * r * gamma[d];", "n[d] = x[d] * r;", 0),
      ("    free(n);\n    *rstd = r;",
       "    for (int d = 0; d < D; ++d) y[d] *= gamma[d];\n    free(n);\n    *rstd = r;", 0)]),
    ("freq_exponent_without_2", [("-2.0 * (double)i / (double)R",
                                  "-1.0 * (double)i / (double)R", 0)]),
    ("freq_over_i_plus_1", [("-2.0 * (double)i / (double)R",
                             "-2.0 * (double)(i + 1) / (double)R", 0)]),
    ("sin_sign_first", [("y[i] = n[i] * c - n[i + half] * s;",
                         "y[i] = n[i] * c + n[i + half] * s;", 0)]),
    ("sin_sign_second", [("y[i + half] = n[i + half] * c + n[i] * s;",
                          "y[i + half] = n[i + half] * c - n[i] * s;", 0)]),
    ("interleaved_pairing", [("y[i] = n[i] * c - n[i + half] * s;\n        y[i + half] = n[i + half] * c + n[i] * s;",
                              "y[2 * i] = n[2 * i] * c - n[2 * i + 1] * s;\n        y[2 * i + 1] = n[2 * i + 1] * c + n[2 * i] * s;", 0)]),
    ("position_plus_one_fwd", [("double phi = (double)m * oracle_inv_freq(i, R, theta);",
                                "double phi = (double)(m + 1) * oracle_inv_freq(i, R, theta);", 0)]),
    ("pass_through_zeroed", [("        y[d] = n[d];", "        y[d] = 0.0;", 0)]),
    ("cos_sin_swapped", [("double c = cos(phi), s = sin(phi);",
                          "double c = sin(phi), s = cos(phi);", 0)]),
    ("bwd_unrotate_sign", [("g[i + half] = -dy[i] * s + dy[i + half] * c;",
                            "g[i + half] = dy[i] * s + dy[i + half] * c;", 0)]),
    ("bwd_forward_rotation", [("g[i] = dy[i] * c + dy[i + half] * s;",
                               "g[i] = dy[i] * c - dy[i + half] * s;", 0),
                              ("g[i + half] = -dy[i] * s + dy[i + half] * c;",
                               "g[i + half] = dy[i] * s + dy[i + half] * c;", 0)]),
    ("bwd_position_plus_one", [("double phi = (double)m * oracle_inv_freq(i, R, theta);",
                                "double phi = (double)(m + 1) * oracle_inv_freq(i, R, theta);", 1)]),
    ("bwd_r_squared", [("- r * r * r * x[d] * dot", "- r * r * x[d] * dot", 0)]),
    ("bwd_dot_over_D_dropped", [("* dot / (double)D;", "* dot;", 0)]),
    ("bwd_dot_uses_g", [("dot += h[e] * x[e];", "dot += g[e] * x[e];", 0)]),
    ("bwd_h_without_gamma", [("h[d] = g[d] * gamma[d];", "h[d] = g[d];", 0)]),
    ("dgamma_without_r", [("dgamma[d] += g[d] * x[d] * r;",
                           "dgamma[d] += g[d] * x[d];", 0)]),
    ("dgamma_uses_dy", [("dgamma[d] += g[d] * x[d] * r;",
                         "dgamma[d] += dy[d] * x[d] * r;", 0)]),
    ("k_rows_use_gamma_q", [("oracle_fwd_row(k + row * D, gamma_k,",
                             "oracle_fwd_row(k + row * D, gamma_q,", 0)]),
    ("positions_ignored", [("oracle_fwd_row(q + row * D, gamma_q, D, R, theta, eps, m[t],",
                            "oracle_fwd_row(q + row * D, gamma_q, D, R, theta, eps, (int64_t)t,", 0)]),
    ("bwd_k_dgamma_into_q", [("theta, eps, m[t], dk + row * D, dgamma_k);",
                              "theta, eps, m[t], dk + row * D, dgamma_q);", 0)]),
    ("ln_mean_not_subtracted", [("            nr[d] = (xr[d] - mu) * r * gamma[d];",
                                 "            nr[d] = xr[d] * r * gamma[d];", 0)]),
    ("ln_variance_not_centred", [("        var += (x[d] - mu) * (x[d] - mu);",
                                  "        var += x[d] * x[d];", 0)]),
    ("ln_mean_over_D_minus_1", [("    return s / (double)D;", "    return s / (double)(D - 1);", 0)]),
    ("ln_bwd_mean_h_dropped", [("r * (h[d] - mean_h - xh[d] * mean_hx);",
                                "r * (h[d] - xh[d] * mean_hx);", 0)]),
    ("ln_bwd_projection_dropped", [("r * (h[d] - mean_h - xh[d] * mean_hx);",
                                    "r * (h[d] - mean_h);", 0)]),
    ("ln_bwd_xh_not_centred", [("            xh[d] = (xr[d] - mu) * r;", "            xh[d] = xr[d] * r;", 0)]),
    ("ln_bwd_unrotate_sign", [("            g[i + half] = -dyr[i] * s + dyr[i + half] * c;",
                               "            g[i + half] = dyr[i] * s + dyr[i + half] * c;", 0)]),
    ("lw_mean_over_D_only", [("        double r = 1.0 / sqrt(ss / (double)HD + eps);\n        rstd[t] = r;",
                              "        double r = 1.0 / sqrt(ss / (double)D + eps);\n        rstd[t] = r;", 0)]),
    ("lw_gamma_per_dim_only", [("                yr[d] = xr[d] * r * gamma[h * D + d];",
                                "                yr[d] = xr[d] * r * gamma[d];", 0)]),
    ("lw_bwd_dot_dropped", [("dx[t * HD + e] = r * (g[e] * gamma[e] - xt[e] * r * dot / (double)HD);",
                             "dx[t * HD + e] = r * (g[e] * gamma[e]);", 0)]),
    ("lw_bwd_dgamma_without_r", [("            dgamma[e] += g[e] * xt[e] * r;",
                                  "            dgamma[e] += g[e] * xt[e];", 0)]),
    ("rope_inverse_ignored", [("            s = -s;", "            s = s;", 0)]),
    ("rope_sin_sign_first", [("yr[i] = xr[i] * c - xr[i + half] * s;",
                              "yr[i] = xr[i] * c + xr[i + half] * s;", 0)]),
    ("rope_pass_through_zeroed", [("            yr[d] = xr[d];", "            yr[d] = 0.0;", 0)]),
    ("rope_position_plus_one", [("double phi = (double)m[j] * oracle_inv_freq(i, R, theta);",
                                 "double phi = (double)(m[j] + 1) * oracle_inv_freq(i, R, theta);", 0)]),
]


def _replace_nth(src, old, new, n):
    at = -1
    for _ in range(n + 1):
        at = src.find(old, at + 1)
        assert at >= 0, f"mutation anchor not found: {old!r}"
    return src[:at] + new + src[at + len(old):]


@pytest.mark.parametrize("name,edits", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(tmp_path, name, edits):
    with open(obuild.SRC) as f:
        src = f.read()
    for old, new, n in edits:
        src = _replace_nth(src, old, new, n)
    csrc = os.path.join(tmp_path, "mutant.c")
    with open(csrc, "w") as f:
        f.write(src)
    lib = obuild.build(csrc, os.path.join(tmp_path, "libmutant.so"))
    orc = oracle.Oracle(lib)
    failed = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(orc)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake {name!r}"
