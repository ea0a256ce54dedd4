"""Each plausible mistake planted in a copy of the oracle's source must make
at least one pin fail (so the pins would catch it in the real oracle)."""
import os

import pytest

import oracle
from oracle.build import SRC, build_variant
import oracle_pins as P

# (name, original text, mutated text): all edits stay memory-safe.
MUTANTS = [
    ("interp_direction", "x.wa = (real)(1.0 - g[k].w);", "x.wa = (real)g[k].w;"),
    ("interp_second_row", "x.b = i - g[k].lo - 1;", "x.b = i - g[k].lo;"),
    ("drop_rule", "if (i - g[k].c < 0) continue;", "if (i - g[k].c < 1) continue;"),
    ("window_shift", "int64_t j = i - t;", "int64_t j = i - t - 1;"),
    ("sink_future", "if ((int64_t)s > i) continue;", "if ((int64_t)s > i + 1) continue;"),
    ("rope_sign", "out[j] = a * cs - b * sn;", "out[j] = a * cs + b * sn;"),
    ("rope_freq", "double theta = pow(base, -2.0 * (double)j / (double)D);\n    double ang = (double)pos * theta;\n    real cs = (real)cos(ang), sn = (real)sin(ang);\n    real a = x[j], b = x[j + half];\n    out[j] = a * cs - b * sn;",
     "double theta = pow(base, -1.0 * (double)j / (double)D);\n    double ang = (double)pos * theta;\n    real cs = (real)cos(ang), sn = (real)sin(ang);\n    real a = x[j], b = x[j + half];\n    out[j] = a * cs - b * sn;"),
    ("rope_t_sign", "out[j] = a * cs + b * sn;", "out[j] = a * cs - b * sn;"),
    ("lse_no_log", "LSE[u * T + i] = any_nan ? (real)NAN : mx + (real)log((double)sum)",
     "LSE[u * T + i] = any_nan ? (real)NAN : mx"),
    ("decode_lse_no_log", "LSE1[u] = any_nan ? (real)NAN : mx + (real)log((double)sum)",
     "LSE1[u] = any_nan ? (real)NAN : mx"),
    ("geometry_round", "float fl = floorf(d);", "float fl = roundf(d);"),
    ("dq_no_scale", "dQ[base_off + i * D + d] *= (real)s;", "dQ[base_off + i * D + d] *= (real)1;"),
    ("dk_second_weight", "dKr[mb[m].b * D + d] += mb[m].wb * gs * qh[d];",
     "dKr[mb[m].b * D + d] += mb[m].wa * gs * qh[d];"),
    ("dv_second_row", "dVu[mb[m].b * D + d] += mb[m].wb * pm * go[d];",
     "dVu[mb[m].a * D + d] += mb[m].wb * pm * go[d];"),
    ("dalpha_v_term", "+ pm * go[d] * (vb[d] - va[d]);", ";"),
    ("dalpha_sign", "t += gs * qh[d] * (kb[d] - ka[d])", "t += gs * qh[d] * (ka[d] - kb[d])"),
    ("dalpha_no_f", "dal += (real)g[mb[m].k].f * t;", "dal += t;"),
    ("dsigma_no_D", "const real gs = pm * (dp[m] - Dsum);", "const real gs = pm * dp[m];"),
    ("theta_map_offset", "alpha[l] = (real)(0.5 + 1.0 / (1.0 + exp(-(double)theta[l])));",
     "alpha[l] = (real)(1.0 / (1.0 + exp(-(double)theta[l])));"),
    ("dtheta_no_derivative", "dtheta[l] = (real)((double)dalpha[l] * s * (1.0 - s));",
     "dtheta[l] = (real)((double)dalpha[l] * s);"),
    ("decode_key_position", "rope_row(Ku + mb[m].a * D, mb[m].a, D, rope_base, ka);",
     "rope_row(Ku + mb[m].a * D, pos, D, rope_base, ka);"),
    ("decode_second_key_weight", "v += mb[m].wb * dot(qh, kb, D);", "v += mb[m].wa * dot(qh, kb, D);"),
    ("prior_on_window", "sc[m] = dot(qh, row, D);\n        if (beta && mb[m].kind == 2)",
     "sc[m] = dot(qh, row, D);\n        if (beta && mb[m].kind != 1)"),
    ("prior_sign", "sc[m] = dot(qh, row, D);\n        if (beta && mb[m].kind == 2) sc[m] += beta",
     "sc[m] = dot(qh, row, D);\n        if (beta && mb[m].kind == 2) sc[m] -= beta"),
    ("prior_key_index", "sc[m] = dot(qh, row, D);\n        if (beta && mb[m].kind == 2) sc[m] += beta[u * T + i];",
     "sc[m] = dot(qh, row, D);\n        if (beta && mb[m].kind == 2) sc[m] += beta[u * T + mb[m].a];"),
    ("bwd_prior_missing", "sc[m] = dot(qh, krow + m * D, D);\n        if (beta && mb[m].kind == 2)",
     "sc[m] = dot(qh, krow + m * D, D);\n        if (beta && mb[m].kind == 99)"),
    ("dbeta_all_members", "if (mb[m].kind == 2) dbet += gs;", "dbet += gs;"),
    ("dbeta_uses_p", "if (mb[m].kind == 2) dbet += gs;", "if (mb[m].kind == 2) dbet += pm;"),
    ("decode_prior_on_window", "if (beta1 && mb[m].kind == 2) v += beta1[u];",
     "if (beta1 && mb[m].kind != 1) v += beta1[u];"),
    ("decode_query_scale", "for (int d = 0; d < D; ++d) qh[d] = (real)s * qh[d];\n    int n = members_of(pos",
     "for (int d = 0; d < D; ++d) qh[d] = qh[d];\n    int n = members_of(pos"),
]


@pytest.fixture(scope="module")
def source():
    with open(SRC) as f:
        return f.read()


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, source, name, old, new):
    assert source.count(old) == 1, f"mutation anchor for {name} not unique"
    lib = build_variant(source.replace(old, new), str(tmp_path), name)
    orc = oracle.Oracle(lib)
    failed = []
    for pin in P.ALL_PINS:
        try:
            pin(orc)
        except AssertionError:
            failed.append(pin.__name__)
            break
    assert failed, f"no pin caught mutant {name}"
