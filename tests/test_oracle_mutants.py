"""Plant plausible mistakes in copies of the oracle (on the CPU) and check that
each one fails at least one pin.  This is what makes the pins worth trusting:
a dropped term, a wrong sign, a transposed operand or an off-by-one in the
oracle cannot pass them."""
import pytest

import oracle
from tests import oracle_pins

with open(oracle.SRC) as _fh:
    SRC = _fh.read()

# (name, text in the oracle, replacement)
MUTANTS = [
    ("silu_sign", "return z / (1.0 + exp(-z));", "return z / (1.0 + exp(z));"),
    ("strict_threshold", "int on = ((float)s >= tau);", "int on = ((float)s > tau);"),
    ("tie_to_higher_index", "if (best < 0 || p[e] > p[best]) best = e;",
     "if (best < 0 || p[e] >= p[best]) best = e;"),
    ("drop_shared", "for (int s = 0; s < S; ++s) {", "for (int s = 0; s < 0; ++s) {"),
    ("gate_transposed", "for (int j = 0; j < f; ++j) g[j] += xi * bf16_to_double(rg[j]);",
     "for (int j = 0; j < f; ++j) g[j] += xi * bf16_to_double(wg[(size_t)j * d + i]);"),
    ("drop_router_weight", "yt[i] += w[r] * h * bf16_to_double",
     "yt[i] += h * bf16_to_double"),
    ("down_uses_u_not_h", "double h = a * u[j];", "double h = u[j];"),
    ("score_from_g", "double s = fabs(a);", "double s = fabs(g[j]);"),
    ("unnormalised_softmax", "for (int e = 0; e < E; ++e) p[e] /= sum;",
     "for (int e = 0; e < E; ++e) p[e] /= 1.0;"),
    ("no_mask", "if (!on) continue;", ";"),
    ("down_transposed", "yt[i] += w[r] * h * bf16_to_double(down[(size_t)j * d + i]);",
     "yt[i] += w[r] * h * bf16_to_double(down[(size_t)i * f + j]);"),
    ("router_transposed", "bf16_to_double(wr[(size_t)e * d + i]);",
     "bf16_to_double(wr[(size_t)i * E + e]);"),
    ("calibration_off_by_one", "double tau = c[m];", "double tau = c[m > 0 ? m - 1 : 0];"),
    ("up_from_gate", "for (int j = 0; j < f; ++j) u[j] += xi * bf16_to_double(ru[j]);",
     "for (int j = 0; j < f; ++j) u[j] += xi * bf16_to_double(rg[j]);"),
    ("mask_input_ignored", "if (active_in) on = (active_in[o] != 0);", ";"),
    ("mask_input_inverted", "if (active_in) on = (active_in[o] != 0);", "if (active_in) on = (active_in[o] == 0);"),
    ("shared_mask_ignored", "if (!((float)ss >= tau_shared)) continue;", ";"),
    ("shared_mask_uses_routed_tau", "if (!((float)ss >= tau_shared)) continue;",
     "if (!((float)ss >= tau)) continue;"),
    ("shared_mask_strict", "if (!((float)ss >= tau_shared)) continue;", "if (!((float)ss > tau_shared)) continue;"),
    ("shared_weighted", "for (int i = 0; i < d; ++i) yt[i] += h * bf16_to_double(down[(size_t)j * d + i]);",
     "for (int i = 0; i < d; ++i) yt[i] += 0.5 * h * bf16_to_double(down[(size_t)j * d + i]);"),
    ("rank_tie_to_higher_index", "return (a->j > b->j) - (a->j < b->j);", "return (a->j < b->j) - (a->j > b->j);"),
    ("rank_ascending", "if (va > vb) return -1;\n    if (va < vb) return 1;",
     "if (va > vb) return 1;\n    if (va < vb) return -1;"),
    ("rank_keeps_one_more", "for (int q = 0; q < n && q < r; ++q) mp[e[q].j] = 1;",
     "for (int q = 0; q < n && q <= r; ++q) mp[e[q].j] = 1;"),
    ("rank_keeps_nan", "if (sp[j] == sp[j]) {   /* not NaN */", "if (1) {"),
    ("rank_in_double", "const float va = (float)a->v, vb = (float)b->v;", "const double va = a->v, vb = b->v;"),
    ("capacity_tie_to_higher_token", "if (wq > wp || (wq == wp && q / k < tp)) ++better;",
     "if (wq > wp || (wq == wp && q / k > tp)) ++better;"),
    ("capacity_keeps_lowest", "if (wq > wp || (wq == wp && q / k < tp)) ++better;",
     "if (wq < wp || (wq == wp && q / k < tp)) ++better;"),
    ("capacity_keeps_one_more", "keep[p] = (uint8_t)(better < C);", "keep[p] = (uint8_t)(better <= C);"),
    ("capacity_across_experts", "if (q == p || idx[q] != e) continue;", "if (q == p) continue;"),
    ("capacity_in_double", "const float wq = (float)w[q];", "const double wq = w[q];"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new):
    assert SRC.count(old) == 1, f"mutation site for {name} not unique/present"
    variant = oracle.build_variant(SRC.replace(old, new), str(tmp_path))
    failures = {k: v for k, v in oracle_pins.run_all(variant).items() if v}
    assert failures, f"planted mistake '{name}' passed every pin"


def test_unmutated_copy_passes(tmp_path):
    variant = oracle.build_variant(SRC, str(tmp_path))
    assert not any(oracle_pins.run_all(variant).values())
