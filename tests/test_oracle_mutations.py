"""Plant plausible mistakes in copies of the oracle (on the CPU) and check that
the pins catch every one of them."""
import os
import subprocess
import tempfile

import pytest

import oracle
from oracle_pins import ALL_PINS

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

# (name, exact text in oracle.c, replacement)
MUTANTS = [
    ("relu_dropped", "double relu = dot > 0.0 ? dot : 0.0;", "double relu = dot;"),
    ("head_weight_dropped", "s += bf16_to_f64(w_t[h]) * relu;", "s += relu;"),
    ("score_scale_dropped", "return s / sqrt((double)p->idx_dim);", "return s;"),
    ("causal_off_by_one", "if (j > t) continue;", "if (j > t + 1) continue;"),
    ("block_sum_not_max", "if (s > best) best = s;", "best = (best < 0.0 ? 0.0 : best) + s;"),
    ("key_dim_dropped", "for (int c = 0; c < p->idx_dim; ++c) dot +=", "for (int c = 1; c < p->idx_dim; ++c) dot +="),
    ("rope_sign", "y[i] = m * (x[i] * ca - x[i + half] * sa);", "y[i] = m * (x[i] * ca + x[i + half] * sa);"),
    ("rope_pairing", "y[i + half] = m * (x[i + half] * ca + x[i] * sa);",
     "y[i + half] = m * (x[i + half] * ca + x[(i + 1) % half] * sa);"),
    ("rope_freq", "pow(p->rope_theta, -2.0 * (double)i / d)", "pow(p->rope_theta, -1.0 * (double)i / d)"),
    ("yarn_scale_dropped", "return p->yarn_factor > 1.0 ? 0.1 * log(p->yarn_factor) + 1.0 : 1.0;", "return 1.0;"),
    ("yarn_ramp_reversed", "return f / s * ramp + f * (1.0 - ramp);", "return f * ramp + f / s * (1.0 - ramp);"),
    ("yarn_factor_multiplies", "return f / s * ramp + f * (1.0 - ramp);", "return f * s * ramp + f * (1.0 - ramp);"),
    ("tie_to_higher_index", "return (x->idx > y->idx) - (x->idx < y->idx);", "return (x->idx < y->idx) - (x->idx > y->idx);"),
    ("prev_block_not_forced", "for (int i = 0; i < budget - 2; ++i) sel[n++] = (int32_t)c[i].idx;\n  sel[n++] = (int32_t)(qb - 1);",
     "for (int i = 0; i < budget - 1; ++i) sel[n++] = (int32_t)c[i].idx;"),
    ("select_ascending_score", "if (x->s > y->s) return -1;\n  if (x->s < y->s) return 1;", "if (x->s < y->s) return -1;\n  if (x->s > y->s) return 1;"),
    ("attn_scale", "1.0 / sqrt((double)d)", "1.0 / (double)d"),
    ("gqa_map", "int g = h / (H / G);", "int g = h % G;"),
    ("lse_max_dropped", "lse[h] = m + log(z);", "lse[h] = log(z);"),
    ("causal_attn_off_by_one", "if (j <= t) js[n++] = j;", "if (j <= t + 1) js[n++] = j;"),
    ("value_head_swap", "vv[(e * G + g) * d + c] = bf16_to_f64(v[(js[e] * G + g) * d + c]);",
     "vv[(e * G + g) * d + c] = bf16_to_f64(v[(js[e] * G + (G - 1 - g)) * d + c]);"),
    ("mean_not_divided", "mean[c] = idx_operand(p, sum / (double)n);", "mean[c] = idx_operand(p, sum);"),
    ("operands_not_rounded_to_bf16", "return p->idx_exact ? v : bf16_to_f64(bf16_round_nearest_even(v));",
     "return v;"),
    ("mean_ties_away_from_zero", "(above == below && fmod(n_lo, 2.0) != 0.0)", "(above == below)"),
    ("idx_rope_key_at_block_end", "rope_vec(p, mean, p->idx_dim, p->idx_pos0 + kb * p->block, kbar);",
     "rope_vec(p, mean, p->idx_dim, p->idx_pos0 + kb * p->block + p->block - 1, kbar);"),
    ("idx_rope_query_not_rotated", "rope_vec(p, x, p->idx_dim, p->idx_pos0 + qb * r + i, dst);",
     "rope_vec(p, x, p->idx_dim, 0, dst);"),
    ("idx_rope_frequency", "const double a = (double)pos * rope_freq(p, i);",
     "const double a = (double)pos * rope_freq(p, i + 1);"),
    ("mean_pool_relu_dropped", "s += bf16_to_f64(w_blk[(int64_t)i * p->idx_heads + h]) * (dot > 0.0 ? dot : 0.0);",
     "s += bf16_to_f64(w_blk[(int64_t)i * p->idx_heads + h]) * dot;"),
    ("reuse_own_block_not_forced", "  in_set[qb] = 1;\n", "\n"),
    ("reuse_prev_block_not_forced", "  if (qb >= 1) in_set[qb - 1] = 1;\n", "\n"),
    ("reuse_row_dropped", "    in_set[sel_in[i]] = 1;", "    in_set[sel_in[i]] = 0;"),
    ("decode_new_key_position", "oracle_rope(p, x, L, kr + (e * G + g) * d);", "oracle_rope(p, x, L - 1, kr + (e * G + g) * d);"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, old, new):
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor not found: {name}"
    mutated = src.replace(old, new)
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "m.c")
        so = os.path.join(d, "m.so")
        open(c, "w").write(mutated)
        subprocess.run(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11", c, "-o", so, "-lm"], check=True)
        O = oracle.Oracle(L=oracle.load_variant(so))
        failed = []
        for pin in ALL_PINS:
            try:
                pin(O)
            except AssertionError:
                failed.append(pin.__name__)
        assert failed, f"mutant {name} passed every pin"
