"""Plant plausible mistakes in a copy of the oracle and show that the pins
catch every one of them (CPU only; the real oracle is never modified)."""
import os
import subprocess

import pytest

import oracle
import oracle_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "attn_oracle.c")

# (name, text in attn_oracle.c, replacement)
MUTATIONS = [
    ("drop_scale", "s[j] = p->scale * acc;", "s[j] = acc;"),
    ("wrong_group_index", "const int g = h / (p->n_q / p->n_kv);", "const int g = h % p->n_kv;"),
    ("causal_off_by_one", "int64_t end = i + ((int64_t)p->Skv - (int64_t)p->Sq) + 1;",
     "int64_t end = i + ((int64_t)p->Skv - (int64_t)p->Sq);"),
    ("causal_top_left", "int64_t end = i + ((int64_t)p->Skv - (int64_t)p->Sq) + 1;",
     "int64_t end = i + 1;"),
    ("no_max_subtraction", "const double e = exp(s[j] - m);", "const double e = exp(s[j]); m = 0.0;"),
    ("lse_log2", "*lse_out = m + log(l);", "*lse_out = m + log2(l);"),
    ("lse_without_max", "*lse_out = m + log(l);", "*lse_out = log(l);"),
    ("no_normalisation", "for (int c = 0; c < p->d_v; ++c) o_row[c] /= l;", ""),
    ("keys_as_values", "const double *vj = vb + j * p->v_ss;", "const double *vj = kb + j * p->k_ss;"),
    ("value_head_ungrouped", "const double *vb = p->v + b * p->v_sb + g * p->v_sh;",
     "const double *vb = p->v + b * p->v_sb + (h % p->n_kv) * p->v_sh;"),
    ("ignore_seqlens", "if (p->seqlens) {", "if (0) {"),
    ("online_no_rescale", "for (int c = 0; c < d_v; ++c) ar[c] *= alpha;", ""),
    ("online_l_no_rescale", "l[r] = alpha * l[r] + rowsum;", "l[r] = l[r] + rowsum;"),
    ("online_rescale_sign", "const double alpha = exp(m[r] - m_new);",
     "const double alpha = exp(m_new - m[r]);"),
    ("online_lse_stale", "lse[row] = m[r] + log(l[r]);", "lse[row] = log(l[r]);"),
    ("window_off_by_one", "return (end - 1 - j < p->window) || (j < p->n_sink);",
     "return (end - 1 - j <= p->window) || (j < p->n_sink);"),
    ("window_sinks_ignored", "return (end - 1 - j < p->window) || (j < p->n_sink);",
     "return (end - 1 - j < p->window);"),
    ("window_anchored_at_row_not_position", "return (end - 1 - j < p->window) || (j < p->n_sink);",
     "return (end - 1 - j - (p->Skv - p->Sq) < p->window) || (j < p->n_sink);"),
    ("rope_sin_sign", "oi[2 * j] = xe * c - xo * s;", "oi[2 * j] = xe * c + xo * s;"),
    ("rope_rotate_half", "const double xe = xi[2 * j], xo = xi[2 * j + 1];",
     "const double xe = xi[j], xo = xi[j + half];"),
    ("rope_theta_exponent", "pow(base, -2.0 * (double)j / (double)d)", "pow(base, -(double)j / (double)d)"),
    ("rope_position_shift", "const int m = pos[i];", "const int m = pos[i] > 0 ? pos[i] - 1 : 0;"),
    ("rope_cos_sin_swapped", "cos_t[(int64_t)m * half + j] = cos(a);", "cos_t[(int64_t)m * half + j] = sin(a);"),
]


def _build_mutant(tmp_path, name, old, new):
    text = open(SRC).read()
    assert text.count(old) >= 1, f"mutation {name}: pattern not found"
    src = tmp_path / f"{name}.c"
    src.write_text(text.replace(old, new, 1))
    so = tmp_path / f"lib{name}.so"
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-fopenmp", str(src), "-o",
                    str(so), "-lm"], check=True)
    return oracle.load(str(so))


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_mutation_is_caught(tmp_path, name, old, new):
    lib = _build_mutant(tmp_path, name, old, new)
    caught = []
    for check in oracle_pins.ALL_CHECKS:
        try:
            check(lib)
        except (AssertionError, ValueError, FloatingPointError):
            caught.append(check.__name__)
    assert caught, f"no pin catches the planted mistake {name}"
