"""Planted mistakes in the CPU oracle must each trip one of the pins.

Each mutant is a copy of ``oracle/lsa_oracle.c`` with one plausible slip (a dropped
term, a flipped sign or comparison, a transposed operand, a wrong index), compiled
into a temporary library and run through the pins in dependency order; the first
pin that fails kills the mutant.  Pins run cheapest-first so that a broken
primitive is caught before a composite routine could be driven out of bounds.
"""
import os
import shutil
import tempfile

import pytest

from oracle import oracle as orc
from tests import oracle_pins as P

ORDER = [
    P.pin_splitmix64_published_vectors, P.pin_init_rule, P.pin_projection_matches_numpy,
    P.pin_distances_closed_form, P.pin_balanced_assign_bruteforce,
    P.pin_balanced_assign_vs_deferred_acceptance, P.pin_tree_invariants,
    P.pin_tree_first_step_from_init, P.pin_tree_rounds_from_trace, P.pin_tree_independent_rebuild,
    P.pin_tree_deterministic_and_seeded,
    P.pin_select_beam_walk, P.pin_select_full_beam_equals_flat,
    P.pin_attention_equals_sdpa, P.pin_attention_special_cases,
    P.pin_backward_autograd, P.pin_backward_finite_differences,
    P.pin_attention_sink_window, P.pin_backward_sink_window_autograd, P.pin_tree_pooled, P.pin_tree_append,
]
assert sorted(f.__name__ for f in ORDER) == sorted(f.__name__ for f in P.ALL_PINS)

# (name, original text, planted text): each original occurs exactly once in the source
MUTANTS = [
    ("mixer shift", "z = (z ^ (z >> 30))", "z = (z ^ (z >> 29))"),
    ("init picks largest hash", "if (best < 0 || h < best_h)", "if (best < 0 || h > best_h)"),
    ("projection transposed W", "acc += X[i * d + j] * W[(int64_t)j * r + k];",
     "acc += X[i * d + j] * W[(int64_t)k * d + j];"),
    ("query mean not divided", "mean[j] = s / (double)G;", "mean[j] = s;"),
    ("distance not squared", "acc += diff * diff;", "acc += diff < 0 ? -diff : diff;"),
    ("capacity off by one", "count[p->c] < cap", "count[p->c] <= cap"),
    ("position tie-break reversed", "if (x->pos < y->pos) return -1;\n  if (x->pos > y->pos) return 1;",
     "if (x->pos > y->pos) return -1;\n  if (x->pos < y->pos) return 1;"),
    ("mean over wrong count", "mu[(int64_t)c * r + k] / (double)cnt[c]",
     "mu[(int64_t)c * r + k] / (double)(cnt[c] + 1)"),
    ("init of every level uses level 0", "e = orc_level_init(Zs, pos, m, r, b, seed, l, mu);",
     "e = orc_level_init(Zs, pos, m, r, b, seed, 0, mu);"),
    ("means updated only after the last round", "        orc_means(Zs, m, r, a, b, mu);\n      }",
     "        if (t == iters - 1) orc_means(Zs, m, r, a, b, mu);\n      }"),
    ("only the first and last rounds run", "for (int32_t t = 0; t < iters && e == ORC_OK; ++t) {",
     "for (int32_t t = 0; t < iters && e == ORC_OK; t = (t == 0 ? iters - 1 : t + 1)) {"),
    ("one round short", "for (int32_t t = 0; t < iters && e == ORC_OK; ++t) {",
     "for (int32_t t = 0; t < iters - 1 && e == ORC_OK; ++t) {"),
    ("children numbered transposed", "next[(s * b + j) * cap + fill[j]] = pos[i];",
     "next[(j * segs + s) * cap + fill[j]] = pos[i];"),
    ("min position as max", "if (pos[i] < min_pos[node_off + s * b + j])",
     "if (pos[i] > min_pos[node_off + s * b + j] || min_pos[node_off + s * b + j] == INT32_MAX)"),
    ("beam keeps lowest scores", "if (x->s > y->s) return -1;\n  if (x->s < y->s) return 1;",
     "if (x->s < y->s) return -1;\n  if (x->s > y->s) return 1;"),
    ("child ids not scaled", "ids[n_ids++] = kept[k] * branching[l + 1] + j;",
     "ids[n_ids++] = kept[k] + j;"),
    ("node eligibility strict", "min_pos[node_off[l] + id] > q_pos[t]",
     "min_pos[node_off[l] + id] >= q_pos[t]"),
    ("leaf slice not scaled", "leaf_index[kept[k] * leaf_size + q]", "leaf_index[kept[k] + q]"),
    ("causal mask excludes diagonal", "if (causal && j > q_pos[t]) continue;\n    out[cnt++] = j;\n  }\n  for",
     "if (causal && j >= q_pos[t]) continue;\n    out[cnt++] = j;\n  }\n  for"),
    ("tail starts one late", "for (int64_t j = tail_begin; j < tail_end; ++j)",
     "for (int64_t j = tail_begin + 1; j < tail_end; ++j)"),
    ("logit not scaled", "logit[k] = scale * s;", "logit[k] = s;"),
    ("softmax not normalised", "double p = exp(logit[k] - mx) / l;", "double p = exp(logit[k] - mx);"),
    ("LSE drops the max", "LSE[t * G + h] = mx + log(l);", "LSE[t * G + h] = log(l);"),
    ("softmax gradient drops delta", "const double ds = p[k] * (dp[k] - delta);",
     "const double ds = p[k] * dp[k];"),
    ("dK sign flipped", "gk[j] += scale * ds * q[j];", "gk[j] -= scale * ds * q[j];"),
    ("dV ignores probabilities", "gv[j] += p[k] * go[j];", "gv[j] += go[j];"),
    ("dQ unscaled", "gq[j] += scale * ds * kr[j];", "gq[j] += ds * kr[j];"),
    ("window one key short", "for (int64_t j = (int64_t)q_pos[t] - window + 1; j <= q_pos[t]; ++j)",
     "for (int64_t j = (int64_t)q_pos[t] - window + 2; j <= q_pos[t]; ++j)"),
    ("sink ignores causality", "if (j <= q_pos[t]) out[cnt++] = j;", "out[cnt++] = j;"),
    ("repeated key counted twice", "if (u == 0 || out[k] != out[u - 1]) out[u++] = out[k];", "out[u++] = out[k];"),
    ("pool drops a key", "for (int32_t i = 0; i < p; ++i) s += Z[(j * p + i) * r + c];",
     "for (int32_t i = 1; i < p; ++i) s += Z[(j * p + i) * r + c];"),
    ("pool sums instead of averaging", "Zp[j * r + c] = s / p;", "Zp[j * r + c] = s;"),
    ("pooled keys not expanded", "leaf_index[s * p + i] = blocks[s] * p + i;", "leaf_index[s * p + i] = blocks[s] + i;"),
    ("pooled min_pos left in blocks", "for (int64_t k = 0; k < nodes; ++k) min_pos[k] *= p;",
     "for (int64_t k = 0; k < nodes; ++k) min_pos[k] *= 1;"),
    ("appended root not averaged", "cent[(new_off + old_nodes) * r + c] = s / (double)U;",
     "cent[(new_off + old_nodes) * r + c] = s / (double)(U - 1);"),
    ("appended min_pos not shifted", "min_pos[new_off + old_nodes + k] = sm[sub_off + k] + (int32_t)n_old;",
     "min_pos[new_off + old_nodes + k] = sm[sub_off + k];"),
    ("appended keys not shifted", "leaf_index[n_old + i] = sl[i] + (int32_t)n_old;", "leaf_index[n_old + i] = sl[i];"),
    ("subtree centroids copied from the old nodes",
     "memcpy(&cent[(new_off + old_nodes) * r], &sc[sub_off * r], sizeof(double) * sub_nodes * r);",
     "memcpy(&cent[(new_off + old_nodes) * r], &cent[new_off * r], sizeof(double) * sub_nodes * r);"),
]


@pytest.fixture(scope="module")
def workdir():
    d = tempfile.mkdtemp(prefix="lsa_mutants_")
    yield d
    shutil.rmtree(d, ignore_errors=True)


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(workdir, name, old, new):
    src = open(orc._SRC).read()
    assert src.count(old) == 1, f"mutation site for {name!r} not unique"
    tag = "".join(ch if ch.isalnum() else "_" for ch in name)
    c_path = os.path.join(workdir, f"m_{tag}.c")
    so_path = os.path.join(workdir, f"m_{tag}.so")
    with open(c_path, "w") as f:
        f.write(src.replace(old, new))
    orc.build(force=True, src=c_path, out=so_path)
    caught = None
    with orc.using(so_path):
        for pin in ORDER:
            try:
                pin()
            except (AssertionError, orc.OracleError):
                caught = pin.__name__
                break
    assert caught is not None, f"mutant {name!r} survived every pin"
