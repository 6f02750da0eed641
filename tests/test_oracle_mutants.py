"""Plant one plausible mistake at a time in a COPY of the oracle source and
check that at least one pin fails for each (CPU only; the committed oracle is
never edited)."""
import pytest

import oracle
from oracle_pins import PINS

# (name, text in oracle.c, replacement); a list pairs several edits
MUTANTS = [
    ("interleaved_head_map", "int g = h / G;", "int g = h % p->h_kv;"),
    ("dropped_scale", "return p->scale * acc;", "return acc;"),
    ("no_max_shift", "double w = exp(s_buf[j - lo] - M);", "double w = exp(s_buf[j - lo]);"),
    ("merge_sign", "double a = exp(M - mc), bw = exp(mi - mc);", "double a = exp(mc - M), bw = exp(mi - mc);"),
    ("no_normalise", "dst[t] = l > 0.0 ? o_tmp[t] / l : 0.0;", "dst[t] = o_tmp[t];"),
    ("k_for_v", "o_out[t] += w * elem(p->v, vi + t, p->dtype);", "o_out[t] += w * elem(p->k, vi + t, p->dtype);"),
    ("split_off_by_one", "int64_t a = (int64_t)i * L, e = a + L;", "int64_t a = (int64_t)i * L, e = a + L - 1;"),
    ("merge_no_empty_guard", ["if (mi == -INFINITY) continue;", "if (M == -INFINITY) {"],
     ["", "if (0) {"]),
    ("merge_drops_l_term", "L = L * a + l[idx] * bw;", "L = L + l[idx] * bw;"),
    ("q_k_index_swap", "int64_t ki = ((p->row_off[b] + j) * p->h_kv + g) * p->d;",
     "int64_t ki = ((p->row_off[b] + j) * p->h_kv + (h % p->h_kv)) * p->d;"),
    ("ceil_as_floor", "(S + p->n_splits - 1) / p->n_splits", "S / p->n_splits"),
    ("wrong_row_offset", "row_off[b] = acc;", "row_off[b] = b * (int64_t)p->seqlens[0];"),
    ("prefill_excludes_diagonal", "range_triplet_at(p, b, h, i, 0, (int64_t)i + 1,",
     "range_triplet_at(p, b, h, i, 0, (int64_t)i + (i == 0),"),
    ("prefill_query_row_of_first_position", "int64_t qrow = p->causal ? p->row_off[b] + i : (int64_t)b;",
     "int64_t qrow = p->causal ? p->row_off[b] : (int64_t)b;"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(tmp_path, name, old, new):
    src = oracle.source()
    olds, news = (old, new) if isinstance(old, list) else ([old], [new])
    for o, n in zip(olds, news):
        assert o in src, f"mutation target for {name} not found: {o}"
        src = src.replace(o, n)
    orc = oracle.compile_variant(src, str(tmp_path / f"mut_{name}.so"))
    failed = []
    for pin in PINS:
        try:
            pin(orc)
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake {name}"
