"""Plant plausible mistakes in copies of the oracle and check that the pins catch each one.

Every mutant is a one-line edit of dao.c compiled into a separate library; the
real oracle is untouched.  A mutant that passes the whole pin battery would mean
the pins leave that part of the oracle unchecked.
"""

import os

import pytest

import oracle
import oracle_pins as P

MUTANTS = [
    ("gqa head mapping", "const int32_t g = h / group;", "const int32_t g = h % num_kv_heads;"),
    ("score without scale", "s[t] = scale * dot;", "s[t] = dot;"),
    ("query head index", "q + ((int64_t)b * num_q_heads + h) * head_dim", "q + ((int64_t)b * num_q_heads + 0) * head_dim"),
    ("page slot of K", "const int64_t kt = (((int64_t)page * num_kv_heads + g) * page_size + t % page_size)",
     "const int64_t kt = (((int64_t)page * num_kv_heads + g) * page_size + (t + 1) % page_size)"),
    ("kv head stride of V", "const int64_t vt = (((int64_t)page * num_kv_heads + g)",
     "const int64_t vt = (((int64_t)page * num_kv_heads + 0)"),
    ("V read from K", "o[j] += w * kv_elem(kv, 1, vt + j, g);", "o[j] += w * kv_elem(kv, 0, vt + j, g);"),
    ("fp8 exponent bias", "else mag = ldexp((double)(8 + m), e - 10);", "else mag = ldexp((double)(8 + m), e - 11);"),
    ("fp8 subnormal step", "if (e == 0) mag = ldexp((double)m, -9);", "if (e == 0) mag = ldexp((double)m, -10);"),
    ("fp8 V scaled by K's scale", "const double sc = is_v ? kv->v_scale[g] : kv->k_scale[g];",
     "const double sc = kv->k_scale[g];"),
    ("fp8 scale ignored", "return sc * e4m3_to_double(", "return e4m3_to_double("),
    ("multi-query causal offset", "const int64_t li = L - q_len + i + 1;", "const int64_t li = L - q_len + i;"),
    ("multi-query wrong block-table row", "block_table + (int64_t)b * max_pages_per_req,\n",
     "block_table + (int64_t)0 * max_pages_per_req,\n"),
    ("block table row", "block_table[(int64_t)b * max_pages_per_req + t / page_size];\n      if",
     "block_table[(int64_t)b + t / page_size];\n      if"),
    ("lse without max", "lse[i] = m + log(l);", "lse[i] = log(l);"),
    ("output not normalised", "const double w = exp(s[t] - m) / l;", "const double w = exp(s[t] - m);"),
    ("exp sign", "l += exp(s[t] - m);", "l += exp(m - s[t]);"),
    ("combine weight", "const double w = exp(lse_parts[i] - total);", "const double w = exp(lse_parts[i] - m);"),
    ("combine max", "if (lse_parts[i] > m) m = lse_parts[i];", "if (lse_parts[i] < m || m == -INFINITY) m = lse_parts[i];"),
    ("owner formula", "((u + 1) * C - 1) / U", "(u * C) / U"),
    ("tile count floor", "return (l + tile_tokens - 1) / tile_tokens;", "return l / tile_tokens;"),
    ("segment split on request only", "if (r != prev_r || c != prev_c) {", "if (r != prev_r) {"),
    ("cta_seg_begin off by one", "count += (seg_cta[s] < c);", "count += (seg_cta[s] <= c);"),
    ("static chunk floor", "const int64_t chunk = (max_tiles + splits - 1) / splits;",
     "const int64_t chunk = max_tiles / splits + (max_tiles < splits);"),
    ("bad length kept", "if (len < 0 || (int64_t)len > capacity) return 0;", "if (len < 0) return 0;"),
    ("start units for empty requests", "(int32_t)(n > 0 ? n + start_cost : 0)", "(int32_t)(n + start_cost)"),
    ("start units after the tiles", "const int64_t t = u - req_tile_prefix[r] - start_cost;",
     "const int64_t t = u - req_tile_prefix[r];"),
    ("weighted ranges over all units", "first[c] = c + (U - C) * Wc / W;", "first[c] = c + U * Wc / W;"),
    ("weighted owner at a range's first unit", "while (first[cw + 1] <= u) ++cw;", "while (first[cw + 1] < u) ++cw;"),
]


def battery(lib):
    failures = []
    for pin in P.ATTENTION_PINS + P.PLAN_PINS:
        try:
            if pin is P.pin_plan_brute_force:
                pin(lib=lib, exhaustive_batch=2, max_len=4)
            else:
                pin(lib=lib)
        except (AssertionError, ValueError, StopIteration) as e:
            failures.append(pin.__name__)
    return failures


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(name, old, new, tmp_path, oracle_lib):
    src = oracle.source_text()
    assert src.count(old) == 1, f"mutation site for '{name}' not unique in dao.c"
    path = oracle.compile_variant(src.replace(old, new), os.path.join(tmp_path, "libdao_mutant.so"))
    lib = oracle._bind(path)
    caught = battery(lib)
    assert caught, f"no pin caught the planted mistake '{name}'"
