"""Strength of the oracle's pins: each plausible mistake below is planted in a
copy of the oracle's C source (on the CPU, in a temporary directory), and the
oracle's own CPU tests must then fail.  A mistake that every pin lets through
would be a mistake the CUDA path could share unnoticed.

The mistakes cover each step the oracle restates: the E2M1 / E4M3 value
definitions and round-to-nearest-even encoders, the block quantisation (scale
= E4M3(amax / 6), nibble order, code = E2M1(x / s)), the index-key encoding,
the scoring s_t = sum_h w_h max(0, q_h . k_t), the top-n selection, the Full
and Reindex selections, the paged slot map, the causal query position, and the
sparse + window attention (window bounds, future entries, scale, softmax
normaliser, log-sum-exp) and its layer-local window rows (ring slot, which
positions take a ring row), the append-time pool update and the merge of
attention partials over disjoint parts."""
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "csa2_ref.c")
PIN_TESTS = ["tests/test_oracle_formats.py", "tests/test_oracle_index.py", "tests/test_oracle_attn.py"]

MUTATIONS = [
    ("ties_round_up", "(d1 == d0 && ((lo + 1) & 1) == 0)", "(d1 == d0)"),
    ("e4m3_saturates_low", "nearest_code(fabs(x), ref_e4m3_value, 0x7E)", "nearest_code(fabs(x), ref_e4m3_value, 0x7D)"),
    ("e4m3_subnormal_scale", "        mag = ldexp((double)m / 8.0, 1 - 7);", "        mag = ldexp((double)m / 8.0, -7);"),
    ("e2m1_subnormal_value", "        mag = ldexp((double)m / 2.0, 1 - 1);", "        mag = ldexp((double)m, 1 - 1);"),
    ("negative_zero_loses_sign", "return (uint8_t)((signbit(x) ? 8 : 0) | code);", "return (uint8_t)((x < 0 ? 8 : 0) | code);"),
    ("amax_signed", "        float a = fabsf(x[i]);\n", "        float a = x[i];\n"),
    ("scale_amax_over_4", "    volatile float six = 6.0f;", "    volatile float six = 4.0f;"),
    ("scale_not_rounded", "    volatile float s = (float)ref_e4m3_value(sc);", "    volatile float s = sf;"),
    ("nibbles_swapped", "(uint8_t)((codes[2 * j] & 0xF) | ((codes[2 * j + 1] & 0xF) << 4))",
     "(uint8_t)((codes[2 * j + 1] & 0xF) | ((codes[2 * j] & 0xF) << 4))"),
    ("dequant_scale_per_32", "double s = ref_e4m3_value(row[D / 2 + d / 16]);", "double s = ref_e4m3_value(row[D / 2 + d / 32]);"),
    ("index_key_scaled", "[slot * c->idx_dim + d] = ref_e4m3_encode(v);", "[slot * c->idx_dim + d] = ref_e4m3_encode(v * 1.0625f);"),
    ("relu_dropped", "s += (double)w[h] * (dot > 0.0 ? dot : 0.0);", "s += (double)w[h] * dot;"),
    ("head_weight_dropped", "s += (double)w[h] * (dot > 0.0 ? dot : 0.0);", "s += (dot > 0.0 ? dot : 0.0);"),
    ("select_ascending", "    if (x->s > y->s) return -1;\n    if (x->s < y->s) return 1;",
     "    if (x->s < y->s) return -1;\n    if (x->s > y->s) return 1;"),
    ("full_skips_p", "    if (!rc) rc = ref_select_top(s, NULL, n, pool_k, pool_idx);\n    if (!rc) rc = ref_select_top(s, NULL, n, top_k, topk_idx);",
     "    if (!rc) rc = ref_select_top(s, NULL, n - 1, pool_k, pool_idx);\n    if (!rc) rc = ref_select_top(s, NULL, n - 1, top_k, topk_idx);"),
    ("reindex_returns_ranks", "w, s);\n    if (!rc) rc = ref_select_top(s, pos, n, top_k, topk_idx);",
     "w, s);\n    if (!rc) rc = ref_select_top(s, NULL, n, top_k, topk_idx);"),
    ("paged_slot_drops_offset", "        slot = (int64_t)phys * c->page_size + t % c->page_size;",
     "        slot = (int64_t)phys * c->page_size;"),
    ("query_position_one_early", "return (int64_t)c->seq_lens[b] - T + j;", "return (int64_t)c->seq_lens[b] - T + j - 1;"),
    ("window_one_short", "    int64_t lo = p - window + 1;\n    if (lo < 0) lo = 0;\n    for (int64_t t = lo;",
     "    int64_t lo = p - window + 2;\n    if (lo < 0) lo = 0;\n    for (int64_t t = lo;"),
    ("future_entry_clipped_to_p", "        if (t >= 0 && t <= p) in_s[t] = 1;", "        if (t >= 0) in_s[t < p ? t : p] = 1;"),
    ("scale_one_over_d", "    if (sm_scale <= 0.0) sm_scale = 1.0 / sqrt((double)D);\n    /* membership",
     "    if (sm_scale <= 0.0) sm_scale = 1.0 / (double)D;\n    /* membership"),
    ("softmax_normaliser_off", "        for (int64_t i = 0; i < nS; ++i) { z[i] = exp(z[i] - m); l += z[i]; }",
     "        for (int64_t i = 0; i < nS; ++i) { z[i] = exp(z[i] - m); l += z[i] * 0.999; }"),
    ("query_channels_swapped", "        for (int d = 0; d < D; ++d) qd[d] = (double)bf16_to_f32(q[(int64_t)h * D + d]);",
     "        for (int d = 0; d < D; ++d) qd[d] = (double)bf16_to_f32(q[(int64_t)h * D + (d ^ 1)]);"),
    ("lse_without_max", "        if (lse) lse[h] = m + log(l);\n    }\n    free(in_s);",
     "        if (lse) lse[h] = log(l);\n    }\n    free(in_s);"),
    ("ring_slot_shifted", "ring + ((int64_t)b * ring_len + t % ring_len) * D;",
     "ring + ((int64_t)b * ring_len + (t + 1) % ring_len) * D;"),
    ("ring_rows_for_every_position", "        if (ring && window > 0 && t >= lo) {", "        if (ring && window > 0) {"),
    ("pool_update_forgets_pool", "        if (pool_prev[i] < 0) continue;\n        if (pool_prev[i] >= t_new0",
     "        if (pool_prev[i] < 0 || i >= 0) continue;\n        if (pool_prev[i] >= t_new0"),
    ("merge_weights_unnormalised", "            double wgt = exp(lses[(int64_t)i * H + h] - l);",
     "            double wgt = exp(lses[(int64_t)i * H + h] - m);"),
    ("pool_update_misses_p", "    for (int64_t t = t_new0; t <= p && !rc; ++t) pos[n++] = (int32_t)t;",
     "    for (int64_t t = t_new0; t < p && !rc; ++t) pos[n++] = (int32_t)t;"),
]


def _copy_tree(dst):
    ign = shutil.ignore_patterns("__pycache__", "*.so", "*.so.tmp*", "csrc")
    for d in ("oracle", "tests", "fp4_sparse_attention_csa2_b200"):
        shutil.copytree(os.path.join(ROOT, d), os.path.join(dst, d), ignore=ign)


def _run_mutation(base, name, old, new):
    """Plant one mistake in a copy of the oracle and run the pins on it:
    (exit status, last line of the pytest report)."""
    d = os.path.join(base, name)
    _copy_tree(d)
    path = os.path.join(d, "oracle", "csa2_ref.c")
    with open(path) as f:
        src = f.read()
    if src.count(old) != 1:
        return None, "the mutation does not apply"
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    r = subprocess.run([sys.executable, "-m", "pytest", *PIN_TESTS, "-x", "-q", "-p", "no:cacheprovider"],
                       cwd=d, capture_output=True, text=True, timeout=600)
    return r.returncode, (r.stdout.strip().splitlines() or [""])[-1]


@pytest.fixture(scope="module")
def outcomes(tmp_path_factory):
    # every planted mistake in its own copy, several at a time
    base = str(tmp_path_factory.mktemp("mutations"))
    with ThreadPoolExecutor(max_workers=max(1, min(8, os.cpu_count() or 1))) as ex:
        futs = {name: ex.submit(_run_mutation, base, name, old, new) for name, old, new in MUTATIONS}
        return {name: f.result() for name, f in futs.items()}


def test_every_mutation_applies_to_the_current_source():
    src = open(SRC).read()
    for name, old, _ in MUTATIONS:
        assert src.count(old) == 1, name


@pytest.mark.parametrize("name", [m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(name, outcomes):
    rc, tail = outcomes[name]
    # exit status 1 with a failed test: the copy built and ran, and a pin caught the mistake
    assert rc == 1 and " failed" in tail, "%s: the pins let the planted mistake through (%s)" % (name, tail)
