"""Mutation check of the oracle's pins: each test compiles a copy of the
oracle's C source with one plausible mistake planted in it (on the CPU, in a
temporary directory) and requires that at least one pin from
``test_oracle_pins`` rejects the broken copy.  A mutant that no pin catches
would mean the pins leave that part of the oracle unchecked.
"""
import json
import os
import subprocess

import pytest

import oracle
import test_oracle_pins as pins
import test_oracle_row as row_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "monarch_oracle.c")

# (name, original text, replacement) -- every occurrence is replaced.
MUTANTS = [
    ("scale_1_over_d", "1.0 / sqrt((double)d)", "1.0 / (double)d"),
    ("no_scale", "1.0 / sqrt((double)d)", "1.0"),
    ("wrong_sign", "logit[j] = scale * acc;", "logit[j] = -scale * acc;"),
    ("unnormalised", "double p = logit[j] / z;", "double p = logit[j];"),
    ("dropped_feature", "for (int c = 0; c < d; ++c) acc += q[c] * krows[j][c];",
     "for (int c = 1; c < d; ++c) acc += q[c] * krows[j][c];"),
    ("shifted_value_column", "y[c] += p * vrows[j][c];", "y[c] += p * vrows[j][(c + 1) % d];"),
    ("stage2_values_are_v", "if (!st) st = stage2_groups(q, k, y1, out,",
     "if (!st) st = stage2_groups(q, k, v, out,"),
    ("stage1_blocks_position_major", "return b * (long)H * W + i;", "return i * (long)T + b;"),
    ("stage2_keys_contiguous", "kr[i] = kb + (i * gs + g) * d;", "kr[i] = kb + (g * gl + i) * d;"),
    ("stage2_query_is_key", "attend_one(qb + (i * gs + g) * d, kr, vr, gl,",
     "attend_one(kb + (i * gs + g) * d, kr, vr, gl,"),
    ("tile_rows_interleaved", "long h = ti * tile_h + hl, w = tj * tile_w + wl;",
     "long h = ti + hl * (H / tile_h), w = tj * tile_w + wl;"),
    ("tile_cols_interleaved", "long h = ti * tile_h + hl, w = tj * tile_w + wl;",
     "long h = ti * tile_h + hl, w = tj + wl * (W / tile_w);"),
    ("stage_order_swapped",
     "st = oracle_monarch_stage1(q, k, v, y1, B, heads, T, H, W, d, fact, tile_h, tile_w);\n"
     "    if (!st) st = stage2_groups(q, k, y1, out, B, heads, (long)T * H * W, stage2_stride(H, W, fact), d);",
     "st = stage2_groups(q, k, v, y1, B, heads, (long)T * H * W, stage2_stride(H, W, fact), d);\n"
     "    if (!st) st = oracle_monarch_stage1(q, k, y1, out, B, heads, T, H, W, d, fact, tile_h, tile_w);"),
    # the (f*h, w) split
    ("row_groups_are_positions", "return fact == ORACLE_FACT_ROW ? (long)W : (long)H * W;",
     "return (long)H * W;"),
    ("row_blocks_are_frames",
     "} else if (fact == ORACLE_FACT_ROW) {\n        *nblocks = (long)T * H;\n        *blocklen = W;",
     "} else if (fact == ORACLE_FACT_ROW) {\n        *nblocks = T;\n        *blocklen = (long)H * W;"),
]

GOLDEN = json.load(open(pins.GOLDEN))["cases"]

# The pins, as (label, callable) with fixed parameters.
PROBES = [(f"golden:{c['name']}", (lambda c=c: pins.test_hand_derived_golden(c))) for c in GOLDEN] + [
    ("single_frame", lambda: pins.test_single_frame_is_dense_attention(4, 5, 8)),
    ("single_position", lambda: pins.test_single_position_is_dense_attention_across_frames(5, 8)),
    ("brute_frame", lambda: pins.test_brute_force_effective_matrix(*pins.BRUTE_SHAPES[0])),
    ("brute_tiled", lambda: pins.test_brute_force_effective_matrix(*pins.BRUTE_SHAPES[2])),
    ("zero_qk", pins.test_zero_qk_gives_global_mean),
    ("zero_qk_tiled", pins.test_zero_qk_tiled_gives_tile_mean),
    ("transpose", lambda: pins.test_transpose_h_w(1, 2, 3)),
    ("numpy", lambda: pins.test_numpy_restatement_small((1, 2, 6, 4, 6, 1, 2, 3))),
    ("row_brute", lambda: row_pins.test_brute_force_effective_matrix(2, 3, 4, 4)),
    ("row_single_column", row_pins.test_single_column_is_dense_attention),
]


def _build_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert old in src, f"mutant {name}: pattern not found in the oracle source"
    mut = src.replace(old, new)
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"lib{name}.so"
    c.write_text(mut)
    subprocess.run(["gcc", "-O1", "-fPIC", "-shared", "-std=c11", "-o", str(so), str(c), "-lm"],
                   check=True)
    return str(so)


def test_unmutated_passes_every_probe():
    for label, fn in PROBES:
        fn()


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, name, old, new):
    so = _build_mutant(tmp_path, name, old, new)
    prev = oracle.use_library(so)
    caught = []
    try:
        for label, fn in PROBES:
            try:
                fn()
            except (AssertionError, ValueError, FloatingPointError):
                caught.append(label)
    finally:
        oracle.restore_library(prev)
    assert caught, f"no pin rejects the planted mistake '{name}'"


# ---------------------------------------------------------------- gradients

import test_oracle_bwd as bwd_pins

BWD_MUTANTS = [
    ("bwd_no_jacobian_mean", "double dl = logit[j] * (dp[j] - pdp);", "double dl = logit[j] * dp[j];"),
    ("bwd_dk_unscaled", "dkrows[j][c] += scale * dl * q[c];", "dkrows[j][c] += dl * q[c];"),
    ("bwd_dq_uses_values", "dq[c] += scale * dl * krows[j][c];", "dq[c] += scale * dl * vrows[j][c];"),
    ("bwd_stage1_upstream_is_dout", "attend_one_bwd(q + row, kr, vr, len, d, scale, dy1 + row,",
     "attend_one_bwd(q + row, kr, vr, len, d, scale, dout + row,"),
    ("bwd_stage2_values_are_v", "vr[i] = y1 + row;", "vr[i] = v + row;"),
    ("bwd_dv_unweighted", "dvrows[j][c] += logit[j] * dy[c];", "dvrows[j][c] += dy[c];"),
    ("bwd_stage2_dk_misplaced", "dkr[i] = dk + row;", "dkr[i] = dv + row;"),
]

BWD_PROBES = [
    ("bwd_value_frame", lambda: bwd_pins.test_value_gradient_is_monarch_transpose(*pins.BRUTE_SHAPES[0])),
    ("bwd_value_tiled", lambda: bwd_pins.test_value_gradient_is_monarch_transpose(*pins.BRUTE_SHAPES[2])),
    ("bwd_fd_frame", lambda: bwd_pins.test_finite_differences(*bwd_pins.FD_SHAPES[0])),
    ("bwd_fd_tiled", lambda: bwd_pins.test_finite_differences(*bwd_pins.FD_SHAPES[1])),
    ("bwd_single_frame", lambda: bwd_pins.test_single_frame_gradients_are_dense_attention_gradients(3, 5, 8)),
    ("bwd_single_position", lambda: bwd_pins.test_single_position_gradients_are_dense_attention_gradients(5, 8)),
]


def test_unmutated_passes_every_gradient_probe():
    for label, fn in BWD_PROBES:
        fn()


@pytest.mark.parametrize("name,old,new", BWD_MUTANTS, ids=[m[0] for m in BWD_MUTANTS])
def test_gradient_pins_catch_mutant(tmp_path, name, old, new):
    so = _build_mutant(tmp_path, name, old, new)
    prev = oracle.use_library(so)
    caught = []
    try:
        for label, fn in BWD_PROBES:
            try:
                fn()
            except (AssertionError, ValueError, FloatingPointError):
                caught.append(label)
    finally:
        oracle.restore_library(prev)
    assert caught, f"no gradient pin rejects the planted mistake '{name}'"


# ---------------------------------------------------------------- autoregressive chunks

import test_oracle_chunk as chunk_pins

CHUNK_MUTANTS = [
    ("chunk_cache_values_are_keys", "vr[t] = y1_cache + (bh * No + t * HW + pos) * d;",
     "vr[t] = k_cache + (bh * No + t * HW + pos) * d;"),
    ("chunk_new_values_are_v", "vr[T_old + t] = y1_new + (bh * Nn + t * HW + pos) * d;",
     "vr[T_old + t] = v + (bh * Nn + t * HW + pos) * d;"),
    ("chunk_context_dropped", "attend_one(q + row, kr, vr, tot, d, scale, logit, out + row);",
     "attend_one(q + row, kr + T_old, vr + T_old, T_new, d, scale, logit, out + row);"),
    ("chunk_cache_rows_frame_major_off_by_one", "kr[t] = k_cache + (bh * No + t * HW + pos) * d;",
     "kr[t] = k_cache + (bh * No + ((t + 1) % T_old) * HW + pos) * d;"),
]

CHUNK_PROBES = [(f"chunk_case{i}", (lambda c=c: chunk_pins.test_last_chunk_equals_full_forward_rows(*c)))
                for i, c in enumerate(chunk_pins.CASES)] + [
    ("chunk_no_context", chunk_pins.test_no_context_is_the_plain_forward),
]


@pytest.mark.parametrize("name,old,new", CHUNK_MUTANTS, ids=[m[0] for m in CHUNK_MUTANTS])
def test_chunk_pins_catch_mutant(tmp_path, name, old, new):
    so = _build_mutant(tmp_path, name, old, new)
    prev = oracle.use_library(so)
    caught = []
    try:
        for label, fn in CHUNK_PROBES:
            try:
                fn()
            except (AssertionError, ValueError, FloatingPointError):
                caught.append(label)
    finally:
        oracle.restore_library(prev)
    assert caught, f"no chunk pin rejects the planted mistake '{name}'"
