"""Planted mistakes in the oracle, on the CPU.

Each mutant is a copy of oracle/lcsa_oracle.cpp with one plausible error (a
dropped term, a wrong sign, index, axis or operand, an off-by-one), compiled
to a temporary library that the oracle package loads through LCSA_ORACLE_LIB.
The oracle's pins (tests/test_oracle_pins.py, tests/test_parameters.py) must
fail against every mutant and pass against an unmodified copy built the same
way: a pin set that let a mutant through would not pin the oracle.
"""
import concurrent.futures as cf
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "lcsa_oracle.cpp")
PINS = [os.path.join(ROOT, "tests", "test_oracle_pins.py"), os.path.join(ROOT, "tests", "test_parameters.py")]

# name: [(exact text in lcsa_oracle.cpp, replacement), ...] applied in order
MUTANTS = {
    # RMSNorm (token scope): sum of squares instead of their mean
    "norm_mean_dropped": [("ss / double(d.C) + g.rms_eps", "ss + g.rms_eps")],
    # RMSNorm: eps added outside the square root
    "norm_eps_outside_root": [("1.0 / std::sqrt(ss / double(d.C) + g.rms_eps)",
                               "1.0 / (std::sqrt(ss / double(d.C)) + g.rms_eps)")],
    # head scope normalised over every channel of the token
    "head_norm_over_token": [("ss / double(D) + g.rms_eps", "ss / double(d.C) + g.rms_eps")],
    # gain not applied (token scope)
    "gain_dropped": [("out[c] = out[c] * inv * double(gamma[c]);", "out[c] = out[c] * inv;")],
    # rotation: wrong sign of one term (no longer a rotation)
    "rotation_sign": [("a * cs[j] - b * sn[j]", "a * cs[j] + b * sn[j]")],
    # rotation by the opposite angle (still a rotation)
    "rotation_direction": [("a * cs[j] - b * sn[j]", "a * cs[j] + b * sn[j]"),
                           ("a * sn[j] + b * cs[j]", "-a * sn[j] + b * cs[j]")],
    # frame-axis frequencies computed with the row axis' dimension count
    "frame_axis_dims": [("expo = 2.0 * j / dims_t;", "expo = 2.0 * j / dims_h;")],
    # row and column axes exchanged
    "row_col_axes_swapped": [("pos = double(y);", "pos = double(@X@);"),
                             ("pos = double(xcol);", "pos = double(y);"),
                             ("pos = double(@X@);", "pos = double(xcol);")],
    # frequencies growing instead of decaying
    "frequency_exponent_sign": [("std::pow(10000.0, -expo)", "std::pow(10000.0, expo)")],
    # query frames placed at the start of the KV window instead of its end
    "query_frames_first": [("double(is_q ? (g.kv_frames - g.q_frames) : 0)", "double(0)")],
    # the absolute frame offset ignored
    "frame_offset_ignored": [("double(g.kv_frame_offset) + ", "0.0 + ")],
    # pooled sum instead of mean
    "pool_sum_not_mean": [("acc[h * D + e] / double(d.nb)", "acc[h * D + e]")],
    # window one block too narrow in one direction
    "window_row_strict": [("std::llabs(dh) <= r", "std::llabs(dh) < r")],
    # window radius from the diameter without the centre block
    "window_radius": [("int64_t r = (g.local_range - 1) / 2;", "int64_t r = (g.local_range + 1) / 2;")],
    # ties to the higher block index
    "ties_to_higher_index": [("return a.second < b.second;", "return a.second > b.second;")],
    # one block too many kept
    "budget_plus_one": [("std::min<int64_t>(g.topk, int64_t(cand.size()))",
                         "std::min<int64_t>(g.topk + 1, int64_t(cand.size()))")],
    # kept blocks emitted in score order instead of ascending index
    "kept_not_ascending": [("std::sort(sel.begin(), sel.end());", "")],
    # softmax scale dropped
    "softmax_scale_dropped": [("logit[j] = s * g.softmax_scale;", "logit[j] = s;")],
    # softmax weights not normalised
    "weights_not_normalised": [("double p = logit[j] / l;", "double p = logit[j];")],
    # keys used as values (transposed operand)
    "values_are_keys": [("o[e] += p * vh[j * D + e];", "o[e] += p * kh[j * D + e];")],
    # tokens of a block taken column-major
    "block_tokens_column_major": [("int64_t yy = (i / g.block_w) % g.block_h;", "int64_t yy = i % g.block_h;"),
                                  ("int64_t xx = i % g.block_w;", "int64_t xx = (i / g.block_h) % g.block_w;")],
    # budget rule with the latent grid not scaled to pixels
    "budget_pixel_scale": [("double H = 16.0 * grid_h, W = 16.0 * grid_w;", "double H = 8.0 * grid_h, W = 8.0 * grid_w;")],
    # budget rounded instead of floored
    "budget_rounded": [("std::floor(num / (H * W))", "std::round(num / (H * W))")],
    # eps dropped from the norm
    "norm_eps_dropped": [("ss / double(d.C) + g.rms_eps", "ss / double(d.C)")],
    # a token's row and column taken with the grid's sides exchanged
    "token_row_from_height": [("int64_t y = (tok / g.grid_w) % g.grid_h;", "int64_t y = (tok / g.grid_h) % g.grid_w;")],
    "token_column_from_height": [("int64_t xcol = tok % g.grid_w;", "int64_t xcol = tok % g.grid_h;")],
    # rotation pairs (j, j + d/2) instead of (2j, 2j+1)
    "rotation_pairs_half_split": [
        ("double a = out[h * D + 2 * j], b = out[h * D + 2 * j + 1];",
         "double a = out[h * D + j], b = out[h * D + j + D / 2];"),
        ("out[h * D + 2 * j] = a * cs[j] - b * sn[j];", "out[h * D + j] = a * cs[j] - b * sn[j];"),
        ("out[h * D + 2 * j + 1] = a * sn[j] + b * cs[j];", "out[h * D + j + D / 2] = a * sn[j] + b * cs[j];")],
    # pooled output laid out head-major over the batch
    "pooled_layout_head_batch": [("pooled[((b * g.heads + h) * nblk + blk) * D + e]",
                                  "pooled[((h * g.batch + b) * nblk + blk) * D + e]")],
    # attention rows split into (batch, head) the wrong way round
    "attention_row_split": [("int64_t b = bh / g.heads, h = bh % g.heads;",
                             "int64_t b = bh % g.batch, h = bh / g.batch;")],
    # query tokens addressed with the key tensor's batch stride
    "query_batch_stride": [("q + (b * d.Lq + tok) * d.C", "q + (b * d.Lkv + tok) * d.C")],
    # values of head 0 for every head
    "values_head_zero": [("v[(b * d.Lkv + tok) * d.C + h * D + e]", "v[(b * d.Lkv + tok) * d.C + e]")],
    # pooled keys of the first (batch, head) for every row
    "score_keys_of_head_zero": [("const double* kk = pk + (bh * d.nKB + kb) * D;", "const double* kk = pk + kb * D;")],
    # score matrix without the window's -inf
    "scores_unmasked": [("scores[row * d.nKB + kb] = ok ? s : -std::numeric_limits<double>::infinity();",
                         "scores[row * d.nKB + kb] = s;")],
    # window column distance against the key's block row
    "window_column_index": [("dw = qrem % d.nWb - krem % d.nWb", "dw = qrem % d.nWb - krem / d.nWb")],
    # gap measured from the best score instead of the k-th
    "gap_from_best": [("cand[keff - 1].first - cand[keff].first", "cand[0].first - cand[keff].first")],
    # head scope: every head takes the first head's gains
    "head_gain_of_head_zero": [("out[h * D + e] * inv * double(gamma[h * D + e])", "out[h * D + e] * inv * double(gamma[e])")],
    # the absolute frame offset given to the keys only
    "frame_offset_keys_only": [("double t_abs = double(g.kv_frame_offset) + double(is_q ? (g.kv_frames - g.q_frames) : 0)",
                                "double t_abs = double(is_q ? 0 : g.kv_frame_offset) + "
                                "double(is_q ? (g.kv_frames - g.q_frames) : 0)")],
    # window restricted to the query's own frame
    "window_same_frame_only": [("if (g.local_range <= 0) return true;",
                                "if (qb / d.bpf != kb / d.bpf) return false;\n  if (g.local_range <= 0) return true;")],
    # pooling rotates query blocks at key positions
    "pool_query_flag_dropped": [("norm_rope_token(g, d, x + (b * L + tok) * d.C, gamma, is_q != 0, tok, v.data());",
                                 "norm_rope_token(g, d, x + (b * L + tok) * d.C, gamma, false, tok, v.data());")],
    # attention rotates queries at key positions
    "attention_query_flag_dropped": [("gamma_q, true, tok, tokvec.data());", "gamma_q, false, tok, tokvec.data());")],
}


def _mutate(text, edits):
    for old, new in edits:
        assert text.count(old) == 1, "mutation target not found exactly once: %r" % old
        text = text.replace(old, new)
    return text


def _compile(name, text, tmp):
    src = os.path.join(tmp, name + ".cpp")
    lib = os.path.join(tmp, "lib" + name + ".so")
    with open(src, "w") as f:
        f.write(text)
    subprocess.run(["g++", "-std=c++17", "-O2", "-fPIC", "-shared", "-pthread", "-o", lib, src], check=True,
                   capture_output=True)
    return lib


def _pins_pass(lib):
    env = dict(os.environ, LCSA_ORACLE_LIB=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", "-m", "not gpu"] + PINS,
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode == 0, r.stdout[-1500:]


def test_pins_catch_every_planted_mistake(tmp_path):
    with open(SRC) as f:
        original = f.read()
    sources = {"unmodified": original}
    sources.update({name: _mutate(original, edits) for name, edits in MUTANTS.items()})
    with cf.ThreadPoolExecutor(8) as ex:
        libs = dict(zip(sources, ex.map(lambda kv: _compile(kv[0], kv[1], str(tmp_path)), sources.items())))
        results = dict(zip(libs, ex.map(_pins_pass, libs.values())))
    ok, log = results.pop("unmodified")
    assert ok, "the pins fail on an unmodified copy of the oracle:\n" + log
    survivors = sorted(name for name, (passed, _) in results.items() if passed)
    assert not survivors, "mutants the pins do not catch: %s" % survivors
