"""Planted mistakes in copies of the oracle must fail its pins (CPU only).

Each mutant is a textual change to a temporary copy of oracle/h3_oracle.c:
a dropped term, a wrong index, a transposed layout, a changed order or
precision, a rounding step skipped.  The copy is compiled with the oracle's own flags and the pins of
tests/oracle_pins.py run against it in a child process (a mutant that writes
out of bounds may crash the child; that also counts as caught).
"""
import os
import subprocess
import sys

import pytest

import oracle
from oracle import build as obuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTANTS = [
    ("remainder_to_last_ranks",
     "starts[i] + q + (i < rem ? 1 : 0)", "starts[i] + q + (i >= w - rem ? 1 : 0)"),
    ("clip_not_rebased", "local_bounds[n] = a - ts;", "local_bounds[n] = a;"),
    ("clip_keeps_empty_pieces", "if (a < b) {", "if (a <= b) {"),
    ("clip_end_not_rebased", "local_bounds[n] = te - ts;", "local_bounds[n] = te;"),
    ("s2h_plane_major_dest",
     "int64_t dst = ((t * P + p) * Hj + hl) * D + d;\n                        recv[j][dst]",
     "int64_t dst = ((p * T + t) * Hj + hl) * D + d;\n                        recv[j][dst]"),
    ("s2h_head_not_rebased",
     "int64_t dst = ((t * P + p) * Hj + hl) * D + d;\n                        recv[j][dst]",
     "int64_t dst = ((t * P + p) * Hj + (hl % Hj)) * D + (d + h) % D;\n                        recv[j][dst]"),
    ("h2s_wrong_token_base",
     "int64_t src = ((t * P + p) * Hj + hl) * D + d;\n                        recv[r][dst]",
     "int64_t src = ((tl * P + p) * Hj + hl) * D + d;\n                        recv[r][dst]"),
    ("h2s_swapped_plane_head",
     "int64_t dst = ((tl * P + p) * H + h) * D + d;\n                        int64_t src",
     "int64_t dst = ((tl * H + h) * P + p) * D + d;\n                        int64_t src"),
    ("locate_drops_head_start", "(hs[j] + hl)) * D + d;", "(hl)) * D + d;"),
    ("locate_h2s_local_token", "(((ts[r] + tl) * P + p) * Hj", "(((tl) * P + p) * Hj"),
    ("reduce_reverse_order",
     "float acc = h3o_bf16_to_f32(vals[0]);\n    for (int32_t w = 1; w < W; ++w)\n        acc = acc + h3o_bf16_to_f32(vals[w]);",
     "float acc = h3o_bf16_to_f32(vals[W - 1]);\n    for (int32_t w = W - 2; w >= 0; --w)\n        acc = acc + h3o_bf16_to_f32(vals[w]);"),
    ("reduce_from_plus_zero",
     "float acc = h3o_bf16_to_f32(vals[0]);\n    for (int32_t w = 1; w < W; ++w)",
     "float acc = 0.0f;\n    for (int32_t w = 0; w < W; ++w)"),
    ("reduce_bias_first",
     "float acc = h3o_bf16_to_f32(vals[0]);\n    for (int32_t w = 1; w < W; ++w)\n        acc = acc + h3o_bf16_to_f32(vals[w]);\n    if (bias_val)\n        acc = acc + h3o_bf16_to_f32(*bias_val);",
     "float acc = bias_val ? h3o_bf16_to_f32(*bias_val) : 0.0f;\n    for (int32_t w = 0; w < W; ++w)\n        acc = acc + h3o_bf16_to_f32(vals[w]);"),
    ("reduce_bias_per_rank",
     "        acc = acc + h3o_bf16_to_f32(vals[w]);\n    if (bias_val)",
     "        acc = acc + h3o_bf16_to_f32(vals[w]) + (bias_val ? h3o_bf16_to_f32(*bias_val) : 0.0f);\n    if (bias_val)"),
    ("reduce_in_double", "    float acc = h3o_bf16_to_f32(vals[0]);", "    double acc = h3o_bf16_to_f32(vals[0]);"),
    ("reduce_rounds_each_step",
     "        acc = acc + h3o_bf16_to_f32(vals[w]);\n    if (bias_val)",
     "        acc = h3o_bf16_to_f32(h3o_f32_to_bf16_rne(acc + h3o_bf16_to_f32(vals[w])));\n    if (bias_val)"),
    ("scatter_wrong_row",
     "vals[w] = partials[w][t * C + c];\n                out[r][tl * C + c]",
     "vals[w] = partials[w][tl * C + c];\n                out[r][tl * C + c]"),
    ("rne_ties_away", "else if (dropped == 0x8000u && (kept & 1u))", "else if (dropped == 0x8000u)"),
    ("rne_truncates", "if (dropped > 0x8000u)\n        kept", "if (dropped > 0xFFFFu)\n        kept"),
    ("nan_becomes_inf", "if (exponent == 0xFFu && mantissa != 0u)", "if (0)"),
    ("gather_wrong_local_row", "out[j][t * C + c] = in[r][(t - ts[r]) * C + c];",
     "out[j][t * C + c] = in[r][(t % (ts[r + 1] - ts[r])) * C + c];"),
    ("gather_from_own_rank", "out[j][t * C + c] = in[r][(t - ts[r]) * C + c];",
     "out[j][t * C + c] = in[j][((t - ts[r]) % (ts[j + 1] - ts[j])) * C + c];"),
    ("plane_major_seq_shifts_channel", "return ((p * Tr + tl) * H + h) * D + d;",
     "return ((p * Tr + tl) * H + h) * D + (d + p) % D;"),
    ("plane_major_head_swapped", "return ((p * T + t) * Hj + hl) * D + d;",
     "return ((t * P + p) * Hj + hl) * D + d;"),
    ("gated_piece_never_advances", "            while (piece + 1 < pieces && tl >= local_bounds[piece + 1])\n                ++piece;",
     "            while (0)\n                ++piece;"),
    ("gated_uses_rank_as_segment", "            int64_t k = seg_ids[piece];", "            int64_t k = r % n_segs;"),
    ("gated_product_dropped", "float sum = h3o_bf16_to_f32(x[r][tl * C + c]) + prod;",
     "float sum = h3o_bf16_to_f32(x[r][tl * C + c]) + g;"),
    ("widen_drops_sign", "uint32_t u = ((uint32_t)b) << 16;", "uint32_t u = ((uint32_t)(b & 0x7FFFu)) << 16;"),
    ("gated_gates_unrounded_sum", "float prod = g * h3o_bf16_to_f32(y);",
     "float yu = h3o_bf16_to_f32(vals[0]);\n"
     "                for (int32_t w2 = 1; w2 < W; ++w2)\n"
     "                    yu = yu + h3o_bf16_to_f32(vals[w2]);\n"
     "                if (bias)\n"
     "                    yu = yu + h3o_bf16_to_f32(bias[c]);\n"
     "                (void)y;\n"
     "                float prod = g * yu;"),
    ("gated_residual_dropped", "float sum = h3o_bf16_to_f32(x[r][tl * C + c]) + prod;",
     "float sum = prod;"),
    ("gated_bias_dropped", "uint16_t y = reduce_one(vals, W, bias ? &bias[c] : NULL);",
     "uint16_t y = reduce_one(vals, W, NULL);"),
    ("gated_gate_row_by_token", "float g = h3o_bf16_to_f32(gate[k * C + c]);",
     "float g = h3o_bf16_to_f32(gate[(t % n_segs) * C + c]);"),
    ("owner_boundary_inclusive", "        if (x < starts[i + 1])\n            return i;",
     "        if (x <= starts[i + 1])\n            return i;"),
    ("reduce_rows_drops_bias", "out[t * C + c] = reduce_one(vals, W, bias ? &bias[c] : NULL);",
     "out[t * C + c] = reduce_one(vals, W, NULL);"),
]

_CHILD = r"""
import sys
sys.path.insert(0, {root!r})
import oracle
from tests import oracle_pins as P
o = oracle.load({lib!r})
failed = P.run_all(o)
print("FAILED:", failed)
sys.exit(3 if failed else 0)
"""


def _run_pins(lib_path: str) -> subprocess.CompletedProcess:
    code = _CHILD.format(root=ROOT, lib=lib_path)
    return subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                          timeout=300)


def _compile(tmp_path, name: str, text: str) -> str:
    src = tmp_path / f"{name}.c"
    src.write_text(text)
    out = str(tmp_path / f"lib_{name}.so")
    obuild.build(str(src), out, extra=["-Wno-error"])
    return out


def test_unmutated_copy_passes(tmp_path):
    with open(oracle.SRC_PATH) as f:
        text = f.read()
    res = _run_pins(_compile(tmp_path, "control", text))
    assert res.returncode == 0, res.stdout + res.stderr


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new):
    with open(oracle.SRC_PATH) as f:
        text = f.read()
    assert text.count(old) >= 1, f"mutation anchor not found: {name}"
    mutated = text.replace(old, new, 1)
    res = _run_pins(_compile(tmp_path, name, mutated))
    assert res.returncode != 0, f"mutant {name} passed every pin:\n{res.stdout}"
