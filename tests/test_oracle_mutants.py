"""The oracle's pins can fail: plausible mistakes, planted one at a time in
the oracle on the CPU, must each make at least one pin of ``tests/test_oracle_*.py``
fail.

Each mutant rewrites one expression in the source of one oracle function (or
one module constant), installs the rewritten function in the oracle module for
the duration of the test, and runs the pins of the listed pin modules (their
parametrizations expanded, fixtures-free cases only) until one fails. A mutant
that every pin accepts is a gap in the pins. The source pattern of every
mutant must still be present in the oracle, so the table follows the code.

The mistakes are the kinds a reader checks a definition for: an off-by-one or
wrongly aligned mask, a dropped factor, a transposed or swapped operand, a wrong
base or sign, a wrong index mapping, a wrong range, bias or rounding rule, and
a wrong block extent or nibble order."""

import inspect
import textwrap

import numpy as np
import pytest

from oracle import attention as oattn
from oracle import e4m3 as oe4m3
from oracle import nvfp4 as onvfp4
from oracle import online_softmax as oonline
from oracle import quant as oquant
from tests import test_oracle_attention as pins_attention
from tests import test_oracle_e4m3 as pins_e4m3
from tests import test_oracle_nvfp4 as pins_nvfp4
from tests import test_oracle_online_softmax as pins_online
from tests import test_oracle_quant as pins_quant
from tests import test_oracle_smooth as pins_smooth

ATT = (pins_attention,)
QUANT = (pins_quant, pins_smooth)

# (name, oracle module, function or None for a constant, old, new, pin modules)
MUTANTS = [
    # attention: masks
    ("causal_off_by_one", oattn, "visible_mask", "vis &= j <= i + (Skv - Sq)", "vis &= j < i + (Skv - Sq)", ATT),
    ("causal_top_left", oattn, "visible_mask", "vis &= j <= i + (Skv - Sq)", "vis &= j <= i", ATT),
    ("block_rows_twice_as_tall", oattn, "visible_mask", "rows = np.arange(Sq) // block",
     "rows = np.arange(Sq) // (2 * block)", ATT),
    ("block_mask_transposed", oattn, "visible_mask", "bm[rows[:, None], cols[None, :]]",
     "bm[np.minimum(cols[None, :], bm.shape[0] - 1), np.minimum(rows[:, None], bm.shape[1] - 1)]", ATT),
    ("rows_causal_top_left", oattn, "attention_rows", "vis &= j <= rows[:, None] + (Skv - Sq)",
     "vis &= j <= rows[:, None]", ATT),
    # attention: arithmetic
    ("gqa_heads_interleaved", oattn, "attention", "h = hk * group + g", "h = g * Hkv + hk", ATT),
    ("softmax_scale_dropped", oattn, "attention", "s = softmax_scale * np.matmul(q[b, r0:r1, h, :], kk.T)",
     "s = np.matmul(q[b, r0:r1, h, :], kk.T)", ATT),
    ("keys_for_values", oattn, "attention", "np.matmul(p, vv)", "np.matmul(p, kk[:, :Dv])", ATT),
    ("lse_base_two", oattn, "attention", "m[:, 0] + np.log(np.where(", "m[:, 0] + np.log2(np.where(", ATT),
    ("max_added", oattn, "attention", "e = np.exp(s - m_safe)", "e = np.exp(s + m_safe)", ATT),
    ("normaliser_dropped", oattn, "attention", "p = np.divide(e, l, out=np.zeros_like(e), where=l > 0)",
     "p = e", ATT),
    ("lse_without_max", oattn, "attention", "m[:, 0] + np.log(np.where(", "np.log(np.where(", ATT),
    ("hidden_rows_divided_by_zero", oattn, "attention", "p = np.divide(e, l, out=np.zeros_like(e), where=l > 0)",
     "p = e / l", ATT),
    ("probabilities_scale_dropped", oattn, "probabilities", "s = softmax_scale * (q @ k.T)", "s = q @ k.T", ATT),
    ("rows_scale_dropped", oattn, "attention_rows", "s = softmax_scale * (q @ k.T)", "s = q @ k.T", ATT),
    ("row_chunk_drops_a_row", oattn, "attention", "r1 = min(Sq, r0 + ROW_CHUNK)",
     "r1 = min(Sq, r0 + ROW_CHUNK - 1)", ATT),
    ("row_chunk_mask_from_first_chunk", oattn, "attention", "vis = vis_full[r0:r1]", "vis = vis_full[:r1 - r0]",
     ATT),
    # attention: paged gather
    ("page_row_off_by_one", oattn, "gather_paged", "(t % page_size)[None, :]", "((t + 1) % page_size)[None, :]",
     ATT),
    ("page_by_token", oattn, "gather_paged", "pages = pt[:, t // page_size]", "pages = pt[:, t % pt.shape[1]]",
     ATT),
    # quantizer
    ("scale_by_reciprocal", oquant, "scale_from_amax", "scale = (amax_f32 / r).astype(np.float32)",
     "scale = (amax_f32 * np.float32(np.float32(1.0) / r)).astype(np.float32)", QUANT),
    ("zero_amax_zero_scale", oquant, "scale_from_amax",
     "np.where(amax_f32 == 0, np.float32(1.0), scale)", "scale", QUANT),
    ("int8_ties_away", oquant, "codes_with_scale", "np.clip(np.rint(q), -127, 127)",
     "np.clip(np.trunc(q + np.copysign(np.float32(0.5), q)), -127, 127)", QUANT),
    ("int8_range_128", oquant, None, "RANGE", {"int8": 128.0, "e4m3": 448.0}, QUANT),
    ("e4m3_range_240", oquant, None, "RANGE", {"int8": 127.0, "e4m3": 240.0}, QUANT),
    ("signed_block_amax", oquant, "quantize_blockwise", "s = scale_from_amax(np.max(np.abs(blk)), out_dtype)",
     "s = scale_from_amax(np.max(blk), out_dtype)", QUANT),
    ("token_block_one_row_long", oquant, "quantize_blockwise",
     "s0, s1 = i * rows_per_block, min(S, (i + 1) * rows_per_block)",
     "s0, s1 = i * rows_per_block, min(S, (i + 1) * rows_per_block + 1)", QUANT),
    ("per_head_first_token_only", oquant, "quantize_blockwise", "blk = x[b, :, h, :]", "blk = x[b, :1, h, :]",
     QUANT),
    ("shift_added", oquant, "quantize_blockwise", "x = (x - sh[:, None, :, :])", "x = (x + sh[:, None, :, :])",
     QUANT),
    ("mean_over_s_minus_one", oquant, "channel_mean", "(total / np.float64(S))", "(total / np.float64(max(S - 1, 1)))",
     QUANT),
    ("mean_summed_in_float32", oquant, "channel_mean", "total = x.astype(np.float64).sum(axis=1)",
     "total = x.sum(axis=1, dtype=np.float32).astype(np.float64)", QUANT),
    ("dequant_next_block_scale", oquant, "dequantize", "idx = np.arange(S) // rows_per_block",
     "idx = np.minimum(np.arange(S) // rows_per_block + 1, sc.shape[2] - 1)", QUANT),
    ("dequant_per_head_one_scale_per_batch", oquant, "dequantize", "return vals * sc[:, None, :, None]",
     "return vals * sc.max(axis=1)[:, None, None, None]", QUANT),
    ("dequant_per_channel_scales_by_token", oquant, "dequantize", "return vals * sc[:, None, :, :]",
     "return vals * sc[:, :1, :, :]", QUANT),
    # E4M3 codec
    ("e4m3_bias_8", oe4m3, "decode", "np.exp2(exp_field.astype(np.float64) - 7.0)",
     "np.exp2(exp_field.astype(np.float64) - 8.0)", (pins_e4m3,)),
    ("e4m3_ties_away", oe4m3, "encode", "steps = np.rint(a / quantum)", "steps = np.floor(a / quantum + 0.5)",
     (pins_e4m3,)),
    ("e4m3_overflow_not_saturated", oe4m3, "encode", "r = np.minimum(r, MAX)", "r = np.where(r > MAX, 480.0, r)",
     (pins_e4m3,)),
    ("e4m3_subnormal_step_halved", oe4m3, "encode", "e = np.maximum(e, -6)", "e = np.maximum(e, -7)",
     (pins_e4m3,)),
    ("e4m3_nan_code_finite", oe4m3, "decode", "val = np.where((exp_field == 0xF) & ((c & 0x7) == 0x7), np.nan, val)",
     "val = val", (pins_e4m3,)),
    ("e4m3_negative_zero_unsigned", oe4m3, "encode", "neg = np.signbit(x)", "neg = x < 0", (pins_e4m3,)),
    # online softmax with rounded P
    ("rescale_on_every_rise", oonline, "_tile_pass", "& (m_tile > m + tau)", "& (m_tile > m)",
     (pins_online,)),
    ("rescale_skips_row_sum", oonline, "_tile_pass", "l *= alpha", "l *= 1.0", (pins_online,)),
    ("rescale_skips_o", oonline, "_tile_pass", "acc *= alpha[:, None]", "acc *= 1.0", (pins_online,)),
    ("row_sum_correction_dropped", oonline, "_tile_pass", "l += p.sum(axis=1) + corr",
     "l += p.sum(axis=1)", (pins_online,)),
    ("p_scale_not_applied", oonline, "attention_rounded_p",
     'g = 1.0 if p_mode in ("bf16", "exact") else 1.0 / sfp', "g = 1.0", (pins_online,)),
    ("low_term_dropped", oonline, "_tile_pass", "stored, corr = hi + lo, 0.0", "stored, corr = hi, 0.0",
     (pins_online,)),
    ("bf16_truncates", oonline, "_round_bf16", "u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000",
     "u = u & 0xFFFF0000", (pins_online,)),
    ("tau_rounded_up", oonline, "tau_for", "math.floor(math.log2(448.0 * sf_p))",
     "math.ceil(math.log2(448.0 * sf_p))", (pins_online,)),
    ("lse_without_p_scale", oonline, "attention_rounded_p", "np.log2(np.where(alive, l, 1.0) / g)",
     "np.log2(np.where(alive, l, 1.0))", (pins_online,)),
    ("p_scale_of_first_block", oonline, "attention_rounded_p", "sfp_arr[b, h, r0 // p_block]", "sfp_arr[b, h, 0]",
     (pins_online,)),
    ("merge_without_max_weights", oonline, "attention_rounded_p",
     "w = [np.where(pl > 0, np.exp2(np.where(pl > 0, pm - m_use, 0.0)), 0.0) for _, pl, pm in parts]",
     "w = [np.where(pl > 0, 1.0, 0.0) for _, pl, pm in parts]", (pins_online,)),
    ("deal_by_halves", oonline, "_deal", "return kept[0::2], kept[1::2]",
     "return kept[:(len(kept) + 1) // 2], kept[(len(kept) + 1) // 2:]", (pins_online,)),
    ("kept_tiles_first_row_bound", oonline, "_kept_tiles",
     "last = min(qblk * tile + tile - 1, Sq - 1) + (Skv - Sq)", "last = qblk * tile + (Skv - Sq)", (pins_online,)),
    ("decode_per_rounded_down", oonline, "_split_groups", "per = -(-total // n_splits) if total else 0",
     "per = max(1, total // n_splits) if total else 0", (pins_online,)),
    ("decode_interleave_by_halves", oonline, "_split_groups", "groups += [mine[0::2], mine[1::2]] if interleave",
     "groups += [mine[:len(mine) // 2], mine[len(mine) // 2:]] if interleave", (pins_online,)),
    ("decode_merge_base_two", oonline, "decode_rounded_p", "np.exp(lse_j - np.where(alive, mx, 0.0)[None])",
     "np.exp2(lse_j - np.where(alive, mx, 0.0)[None])", (pins_online,)),
    ("decode_head_major_packing", oonline, "decode_rounded_p", "tok, head = rows // G, hk * G + rows % G",
     "tok, head = rows % Sq, hk * G + rows // Sq", (pins_online,)),
    ("decode_mask_row_by_tile", oonline, "decode_rounded_p", "bm[tok0 // TILE, c]", "bm[min(u, bm.shape[0] - 1), c]",
     (pins_online,)),
    # NVFP4
    ("nvfp4_token_scale_448", onvfp4, None, "ROW_RANGE", np.float32(448.0), (pins_nvfp4,)),
    ("e2m1_ties_down", onvfp4, "e2m1_encode", "better = (d < best) | ((d == best) & (c % 2 == 0))",
     "better = (d < best)", (pins_nvfp4,)),
    ("zero_row_token_scale_zero", onvfp4, "quantize_per_token",
     "s_t = np.float32(1.0) if amax == 0 else np.float32(amax / ROW_RANGE)", "s_t = np.float32(amax / ROW_RANGE)",
     (pins_nvfp4,)),
    ("nibbles_swapped", onvfp4, "quantize_per_token", "packed = (codes4[:, 0::2] | (codes4[:, 1::2] << 4))",
     "packed = (codes4[:, 1::2] | (codes4[:, 0::2] << 4))", (pins_nvfp4,)),
    ("nvfp4_dequant_nibbles_swapped", onvfp4, "dequantize", "c[:, 0::2] = packed & 0xF",
     "c[:, 0::2] = packed >> 4", (pins_nvfp4,)),
    ("block_scale_without_e2m1_max", onvfp4, "quantize_per_token",
     "q = np.float32(np.float32(amax_b / s_t) / np.float32(6.0))", "q = np.float32(amax_b / s_t)", (pins_nvfp4,)),
]


def pin_cases(module):
    """(name, function, kwargs) for every fixture-free case of a pin module."""
    for name, fn in sorted(vars(module).items()):
        if not name.startswith("test_") or not callable(fn):
            continue
        combos = [{}]
        for mark in getattr(fn, "pytestmark", []):
            if mark.name != "parametrize":
                continue
            argnames, values = mark.args[0], mark.args[1]
            names = [a.strip() for a in argnames.split(",")] if isinstance(argnames, str) else list(argnames)
            expanded = []
            for combo in combos:
                for val in values:
                    val = getattr(val, "values", val)  # pytest.param(...)
                    vals = tuple(val) if len(names) > 1 else (val,)
                    expanded.append({**combo, **dict(zip(names, vals))})
            combos = expanded
        params = set(inspect.signature(fn).parameters)
        for combo in combos:
            if params <= set(combo):
                yield name, fn, {k: combo[k] for k in params}


def first_failure(modules):
    """Runs the pins of the modules in order; returns the first failing case or None."""
    for module in modules:
        for name, fn, kwargs in pin_cases(module):
            try:
                fn(**kwargs)
            except pytest.skip.Exception:
                continue
            except (Exception, pytest.fail.Exception) as e:  # an assertion, or the mutant broke the call
                return f"{module.__name__}.{name}{kwargs or ''}: {type(e).__name__}"
    return None


def install(monkeypatch, module, func, old, new):
    if func is None:  # a module constant
        assert hasattr(module, old)
        monkeypatch.setattr(module, old, new)
        return
    src = textwrap.dedent(inspect.getsource(getattr(module, func)))
    assert src.count(old) == 1, f"pattern not found once in {module.__name__}.{func}: {old!r}"
    namespace = dict(vars(module))
    exec(compile(src.replace(old, new), f"<mutant of {module.__name__}.{func}>", "exec"), namespace)
    monkeypatch.setattr(module, func, namespace[func])


def test_unmutated_oracle_passes_every_pin():
    """The harness itself: the real oracle passes every case it runs."""
    mods = (pins_attention, pins_quant, pins_smooth, pins_e4m3, pins_nvfp4, pins_online)
    assert sum(1 for m in mods for _ in pin_cases(m)) > 60
    assert first_failure(mods) is None


@pytest.mark.parametrize("name,module,func,old,new,pins", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(monkeypatch, name, module, func, old, new, pins):
    install(monkeypatch, module, func, old, new)
    with np.errstate(all="ignore"):
        caught = first_failure(pins)
    assert caught is not None, f"no pin fails with the mutant {name}"
