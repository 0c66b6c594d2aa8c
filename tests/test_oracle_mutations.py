"""The oracle's pins catch plausible mistakes: each case below plants one
mistake in the oracle (monkeypatched, on the CPU, for this test only) and
checks that at least one pin of tests/test_oracle_*.py then fails.  A pin
set that let a planted mistake through would not pin the oracle."""
import math

import numpy as np
import pytest

import test_oracle_attention as TA
import test_oracle_formats as TF
import test_oracle_projection as TP
from oracle import attention, formats, fp8, merge, projection, rope


# ---------------------------------------------------------------- planted mistakes

def _rotation_sign(x, c, s):
    x = np.asarray(x, dtype=np.float64)
    out = np.empty_like(x)
    out[..., 0::2] = x[..., 0::2] * c + x[..., 1::2] * s        # turns by -phi
    out[..., 1::2] = -x[..., 0::2] * s + x[..., 1::2] * c
    return out


def _frequency_exponent(axes=rope.DEFAULT_AXES, theta=rope.DEFAULT_THETA):
    axis_of_pair, omega = [], []
    for a, d in enumerate(axes):
        for i in range(d // 2):
            axis_of_pair.append(a)
            omega.append(theta ** (-1.0 * i / d))                  # -i/d instead of -2i/d
    return np.asarray(axis_of_pair), np.asarray(omega)


def _axis_order(axes=rope.DEFAULT_AXES, theta=rope.DEFAULT_THETA):
    axis_of_pair, omega = _ORIG["frequencies"](axes, theta)
    return 2 - axis_of_pair, omega                                  # positions of (w, h, t) for slices (t, h, w)


def _pair_layout(x, c, s):
    x = np.asarray(x, dtype=np.float64)
    h = x.shape[-1] // 2                                            # half-split pairs (j, j + D/2)
    out = np.empty_like(x)
    out[..., :h] = x[..., :h] * c - x[..., h:] * s
    out[..., h:] = x[..., :h] * s + x[..., h:] * c
    return out


def _softmax_scale(q_rows, k, v, scale, allowed=None):
    return _ORIG["attention_rows"](q_rows, k, v, scale * math.sqrt(2.0), allowed)


def _lse_without_max(q_rows, k, v, scale, allowed=None):
    o, l = _ORIG["attention_rows"](q_rows, k, v, scale, allowed)
    s = (q_rows @ k.T) * scale
    return o, l - s.max(axis=1)                                     # log sum exp(s - m), the max not added back


def _value_rows_shifted(q_rows, k, v, scale, allowed=None):
    return _ORIG["attention_rows"](q_rows, k, np.roll(v, 1, axis=0), scale, allowed)


def _merge_unnormalised(outs, lses):
    o, l = _ORIG["merge"](outs, lses)
    lses = np.stack([np.asarray(x, dtype=np.float64) for x in lses])
    return o * np.exp(lses - l[None, :]).max(axis=0)[:, None], l  # drops the 1 / sum of weights


def _fp8_max_240(x32, block=fp8.BLOCK):
    x32 = np.asarray(x32, dtype=np.float32)
    return (_ORIG["block_scales"](x32, block) * np.float32(448.0 / 240.0)).astype(np.float32)


def _round_half_up(x, sig_bits, min_exp):
    x = np.asarray(x, dtype=np.float64)
    ax = np.abs(x)
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    e = np.maximum(e, min_exp)
    step = np.ldexp(1.0, (e - (sig_bits - 1)).astype(np.int64))
    return np.sign(x) * np.floor(ax / step + 0.5) * step             # ties away from zero


def _split_remainder_unrounded(r):
    hi = _ORIG["round_fp16"](np.asarray(r, dtype=np.float64))
    return hi, np.asarray(r, dtype=np.float64) - hi                   # lo not rounded to fp16


def _split_truncated(r):
    r = np.asarray(r, dtype=np.float64)
    _, e = np.frexp(np.abs(r))
    step = np.ldexp(1.0, np.maximum(e - 1, -14) - 10)
    hi = np.trunc(r / step) * step                                    # hi chopped instead of rounded
    return hi, _ORIG["round_fp16"](r - hi)


def _fp32_chopped(x):
    x = np.asarray(x, dtype=np.float64)
    return x.astype(np.float32).astype(np.float64) * (1.0 - 2.0 ** -24)


def _projection_head_major(x, w, bias=None, H=24, D=128):
    y = np.einsum("bnc,oc->bno", attention.to_f64(x), attention.to_f64(w))
    if bias is not None:
        y = y + attention.to_f64(bias)[None, None, :]
    B, N, _ = y.shape
    y = y.reshape(B, N, H, 3, D).transpose(3, 0, 2, 1, 4)            # features read as (h, s, d)
    return y[0], y[1], y[2]


def _projection_without_bias(x, w, bias=None, H=24, D=128):
    return _ORIG["project"](x, w, None, H=H, D=D)


_ORIG = {"project": projection.project, "round_fp16": formats.round_fp16, "frequencies": rope.frequencies, "attention_rows": attention.attention_rows, "merge": merge.merge,
         "block_scales": fp8.block_scales}

# pins, as callables without arguments
P_BRUTE = [lambda: TA.test_brute_force_50_digits(12, (2, 2, 4), 1), lambda: TA.test_brute_force_50_digits(16, (4, 6, 6), 2)]
P_ROPE = [TA.test_rope_rotation_direction, TA.test_rope_relative_position,
          lambda: TA.test_rope_single_pair_logit_is_cos_of_angle(18, 1, 10.0 ** (-1.0 / 7.0)),
          lambda: TA.test_rope_single_pair_logit_is_cos_of_angle(2, 0, 10.0 ** (-1.0 / 2.0))]
P_ATTN = [TA.test_rows_sum_to_one, TA.test_zero_query_gives_column_mean_and_log_n,
          TA.test_dominant_key_returns_its_value_row, lambda: TA.test_matches_library_sdpa_without_rope(64)]
P_MERGE = [TA.test_merge_of_key_slices_equals_full_attention, TA.test_merge_weights_follow_the_softmax_of_the_lses]
P_PROJ = [TP.test_project_matches_exact_rational_sums, TP.test_project_regroups_features_into_q_k_v_heads]
P_SPLIT = [TF.test_split_fp16_terms, TF.test_round_fp32_matches_library_cast_and_ties_to_even]
P_FP8 = [TF.test_block_quantisation_properties, TF.test_e4m3_midpoints_round_to_even_and_saturate,
         TF.test_e4m3_encode_matches_library_cast, TF.test_e4m3_landmark_codes]

MUTATIONS = [
    ("rotation sign", rope, "rotate_with_table", _rotation_sign, P_ROPE + P_BRUTE),
    ("frequency exponent", rope, "frequencies", _frequency_exponent, P_ROPE + P_BRUTE),
    ("axis order", rope, "frequencies", _axis_order, P_ROPE + P_BRUTE),
    ("half-split pair layout", rope, "rotate_with_table", _pair_layout, P_ROPE + P_BRUTE),
    ("softmax scale", attention, "attention_rows", _softmax_scale, P_ATTN + P_BRUTE),
    ("LSE without the max", attention, "attention_rows", _lse_without_max, P_ATTN + P_BRUTE),
    ("value rows shifted", attention, "attention_rows", _value_rows_shifted, P_ATTN + P_BRUTE),
    ("merge not renormalised", merge, "merge", _merge_unnormalised, P_MERGE),
    ("E4M3 scale from 240", fp8, "block_scales", _fp8_max_240, P_FP8),
    ("rounding ties away from zero", formats, "_round_nearest_even", _round_half_up, P_FP8),
    ("split remainder not rounded", formats, "split_fp16", _split_remainder_unrounded, P_SPLIT),
    ("split hi chopped", formats, "split_fp16", _split_truncated, P_SPLIT),
    ("fp32 rounding biased", formats, "round_fp32", _fp32_chopped, P_SPLIT),
    ("projection features read head-major", projection, "project", _projection_head_major, P_PROJ),
    ("projection bias dropped", projection, "project", _projection_without_bias, P_PROJ),
]


@pytest.mark.parametrize("name,module,attr,bad,pins", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_fails_a_pin(name, module, attr, bad, pins, monkeypatch):
    monkeypatch.setattr(module, attr, bad)
    caught = 0
    for pin in pins:
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught >= 1, "no pin caught the planted mistake: %s" % name


def test_pins_pass_on_the_unmodified_oracle():
    for pin in P_BRUTE + P_ROPE + P_ATTN + P_MERGE + P_FP8 + P_SPLIT + P_PROJ:
        pin()
