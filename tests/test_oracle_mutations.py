"""The oracle's pins catch plausible mistakes (CPU only).

Each case plants one mistake in a copy of the oracle (its C source, or the
Python layer that composes the steps): a dropped term, a wrong sign, index or
reduction order, a missed rounding point, a wrong constant. The case then runs
the pin tests (``test_oracle_pins.py``) against the copy, and at least one of
them must fail (pytest's exit code 1: a test failed, not a crash or a
collection error). An unmodified copy must pass, so that a failure means the
pins saw the mistake and not that the harness is broken.
"""

import os
import shutil
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PINS = os.path.join(ROOT, "tests", "test_oracle_pins.py")

TRUNC_H = ("{ float hv_ = silu_f32(g) * u; uint32_t hu_; memcpy(&hu_, &hv_, 4); "
           "hrow[j] = (uint16_t)(hu_ >> 16); }")
TRUNC_OUT = ("{ uint32_t ou_; memcpy(&ou_, &acc, 4); out[(size_t)t * H + o] = (uint16_t)(ou_ >> 16); }")

# (name, text in moe_oracle.c, replacement); names starting "py_" edit __init__.py instead
MUTATIONS = [
    # router logits: reduction order and arithmetic
    ("sequential_logit", "for (int o = LANES / 2; o >= 1; o /= 2)",
     "for (int s = 1; s < LANES; ++s) p[0] += p[s]; for (int o = 0; o >= 1; o /= 2)"),
    ("tree_levels_reversed", "for (int o = LANES / 2; o >= 1; o /= 2)", "for (int o = 1; o <= LANES / 2; o *= 2)"),
    ("contiguous_blocks_per_lane", "for (int h = j; h < H; h += LANES) acc",
     "for (int h = j * (H / LANES); h < (j + 1) * (H / LANES); ++h) acc"),
    ("eight_element_chunks_per_lane",
     "for (int h = j; h < H; h += LANES) acc = fmaf(bf16_to_f32(xrow[h]), wrow[h], acc);",
     "for (int c = j; c * 8 < H; c += LANES) for (int h = c * 8; h < c * 8 + 8; ++h) "
     "acc = fmaf(bf16_to_f32(xrow[h]), wrow[h], acc);"),
    ("sixteen_lanes", "#define LANES 32", "#define LANES 16"),
    ("decreasing_h_in_lane", "for (int h = j; h < H; h += LANES) acc",
     "for (int h = j + ((H - 1 - j) / LANES) * LANES; h >= 0; h -= LANES) acc"),
    ("no_fma_in_logit", "for (int h = j; h < H; h += LANES) acc = fmaf(bf16_to_f32(xrow[h]), wrow[h], acc);",
     "for (int h = j; h < H; h += LANES) acc = acc + bf16_to_f32(xrow[h]) * wrow[h];"),
    ("dropped_bias", "if (bias) l = l + bias[e];", "if (bias) l = l;"),
    # top-k, weights, permutation
    ("ties_to_higher_index", "while (j >= 0 && l[order[j]] < l[v])", "while (j >= 0 && l[order[j]] <= l[v])"),
    ("weights_over_all_experts", "for (int k = 0; k < K; ++k) den += exp(", "for (int k = 0; k < E; ++k) den += exp("),
    ("tokens_reversed_in_permutation", "for (int t = 0; t < T; ++t) /* tokens", "for (int t = T-1; t >= 0; --t) /* tokens"),
    # bf16 FFN
    ("gate_up_swapped", "const uint16_t* wu = wgu + (size_t)(I + j) * H;", "const uint16_t* wu = wgu + (size_t)(j) * H;"),
    ("silu_sign", "return g / (1.0f + expf(-g));", "return g / (1.0f + expf(g));"),
    ("down_transposed", "const uint16_t* wd = wdn + (size_t)o * I;", "const uint16_t* wd = wdn + (size_t)(o % I) * I;"),
    ("routing_weight_dropped", "y[o] = weight * acc;", "y[o] = acc;"),
    ("h_truncated_not_rounded", "hrow[j] = f32_to_bf16(silu_f32(g) * u);", TRUNC_H),
    # combine
    ("combine_reversed", "for (int k = 1; k < K; ++k) acc = acc + y_pair", "for (int k = K-1; k >= 1; --k) acc = acc + y_pair"),
    ("combine_rounds_each_term", "acc = acc + y_pair[(size_t)inv[(size_t)t * K + k] * H + o];",
     "acc = acc + bf16_to_f32(f32_to_bf16(y_pair[(size_t)inv[(size_t)t * K + k] * H + o]));"),
    ("output_truncated_not_rounded", "out[(size_t)t * H + o] = f32_to_bf16(acc);", TRUNC_OUT),
    # FP8
    ("e4m3_round_half_up", "double q = nearbyint((m - 1.0) * 8.0);", "double q = floor((m - 1.0) * 8.0 + 0.5);"),
    ("quantiser_reciprocal_multiply", "float t = v / s;", "float t = v * (1.0f / s);"),
    ("quantiser_e4m3fnuz_max", "amax / 448.0f", "amax / 240.0f"),
    ("quantiser_zero_block_scale", "float s = (amax == 0.0f) ? 1.0f : amax / 448.0f;", "float s = amax / 448.0f;"),
    ("fp8_activation_scale_dropped", "acc = fmaf(part, sa[kb] * sw[kb], acc);", "acc = fmaf(part, sw[kb], acc);"),
    ("fp8_weight_block_row", "sgu[e] + (size_t)(rg / 128) * (H / 128)", "sgu[e] + (size_t)(rg / 256) * (H / 128)"),
    # MX (MXFP4 weights, MX e4m3 activations)
    ("e2m1_round_half_up", "double q = nearbyint((m - 1.0) * 2.0);", "double q = floor((m - 1.0) * 2.0 + 0.5);"),
    ("mx_e2m1_emax_3", "const int emax = elem == 0 ? 2 : 8;", "const int emax = elem == 0 ? 3 : 8;"),
    ("mx_scale_applied_upside_down", "ldexp((double)bf16_to_f32(v[i]), -sexp)", "ldexp((double)bf16_to_f32(v[i]), sexp)"),
    ("mx_zero_block_scale", "int sexp = -127;", "int sexp = 0;"),
    ("mx_activation_scale_dropped", "(int)sw[b] + (int)sa[b] - 254", "(int)sw[b] - 127"),
    # composition of the steps
    ("py_weights_of_the_wrong_slot", "pw = w64[sel].reshape(-1)", "pw = w64[sel][:, ::-1].reshape(-1)"),
    ("py_pairs_of_the_wrong_token", "pt = np.repeat(sel, K)", "pt = np.tile(sel, K)"),
]


def _run_pins(tmp_path, name, old=None, new=None):
    d = tmp_path / name
    shutil.copytree(os.path.join(ROOT, "oracle"), d / "oracle",
                    ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    src = d / "oracle" / ("__init__.py" if name.startswith("py_") else "moe_oracle.c")
    if old is not None:
        s = src.read_text()
        assert s.count(old) >= 1, f"{name}: text not found in the oracle"
        src.write_text(s.replace(old, new, 1))
    env = dict(os.environ, PYTHONPATH=os.pathsep.join([str(d), ROOT]))
    return subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", PINS],
                          cwd=str(d), env=env, capture_output=True, text=True, timeout=900)


def test_unmodified_copy_passes_the_pins(tmp_path):
    r = _run_pins(tmp_path, "control")
    assert r.returncode == 0, r.stdout[-3000:]


def test_every_planted_mistake_fails_a_pin(tmp_path):
    """All mutants at once (one process each, run side by side)."""
    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(max_workers=max(2, (os.cpu_count() or 2))) as ex:
        runs = list(ex.map(lambda m: (m[0], _run_pins(tmp_path, *m)), MUTATIONS))
    survived = [name for name, r in runs if r.returncode == 0]
    crashed = [(name, r.returncode, r.stderr[-500:]) for name, r in runs if r.returncode not in (0, 1)]
    assert not survived, f"mistakes that no pin caught: {survived}"
    assert not crashed, f"mutants that did not run to a pin failure: {crashed}"
    assert len(runs) == len({m[0] for m in MUTATIONS}) == len(MUTATIONS)
