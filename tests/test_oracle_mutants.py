"""The oracle's pins catch plausible mistakes.

Each case plants one mistake (a dropped term, a wrong sign, an off-by-one, a
wrong index or operand) in a temporary copy of the C oracle, builds it with
the oracle's own compiler flags, loads it in place of the real library and
runs the pins of test_oracle_pins.py against it: at least one pin must fail.
The few steps the oracle takes in Python (the rows of a long forward, the
prefill -> ring handoff) are mutated the same way, in a copy of the function
swapped in for one case.  The oracle's source is never changed, and every
planted mistake keeps all memory accesses inside their buffers.
"""
import contextlib
import inspect
import os
import shutil
import textwrap

import pytest

import oracle
import test_oracle_pins as pins
from oracle.build import SRC, compile_lib

# (name, [(text in swa_oracle.c, replacement)]): each text is replaced at its
# first occurrence, which is the one the comment names.
MUTANTS = [
    # RMSNorm (rms_norm)
    ("rmsnorm_eps_dropped", [("sqrt(ss / D + eps)", "sqrt(ss / D)")]),
    ("rmsnorm_mean_over_D_minus_1", [("sqrt(ss / D + eps)", "sqrt(ss / (D - 1) + eps)")]),
    ("rmsnorm_weight_dropped", [("y[d] = xhat[d] * w[d];", "y[d] = xhat[d];")]),
    # RoPE (rope_apply, then rope_apply_transpose)
    ("rope_sign", [("y[j] = a * c - b * s;", "y[j] = a * c + b * s;")]),
    ("rope_frequency_exponent", [("pow(base, -2.0 * j / R)", "pow(base, -1.0 * j / R)")]),
    ("rope_transpose_sign", [("dy[j] = a * c + b * s;", "dy[j] = a * c - b * s;")]),
    # forward (oracle_fwd)
    ("fwd_key_position_off_by_one",
     [("rope_apply(y, R, base, (double)(pos0 + t));", "rope_apply(y, R, base, (double)(pos0 + t + 1));")]),
    ("fwd_window_one_short", [("int64_t j0 = i - W + 1;", "int64_t j0 = i - W + 2;")]),
    ("fwd_gqa_head_mapping", [("int kvh = h / group;", "int kvh = h % Hkv;")]),
    ("fwd_scale_dropped",
     [("s[j - j0] = scale * dot(qp, kp + IDX4(b, j, kvh, 0, T, Hkv, D), D);",
       "s[j - j0] = dot(qp, kp + IDX4(b, j, kvh, 0, T, Hkv, D), D);")]),
    ("fwd_gate_sign", [("oi[d] = a[d] * sigmoid(gi[d]);", "oi[d] = a[d] * sigmoid(-gi[d]);")]),
    ("fwd_lse_without_max", [("* Hq + h] = m + log(l);", "* Hq + h] = log(l);")]),
    ("fwd_exp_without_max", [("s[j - j0] = exp(s[j - j0] - m);", "s[j - j0] = exp(s[j - j0]);")]),
    # backward (oracle_bwd, norm_rope_backward)
    ("bwd_key_position_off_by_one",
     [("rope_apply(kp + t * D, R, base, (double)t);", "rope_apply(kp + t * D, R, base, (double)(t + 1));")]),
    ("bwd_jacobian_mean_term_dropped",
     [("dx[d] = (dy[d] * w[d] - xhat[d] * mean) / r;", "dx[d] = (dy[d] * w[d]) / r;")]),
    ("bwd_dw_weighted", [("dw_acc[d] += dy[d] * xhat[d];", "dw_acc[d] += dy[d] * w[d] * xhat[d];")]),
    ("bwd_ds_without_rowsum",
     [("double ds = P[j - j0] * (dp[j - j0] - Dsum);", "double ds = P[j - j0] * dp[j - j0];")]),
    ("bwd_dg_sigmoid_derivative",
     [("dgi[d] = dOi[d] * a[d] * sg * (1.0 - sg);", "dgi[d] = dOi[d] * a[d] * sg;")]),
    ("bwd_dv_ungated", [("dvj[d] += P[j - j0] * dA[d];", "dvj[d] += P[j - j0] * dOi[d];")]),
    ("bwd_dk_scale_dropped",
     [("dkp[j * D + d] += scale * ds * qp[d];", "dkp[j * D + d] += ds * qp[d];")]),
    ("bwd_dq_uses_query_not_key",
     [("dqp[d] += scale * ds * kp[j * D + d];", "dqp[d] += scale * ds * qp[d];")]),
    # decode (oracle_decode)
    ("decode_ring_slot", [("int64_t slot = p % W;", "int64_t slot = (p + 1) % W;")]),
    ("decode_position_zero_invalid", [("valid[si] = ps >= 0;", "valid[si] = ps > 0;")]),
    ("decode_query_position",
     [("rope_apply(qp, R, base, (double)p);", "rope_apply(qp, R, base, (double)(p + 1));")]),
    ("decode_caches_k_as_v",
     [("vc[d] = oracle_bf16_bits(v_new[(n * Hkv + h) * D + d]);",
       "vc[d] = oracle_bf16_bits(k_new[(n * Hkv + h) * D + d]);")]),
    # bf16 rounding and the footprint
    ("bf16_ties_away", [("nearbyint(x / q) * q", "floor(x / q + 0.5) * q")]),
    ("bf16_subnormal_floor", [("if (qe < -133) qe = -133;", "if (qe < -126) qe = -126;")]),
    ("kv_footprint_one_vector", [("return 2 * layers * kv_heads", "return layers * kv_heads")]),
]

# (name, oracle function, [(text in its source, replacement)])
PY_MUTANTS = [
    ("prefill_ring_drops_oldest", "prefill_to_ring",
     [("range(max(0, T - W), T)", "range(max(0, T - W + 1), T)")]),
    ("prefill_ring_slot_as_position", "prefill_to_ring",
     [("np.full(B, float(p))", "np.full(B, float(s))")]),
    ("fwd_rows_keys_start_one_late", "fwd_rows",
     [("kb = max(0, t0 - W + 1)", "kb = max(0, t0 - W + 2)")]),
    ("global_decode_skips_new_key", "global_decode",
     [("kc[n, kvh, :p + 1]", "kc[n, kvh, :p]"), ("vc[n, kvh, :p + 1]", "vc[n, kvh, :p]")]),
    ("global_decode_gqa_mapping", "global_decode", [("kvh = h // group", "kvh = h % Hkv")]),
    ("global_decode_query_position", "global_decode",
     [("qp = norm_rope(q[n][None], wq, at,", "qp = norm_rope(q[n][None], wq, at + 1,")]),
    ("global_decode_caches_k_as_v", "global_decode",
     [("vc[n, :, p, :] = bf16_round_array(v_new[n])",
       "vc[n, :, p, :] = bf16_round_array(k_new[n])")]),
    ("global_decode_scale_dropped", "global_decode",
     [("s = sc * (keys @ qp[h])", "s = keys @ qp[h]")]),
    ("ring_varlen_position_offset_dropped", "prefill_to_ring_varlen",
     [("np.array([float(p)])", "np.array([float(p - p0)])")]),
    ("ring_varlen_drops_oldest", "prefill_to_ring_varlen",
     [("range(max(p0, p0 + n - W), p0 + n)", "range(max(p0, p0 + n - W + 1), p0 + n)")]),
    ("e4m3_bias_8", "e4m3_to_f64", [("e.astype(np.float64) - 7.0", "e.astype(np.float64) - 8.0")]),
    ("e4m3_subnormal_scale", "e4m3_to_f64", [("m * 2.0 ** -9", "m * 2.0 ** -10")]),
]

PINS = (
    [(f"fwd_bruteforce{args}", pins.test_fwd_matches_dense_bruteforce, args) for args in [
        (2, 5, 4, 2, 3), (1, 40, 8, 8, 7), (1, 33, 2, 1, 1), (1, 1, 4, 1, 128),
        (1, 129, 8, 2, 128), (2, 200, 4, 1, 64)]]
    + [(f.__name__, f, ()) for f in [
        pins.test_fwd_other_head_dim_and_rot_dim, pins.test_window_ge_T_is_causal_sdpa,
        pins.test_window_one_is_v_times_gate_and_ignores_q_k_w, pins.test_saturated_gates,
        pins.test_lse_is_log_normaliser, pins.test_gate_worked_example,
        pins.test_window_includes_self_worked_example, pins.test_long_positions_chunked_equals_full,
        pins.test_rmsnorm_mean_square_closed_form, pins.test_rope_invariants,
        pins.test_rope_relative_position_invariance, pins.test_bwd_central_finite_differences,
        pins.test_bwd_matches_torch_autograd, pins.test_decode_matches_dense_over_ring_contents,
        pins.test_bf16_rounding_matches_torch_rne, pins.test_kv_footprint_worked_numbers]]
    + [(f"decode_equals_prefill_row({p})", pins.test_decode_equals_prefill_row, (p,))
       for p in (0, 5, 127, 128, 300)]
    + [(f"prefill_to_ring({T})", pins.test_prefill_to_ring_equals_sequential_decode, (T,))
       for T in (1, 131)]
    + [("global_decode_dense", pins.test_global_decode_matches_dense_over_cache_contents, ())]
    + [("e4m3_decoding", pins.test_e4m3_decoding_matches_torch_and_the_encoding, ())]
    + [(f"ring_varlen({c})", pins.test_prefill_to_ring_varlen_equals_sequential_decode, (c,))
       for c in ("ragged", "continued")]
    + [(f"global_decode_ring({p})", pins.test_global_decode_equals_ring_decode_inside_the_window,
        (p,)) for p in (0, 77)]
    + [(f"global_decode_prefill({p})", pins.test_global_decode_equals_causal_prefill_row, (p,))
       for p in (5, 200)]
)


def build_variant(tmp_path, edits):
    src = open(SRC, encoding="utf-8").read()
    for old, new in edits:
        assert old in src, f"mutation site not found: {old}"
        src = src.replace(old, new, 1)
    path = os.path.join(str(tmp_path), "swa_oracle_variant.c")
    with open(path, "w", encoding="utf-8") as f:
        f.write(src)
    return compile_lib(path, os.path.join(str(tmp_path), "liboracle_variant.so"))


@contextlib.contextmanager
def oracle_library(path):
    """Route every oracle call to the library at `path` for the duration."""
    saved_lib, saved_build = oracle._lib, oracle._build
    oracle._lib, oracle._build = None, (lambda: path)
    try:
        yield
    finally:
        oracle._lib, oracle._build = saved_lib, saved_build


@contextlib.contextmanager
def oracle_function(name, edits):
    """Swap in a copy of oracle.<name> with `edits` applied to its source."""
    src = textwrap.dedent(inspect.getsource(getattr(oracle, name)))
    for old, new in edits:
        assert old in src, f"mutation site not found: {old}"
        src = src.replace(old, new, 1)
    ns = dict(vars(oracle))
    exec(compile(src, f"<{name} variant>", "exec"), ns)
    saved = getattr(oracle, name)
    setattr(oracle, name, ns[name])
    try:
        yield
    finally:
        setattr(oracle, name, saved)


def failing_pins(stop_at_first):
    failed = []
    for name, fn, args in PINS:
        try:
            fn(*args)
        except Exception:  # an assertion, or NaNs / infs a pin refuses
            failed.append(name)
            if stop_at_first:
                break
    return failed


pytestmark = pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")


def test_unmodified_copy_passes_every_pin(tmp_path):
    """The harness itself: unedited copies, built or swapped in this way,
    pass all the pins."""
    with oracle_library(build_variant(tmp_path, [])):
        assert failing_pins(stop_at_first=False) == []
    with oracle_function("prefill_to_ring", []), oracle_function("fwd_rows", []), \
            oracle_function("global_decode", []), oracle_function("e4m3_to_f64", []), \
            oracle_function("prefill_to_ring_varlen", []):
        assert failing_pins(stop_at_first=False) == []


@pytest.mark.parametrize("name,edits", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_fails_a_pin(tmp_path, name, edits):
    with oracle_library(build_variant(tmp_path, edits)):
        assert failing_pins(stop_at_first=True), f"no pin catches the planted mistake {name}"


@pytest.mark.parametrize("name,func,edits", PY_MUTANTS, ids=[m[0] for m in PY_MUTANTS])
def test_planted_mistake_in_python_step_fails_a_pin(name, func, edits):
    with oracle_function(func, edits):
        assert failing_pins(stop_at_first=True), f"no pin catches the planted mistake {name}"
