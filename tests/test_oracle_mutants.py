"""Plants typical slips in a copy of the oracle and checks that the pins catch each one.

Every mutant is a one-line edit of ``oracle/attention.py``'s source (a dropped term, a wrong
sign, a wrong index, a transposed operand, an off-by-one). The edited copy is loaded as a
separate module on the CPU and handed to the pin tests in place of the real oracle; the
test passes only if at least one pin then fails. The real oracle is never modified.
"""
import importlib.util
import inspect
import os
import types

import pytest

import oracle.attention as real
import tests.test_oracle_pins as pins

SRC = inspect.getsource(real)

MUTANTS = {
    "rope_sign": ("x * cos - y * sin, x * sin + y * cos", "x * cos + y * sin, -x * sin + y * cos"),
    "rope_freq": ("-2.0 * pair / hd", "-1.0 * pair / hd"),
    "rope_pairing_halves": ("pairs = t.reshape(t.shape[:-1] + (hd // 2, 2))",
                            "pairs = t.reshape(t.shape[:-1] + (2, hd // 2)).swapaxes(-1, -2)"),
    "rope_positions_shift": ("p = np.asarray(positions, dtype=F64).reshape(-1, 1)",
                             "p = np.asarray(positions, dtype=F64).reshape(-1, 1) + 1"),
    "alibi_slope_index": ("-8.0 * (h + 1.0) / H", "-8.0 * h / H"),
    "alibi_sign": ("s = s - float(slopes[h]) * np.abs(i - j)", "s = s + float(slopes[h]) * np.abs(i - j)"),
    "gqa_modulo": ("g = h // group                            # key/value head serving query head h",
                   "g = h % KV"),
    "window_off_by_one": ("ok &= (i - j) < window", "ok &= (i - j) <= window"),
    "causal_strict": ("ok &= j <= i", "ok &= j < i"),
    "scale_dropped": ("s = qh[b, h] @ kh[b, g].T / np.sqrt(hd)", "s = qh[b, h] @ kh[b, g].T"),
    "scale_by_hd": ("s = qh[b, h] @ kh[b, g].T / np.sqrt(hd)", "s = qh[b, h] @ kh[b, g].T / hd"),
    "softmax_no_max_shift_lse": ("m[..., 0] + np.log(safe[..., 0])", "np.log(safe[..., 0])"),
    "k_not_rotated": ("kh = rope(kh, pos, rope_base)", "kh = kh"),
    "values_rotated": ("    else:\n        qh = qh[:, :, rows]",
                       "        vh = rope(vh, pos, rope_base)\n    else:\n        qh = qh[:, :, rows]"),
    "decode_qpos_shift": ("qb = rope(qb[:, None, :], [p], rope_base)[:, 0, :]",
                          "qb = rope(qb[:, None, :], [p - 1], rope_base)[:, 0, :]"),
    "decode_window": ("ok = (p - j) < window if window > 0", "ok = (p - j) <= window if window > 0"),
    "chunk_position_shift": ("P = int(qpos0[b]) + np.arange(Tq)                    # query positions",
                             "P = int(qpos0[b]) + np.arange(Tq) + 1"),
    "chunk_keys_beyond_length": ("kb = _f64(kcache[b, :L]).transpose(1, 0, 2)          # [KV,L,hd]",
                                 "kb = _f64(kcache[b, :L + 1]).transpose(1, 0, 2)"),
    "kv_write_rotation_position": ("kb = rope(kb, p, rope_base)\n        kc[b, p]",
                                   "kb = rope(kb, p + 1, rope_base)\n        kc[b, p]"),
    "paged_row_index": ("return pages[page, j % page_size]", "return pages[page, (j + 1) % page_size]"),
    "paged_block_index": ("page = np.asarray(block_table)[b][j // page_size]",
                          "page = np.asarray(block_table)[b][j % page_size]"),
    "latent_scale_by_dc": ("s = k @ q[b, h] / np.sqrt(hd)", "s = k @ q[b, h] / np.sqrt(c.shape[2])"),
    "latent_value_projection": ("v = c[b, :L] @ W_uv[h]", "v = c[b, :L] @ W_uk[h]"),
    "rmsnorm_mean_not_rms": ("rms = np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)",
                             "rms = np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)"),
    "rmsnorm_eps_outside_root": ("rms = np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)",
                                 "rms = np.sqrt(np.mean(x * x, axis=-1, keepdims=True)) + eps"),
    "rmsnorm_default_eps": ("def rmsnorm(x, gamma, eps: float = 1e-6)", "def rmsnorm(x, gamma, eps: float = 1e-5)"),
    "fused_default_eps": ("window: int = 0, slopes=None, eps: float = 1e-6, rows=None):",
                          "window: int = 0, slopes=None, eps: float = 1e-8, rows=None):"),
    "fused_no_residual": ("out = (x if rows is None else x[:, np.asarray(rows)]) + ctx.reshape(B, R, H * hd) @ Wo",
                          "out = ctx.reshape(B, R, H * hd) @ Wo"),
    "fused_qkv_split": ("k = qkv[..., H * hd:(H + KV) * hd].reshape(B, T, KV, hd)",
                        "k = qkv[..., (H + KV) * hd:].reshape(B, T, KV, hd)"),
    "block_wq_transposed": ("q = (x @ Wq).reshape(B, T, H, hd)", "q = (x @ Wq.T).reshape(B, T, H, hd)"),
    "block_head_split": ("q = (x @ Wq).reshape(B, T, H, hd)",
                         "q = (x @ Wq).reshape(B, T, hd, H).swapaxes(2, 3)"),
}

PIN_TESTS = [
    ("test_rope_closed_forms", True), ("test_rope_identity_at_zero_and_norm", False),
    ("test_rope_relative", False), ("test_rope_matches_complex_view", False),
    ("test_alibi_slopes_fixture", True), ("test_alibi_geometric_weights", False),
    ("test_window_one_returns_own_value", False), ("test_single_token", False),
    ("test_zero_query_prefix_mean", False), ("test_weights_sum_to_one", False),
    ("test_scale_is_inverse_sqrt_hd", False), ("test_gqa_equals_mha_with_repeated_heads", False),
    ("test_lab_properties", True), ("test_decode_token_by_token_equals_full", False),
    ("test_decode_brute_force_and_empty_cache", False), ("test_chunked_prefill_equals_full", False),
    ("test_chunk_brute_force_and_cache_route", False),
    ("test_chunk_of_one_row_is_a_decode_step_and_empty_cache", False),
    ("test_paged_decode_brute_force_and_page_order", False),
    ("test_latent_fold_leaves_scores_and_outputs_unchanged", False),
    ("test_rmsnorm_closed_forms", False),
    ("test_fused_block_is_residual_plus_the_plain_block_on_normalised_input", False),
]


def _load_mutant(name):
    old, new = MUTANTS[name]
    assert SRC.count(old) >= 1, f"mutant {name}: pattern not found in the oracle source"
    mod = types.ModuleType(f"oracle_mutant_{name}")
    mod.__file__ = real.__file__
    exec(compile(SRC.replace(old, new, 1), f"<mutant {name}>", "exec"), mod.__dict__)
    return mod


def _caught(mod, golden_dir, monkeypatch):
    monkeypatch.setattr(pins, "A", mod)
    for test_name, wants_golden in PIN_TESTS:
        fn = getattr(pins, test_name)
        try:
            fn(golden_dir) if wants_golden else fn()
        except Exception:
            return test_name
    # the parametrised cross-route checks
    for flags in pins.FLAGS:
        for shape in [(1, 5, 4, 2, 8), (2, 7, 4, 1, 6)]:
            try:
                pins.test_brute_force_agrees(flags, shape)
            except Exception:
                return "test_brute_force_agrees"
    for pos0 in (0, 100):
        try:
            pins.test_block_brute_force(pos0)
        except Exception:
            return "test_block_brute_force"
    return None


@pytest.mark.filterwarnings("ignore::RuntimeWarning")
@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, golden_dir, monkeypatch):
    mod = _load_mutant(name)
    assert _caught(mod, golden_dir, monkeypatch) is not None, f"no pin catches mutant {name}"


def test_unmutated_copy_passes(golden_dir, monkeypatch):
    mod = types.ModuleType("oracle_copy")
    exec(compile(SRC, "<oracle copy>", "exec"), mod.__dict__)
    assert _caught(mod, golden_dir, monkeypatch) is None
