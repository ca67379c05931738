"""The CPU oracle against brute force, closed forms, invariants and the pages' budget.

Also plants mistakes in copies of the oracle (on the CPU) and checks that
each one is caught by at least one pin.
"""
import importlib.util
import os
import sys

import pytest

from oracle_pins import ALL_PINS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE_SRC = os.path.join(ROOT, "oracle", "kvpop_oracle.py")

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import oracle  # noqa: E402


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pins(pin):
    pin(oracle)


# Each mutant: (name, original text, replacement).  Every original must occur in the source.
MUTANTS = [
    ("window_strict", "rows - cols >= W", "rows - cols > W"),
    ("causal_excludes_self", "cols <= rows, S, -np.inf", "cols < rows, S, -np.inf"),
    ("causal_mask_dropped", "S = np.where(cols <= rows, S, -np.inf)", "S = S"),
    ("gqa_wrong_group_target", "h = g // G\n", "h = g % Hkv\n"),
    ("gqa_wrong_group_lse", "kh = q[s:s + L, g, :], k[s:s + L, g // G, :]",
     "kh = q[s:s + L, g, :], k[s:s + L, g % Hkv, :]"),
    ("scale_dropped", "S = scale * (qg[r0:r1] @ kh[:r1].T)", "S = (qg[r0:r1] @ kh[:r1].T)"),
    ("operands_transposed", "S = scale * (qg[r0:r1] @ kh[:r1].T)", "S = scale * (kh[r0:r1] @ qg[:r1].T)"),
    ("group_mean_not_sum", "col_sum = F.sum(axis=0)", "col_sum = F.sum(axis=0) / G"),
    ("lse_max_dropped", "lse = (m + np.log(Z))[:, 0]", "lse = (np.log(Z))[:, 0]"),
    ("softmax_unnormalised", "A = P / Z", "A = P"),
    ("keep_tie_break_reversed", "np.lexsort((pos, -sc))", "np.lexsort((-pos, -sc))"),
    ("keep_smallest_not_largest", "np.lexsort((pos, -sc))", "np.lexsort((pos, sc))"),
    ("keep_window_short", "keep[h, s + L - W:s + L] = 1", "keep[h, s + L - W + 1:s + L] = 1"),
    ("keep_no_sinks", "keep[h, s:s + S] = 1", "pass"),
    ("keep_off_by_one_k", "order[:k_top]", "order[:k_top - 1]"),
    ("keep_all_when_short_dropped", "if L <= B:", "if L < 0:"),
    ("threshold_window_off_by_one", "hi = t - W                                     # last candidate position",
     "hi = t - W - 1"),
    ("threshold_kth_off_by_one", "kth = order[k_top - 1]", "kth = order[k_top]"),
    ("threshold_tie_reversed", "order = np.lexsort((pos, -sc))\n                kth", "order = np.lexsort((-pos, -sc))\n                kth"),
    ("threshold_sinks_included", "pos = np.arange(S, hi + 1)", "pos = np.arange(0, hi + 1)"),
    ("compact_drops_last", "p = p[:capacity]", "p = p[:capacity - 1]"),
    ("decode_wrong_group", "            h = g // G\n            n = int(count[b, h])", "            h = g % Hkv\n            n = int(count[b, h])"),
    ("decode_unnormalised", "out[b, g] = (w / Z) @ vc[b, h, :n]", "out[b, g] = w @ vc[b, h, :n]"),
    ("decode_scale_dropped", "logits = scale * (kc[b, h, :n] @ q[b, g])", "logits = (kc[b, h, :n] @ q[b, g])"),
    ("bf16_decoded_wrongly", "<< np.uint32(16)", "<< np.uint32(15)"),
    ("target_overwritten_not_summed", "target[h, s + j_lo:s + r1] += col_sum[j_lo:]",
     "target[h, s + j_lo:s + r1] = col_sum[j_lo:]"),
    ("target_last_row_dropped", "for r0 in range(i_start, L, ROW_BLOCK):\n                r1 = min(r0 + ROW_BLOCK, L)",
     "for r0 in range(i_start, L, ROW_BLOCK):\n                r1 = min(r0 + ROW_BLOCK, L - 1)"),
    ("far_mass_unwindowed", "far[g, s + r0:s + r1] = F.sum(axis=1)", "far[g, s + r0:s + r1] = A.sum(axis=1)"),
    ("key_lo_rows_skipped", "i_start = min(L, j_lo + W) if key_lo", "i_start = min(L, j_lo + W + 1) if key_lo"),
    ("keep_candidates_overlap_window", "lo, hi = S, L - W ", "lo, hi = S, L - W + 1 "),
    ("keep_nan_ranked_first",
     "sc = score[h, s + lo:s + hi].astype(np.float64)\n            order",
     "sc = np.nan_to_num(score[h, s + lo:s + hi].astype(np.float64), nan=np.inf)\n            order"),
    ("keep_budget_unchecked", "if B < S + W:", "if B < 0:"),
    ("threshold_defined_one_step_late", "if len(pos) < k_top:", "if len(pos) <= k_top:"),
    ("threshold_k0_keeps_all", "thr_s[h, s0 + t] = np.inf", "thr_s[h, s0 + t] = -np.inf"),
    ("threshold_nan_ranked_first", "sc = score[h, s0 + S:s0 + hi + 1].astype(np.float64)",
     "sc = np.nan_to_num(score[h, s0 + S:s0 + hi + 1].astype(np.float64), nan=np.inf)"),
    ("threshold_budget_unchecked", "if k_top < 0:", "if k_top < -10**9:"),
    ("compact_count_capped", "cnt[b, h] = len(p)\n            p = p[:capacity]",
     "p = p[:capacity]\n            cnt[b, h] = len(p)"),
    ("decode_count_ignored", "n = int(count[b, h])\n            if n == 0", "n = kc.shape[2]\n            if int(count[b, h]) == 0"),
    ("decode_lse_max_dropped", "lse[b, g] = m + np.log(Z)", "lse[b, g] = np.log(Z)"),
]


def _load_mutant(name, old, new, tmp_path):
    src = open(ORACLE_SRC).read()
    assert old in src, f"mutant {name}: text not found in the oracle"
    path = tmp_path / f"oracle_mutant_{name}.py"
    path.write_text(src.replace(old, new))
    spec = importlib.util.spec_from_file_location(f"oracle_mutant_{name}", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_oracle_mutants_are_caught(name, old, new, tmp_path):
    mod = _load_mutant(name, old, new, tmp_path)
    caught = []
    for pin in ALL_PINS:
        try:
            pin(mod)
        except Exception:  # an assertion, or the mutant crashing on the pin's input
            caught.append(pin.__name__)
    assert caught, f"planted mistake {name} passed every pin"
