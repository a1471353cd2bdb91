"""Planted mistakes in the oracles, caught by their pins.

Each case below writes one plausible slip (a dropped term, a flipped sign, a
wrong index, bound or head mapping, a transposed or swapped operand, a missing
scale factor, a lost de-duplication, a wrong tie order) into a copy of one
oracle module's source, runs that copy in place of the real one, and requires
at least one pin of the module's pin file (``test_oracle``,
``test_selector_oracle``, ``test_bitmap_oracle``) to fail on it.  The pins
compare with things other than the oracle (hand-worked values, a brute-force
per-pair loop, PyTorch's causal attention, closed forms, finite differences,
invariants, special cases that reduce to a sort), so this shows that every
formula the oracles state is held by something outside them.  The mistakes are
planted on the CPU, in the oracles only.
"""

import pathlib
import types

import pytest

import oracle
import test_bitmap_oracle as bitmap_pins
import test_oracle as pins
import test_selector_oracle as selector_pins

ORACLE_DIR = pathlib.Path(oracle.__file__).parent

# ---------------------------------------------------------------------------
# attention oracle: the pins reach it through the ``oracle`` package
# ---------------------------------------------------------------------------

ATTENTION_PINS = [
    ("hand-worked example", pins.test_hand_worked_example),
    ("brute force G=2", lambda: pins.test_brute_force_pair_loop(24, 24, 4, 2, 16)),
    ("brute force T!=T_kv", lambda: pins.test_brute_force_pair_loop(10, 14, 12, 1, 24)),
    ("causal = SDPA, 24Q/2KV", lambda: pins.test_causal_routes_equal_causal_attention(20, 24, 2)),
    ("padding rows", pins.test_padding_rows_zero_output_and_gradients),
    ("duplicates/invalid = set", pins.test_duplicates_and_invalid_ids_are_a_set),
    ("route order", pins.test_route_order_is_irrelevant),
    ("single-route closed form", pins.test_single_route_closed_form),
    ("lse = logsumexp", pins.test_all_keys_lse_is_logsumexp),
    ("finite differences", pins.test_backward_matches_finite_differences),
    ("rows = dense, seq32k recipe", lambda: pins.test_row_form_matches_dense_form("seq32k", 192)),
    ("rows = dense, cp128k recipe", lambda: pins.test_row_form_matches_dense_form("cp128k", 128)),
    ("non-finite isolation", pins.test_row_form_isolates_unselected_nonfinite_kv),
    ("row lists and quads", pins.test_route_rows_csr_and_quad_lists),
    ("tile lists, 8 keys", lambda: pins.test_key_tile_lists(8)),
    ("tile lists, 128 keys", lambda: pins.test_key_tile_lists(128)),
    ("tiles of 4 = quads", pins.test_key_tile_lists_refine_quads),
    ("query unions, groups of 4", lambda: pins.test_query_union_lists(4)),
    ("query unions, groups of 1", lambda: pins.test_query_union_lists(1)),
]

# name -> (text in the oracle, its mistaken form); every occurrence is replaced,
# so a slip made consistently in the dense and the row forms is covered too
ATTENTION_MUTANTS = {
    "membership drops key 0": ("valid = (r >= 0) & (r < kv_length)", "valid = (r > 0) & (r < kv_length)"),
    "row sets keep duplicates": ("out.append(np.unique(keep))", "out.append(np.sort(keep))"),
    "row lists padded with 0": ("cols = np.full((T, W), -1, dtype=np.int32)", "cols = np.zeros((T, W), dtype=np.int32)"),
    "quad mask bits reversed": ("(1 << (int(j) & 3))", "(1 << (3 - (int(j) & 3)))"),
    "tile index fixed at 128": ("tiles = s // tile", "tiles = s // 128"),
    "tile i0 = last key": ("int(pos[0])", "int(pos[-1])"),
    "lse without the max": ("lse = np.where(nonempty, m + np.log(", "lse = np.where(nonempty, np.log("),
    "empty-row lse 0": ("np.log(np.where(nonempty, l, 1.0)), -np.inf)", "np.log(np.where(nonempty, l, 1.0)), 0.0)"),
    "exp not shifted by max": ("np.exp(np.where(M, S, 0.0) - m[:, None])", "np.exp(np.where(M, S, 0.0))"),
    "softmax not normalised": ("P = E / np.where(nonempty, l, 1.0)[:, None]", "P = E"),
    "forward scores unscaled": ("S = scale * (q[:, h, :] @ k[:, g, :].T)\n        P, lse[:, h]",
                                "S = (q[:, h, :] @ k[:, g, :].T)\n        P, lse[:, h]"),
    "KV head h % G": ("g = h // hpg", "g = h % G"),
    "delta dropped": ("dS = P * (dP - delta[:, None])", "dS = P * dP"),
    "dS sign flipped": ("dS = P * (dP - delta[:, None])", "dS = P * (delta[:, None] - dP)"),
    "delta from dO . dO": ("delta = (do[:, h, :] * out_h).sum(axis=1)", "delta = (do[:, h, :] * do[:, h, :]).sum(axis=1)"),
    "dQ against V": ("dq[:, h, :] = scale * (dS @ k[:, g, :])", "dq[:, h, :] = scale * (dS @ v[:, g, :])"),
    "dQ unscaled": ("dq[:, h, :] = scale * (dS @ k[:, g, :])", "dq[:, h, :] = dS @ k[:, g, :]"),
    "dK unscaled": ("dk[:, g, :] += scale * (dS.T @ q[:, h, :])", "dk[:, g, :] += dS.T @ q[:, h, :]"),
    "dK overwritten per head": ("dk[:, g, :] += scale", "dk[:, g, :] = scale"),
    "dV from untransposed P": ("dv[:, g, :] += P.T @ do[:, h, :]", "dv[:, g, :] += P @ do[:, h, :]"),
    "dV from dS": ("dv[:, g, :] += P.T @ do[:, h, :]", "dv[:, g, :] += dS.T @ do[:, h, :]"),
    "row lse without the max": ("return P, m + np.log(l), P @ Vg", "return P, np.log(l), P @ Vg"),
    "row group one head short": ("hs = slice(g * hpg, (g + 1) * hpg)", "hs = slice(g * hpg, (g + 1) * hpg - 1)"),
    "row dK unscaled": ("dk[R, g, :] += scale * (dS.T @ q[t, hs, :])", "dk[R, g, :] += dS.T @ q[t, hs, :]"),
    "row dQ against V": ("dq[i, hs, :] = scale * (dS @ Kg)", "dq[i, hs, :] = scale * (dS @ Vg)"),
    "sampled-key dV from dS": ("dv[dst, g, :] += P[:, n] @ do[t, hs, :]", "dv[dst, g, :] += dS[:, n] @ do[t, hs, :]"),
    "sampled-key dK unscaled": ("dk[dst, g, :] += scale * (dS[:, n] @ q[t, hs, :])", "dk[dst, g, :] += dS[:, n] @ q[t, hs, :]"),
    "tile run one key long": ("int(pos.size)", "int(pos.size) + 1"),
    "union owner bits shifted": ("own[int(j)] = own.get(int(j), 0) | (1 << q)",
                                 "own[int(j)] = own.get(int(j), 0) | (1 << (q + 1))"),
    "union drops a group's last row": ("for q in range(group):\n            t = group * i + q",
                                       "for q in range(group - 1):\n            t = group * i + q"),
    "union keys unsorted": ("ks = sorted(own)", "ks = list(own)"),
}

# ---------------------------------------------------------------------------
# selector oracle
# ---------------------------------------------------------------------------

SELECTOR_PINS = [
    ("hand-worked example", selector_pins.test_hand_worked_example),
    ("identity keys = sort", selector_pins.test_one_head_identity_keys_reduce_to_a_sort),
    ("homogeneity, head additivity", selector_pins.test_score_homogeneity_and_head_additivity),
    ("ratio-causal candidates", selector_pins.test_ratio_causal_candidates),
    ("packed sequences, route format", selector_pins.test_packed_sequences_and_route_format),
    ("last compressed block", selector_pins.test_candidates_stop_at_the_last_compressed_block),
]

SELECTOR_MUTANTS = {
    "relu dropped": ("np.maximum(dots, 0.0).sum(axis=0)", "dots.sum(axis=0)"),
    "abs for relu": ("np.maximum(dots, 0.0).sum(axis=0)", "np.abs(dots).sum(axis=0)"),
    "score unscaled": ("S[t, :n] = scale * ", "S[t, :n] = "),
    "own block a candidate": ("np.minimum(own_blocks(T, pos, tok_base), NB - blk_base)",
                              "np.minimum(own_blocks(T, pos, tok_base) + 1, NB - blk_base)"),
    "scores ignore blk_base": ("blocks = kbar[blk_base[t]:blk_base[t] + n]", "blocks = kbar[0:n]"),
    "ties to the higher block": ("np.lexsort((c, -S[t, :n]))", "np.lexsort((-c, -S[t, :n]))"),
    "smallest scores kept": ("np.lexsort((c, -S[t, :n]))", "np.lexsort((c, S[t, :n]))"),
    "selection left unsorted": ("pick = np.sort(order[:k])", "pick = order[:k]"),
    "tail is the query alone": ("tail = list(range(int(tok_base[t] + 4 * own), int(pos[t]) + 1))",
                                "tail = [int(pos[t])]"),
    "expansion ignores tok_base": ("toks = [int(tok_base[t] + 4 * c + i)", "toks = [int(4 * c + i)"),
}

# ---------------------------------------------------------------------------
# bitmap-lookup oracle
# ---------------------------------------------------------------------------

BITMAP_PINS = [
    ("hand-worked packed example", bitmap_pins.test_hand_worked_packed_example),
    ("floor division", bitmap_pins.test_floor_division_distinguishes_truncation),
    ("round trip of block routes", bitmap_pins.test_round_trip_of_causal_block_routes),
    ("empty and out of range", bitmap_pins.test_empty_and_out_of_range),
    ("width truncation", bitmap_pins.test_width_truncation_reports_true_counts),
]

BITMAP_MUTANTS = {
    "truncating division": ("np.floor_divide(j - tok_base[t], block_size)",
                            "((j - tok_base[t]) / block_size).astype(np.int64)"),
    "hi exclusive": ("(j <= hi[t])", "(j < hi[t])"),
    "lo ignored": ("ok = (lo[t] <= j) & ", "ok = "),
    "blk_base ignored": ("b = blk_base[t] + np.floor_divide", "b = np.floor_divide"),
    "truncation keeps the largest": ("out[t, :n] = r[:n]", "out[t, :n] = r[r.size - n:]"),
    "counts report the kept width": ("counts[t] = r.size", "counts[t] = min(r.size, width)"),
}

# oracle module -> (pins, mistakes, namespaces whose bindings of its functions are swapped)
SUITES = {
    "qsa_oracle": (ATTENTION_PINS, ATTENTION_MUTANTS, [oracle]),
    "qsa_selector": (SELECTOR_PINS, SELECTOR_MUTANTS, [selector_pins]),
    "qsa_bitmap": (BITMAP_PINS, BITMAP_MUTANTS, [bitmap_pins]),
}
CASES = [(mod, name) for mod, (_, mutants, _) in SUITES.items() for name in mutants]


def _source(mod):
    return (ORACLE_DIR / f"{mod}.py").read_text()


def _install(monkeypatch, mod, source):
    copy = types.ModuleType(f"{mod}_copy")
    exec(compile(source, str(ORACLE_DIR / f"{mod}.py"), "exec"), copy.__dict__)
    swapped = 0
    for ns in SUITES[mod][2]:
        for name in dir(ns):
            fn = getattr(ns, name)
            if callable(fn) and getattr(fn, "__module__", "") == f"oracle.{mod}":
                monkeypatch.setattr(ns, name, getattr(copy, name))
                swapped += 1
    return swapped


@pytest.mark.parametrize("mod", list(SUITES))
def test_unmodified_copy_passes_every_pin(monkeypatch, mod):
    # the harness itself (a fresh copy of the source, swapped in) breaks nothing
    assert _install(monkeypatch, mod, _source(mod)) >= 3
    for _, pin in SUITES[mod][0]:
        pin()


@pytest.mark.parametrize("mod,name", CASES)
def test_planted_mistake_is_caught(monkeypatch, mod, name):
    pins_of, mutants, _ = SUITES[mod]
    old, new = mutants[name]
    source = _source(mod)
    assert old in source, f"{mod} no longer contains {old!r}"
    _install(monkeypatch, mod, source.replace(old, new))
    caught = []
    for pin_name, pin in pins_of:
        try:
            pin()
        except Exception:          # a wrong value, or shapes that no longer fit
            caught.append(pin_name)
            break
    assert caught, f"no pin fails when {mod} has the mistake {name!r}"
