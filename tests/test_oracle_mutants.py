"""Planted mistakes in the expansion, paged-gather and append oracles.

Each mutant is a plausible slip in one oracle function (it lives only in this test, on the
CPU); with it in place, at least one of the pins written for that oracle must fail.  This shows
the pins are tight enough to catch a dropped term, a wrong index or a transposed operand."""
import numpy as np
import pytest

import oracle
from oracle import append_oracle, expand_oracle, paged_oracle

import test_append_oracle as TA
import test_expand_oracle as TE
import test_paged_oracle as TP


def _fails(pins) -> bool:
    for pin in pins:
        try:
            pin()
        except (Exception, pytest.fail.Exception):  # noqa: BLE001 -- any failure means the pin caught it
            return True
    return False


# ---------------------------------------------------------------- expansion
def _expand_mutant(kind):
    rms = oracle.rms_norm

    def f(kv_c, gamma, eps, wkv_b, heads, qk_nope, v_head, batch, seq_len):
        kv = np.asarray(kv_c, dtype=np.float64)
        w = np.asarray(wkv_b, dtype=np.float64)
        if kind == "no_gain":
            x = rms(kv, None, eps)
        elif kind == "sum_not_mean":
            g = np.ones(kv.shape[1]) if gamma is None else np.asarray(gamma, dtype=np.float64)
            x = kv / np.sqrt((kv * kv).sum(axis=1, keepdims=True) + eps) * g
        elif kind == "no_eps":
            x = rms(kv, gamma, 0.0)
        else:
            x = rms(kv, gamma, eps)
        y = x @ w.T
        if kind == "head_minor":
            y = y.reshape(batch, seq_len, qk_nope + v_head, heads).transpose(0, 3, 1, 2)
        elif kind == "no_transpose":
            y = y.reshape(batch, heads, seq_len, qk_nope + v_head)
        else:
            y = y.reshape(batch, seq_len, heads, qk_nope + v_head).transpose(0, 2, 1, 3)
        k, v = y[..., :qk_nope], y[..., qk_nope:]
        if kind == "split_swapped":
            k, v = y[..., v_head:], y[..., :v_head]
        return np.ascontiguousarray(k), np.ascontiguousarray(v)
    return f


EXPAND_PINS = [TE.test_hand_example, TE.test_layout_head_before_token_and_split, TE.test_scale_invariance_without_eps,
               TE.test_linear_in_the_weight,
               lambda: TE.test_expanded_keys_and_values_reproduce_the_attention_oracle([1, 1], [7, 40]),
               lambda: TE.test_expanded_keys_and_values_reproduce_the_attention_oracle([3], [20])]


@pytest.mark.parametrize("kind", ["no_gain", "sum_not_mean", "no_eps", "head_minor", "no_transpose",
                                  "split_swapped"])
def test_expand_pins_catch(monkeypatch, kind):
    assert not _fails(EXPAND_PINS)          # the real oracle passes them
    m = _expand_mutant(kind)
    monkeypatch.setattr(oracle, "expand_kv", m)
    monkeypatch.setattr(expand_oracle, "expand_kv", m)
    assert _fails(EXPAND_PINS), kind


# ---------------------------------------------------------------- paged gather
def _gather_mutant(kind):
    def f(kv_cache, pe_cache, block_table, seqlens_k, page_size):
        kv_cache, pe_cache, table = np.asarray(kv_cache), np.asarray(pe_cache), np.asarray(block_table)
        num_pages = kv_cache.shape[0] // page_size
        kvs, pes, lens, first = [], [], [], 0
        for b, t in enumerate(seqlens_k):
            t = int(t)
            idx = []
            for j in range(t):
                page = int(table[b, j // page_size])
                if kind != "no_bounds" and not 0 <= page < num_pages:
                    raise ValueError("outside")
                if kind == "div_not_mod":
                    row = page * page_size + j // page_size
                elif kind == "no_page_scale":
                    row = page + j % page_size
                elif kind == "packed":
                    row = first + j
                else:
                    row = page * page_size + j % page_size
                idx.append(min(max(row, 0), kv_cache.shape[0] - 1))
            first += t
            kvs.append(kv_cache[idx])
            pes.append(pe_cache[idx])
            lens.append(t)
        cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
        return np.concatenate(kvs), np.concatenate(pes), cu
    return f


PAGED_PINS = [TP.test_gather_hand_example, TP.test_gather_rejects_an_entry_outside_the_cache_that_holds_keys,
              TP.test_gather_identity_table_is_the_packed_cache,
              lambda: TP.test_gather_inverts_a_token_by_token_scatter(3),
              lambda: TP.test_paged_attention_equals_packed_attention(2)]


@pytest.mark.parametrize("kind", ["div_not_mod", "no_page_scale", "packed", "no_bounds"])
def test_paged_pins_catch(monkeypatch, kind):
    assert not _fails(PAGED_PINS)
    m = _gather_mutant(kind)
    monkeypatch.setattr(oracle, "gather_paged", m)
    monkeypatch.setattr(paged_oracle, "gather_paged", m)
    assert _fails(PAGED_PINS), kind


# ---------------------------------------------------------------- append
def _rope_mutant(kind):
    def f(x, positions, base):
        x = np.asarray(x, dtype=np.float64)
        r = x.shape[-1]
        out = np.empty_like(x)
        pos = np.asarray(positions, dtype=np.float64) + (1.0 if kind == "position_plus_one" else 0.0)
        for i in range(r // 2):
            theta = pos * base ** (-2.0 * i / r) * (-1.0 if kind == "negative_angle" else 1.0)
            c, s = np.cos(theta), np.sin(theta)
            if kind == "rotate_half":
                ia, ib = i, i + r // 2
            else:
                ia, ib = 2 * i, 2 * i + 1
            a, b = x[..., ia], x[..., ib]
            out[..., ia] = a * c - b * s
            out[..., ib] = a * s + b * c
        return out
    return f


def _rms_sum(x, gamma, eps):
    x = np.asarray(x, dtype=np.float64)
    g = np.ones(x.shape[-1]) if gamma is None else np.asarray(gamma, dtype=np.float64)
    return x / np.sqrt((x * x).sum(axis=-1, keepdims=True) + eps) * g


APPEND_PINS = [TA.test_rms_norm_closed_forms, TA.test_rms_norm_is_scale_invariant,
               TA.test_rope_closed_form_and_invariants, TA.test_append_writes_only_its_slots,
               TA.test_append_agrees_with_the_workload_generator]


@pytest.mark.parametrize("kind", ["position_plus_one", "negative_angle", "rotate_half", "rms_sum"])
def test_append_pins_catch(monkeypatch, kind):
    assert not _fails(APPEND_PINS)
    if kind == "rms_sum":
        monkeypatch.setattr(oracle, "rms_norm", _rms_sum)
        monkeypatch.setattr(append_oracle, "rms_norm", _rms_sum)
    else:
        m = _rope_mutant(kind)
        monkeypatch.setattr(oracle, "rope_interleaved", m)
        monkeypatch.setattr(append_oracle, "rope_interleaved", m)
    assert _fails(APPEND_PINS), kind


def test_append_slot_off_by_one_is_caught(monkeypatch):
    orig = append_oracle.append_latent

    def off_by_one(kv_new, k_pe_new, gamma, eps, positions, slots, kv_cache, pe_cache, base=10000.0):
        return orig(kv_new, k_pe_new, gamma, eps, positions, np.asarray(slots) + 1, kv_cache, pe_cache, base)
    monkeypatch.setattr(oracle, "append_latent", off_by_one)
    assert _fails(APPEND_PINS)


# ---------------------------------------------------------------- token-granular selection
import test_sparse_oracle as TS  # noqa: E402
from oracle import sparse_oracle  # noqa: E402


def _select_mutant(kind):
    def f(kv_cache, pe_cache, indices, counts):
        kv_cache, pe_cache, idx = np.asarray(kv_cache), np.asarray(pe_cache), np.asarray(indices)
        rows = kv_cache.shape[0]
        kvs, pes, lens = [], [], []
        for b, n in enumerate(counts):
            n = int(n)
            if kind == "count_minus_one":
                n = max(0, n - 1)
            sel = idx[b, :n].astype(np.int64)
            if kind == "plus_one":
                sel = sel + 1
            elif kind == "unique":
                sel = np.unique(sel)
            if kind == "no_bounds":
                sel = np.clip(sel, 0, rows - 1)
            elif np.any((sel < 0) | (sel >= rows)):
                raise ValueError("outside")
            kvs.append(kv_cache[sel])
            pes.append(pe_cache[sel])
            lens.append(len(sel))
        cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
        return np.concatenate(kvs), np.concatenate(pes), cu
    return f


SPARSE_PINS = [TS.test_gather_selected_hand_example, TS.test_selected_row_outside_the_cache_is_an_error,
               TS.test_selecting_every_token_in_any_order_is_dense_decode,
               TS.test_one_selected_token_returns_its_projected_value,
               TS.test_selection_is_attention_over_those_tokens_only]


@pytest.mark.parametrize("kind", ["plus_one", "count_minus_one", "unique", "no_bounds"])
def test_sparse_pins_catch(monkeypatch, kind):
    assert not _fails(SPARSE_PINS)
    m = _select_mutant(kind)
    monkeypatch.setattr(oracle, "gather_selected", m)
    monkeypatch.setattr(sparse_oracle, "gather_selected", m)
    assert _fails(SPARSE_PINS), kind
