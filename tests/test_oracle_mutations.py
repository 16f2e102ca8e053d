"""Planted mistakes in the oracle (on the CPU) must each fail one of its pins.

Every case monkeypatches one plausible slip into an oracle function — a swapped loop, a wrong
divisor, a reversed tie-break, a dropped mask, an off-by-one at the mass cut, an arg-min for an
arg-max — and runs the pin that should catch it.
"""
import math

import numpy as np
import pytest

import oracle.attention
import oracle.attention_bwd
import oracle.bsa
import oracle.packed
import oracle.pool
import oracle.select
import oracle.tiling
from tests import test_oracle_attention as ta
from tests import test_oracle_attention_bwd as tb
from tests import test_oracle_bsa_ratio as tr
from tests import test_oracle_packed as tk
from tests import test_oracle_pool_select as tp
from tests import test_oracle_tiling as tt


def _swapped_partition(T, H, W, tile=(4, 4, 4)):
    order = []
    for a in range(math.ceil(T / 4)):
        for c in range(math.ceil(W / 4)):  # w-tile before h-tile: wrong
            for b in range(math.ceil(H / 4)):
                for t in range(4 * a, min(4 * a + 4, T)):
                    for h in range(4 * b, min(4 * b + 4, H)):
                        for w in range(4 * c, min(4 * c + 4, W)):
                            order.append((t * H + h) * W + w)
    return np.asarray(order)


def _pool_by_64(y, vc):
    B, Lp, nh, D = y.shape
    return np.stack([y[:, 64 * i:64 * i + 64].sum(axis=1) / 64.0 for i in range(Lp // 64)],
                    axis=2).transpose(0, 2, 1, 3)


def _topk_high_tie(row, k):
    idx = np.arange(row.shape[0])
    return np.sort(np.lexsort((-idx, -row))[:min(k, row.shape[0])])


def _mass_no_crossing(row, scale, tau, min_k):
    p = oracle.select.softmax_row(scale * row)
    order = np.lexsort((np.arange(len(row)), -row))
    csum = np.cumsum(p[order])
    m = max(int(np.sum(csum < tau)), min(min_k, len(row)), 1)
    return np.sort(order[:m])


def _keys_all_slots(sets_i, vc, E=64):
    parts = [E * int(j) + np.arange(E) for j in sets_i]
    return np.concatenate(parts) if parts else np.zeros(0, dtype=np.int64)


def _prune_argmin(rows, thresh):
    keep, src, cm = _orig_prune(rows, thresh)
    kept = np.nonzero(keep)[0]
    for i in range(len(src)):
        if not keep[i]:
            c = [float(np.dot(rows[i], rows[j]) / np.linalg.norm(rows[i]) / np.linalg.norm(rows[j]))
                 for j in kept]
            src[i] = kept[int(np.argmin(c))]
    return keep, src, cm


_orig_prune = oracle.bsa.prune_block


def _ratio_keep_most_similar(rows, ratio):
    rows = rows.astype(np.float64)
    n = rows.shape[0]
    mu = rows.sum(axis=0) / n
    cmean = np.array([oracle.bsa._cos(rows[i], mu) for i in range(n)])
    order = sorted(range(n), key=lambda i: (-cmean[i], i))  # most similar first: wrong
    keep = np.zeros(n, dtype=bool)
    keep[order[:oracle.bsa.keep_size_for_ratio(ratio, n)]] = True
    return keep, oracle.bsa._sources(rows, keep), cmean


def _bwd_no_delta(q_rows, k_rows, v_rows, do_rows, scale):
    q, k, v, do = (np.asarray(a, dtype=np.float64) for a in (q_rows, k_rows, v_rows, do_rows))
    logits = scale * (q @ k.T)
    e = np.exp(logits - logits.max(axis=1, keepdims=True))
    p = e / e.sum(axis=1, keepdims=True)
    ds = p * (do @ v.T)  # the softmax Jacobian's "- dO . o" term dropped: wrong
    return scale * (ds @ k), scale * (ds.T @ q), p.T @ do


def _bwd_dk_unscaled(q_rows, k_rows, v_rows, do_rows, scale):
    dq, dk, dv = _orig_rows_bwd(q_rows, k_rows, v_rows, do_rows, scale)
    return dq, dk / scale, dv  # key gradient without the softmax scale: wrong


_orig_rows_bwd = oracle.attention_bwd.attend_rows_bwd


def _bwd_pruned_keep_own_grad(qt, kt, vt, vc, sets, scale, do, keep=None, src=None):
    B, Lp, nh, D = qt.shape
    dq, dk, dv = (np.zeros((B, Lp, nh, D)) for _ in range(3))
    for b in range(B):
        for h in range(nh):
            for i in range(Lp // 64):
                rows_k = oracle.attention._key_rows(sets[b][h][i], vc)
                kk = np.nonzero(keep[b, h, i][:int(vc[i])])[0]
                rows_q = 64 * i + kk
                g_out = np.asarray(do)[b, rows_q, h]  # pruned rows' gradients dropped: wrong
                gq, gk, gv = _orig_rows_bwd(qt[b, rows_q, h], kt[b, rows_k, h], vt[b, rows_k, h],
                                            g_out, scale)
                dq[b, rows_q, h] = gq
                dk[b, rows_k, h] += gk
                dv[b, rows_k, h] += gv
    return dq, dk, dv


_orig_packed_geometry = oracle.packed.packed_geometry


def _geometry_partial_run_first(segs, tile_shape):
    """Dense segments cut with their partial run first instead of last."""
    geo = _orig_packed_geometry(segs, tile_shape)
    E = geo["E"]
    sr, vc = geo["slot_row"].copy(), geo["vc"].copy()
    t, off = 0, 0
    for s in segs:
        if isinstance(s, int):
            n = -(-s // E)
            sizes = [s - E * (n - 1)] + [E] * (n - 1)
            for sz in sizes:
                sr[E * t:E * (t + 1)] = -1
                sr[E * t:E * t + sz] = np.arange(off, off + sz)
                vc[t] = sz
                off += sz
                t += 1
        else:
            off += s[0] * s[1] * s[2]
    return dict(geo, slot_row=sr, vc=vc)


def _geometry_regions_in_64_shape(segs, tile_shape):
    """Every region tiled with the 64-token shape whatever the tile size."""
    E = int(np.prod(tile_shape))
    geo = _orig_packed_geometry(segs, (4, 4, 4))
    if E == 64:
        return geo
    n = len(geo["vc"])
    sr = np.full(n * E, -1, dtype=np.int64)
    for t in range(n):
        sr[E * t:E * t + 64] = geo["slot_row"][64 * t:64 * (t + 1)]
    return dict(geo, slot_row=sr, E=E)


def _select_ceil(S, geo, keep_rates, exempt=True, dense=False):
    """Per-region keep count rounded up instead of truncated."""
    nT = S.shape[-1]

    def top(row, lo, hi, rate):
        order = sorted(range(lo, hi), key=lambda j: (-row[j], j))
        return order[:min(hi - lo, math.ceil(rate * (hi - lo)))]

    def row_sets(row, i):
        if dense or (exempt and i < geo["n_prefix"]):
            return np.arange(nT)
        if not exempt:
            return np.asarray(sorted(top(row, 0, nT, keep_rates[-1])))
        kept = list(range(geo["n_prefix"]))
        for (lo, hi), r in zip(geo["spans"], keep_rates):
            kept += top(row, lo, hi, r)
        return np.asarray(sorted(kept))

    return [[[row_sets(S[b, h, i], i) for i in range(nT)] for h in range(S.shape[1])]
            for b in range(S.shape[0])]


_orig_select = oracle.packed.select


def _select_prefix_queries_not_exempt(S, geo, keep_rates, exempt=True, dense=False):
    """Prefix query tiles select like video query tiles."""
    return _orig_select(S, dict(geo, n_prefix=0, spans=[(0, geo["n_prefix"])] + list(geo["spans"])),
                        [1.0] + list(keep_rates), exempt, dense)


def _select_rates_reversed(S, geo, keep_rates, exempt=True, dense=False):
    return _orig_select(S, geo, list(keep_rates)[::-1], exempt, dense)


def _rates_generated_first(n_regions, sparsity, ref_keep_rate, exempt):
    r = _orig_rates(n_regions, sparsity, ref_keep_rate, exempt)
    return r[-1:] + r[:-1]


_orig_rates = oracle.packed.span_keep_rates


def _scatter_pads_one(x, geo):
    y = np.ones((x.shape[0], geo["slot_row"].shape[0]) + x.shape[2:], dtype=x.dtype)
    for slot, r in enumerate(geo["slot_row"]):
        if r >= 0:
            y[:, slot] = x[:, r]
    return y


@pytest.mark.parametrize("patch,pin", [
    ((oracle.tiling, "tile_partition_indices", _swapped_partition),
     lambda: tt.test_partition_matches_sort_by_tile_key((5, 9, 9))),
    ((oracle.pool, "tile_mean_pool", _pool_by_64),
     lambda: tp.test_pool_matches_per_token_accumulation((3, 5, 7))),
    ((oracle.select, "select_topk_row", _topk_high_tie), tp.test_topk_ties_go_to_lower_index),
    ((oracle.select, "select_mass_row", _mass_no_crossing), tp.test_mass_bruteforce_minimal_subset),
    ((oracle.attention, "_key_rows", _keys_all_slots),
     lambda: ta.test_full_selection_is_dense_attention((5, 6, 7))),
    ((oracle.bsa, "prune_block", _prune_argmin), ta.test_prune_cosine_against_torch),
    ((oracle.bsa, "prune_block_ratio", _ratio_keep_most_similar),
     tr.test_fan_keeps_the_widest_angles_and_copies_the_nearest_kept_row),
    ((oracle.bsa, "keep_size_for_ratio", lambda ratio, n=64: max(1, int(round(ratio * n)))),
     lambda: tr.test_keep_size(0.2, 12)),
    ((oracle.attention_bwd, "attend_rows_bwd", _bwd_no_delta), tb.test_softmax_identities),
    ((oracle.attention_bwd, "attend_rows_bwd", _bwd_dk_unscaled), tb.test_finite_differences_tiny),
    ((oracle.attention_bwd, "block_sparse_attention_bwd", _bwd_pruned_keep_own_grad),
     tb.test_pruned_rows_route_their_gradient_to_the_source_row),
    ((oracle.packed, "packed_geometry", _geometry_partial_run_first),
     tk.test_geometry_mixed_tile64_fixture),
    ((oracle.packed, "packed_geometry", _geometry_regions_in_64_shape),
     tk.test_geometry_tile128_fixture),
    ((oracle.packed, "select", _select_ceil), tk.test_select_hand_worked_row),
    ((oracle.packed, "select", _select_prefix_queries_not_exempt), tk.test_select_hand_worked_row),
    ((oracle.packed, "select", _select_rates_reversed), tk.test_select_hand_worked_row),
    ((oracle.packed, "span_keep_rates", _rates_generated_first),
     tk.test_token_segments_and_keep_rates_contract),
    ((oracle.packed, "scatter", _scatter_pads_one), tk.test_scatter_gather_round_trip_and_zero_pads),
])
def test_planted_mistake_is_caught(monkeypatch, patch, pin):
    mod, name, fn = patch
    monkeypatch.setattr(mod, name, fn)
    with pytest.raises(AssertionError):
        pin()
