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
import oracle.pool
import oracle.select
import oracle.tiling
from tests import test_oracle_attention as ta
from tests import test_oracle_attention_bwd as tb
from tests import test_oracle_bsa_ratio as tr
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
])
def test_planted_mistake_is_caught(monkeypatch, patch, pin):
    mod, name, fn = patch
    monkeypatch.setattr(mod, name, fn)
    with pytest.raises(AssertionError):
        pin()
