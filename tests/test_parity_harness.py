"""The routing replay of the parity harness accepts the oracle's own routing
and rejects a wrong keep/drop decision even on a level of tiny probabilities
(CPU only: the 'GPU trace' here is written by the test).

A frontier of 150,000 single-token leaves with near-uniform scores puts every
probability near 7e-6, below an absolute 1e-5 band; the harness's band is
relative to the probability at the cut, so a node far from the cut still
counts as a real difference there.
"""
import numpy as np
import pytest

import oracle
from parity import replay_head


def _case():
    rng = np.random.default_rng(42)
    N, d = 150_000, 8
    K = (rng.standard_normal((N, d)) * 0.3).astype(np.float32)
    ref = rng.standard_normal((1, d))
    tree = oracle.build(K, N, ref, 1, 1)
    q = rng.standard_normal(d) * 0.2
    return tree, ref, q, N


def _trace(kept_ids, N):
    ids = np.zeros((1, 1, N), dtype=np.int32)
    cnt = np.zeros((1, 1), dtype=np.int32)
    k = np.sort(np.asarray(kept_ids, dtype=np.int64))
    ids[0, 0, :len(k)] = k
    cnt[0, 0] = len(k)
    return ids, cnt


def test_replay_accepts_oracle_routing_and_rejects_a_far_node():
    tree, ref, q, N = _case()
    p = 0.75
    kept, _ = oracle.route(tree, ref, q, p)
    front = np.arange(N)
    est = tree.estimates(1, front, ref, q)
    k_o, prob, cb, rank = oracle.topp(est, front, p)
    assert prob.max() < 1e-5, "the level must consist of tiny probabilities"
    ids, cnt = _trace(kept[0], N)
    amb, vis, leaves = replay_head(tree, ref, q, p, ids, cnt, 0, N, 1, 1)
    assert amb == 0 and vis == N and np.array_equal(leaves, kept[0])
    # drop the most probable kept node and keep the first dropped one instead:
    # both probabilities are below 1e-5, but the top one is far from the cut
    order = np.argsort(rank)
    top = int(front[order[0]])
    first_out = int(front[order[int(k_o.sum())]])
    wrong = [x for x in kept[0].tolist() if x != top] + [first_out]
    ids, cnt = _trace(wrong, N)
    with pytest.raises(AssertionError):
        replay_head(tree, ref, q, p, ids, cnt, 0, N, 1, 1)


def test_replay_counts_a_boundary_swap_as_ambiguous():
    tree, ref, q, N = _case()
    p = 0.75
    kept, _ = oracle.route(tree, ref, q, p)
    front = np.arange(N)
    est = tree.estimates(1, front, ref, q)
    k_o, prob, cb, rank = oracle.topp(est, front, p)
    order = np.argsort(rank)
    nk = int(k_o.sum())
    last_in, first_out = int(front[order[nk - 1]]), int(front[order[nk]])
    swapped = [x for x in kept[0].tolist() if x != last_in] + [first_out]
    ids, cnt = _trace(swapped, N)
    amb, _, _ = replay_head(tree, ref, q, p, ids, cnt, 0, N, 1, 1)
    assert amb == 2
