"""The benchmark's algorithmic byte counts (the roofline's numerator) on a
hand-worked tree: 64 or 61 tokens, chunk 4, depth 2, d = 8, R = 2, one KV
head with two query heads, bf16 rows."""
import importlib.util
import os
import types

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
_spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
bench = importlib.util.module_from_spec(_spec)
_spec.loader.exec_module(bench)

W = types.SimpleNamespace(c=4, D=2, d=8, R=2, group=2, h_kv=1, h_q=2, kv_dtype="bf16")
NODE = 2 * (8 + 1) * 4  # g row and plane offset of each of R planes, fp32


def _trace(kept_top, kept_leaves):
    """trace_ids[l - 1, h] = ids kept at level l by head h."""
    cap = 8
    ids = np.full((2, 2, cap), -1, dtype=np.int32)
    cnt = np.zeros((2, 2), dtype=np.int32)
    for h in range(2):
        for lvl, kept in ((1, kept_top[h]), (0, kept_leaves[h])):
            ids[lvl, h, :len(kept)] = kept
            cnt[lvl, h] = len(kept)
    return ids, cnt


def test_decode_bytes_union_of_heads_and_sink():
    # head 0 keeps top nodes {0, 2} then leaves {1, 9}; head 1 keeps {2}, {9, 10}
    ids, cnt = _trace([[0, 2], [2]], [[1, 9], [9, 10]])
    route, attn_qo, slots, per_level = bench.step_bytes(W, ids, cnt, 64)
    # level 2: all 4 top nodes; level 1: the children of the union {0, 2}
    assert slots == 4 + 8 and per_level[2] == 4 and per_level[1] == 8
    assert route == 12 * NODE
    # union leaves {1, 9, 10}: 12 tokens, plus the sink (leaf 0 is not kept)
    rows = 13 * 2 * 8 * 2
    assert attn_qo == rows + 2 * 8 * 8


def test_decode_bytes_ragged_tail_and_kept_sink_leaf():
    # 61 tokens: top node 3 covers tokens 48..60, leaf 15 holds token 60 only
    ids, cnt = _trace([[0, 3], [3]], [[0, 15], [15]])
    route, attn_qo, slots, _ = bench.step_bytes(W, ids, cnt, 61)
    assert route == (4 + 8) * NODE and slots == 12
    # leaves {0, 15}: 4 + 1 tokens; token 0 is in leaf 0, so no extra sink row
    assert attn_qo == 5 * 2 * 8 * 2 + 2 * 8 * 8


def test_append_bytes():
    # the 62nd token: its k and v rows, the 2 tokens of leaf 15, the D = 2
    # rewritten nodes (g, m, b of R planes), and the 4 children of node 3
    b = bench.append_bytes(W, 62)
    assert b == 2 * 8 * 2 + 2 * 8 * 2 + 2 * (2 * (8 + 2) * 4) + 4 * NODE
