"""Fixtures printed on the pages (tests/golden/, each with its source)."""
import json
import os

import numpy as np

from oracle import oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def test_indexer_shape_reading_matches_printed_param_count():
    """The indexer parameters printed on the ablation card (difference of the two
    counts) are exactly those of the shape the oracle computes: per layer a query
    projection hidden -> H_I*D_I, ONE key projection hidden -> D_I shared by all
    indexer heads, and a weight projection hidden -> H_I, without biases."""
    g = _load("ablation_card_param_count.json")
    diff = g["params_with_indexers"] - g["params_without_indexers"]
    h, H_I, D_I = g["hidden"], g["indexer_heads"], g["indexer_head_dim"]
    per_layer_shared_key = h * H_I * D_I + h * D_I + h * H_I
    assert g["layers"] * per_layer_shared_key == diff
    # a key per indexer head would not fit the printed count
    per_layer_per_head_key = h * H_I * D_I + h * H_I * D_I + h * H_I
    assert g["layers"] * per_layer_per_head_key != diff
    # and the oracle takes exactly that layout: k_idx [S, D_I], w [T, H_I]
    T = 4
    q = np.ones((T, H_I, D_I), np.float32)
    k = np.ones((T, D_I), np.float32)
    w = np.ones((T, H_I), np.float32)
    sc = O.indexer_scores_prefill(q, k, w)
    assert sc[T - 1, 0] == H_I * D_I


def test_printed_pattern_is_a_valid_stack():
    g = _load("index_topk_pattern_61.json")
    p = g["pattern"]
    assert len(p) == g["num_layers"] and p[0] == "F" and set(p) <= {"F", "S"}
