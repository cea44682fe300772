"""Pins of the greedy-argmax oracle: hand cases from the tie rule, agreement with numpy.argmax
(documented to return the first occurrence of the maximum) by brute force over small vectors
with forced ties, and the LM-head composition against the GEMV oracle."""
import itertools
import json
import os

import numpy as np

import synth
from oracle import argmax as oa
from oracle import qgemv as oq


def test_hand_cases(golden_dir):
    d = json.load(open(os.path.join(golden_dir, "argmax_hand.json")))
    for c in d["cases"]:
        v = np.array(c["logits"], dtype=np.float32)
        assert oa.argmax_lower(v) == c["token"], c["why"]


def test_matches_numpy_first_occurrence_exhaustively():
    """Every vector of length 1..5 over a value set with repeats and signed zeros."""
    values = [-1.0, -0.0, 0.0, 2.0, 2.0000002, -7.5]
    for n in range(1, 6):
        for combo in itertools.product(values, repeat=n):
            v = np.array(combo, dtype=np.float32)
            assert oa.argmax_lower(v) == int(np.argmax(v)), combo


def test_large_random_vectors_with_planted_ties():
    rng = np.random.default_rng(7)
    for _ in range(20):
        v = rng.standard_normal(32000).astype(np.float32)
        m = v.max()
        pos = np.sort(rng.choice(32000, size=3, replace=False))
        v[pos] = m + 1.0                      # three equal maxima: the first one wins
        assert oa.argmax_lower(v) == pos[0] == int(np.argmax(v))


def test_lm_head_greedy_is_argmax_of_the_head():
    rows, cols = 96, 64
    W = synth.q8_0_matrix(rows, cols, 0, "argmax/head").numpy()
    x = synth.normal_f32(0, 3, cols).numpy().astype(np.float64)
    t, m = oa.lm_head_greedy(oq.FMT_Q8_0, W, x, rows, cols)
    y = oq.qgemv(oq.FMT_Q8_0, W, x, rows, cols)
    assert t == int(np.argmax(y)) and m == y[t]
    # a unit vector x = e_j picks the row with the largest d * q_j
    d, q = oq.q8_0_decode(W, rows, cols)
    e = np.zeros(cols)
    e[5] = 1.0
    t, _ = oa.lm_head_greedy(oq.FMT_Q8_0, W, e, rows, cols)
    col = d[:, 0] * q[:, 0, 5]
    assert t == int(np.argmax(col))
