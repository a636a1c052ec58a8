"""Pins for the oracle's SpenseGPT+ scorer and dense-set selection (CPU only).

Fixed independently of the oracle's code:
- a hand-worked case with every term written out;
- the score of an intermediate index moves with it when the intermediate
  indices are permuted (rows of gate/up, columns of down, entries of h_mid);
- each projection's term is homogeneous: scaling h_in by c^2 scales the gate
  and up terms by c, scaling h_mid by c^2 scales the down term by c;
- the terms add: the score with gate and up equals the sum of the scores with
  each alone minus the down-only score;
- the selection is the top-Kd by score with ties to the lower index, listed in
  ascending order (equivalently numpy's lexsort on (index, -score)).
"""
import numpy as np
import pytest

import oracle

E4 = {1.0: 0x38, 2.0: 0x40, 0.5: 0x30, -1.0: 0xB8, 1.5: 0x3C, -2.0: 0xC0, 0.0: 0x00, 4.0: 0x48}


def codes(vals):
    return np.vectorize(lambda v: E4[v])(np.array(vals, np.float64)).astype(np.uint8)


def test_hand_worked_case():
    # I = 2 intermediate indices, H = 2 hidden channels.
    gate = codes([[1.0, -1.0], [2.0, 0.0]])      # rows t
    s_gate = np.array([1.0, 0.5], np.float32)
    up = codes([[0.5, 1.5], [-2.0, 4.0]])
    s_up = np.array([2.0, 1.0], np.float32)
    down = codes([[1.0, 2.0], [0.5, -1.0]])      # rows i (hidden), columns t
    s_down = np.array([1.0, 2.0], np.float32)
    h_in = np.array([4.0, 9.0], np.float32)      # sqrt: 2, 3
    h_mid = np.array([1.0, 16.0], np.float32)    # sqrt: 1, 4
    sc = oracle.score_glu(down, s_down, h_in, h_mid, gate=gate, s_gate=s_gate, up=up, s_up=s_up)
    # t = 0: gate |1*1|*2 + |1*-1|*3 = 5; up |2*.5|*2 + |2*1.5|*3 = 11;
    #        down sqrt(1) * (|1*1| + |2*.5|) = 2          -> 18
    # t = 1: gate |.5*2|*2 + 0 = 2; up |1*-2|*2 + |1*4|*3 = 16;
    #        down sqrt(16) * (|1*2| + |2*-1|) = 16        -> 34
    assert sc.tolist() == [18.0, 34.0]


def random_mlp(seed, I=40, H=24):
    g = np.random.default_rng(seed)
    finite = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    pick = lambda shape: g.choice(finite, size=shape)
    return dict(gate=pick((I, H)), s_gate=g.uniform(0.1, 2, I).astype(np.float32),
                up=pick((I, H)), s_up=g.uniform(0.1, 2, I).astype(np.float32),
                down=pick((H, I)), s_down=g.uniform(0.1, 2, H).astype(np.float32),
                h_in=g.uniform(0, 5, H).astype(np.float32), h_mid=g.uniform(0, 5, I).astype(np.float32))


def score(m, **over):
    d = dict(m, **over)
    return oracle.score_glu(d["down"], d["s_down"], d["h_in"], d["h_mid"], gate=d["gate"], s_gate=d["s_gate"],
                            up=d["up"], s_up=d["s_up"])


def test_scores_follow_a_permutation_of_the_intermediate_indices():
    m = random_mlp(1)
    p = np.random.default_rng(2).permutation(m["h_mid"].shape[0])
    q = dict(m, gate=m["gate"][p], s_gate=m["s_gate"][p], up=m["up"][p], s_up=m["s_up"][p],
             down=np.ascontiguousarray(m["down"][:, p]), h_mid=m["h_mid"][p])
    assert np.allclose(score(q), score(m)[p], rtol=1e-12, atol=0)


def test_each_term_is_homogeneous_in_its_hessian():
    m = random_mlp(3)
    base_in = score(m, h_mid=np.zeros_like(m["h_mid"]))      # gate + up terms only
    base_mid = score(m, h_in=np.zeros_like(m["h_in"]))       # down term only
    assert np.allclose(base_in + base_mid, score(m), rtol=1e-12)
    # (9 h and 4 h are rounded to fp32 before the square root: rtol 1e-6)
    assert np.allclose(score(m, h_in=m["h_in"] * 9, h_mid=np.zeros_like(m["h_mid"])), 3 * base_in, rtol=1e-6)
    assert np.allclose(score(m, h_mid=m["h_mid"] * 4, h_in=np.zeros_like(m["h_in"])), 2 * base_mid, rtol=1e-6)


def test_terms_add():
    m = random_mlp(4)
    both = score(m)
    only_gate = score(m, up=None, s_up=None)
    only_up = score(m, gate=None, s_gate=None)
    none = score(m, gate=None, s_gate=None, up=None, s_up=None)
    assert np.allclose(both, only_gate + only_up - none, rtol=1e-12)


@pytest.mark.parametrize("seed,I,Kd", [(0, 50, 12), (1, 64, 0), (2, 64, 64), (3, 500, 125)])
def test_selection_is_the_top_kd_with_ties_to_the_lower_index(seed, I, Kd):
    g = np.random.default_rng(seed)
    sc = g.integers(0, 10, size=I).astype(np.float64)   # many ties
    got = oracle.select_top(sc, Kd)
    order = np.lexsort((np.arange(I), -sc))              # by score desc, then index asc
    assert np.array_equal(got, np.sort(order[:Kd]).astype(np.int32))
    assert np.all(np.diff(got) > 0)


def test_rejects_bad_arguments():
    with pytest.raises(oracle.OracleError):
        oracle.select_top(np.zeros(4), 5)
