"""Pins of the oracle's bidirectional attention against closed forms and invariants
(not against a retyped formula):

  one key          the output is that key's value row, exactly
  q = 0            every weight is 1/Lk: the output is the mean of V
  two keys         the weight of key 0 is the logistic of (q.k0 - q.k1) / sqrt(dh): fixes
                   the 1/sqrt(dh) scale and which operand is the query
  hard attention   one logit far above the rest: the output is that key's value
  permutations     permuting key/value rows together changes nothing (no mask, no
                   position); permuting query rows permutes the output rows
  shift            adding one vector to every key adds the same amount to every logit
  linearity        linear in V
  heads            with H = 4 and Hkv = 2, heads 0-1 use key/value head 0, heads 2-3 head 1
  query subset     the requested rows of a full-canvas result equal the result for those
                   queries alone (the last layer's case)
"""
import numpy as np

import oracle


def _rand(shape, seed, s=1.0):
    return (np.random.default_rng(seed).standard_normal(shape) * s).astype(np.float32)


def test_one_key_returns_its_value():
    q, k, v = _rand((3, 2, 16), 1), _rand((1, 2, 16), 2), _rand((1, 2, 16), 3)
    o = oracle.attention(q, k, v)
    assert np.array_equal(o, np.broadcast_to(v.astype(np.float64), o.shape))


def test_zero_query_gives_mean_of_values():
    k, v = _rand((9, 1, 8), 4), _rand((9, 1, 8), 5)
    o = oracle.attention(np.zeros((2, 1, 8), np.float32), k, v)
    assert np.allclose(o, v.astype(np.float64).mean(0, keepdims=True), rtol=0, atol=1e-15)


def test_two_keys_logistic_weight_and_scale():
    dh = 64
    q = np.zeros((1, 1, dh), np.float32)
    k = np.zeros((2, 1, dh), np.float32)
    q[0, 0, 0], k[0, 0, 0], k[1, 0, 0] = 2.0, 3.0, -1.0       # logits 6/8 and -2/8
    v = np.zeros((2, 1, dh), np.float32)
    v[0, 0, 1], v[1, 0, 2] = 1.0, 1.0
    o = oracle.attention(q, k, v)[0, 0]
    w0 = 1.0 / (1.0 + np.exp(-(6.0 - (-2.0)) / 8.0))          # logistic(1)
    assert abs(w0 - 0.7310585786300049) < 1e-15               # the textbook value
    assert abs(o[1] - w0) < 1e-15 and abs(o[2] - (1 - w0)) < 1e-15
    # swapping the roles of q and k changes the answer: here q . k is symmetric in
    # value, so use a query that differs per key only through k
    o2 = oracle.attention(k[:1], np.concatenate([q, -q]), v)[0, 0]
    assert not np.allclose(o2, o)


def test_hard_attention():
    k = _rand((6, 1, 8), 6)
    v = _rand((6, 1, 8), 7)
    q = (k[3:4] * 400.0).astype(np.float32)                 # key 3 dominates by far
    o = oracle.attention(q, k, v)
    assert np.allclose(o[0, 0], v[3, 0], rtol=0, atol=1e-9)


def test_key_value_permutation_and_query_permutation():
    q, k, v = _rand((5, 2, 16), 8), _rand((11, 2, 16), 9), _rand((11, 2, 16), 10)
    o = oracle.attention(q, k, v)
    p = np.random.default_rng(11).permutation(11)
    assert np.allclose(oracle.attention(q, k[p], v[p]), o, rtol=0, atol=1e-14)
    pq = np.random.default_rng(12).permutation(5)
    assert np.array_equal(oracle.attention(q[pq], k, v), o[pq])


def test_key_shift_invariance():
    # quarter-integers, so k + c and every dot product are exact
    rng = np.random.default_rng(13)
    q = (rng.integers(-8, 9, (4, 1, 8)) / 4).astype(np.float32)
    k = (rng.integers(-8, 9, (10, 1, 8)) / 4).astype(np.float32)
    c = (rng.integers(-8, 9, (1, 1, 8)) / 4).astype(np.float32)
    v = _rand((10, 1, 8), 15)
    o = oracle.attention(q, k, v)
    assert np.allclose(oracle.attention(q, k + c, v), o, rtol=0, atol=1e-12)


def test_linear_in_values():
    q, k = _rand((3, 2, 8), 17), _rand((7, 2, 8), 18)
    v1, v2 = _rand((7, 2, 8), 19), _rand((7, 2, 8), 20)
    o = oracle.attention(q, k, (v1 + v2).astype(np.float32))
    # v1 + v2 in f32 is exact here only up to rounding; compare against the f64 sum
    o1, o2 = oracle.attention(q, k, v1), oracle.attention(q, k, v2)
    assert np.allclose(o, o1 + o2, rtol=0, atol=1e-6)
    assert np.allclose(oracle.attention(q, k, (2 * v1).astype(np.float32)), 2 * o1, rtol=0, atol=1e-15)


def test_grouped_heads_map():
    q = _rand((3, 4, 8), 21)
    k, v = _rand((6, 2, 8), 22), _rand((6, 2, 8), 23)
    o = oracle.attention(q, k, v)
    for h in range(4):
        g = h // 2
        oh = oracle.attention(q[:, h:h + 1], k[:, g:g + 1], v[:, g:g + 1])
        assert np.array_equal(oh[:, 0], o[:, h])


def test_query_subset_equals_rows_of_full():
    q, k, v = _rand((16, 2, 8), 24), _rand((16, 2, 8), 25), _rand((16, 2, 8), 26)
    full = oracle.attention(q, k, v)
    rows = np.array([9, 3, 15])
    assert np.array_equal(oracle.attention(q[rows], k, v), full[rows])
