"""The Q5_K split form (tests/q5k_split.py) against the oracle's own decoders: every
weight of a Q5_K matrix equals the sum of the two Q4_K-form weights it becomes, in fp64
(d * sc * q - dmin * m is exact in both forms, and 16 d is exact in f16)."""
import numpy as np
import pytest

import oracle
from quantized_int8_gemm_q4_b200 import synth
from tests.q5k_split import split_q5k


@pytest.mark.parametrize("N,K,seed", [(3, 256, 1), (5, 1024, 2), (2, 4096, 3)])
def test_split_weights_sum_to_the_q5k_weights(N, K, seed):
    w5 = synth.q5k_weights(N, K, seed)
    w4 = split_q5k(w5)
    nsb = K // 256
    d5 = oracle.dequant(13, w5, N, K)
    d4 = oracle.dequant(12, w4, N, 2 * K)
    assert np.array_equal(d5, d4[:, :K] + d4[:, K:])


def test_split_blocks_of_extreme_quants():
    """All fifth bits set, largest scales: the high blocks carry 16 d sc exactly."""
    w5 = synth.q5k_weights(1, 256, 4)
    w5[..., 16:48] = 255        # every fifth bit
    w5[..., 48:176] = 255       # every low nibble 15: q = 31
    w4 = split_q5k(w5)
    d5 = oracle.dequant(13, w5, 1, 256)
    d4 = oracle.dequant(12, w4, 1, 512)
    assert np.array_equal(d5, d4[:, :256] + d4[:, 256:])
    assert np.all(w4[0, 1, 16:] == 0x11)
