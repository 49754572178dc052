"""The parallel driver of the oracle returns what the oracle returns.

``oracle_pool.attention_rows_parallel`` only splits the work of
``oracle.attention_rows_ref`` into (segment, head, row-chunk) tasks run in
spawned worker processes; on a small packed case, with chunks that split
segments, it must agree with one direct call to within the summation-order
rounding of float64 (1e-13).
"""

import numpy as np

import oracle
import synth
from oracle_pool import attention_rows_parallel


def test_pool_equals_direct_oracle_call():
    q, k, v, pos, cu = synth.draw_random_case([300, 1, 517, 0, 90], 3, 64, 17, pos_range=64.0)
    rows = np.r_[0:cu[-1]]
    heads = [2, 0]
    O1, L1 = attention_rows_parallel(q, k, v, cu, 0.11, rows, heads, pos, (16, 24, 24),
                                     chunk=128)
    O2, L2 = oracle.attention_rows_ref(q, k, v, cu, 0.11, rows, heads, pos, (16, 24, 24))
    np.testing.assert_allclose(O1, O2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(L1, L2, rtol=0, atol=1e-13)


def test_pool_without_positions_and_sparse_rows():
    q, k, v, pos, cu = synth.draw_random_case([200, 333], 2, 128, 18, pos_range=64.0)
    rows = np.array([0, 5, 199, 200, 201, 532])
    O1, L1 = attention_rows_parallel(q, k, v, cu, 0.09, rows, [1], chunk=2)
    O2, L2 = oracle.attention_rows_ref(q, k, v, cu, 0.09, rows, [1])
    np.testing.assert_allclose(O1, O2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(L1, L2, rtol=0, atol=1e-13)
