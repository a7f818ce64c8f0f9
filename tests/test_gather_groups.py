"""Host logic of aq_gather_qmm's expert grouping (no GPU): pairs that share a
weight matrix become problems of up to 16 / M pairs, in pair order within a
matrix, padded with -1 rows to the largest problem; nothing is grouped when
it would not save a weight read."""
import ctypes

import numpy as np

from group_wise_affine_quant_b200 import _lib

I32 = ctypes.c_int32


def groups(lhs, rhs, M, N=256, K=1024, x_batch=None, cap=4096):
    n = len(rhs)
    x_batch = x_batch or (max(lhs) + 1 if lhs else n)
    xm, ym = (I32 * cap)(), (I32 * cap)()
    mb = ctypes.c_int(0)
    G = _lib.lib().aq_testing_gather_groups(
        (I32 * n)(*lhs) if lhs is not None else None, (I32 * n)(*rhs), n, M, N, K, x_batch, xm, ym,
        cap, ctypes.byref(mb))
    rows = G * mb.value
    return G, mb.value, np.array(xm[:rows]).reshape(G, -1) if G else None, \
        np.array(ym[:rows]).reshape(G, -1) if G else None


def test_groups_by_matrix_in_pair_order():
    lhs = [5, 0, 3, 1, 2]
    rhs = [2, 0, 2, 0, 2]
    G, Mb, xm, ym = groups(lhs, rhs, M=1)
    assert (G, Mb) == (2, 3)
    # matrix 0: pairs 1, 3; matrix 2: pairs 0, 2, 4 (ascending matrix order)
    assert xm.tolist() == [[0, 1, -1], [5, 3, 2]]
    assert ym.tolist() == [[1, 3, -1], [0, 2, 4]]


def test_rows_of_x_per_pair_and_split_groups():
    M = 5                                         # 16 // 5 = 3 pairs per problem
    rhs = [1] * 7
    lhs = [0, 1, 2, 3, 4, 5, 6]
    G, Mb, xm, ym = groups(lhs, rhs, M=M)
    assert (G, Mb) == (3, 15)                     # 3 + 3 + 1 pairs
    assert xm[0].tolist() == list(range(0, 15))   # pairs 0..2: x rows 0..14
    assert xm[2].tolist() == list(range(30, 35)) + [-1] * 10
    assert ym[2].tolist() == list(range(30, 35)) + [-1] * 10


def test_no_grouping_without_a_shared_matrix_or_for_large_m():
    assert groups([0, 1, 2], [0, 1, 2], M=1)[0] == 0          # every matrix once
    assert groups([0, 1], [0, 0], M=9)[0] == 0                # 16 // 9 = 1 pair per problem
    assert groups([0, 1], [0, 0], M=1, N=100)[0] == 0         # y rows not 16-byte multiples
