"""The RMS pass sums a row's squares in its own order -- per 1024-element
round, each lane's 32 contiguous squares as a pairwise tree, an xor butterfly
over the 32 lanes, then the rounds merged like a binary counter and closed
over the set bits of the round count (the zero padding never computed) -- and
claims that this is the contiguous pairwise tree over the row zero-padded to a
power of two, which the RMSNorm reading fixes (ARCQuant page, 방법론, 커널
구현; the reading is pinned in test_oracle_rmsnorm.py).  Here that order is
replayed in binary32 numpy arithmetic and compared with the tree taken level
by level, bit for bit, on rows whose sums depend on the order; a left-to-right
sum differs on them, so the comparison has teeth."""
import numpy as np
import pytest

import workloads


def _squares(rows: int, K: int, seed: int) -> np.ndarray:
    x = workloads.small_operand(rows, K, seed=seed).make().float().numpy()
    x[:, ::97] *= 300.0  # spread the magnitudes so that the order of the additions matters
    return (x * x).astype(np.float32)


def _tree(sq: np.ndarray) -> np.ndarray:
    """Contiguous pairwise tree over each row, zero-padded to a power of two."""
    rows, K = sq.shape
    n = 1 << (K - 1).bit_length()
    a = np.zeros((rows, n), np.float32)
    a[:, :K] = sq
    while a.shape[1] > 1:
        a = a[:, 0::2] + a[:, 1::2]
    return a[:, 0]


def _kernel_order(sq: np.ndarray) -> np.ndarray:
    """The RMS pass's order (lanes, butterfly, rounds, counter, closure)."""
    rows, K = sq.shape
    used = (K + 1023) // 1024
    a = np.zeros((rows, used * 1024), np.float32)
    a[:, :K] = sq
    # [rows, round, lane, group, 8]: lane l of round q holds elements 1024q + 32l .. + 31
    g = a.reshape(rows, used, 32, 4, 8)
    b = g[..., 0::2] + g[..., 1::2]                # (a0+a1, a2+a3, a4+a5, a6+a7)
    c = b[..., 0::2] + b[..., 1::2]                # ((a0+a1)+(a2+a3), (a4+a5)+(a6+a7))
    s8 = c[..., 0] + c[..., 1]                     # the group's pairwise sum
    v = (s8[..., 0] + s8[..., 1]) + (s8[..., 2] + s8[..., 3])  # the lane's 32 elements
    lanes = np.arange(32)
    for o in (1, 2, 4, 8, 16):
        v = v + v[..., lanes ^ o]                  # the xor butterfly: v_l + v_(l^o)
    rsum = v[..., 0]                               # every lane holds the round's subtree
    stk = [None] * 5
    for q in range(used):                          # the binary counter
        t = rsum[:, q]
        for lvl in range(5):
            if not (q >> lvl) & 1:
                stk[lvl] = t
                break
            t = stk[lvl] + t
    total = None
    for lvl in range(5):                           # closure over the set bits of `used`
        if (used >> lvl) & 1:
            total = stk[lvl] if total is None else stk[lvl] + total
    return total


@pytest.mark.parametrize("K", [64, 128, 320, 1024, 1088, 2112, 5120, 7168, 8192, 8256, 12288, 16384])
def test_kernel_order_is_the_padded_pairwise_tree(K):
    sq = _squares(48, K, seed=K)
    assert np.array_equal(_kernel_order(sq).view(np.uint32), _tree(sq).view(np.uint32))


def test_a_left_to_right_sum_differs_on_these_rows():
    sq = _squares(48, 5120, seed=5120)
    seq = np.zeros(sq.shape[0], np.float32)
    for k in range(sq.shape[1]):
        seq = seq + sq[:, k]
    assert not np.array_equal(seq, _tree(sq))
