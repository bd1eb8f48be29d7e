"""The oracle, pinned to what the pages and the mathematics fix (CPU only)."""
import numpy as np
import pytest

import oracle
from oracle_checks import ALL_CHECKS


@pytest.mark.parametrize("check", ALL_CHECKS, ids=lambda c: c.__name__)
def test_pin(check):
    check(oracle._lib())


def test_oracle_rejects_bad_arguments():
    lib = oracle._lib()
    q = np.zeros((1, 4, 8, 64), np.uint16)
    k = np.zeros((1, 3, 8, 64), np.uint16)
    with pytest.raises(oracle.OracleError):      # Hq % Hkv != 0
        oracle.attention(q, k, k, lib=lib)
    k = np.zeros((1, 2, 8, 64), np.uint16)
    with pytest.raises(oracle.OracleError):      # window without causal
        oracle.attention(q, k, k, causal=False, window=4, lib=lib)
    with pytest.raises(oracle.OracleError):      # row id out of range
        oracle.attention(q, k, k, rows=np.array([4 * 8]), lib=lib)
    qd = np.zeros((1, 4, 64), np.uint16)
    pages = np.zeros((2, 2, 16, 64), np.uint16)
    with pytest.raises(oracle.OracleError):      # block-table entry outside the pool
        oracle.decode_paged(qd, pages, pages, np.array([[5]], np.int32), np.array([3], np.int32), lib=lib)
    with pytest.raises(oracle.OracleError):      # seq_len beyond the table
        oracle.decode_paged(qd, pages, pages, np.array([[0]], np.int32), np.array([17], np.int32), lib=lib)
