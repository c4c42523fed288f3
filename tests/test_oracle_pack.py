"""Pins for the oracle's packed formats (CPU only): hand-derived bytes, the
pages' memory accounting, exhaustive enumeration and round trips."""
import itertools

import numpy as np
import pytest

from conftest import GOLDEN, read_golden
import os

FMT = {"i2": 0, "t5": 1}


def _hand_cases():
    with open(os.path.join(GOLDEN, "pack_hand.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            lhs, rhs = line.split(":")
            fmt, K, *codes = lhs.split()
            yield FMT[fmt], int(K), [int(c) for c in codes], [int(b) for b in rhs.split()]


@pytest.mark.parametrize("case", list(_hand_cases()))
def test_hand_packed_bytes(orc, case):
    fmt, K, codes, want = case
    packed = orc.pack(np.array([codes], np.int8), fmt)
    assert packed[0].tolist() == want
    assert orc.unpack(packed, 1, K, fmt)[0].tolist() == codes


def test_row_bytes_and_memory_accounting(orc):
    g = read_golden("memory_accounting.txt")
    params = float(g["params"][0])
    # a 70B-layer-shaped row: K = 8192 (and 28672) weights
    for K in (8192, 28672):
        i2 = orc.packed_row_bytes(K, 0)
        assert i2 == K // 4
        assert params * i2 / K / 1e9 == pytest.approx(float(g["i2_gb"][0]))
        t5 = orc.packed_row_bytes(K, 1)
        assert t5 == -(-(-(-K // 5)) // 16) * 16
        assert params * t5 / K / 1e9 == pytest.approx(float(g["t5_gb_approx"][0]), rel=0.01)
    assert params * 2 / 1e9 == pytest.approx(float(g["fp16_gb"][0]))
    assert 8 / 5 == pytest.approx(float(g["t5_bits_per_w"][0]))
    # the row sizes the workloads use
    table = {(256, 0): 64, (3200, 0): 800, (8640, 0): 2160, (8192, 0): 2048, (28672, 0): 7168,
             (5, 0): 16, (3200, 1): 640, (8640, 1): 1728, (8192, 1): 1648, (28672, 1): 5744,
             (5, 1): 16, (1, 0): 16, (64, 0): 16, (65, 0): 32, (80, 1): 16, (81, 1): 32}
    for (K, fmt), rb in table.items():
        assert orc.packed_row_bytes(K, fmt) == rb, (K, fmt)


def test_two_bit_exhaustive(orc):
    """All 81 groups of four trits: distinct bytes, no byte holds code 11,
    and unpack inverts pack."""
    groups = list(itertools.product((-1, 0, 1), repeat=4))
    codes = np.array(groups, np.int8)                      # 81 rows, K = 4
    packed = orc.pack(codes, 0)
    first = packed[:, 0]
    assert len(set(first.tolist())) == 81
    for b in first.tolist():
        assert all(((b >> (2 * i)) & 3) != 3 for i in range(4))
    assert (packed[:, 1:] == 0x55).all()
    assert np.array_equal(orc.unpack(packed, 81, 4, 0), codes)


def test_base3_exhaustive_is_bijection(orc):
    """All 243 groups of five trits map one-to-one onto the bytes 0..242."""
    groups = list(itertools.product((-1, 0, 1), repeat=5))
    codes = np.array(groups, np.int8)
    packed = orc.pack(codes, 1)
    assert sorted(packed[:, 0].tolist()) == list(range(243))
    assert (packed[:, 1:] == 121).all()
    assert np.array_equal(orc.unpack(packed, 243, 5, 1), codes)


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("K", [1, 2, 3, 4, 5, 7, 15, 16, 63, 64, 65, 79, 80, 81, 129, 256, 3200])
def test_round_trip(orc, fmt, K):
    rng = np.random.default_rng(K * 7 + fmt)
    codes = rng.integers(-1, 2, size=(5, K), dtype=np.int8)
    packed = orc.pack(codes, fmt)
    assert packed.shape == (5, orc.packed_row_bytes(K, fmt))
    assert np.array_equal(orc.unpack(packed, 5, K, fmt), codes)


def test_invalid_codes_rejected(orc):
    with pytest.raises(ValueError):
        orc.pack(np.array([[2, 0, 0, 0]], np.int8), 0)
    bad = np.full((1, 16), 0x55, np.uint8)
    bad[0, 0] = 0b11
    with pytest.raises(ValueError):
        orc.unpack(bad, 1, 4, 0)
    bad = np.full((1, 16), 121, np.uint8)
    bad[0, 0] = 243
    with pytest.raises(ValueError):
        orc.unpack(bad, 1, 5, 1)
    # a padding digit that is not weight 0
    bad = np.full((1, 16), 121, np.uint8)
    bad[0, 3] = 0
    with pytest.raises(ValueError):
        orc.unpack(bad, 1, 5, 1)
