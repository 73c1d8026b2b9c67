"""Exactness of the integer identities the routing and sort kernels rely on, restated on the host
over exhaustive or randomised ranges.  These check the arithmetic the kernels' comments claim
(csrc/sort.cu, csrc/route.cu), not the kernels themselves (the GPU parity tests do that)."""
import struct

import numpy as np


def test_multiply_high_division_is_exact_below_2_16():
    # FastDiv (sort.cu): m = floor((2^32 - 1) / d) + 1; floor(v m / 2^32) = floor(v / d) for v < 2^16 and
    # 1 < d <= 2^16 (d = 2^16 included: the fast RBD plan allows E = 65536).
    v = np.arange(1 << 16, dtype=np.uint64)
    for d in list(range(2, 300)) + [1000, 4095, 4096, 32767, 32768, 65535, 65536]:
        m = np.uint64((0xFFFFFFFF // d) + 1)
        assert np.array_equal((v * m) >> np.uint64(32), v // np.uint64(d)), d


def test_reciprocal_64_division_of_pft_indices():
    # PftSink: kinv = floor((2^64 - 1) / k) + 1; token = high word of i * kinv = floor(i / k) for every
    # 32-bit i (the PFT's assignment index i = t k + j < 2^31).
    r = np.random.default_rng(3)
    for k in range(2, 33):
        kinv = ((1 << 64) - 1) // k + 1
        for i in [0, 1, k - 1, k, k + 1, (1 << 31) - 1, (1 << 31) - 2] + r.integers(0, 1 << 31, 2000).tolist():
            assert (i * kinv) >> 64 == i // k, (i, k)


def test_byte_wise_prefix_by_multiplication():
    # RBD emit: per-node replica counts one byte each (nodes < 8, total <= 32); cnt * 0x0101..01 - cnt
    # holds in byte n the replicas on nodes before n (no carries between bytes).
    r = np.random.default_rng(4)
    for _ in range(5000):
        k = int(r.integers(1, 33))
        nodes = r.integers(0, 8, size=k)
        cnt = 0
        for n in nodes:
            cnt += 1 << (8 * int(n))
        first = (cnt * 0x0101010101010101 - cnt) & ((1 << 64) - 1)
        per = np.bincount(nodes, minlength=8)
        for n in range(8):
            assert (cnt >> (8 * n)) & 0xFF == per[n]
            assert (first >> (8 * n)) & 0xFF == per[:n].sum()


def test_sort_keys_order_by_id_then_slot():
    # RBD: keys id * 256 + slot (id < 2^16, slot < 32); ascending keys = ascending (id, slot), and the
    # padding key INT_MAX sorts after every real key.
    r = np.random.default_rng(5)
    for _ in range(2000):
        k = int(r.integers(1, 33))
        ids = r.integers(0, 1 << 16, size=k)
        ids[r.integers(0, k)] = ids[0]   # a repeated id
        keys = sorted(int(e) << 8 | j for j, e in enumerate(ids)) + [2 ** 31 - 1]
        assert [(x >> 8, x & 0xFF) for x in keys[:-1]] == sorted((int(e), j) for j, e in enumerate(ids))
        assert keys[-1] > keys[-2]


def _sel_key(v, e):
    # route.cu sel_key, bit for bit: float bits made monotonic, -0 -> +0, then ~expert in the low word
    v = np.float32(v)
    if v == 0:
        v = np.float32(0.0)
    u = struct.unpack("<I", struct.pack("<f", v))[0]
    u = (~u & 0xFFFFFFFF) if u & 0x80000000 else (u | 0x80000000)
    return (u << 32) | (~e & 0xFFFFFFFF)


def test_selection_keys_order_by_value_then_lower_expert():
    # Larger key first = larger value first, equal values (also -0 and +0) by lower expert id.
    vals = [-np.inf, -3.5, -1e-30, -0.0, 0.0, 1e-30, 2.0, 2.0, 7.25, np.inf]
    items = [(float(v), e) for e, v in enumerate(vals)]
    r = np.random.default_rng(6)
    items += [(float(np.float32(x)), 100 + i) for i, x in enumerate(r.standard_normal(300))]
    items += [(float(np.float32(x)), 500 + i) for i, x in enumerate(r.choice([-1.0, 0.5, 3.0], 60))]
    by_key = sorted(items, key=lambda it: -_sel_key(*it))
    expect = sorted(items, key=lambda it: (-(it[0] + 0.0), it[1]))
    assert by_key == expect
