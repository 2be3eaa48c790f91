"""Host checks of the B200 weight layout and of the offset-nibble identity the
grouped GEMM relies on (no GPU).

The GEMM feeds each stored uint4b8 nibble u = q + 8 to the FP8 MMA as the
E4M3 byte 0x0u, whose value is u * 2^-9, and removes the offset per group
with the group sum of the activation values.  These tests fix the three facts
that makes exact, using the oracle's E4M3 decoder (itself pinned to the OCP
FP8 points in test_oracle_numerics) and the oracle's packer.
"""
import numpy as np

import oracle
from gpu_helpers import repack_b200


def test_low_nibble_bytes_are_exact_e4m3_multiples_of_2_pow_minus_9():
    u = np.arange(16)
    assert np.array_equal(oracle.e4m3_decode(u.astype(np.uint8)), u * 2.0 ** -9)


def test_repack_puts_elements_in_byte_order_and_is_a_bijection():
    rng = np.random.default_rng(5)
    q = rng.integers(-8, 8, size=(3, 256))
    packed = oracle.pack_uint4b8(q)
    rep = repack_b200(packed).view(np.uint32)
    lo = rep & np.uint32(0x0F0F0F0F)
    hi = (rep >> np.uint32(4)) & np.uint32(0x0F0F0F0F)
    # bytes of lo are elements 0..3 of the word, bytes of hi elements 4..7
    bytes_ = np.stack([lo, hi], axis=-1).astype("<u4").view(np.uint8).reshape(3, 256)
    assert np.array_equal(bytes_.astype(np.int64) - 8, q)
    words = rng.integers(0, 2**32, size=100000, dtype=np.uint64).astype(np.uint32).view(np.int32)
    assert len(np.unique(repack_b200(words))) == len(np.unique(words))


def test_offset_identity_is_exact_per_group():
    rng = np.random.default_rng(9)
    for _ in range(200):
        a = oracle.e4m3_decode(rng.integers(0, 256, size=128).astype(np.uint8))
        a = np.where(np.isnan(a), 0.0, a)
        q = rng.integers(-8, 8, size=128)
        d = np.sum(a * ((q + 8) * 2.0 ** -9))
        assert 512.0 * d - 8.0 * np.sum(a) == np.sum(a * q)
