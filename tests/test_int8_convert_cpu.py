"""The exact int8 -> bf16 conversion the INT8-weight kernels use
(int8_convert.cuh), emulated bit for bit on the host over every byte value:
the sign flip, the byte permute into the mantissa of 2^23, the subtraction of
2^23 + 128, and the pack of two results' upper halves into a bf16 pair. It
must return the signed byte exactly, and the pack must pair the right bytes."""
import numpy as np


def bf16_bits_to_f64(bits):
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


def byte_perm(x: int, y: int, sel: int) -> int:
    """The byte permute of two 32-bit words: result byte i is byte (sel >> 4i) & 7
    of the 8-byte value whose bytes 0-3 are x and 4-7 are y."""
    src = [(x >> (8 * i)) & 0xFF for i in range(4)] + [(y >> (8 * i)) & 0xFF for i in range(4)]
    return sum(src[(sel >> (4 * i)) & 7] << (8 * i) for i in range(4))


def test_f32_route_is_exact_for_every_byte():
    b = np.arange(-128, 128, dtype=np.int64)
    u = ((b & 0xFF) ^ 0x80).astype(np.uint32)
    f = (u | 0x4B000000).view(np.float32)
    v = (f - np.float32(8388736.0)).astype(np.float64)
    assert np.array_equal(v, b.astype(np.float64))


def test_placement_and_pack_through_the_byte_permute():
    """Each byte j of a word lands in the mantissa of 2^23 (selector 0x765j with
    2^23 as the second word) and converts to the byte's value; two converted
    values pack into one bf16 pair (selector 0x7632): the first one's upper
    half low, the second's high, both exact in bf16."""
    rng = np.random.default_rng(7)
    for _ in range(200):
        w = int(rng.integers(0, 2**32, dtype=np.uint64))
        u = w ^ 0x80808080
        vals = []
        for j in range(4):
            bits = byte_perm(u, 0x4B000000, 0x7650 | j)
            f = np.array([bits], dtype=np.uint32).view(np.float32)[0] - np.float32(8388736.0)
            b = (w >> (8 * j)) & 0xFF
            assert float(f) == (b - 256 if b >= 128 else b)
            vals.append(np.array([f], dtype=np.float32).view(np.uint32)[0])
        pair = byte_perm(int(vals[0]), int(vals[1]), 0x7632)
        assert bf16_bits_to_f64([pair & 0xFFFF])[0] == float(np.array([vals[0]], dtype=np.uint32).view(np.float32)[0])
        assert bf16_bits_to_f64([pair >> 16])[0] == float(np.array([vals[1]], dtype=np.uint32).view(np.float32)[0])
