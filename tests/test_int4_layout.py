"""The test-side restatement of the packed 4-bit layout is self-consistent
(CPU only): packing and unpacking are inverse, a hand-placed code lands where
the header's description puts it, and the sizes match the library's."""
import numpy as np

import int4_layout as L


def test_pack_unpack_roundtrip():
    rng = np.random.default_rng(3)
    for K, N in ((256, 16), (512, 272), (1024, 512)):
        codes = rng.integers(0, 16, (K, N)).astype(np.uint8)
        s = rng.standard_normal((K // 64, N)).astype(np.float16)
        lo = rng.standard_normal((K // 64, N)).astype(np.float16)
        W4, S4 = L.pack(codes, s, lo)
        assert W4.size == L.padded_n(N) * K // 2 and S4.size == L.padded_n(N) * K // 64 * 4
        c2, s2, l2 = L.unpack(W4, S4, K, N)
        assert np.array_equal(c2, codes)
        assert np.array_equal(s2.view(np.uint16), s.view(np.uint16))
        assert np.array_equal(l2.view(np.uint16), lo.view(np.uint16))


def test_single_code_position():
    """Code (k, n) = (256 + 32*2 + 8*1 + 3, 256 + 9) goes to block (nt=1, kt=1),
    column r = 9, chunk 2 at position 2 ^ (9 % 8) = 3, word 1, nibble 4 + 1."""
    K, N = 512, 512
    codes = np.zeros((K, N), np.uint8)
    k, n = 256 + 64 + 8 + 3, 256 + 9
    codes[k, n] = 0xB
    W4, _ = L.pack(codes, np.zeros((K // 64, N), np.float16), np.zeros((K // 64, N), np.float16))
    KT = K // 256
    block = (1 * KT + 1) * 32768
    at = block + 9 * 128 + 3 * 16 + 1 * 4                     # word 1 of the chunk
    word = int(np.frombuffer(W4[at:at + 4].tobytes(), "<u4")[0])
    assert word == 0xB << (4 * 5)
    assert np.count_nonzero(W4) == 1


def test_library_sizes_match(tmp_path):
    import int8_quantized_row_b200 as i8
    for K, N in ((256, 16), (12288, 49152), (512, 4800)):
        assert i8.int4_packed_code_bytes(K, N) == L.padded_n(N) * K // 2
        assert i8.int4_packed_scale_bytes(K, N) == L.padded_n(N) * K // 64 * 4
