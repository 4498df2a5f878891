"""The packed 4-bit weight layout of include/int8row.h, restated in numpy for
the tests: unpack the library's W4 / S4 buffers into plain arrays (codes
[K,N], s and lo [K/64,N]) that compare with the oracle's, and pack plain
arrays the same way (to check the unpacker against the description).  Layout
only; none of the codec's arithmetic is here."""
import numpy as np

BLOCK_N, BLOCK_K, G = 256, 256, 64


def padded_n(N):
    return (N + BLOCK_N - 1) // BLOCK_N * BLOCK_N


def _nibble_order():
    """Position (0..7) in a 32-bit word of each of its 8 codes, code e -> nibble."""
    return np.array([e // 2 if e % 2 == 0 else 4 + e // 2 for e in range(8)])


def unpack(W4, S4, K, N):
    """(codes uint8 [K,N], s fp16 [K/64,N], lo fp16 [K/64,N]) from the packed bytes."""
    NP, KT = padded_n(N), K // BLOCK_K
    blocks = np.asarray(W4, np.uint8).reshape(NP // BLOCK_N, KT, BLOCK_N, 8, 16)       # nt, kt, r, chunk pos, byte
    r = np.arange(BLOCK_N)
    chunks = np.empty_like(blocks)
    for c in range(8):
        chunks[:, :, :, c] = blocks[:, :, r, c ^ (r & 7)]
    words = chunks.reshape(NP // BLOCK_N, KT, BLOCK_N, 8, 4, 4).view("<u4")[..., 0]    # nt, kt, r, chunk, word
    nib = _nibble_order()
    codes = np.stack([(words >> np.uint32(4 * nib[e])) & np.uint32(0xF) for e in range(8)], axis=-1)  # ..., word, code
    codes = codes.reshape(NP // BLOCK_N, KT, BLOCK_N, BLOCK_K).astype(np.uint8)        # k = 32c + 8i + e
    codes = codes.transpose(1, 3, 0, 2).reshape(K, NP)[:, :N]
    sl = np.asarray(S4, np.uint8).reshape(NP // BLOCK_N, KT, BLOCK_N, 4, 2, 2).view("<u2")[..., 0]
    sl = sl.transpose(1, 3, 0, 2, 4).reshape(K // G, NP, 2)[:, :N]
    return codes, sl[..., 0].copy().view(np.float16), sl[..., 1].copy().view(np.float16)


def pack(codes, s, lo):
    """The packed (W4, S4) bytes of plain arrays (padding columns zero)."""
    K, N = codes.shape
    NP, KT = padded_n(N), K // BLOCK_K
    c = np.zeros((K, NP), np.uint32)
    c[:, :N] = codes
    c = c.reshape(KT, 8, 4, 8, NP // BLOCK_N, BLOCK_N)                     # kt, chunk, word, code, nt, r
    nib = _nibble_order()
    words = np.zeros((KT, 8, 4, NP // BLOCK_N, BLOCK_N), np.uint32)
    for e in range(8):
        words |= c[:, :, :, e] << np.uint32(4 * nib[e])
    words = words.transpose(3, 0, 4, 1, 2)                                 # nt, kt, r, chunk, word
    chunks = np.ascontiguousarray(words, dtype="<u4").view(np.uint8).reshape(NP // BLOCK_N, KT, BLOCK_N, 8, 16)
    r = np.arange(BLOCK_N)
    placed = np.empty_like(chunks)
    for cc in range(8):
        placed[:, :, r, cc ^ (r & 7)] = chunks[:, :, :, cc]
    sl = np.zeros((K // G, NP, 2), np.uint16)
    sl[:, :N, 0] = np.asarray(s, np.float16).view(np.uint16)
    sl[:, :N, 1] = np.asarray(lo, np.float16).view(np.uint16)
    sl = sl.reshape(KT, 4, NP // BLOCK_N, BLOCK_N, 2).transpose(2, 0, 3, 1, 4)
    return placed.reshape(-1), np.ascontiguousarray(sl, dtype="<u2").view(np.uint8).reshape(-1)
