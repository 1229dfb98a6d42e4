"""CPU check of the test-side reader of the rank-major int4 value layout: blocks written
element by element from the layout's definition (rank row i, 16-byte column
c ^ (i / 2 % 4), nibble ((t & 1) << 2) | ((t >> 1) & 3); scales then zeros per group) are
read back as the token-major words and {scale, zero} params of the oracle's packer."""
import numpy as np

from tests import helpers as H


def _encode_reference(codes_tm, params_tm, G):
    """Write token-major codes [B][T][G*4] and params [B][T][G] (T a multiple of 128) into
    rank-major blocks with plain loops over the definition."""
    B, T, _ = codes_tm.shape
    nb = T // 128
    raw = np.zeros((B, nb, G * 32, 16), np.uint32)
    halves = np.zeros((B, nb, G, 256), np.uint16)
    for b in range(B):
        for tok in range(T):
            blk, t = divmod(tok, 128)
            for i in range(G * 32):
                g, e = divmod(i, 32)
                code = (int(codes_tm[b, tok, g * 4 + e // 8]) >> (4 * (e % 8))) & 15
                word = (((t >> 5) ^ ((i >> 1) & 3)) << 2) + ((t & 31) >> 3)
                nib = ((t & 1) << 2) | ((t >> 1) & 3)
                raw[b, blk, i, word] |= np.uint32(code << (4 * nib))
            for g in range(G):
                pw = int(params_tm[b, tok, g])
                halves[b, blk, g, t] = pw & 0xFFFF
                halves[b, blk, g, 128 + t] = pw >> 16
    return raw, halves


def test_value_layout_reader_round_trips():
    rng = np.random.default_rng(3)
    B, T, G = 2, 256, 3
    codes = rng.integers(0, 2 ** 32, size=(B, T, G * 4), dtype=np.uint64).astype(np.uint32)
    params = rng.integers(0, 2 ** 32, size=(B, T, G), dtype=np.uint64).astype(np.uint32)
    raw, halves = _encode_reference(codes, params, G)
    c, p = H.value_blocks_to_token_major(raw, halves)
    assert np.array_equal(c, codes)
    assert np.array_equal(p, params)


def test_value_layout_columns_are_bank_spread():
    """Eight consecutive rank rows read at the same logical column land in eight distinct
    16-byte columns of a 128-byte line (rows are 64 bytes apart)."""
    for c in range(4):
        cols = set()
        for i in range(8):
            addr = i * 64 + ((c ^ ((i >> 1) & 3)) * 16)
            cols.add(addr % 128)
        assert len(cols) == 8
