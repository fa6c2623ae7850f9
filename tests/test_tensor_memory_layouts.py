"""Host models of index arithmetic in the tensor-memory serving kernels.

1. 2:4 sparsity metadata in tensor memory (kernels_umma.cuh). For a kind::f16 sparse MMA with
   M = 128 and K = 32, the 4-bit code of block b (columns 4b..4b+3, b = 0..7) of row m sits in
   TMEM lane (m % 8) + 8 (b // 4) + 16 (m // 16), at nibble (b % 4) + 4 ((m // 8) % 2) of the
   32-bit column. The kernel builds lane 32 w + l's word from the packed 2:4 metadata words of
   two rows with one byte permute; this checks that every code lands where the layout puts it.
2. 4:8 expansion (kernels_umma.cuh, u8_table_entry): a block's four values in position order
   (v0 v1 in one word, v2 v3 in the other) become a dense chunk of eight bf16 through
   prmt(prmt(v0v1, 0, A[p0 p1]), v2v3, B[p2 p3]) per word; this checks all 70 position sets.
   The four words are the block's four 32-bit columns of the dense tile in tensor memory.
3. 4:8 prefill (kernels_pf48.cuh): the reads of the 64-byte-swizzled box of compressed values.
"""
import itertools
import random


def byte_perm(x, y, s):
    """CUDA __byte_perm: byte n of the result is byte (s >> 4n) & 7 of the 8 bytes (x, y)."""
    src = [(x >> (8 * k)) & 0xFF for k in range(4)] + [(y >> (8 * k)) & 0xFF for k in range(4)]
    return sum(src[(s >> (4 * n)) & 7] << (8 * n) for n in range(4))


def test_2of4_tmem_metadata_words_follow_the_mma_layout():
    rng = random.Random(7)
    # packed 2:4 metadata of one 128-row stage: per row 4 words (one per 32-column K step),
    # nibble q of word j = code of block q of that K step
    meta = [[rng.getrandbits(32) for _ in range(4)] for _ in range(128)]
    lane_words = {}
    for warp in range(4):
        for lane in range(32):
            # the kernel's arithmetic for its TMEM lane 32 warp + lane
            h = (lane >> 3) & 1
            ra = 32 * warp + 16 * (lane >> 4) + (lane & 7)
            esel = 0x7632 if h else 0x5410
            lane_words[32 * warp + lane] = [byte_perm(meta[ra][j], meta[ra + 8][j], esel) for j in range(4)]
    for m in range(128):
        for j in range(4):
            for b in range(8):
                code = (meta[m][j] >> (4 * b)) & 0xF
                dp = (m % 8) + 8 * (b // 4) + 16 * (m // 16)
                nib = (b % 4) + 4 * ((m // 8) % 2)
                assert (lane_words[dp][j] >> (4 * nib)) & 0xF == code, (m, j, b)


def u8_table_entry(q, second):
    """Restates the device function: selectors of the four words of a dense chunk."""
    pa, pb = q & 7, q >> 3
    words = []
    for i in range(4):
        sel = 0
        for h in range(2):
            pos = 2 * i + h
            base, other = (4, 2 * h) if second else (0, 4)
            b0 = base if pos == pa else (base + 2 if pos == pb else other)
            sel |= (b0 | (b0 + 1) << 4) << (8 * h)
        words.append(sel)
    return words


def test_4of8_expansion_tables_rebuild_every_dense_chunk():
    table_a = [u8_table_entry(q, False) for q in range(64)]
    table_b = [u8_table_entry(q, True) for q in range(64)]
    rng = random.Random(3)
    sets = list(itertools.combinations(range(8), 4))
    assert len(sets) == 70
    for pos in sets:
        for _ in range(4):
            v = [rng.randrange(1, 1 << 16) for _ in range(4)]
            lo, hi = v[0] | v[1] << 16, v[2] | v[3] << 16
            code = pos[0] | pos[1] << 3 | pos[2] << 6 | pos[3] << 9  # the packed 4:8 code
            sa, sb = table_a[code & 63], table_b[code >> 6]
            words = [byte_perm(byte_perm(lo, 0, sa[i]), hi, sb[i]) for i in range(4)]
            dense = [0] * 8
            for k, p in enumerate(pos):
                dense[p] = v[k]
            assert words == [dense[2 * i] | dense[2 * i + 1] << 16 for i in range(4)], pos


def test_4of8_zero_filled_code_expands_to_zero():
    """Rows past the matrix arrive zero-filled (values 0, code 0): the chunk must be zero."""
    sa, sb = u8_table_entry(0, False), u8_table_entry(0, True)
    assert [byte_perm(byte_perm(0, 0, sa[i]), 0, sb[i]) for i in range(4)] == [0, 0, 0, 0]


def test_4of8_prefill_value_reads_undo_the_64_byte_swizzle():
    """The 4:8 prefill kernel lands each stage's 128-row x 64-byte box of compressed values
    with the tensor map's 64-byte swizzle (on a 512-byte boundary: 16-byte chunk c of row r at
    chunk c ^ ((r >> 1) & 3)); the thread of row r and part pt reads its chunk at that place,
    and the eight consecutive rows a quarter-warp reads at one part fall on eight distinct
    four-bank groups (no bank conflict)."""
    def landed(off):  # byte offset of logical byte `off` of the box after the 64-byte swizzle
        return off ^ (((off >> 7) & 3) << 4)

    def read_at(r, pt):  # the kernel's address of row r, part pt
        return r * 64 + ((pt ^ ((r >> 1) & 3)) << 4)

    for r in range(128):
        for pt in range(4):
            assert landed(r * 64 + pt * 16) == read_at(r, pt)
    for q0 in range(0, 128, 8):
        for pt in range(4):
            assert len({(read_at(r, pt) // 16) % 8 for r in range(q0, q0 + 8)}) == 8
