"""Host model of the expert-tail pair kernel's tile rule (the constexpr
`tail_tiles_per_block` and `tail_tile_rows` in csrc/grouped_gemm.cu): for
every bucket size up to 2000 rows, the tiles of a column block cover each
bucket row exactly once, a main MMA covers 256 rows (or the whole bucket when
it has at most 256), a tail has 1..128 rows and rides along only with the
last tile, and its MMA width N (rows rounded up to 32) stages a multiple of
16 rows per CTA."""
PAIR_ROWS, BM = 256, 128


def tiles_per_block(cnt):
    if cnt > PAIR_ROWS and cnt % PAIR_ROWS != 0 and cnt % PAIR_ROWS <= BM:
        return cnt // PAIR_ROWS
    return (cnt + PAIR_ROWS - 1) // PAIR_ROWS


def tile_rows(cnt, m, mt):
    left = cnt - m * PAIR_ROWS
    if cnt <= BM:
        return 0, cnt
    return min(PAIR_ROWS, left), (left - PAIR_ROWS if (m == mt - 1 and left > PAIR_ROWS) else 0)


def swap_n(rows):
    return (rows + 31) & ~31


def test_every_row_once_and_tail_shapes():
    for cnt in range(1, 2001):
        mt = tiles_per_block(cnt)
        seen = [0] * cnt
        for m in range(mt):
            main, tail = tile_rows(cnt, m, mt)
            assert main > 0 or tail > 0
            assert main == 0 or main > BM            # no half tiles: small tails ride along
            for r in range(m * PAIR_ROWS, m * PAIR_ROWS + main):
                seen[r] += 1
            if tail:
                assert 0 < tail <= BM and m == mt - 1
                n = swap_n(tail)
                assert n in (32, 64, 96, 128) and n >= tail and (n // 2) % 16 == 0
                start = m * PAIR_ROWS + (PAIR_ROWS if main else 0)
                assert start + tail == cnt
                for r in range(start, cnt):
                    seen[r] += 1
        assert seen == [1] * cnt, cnt


def test_tile_counts_of_typical_buckets():
    # fine-grained buckets of 256 +- 16 rows: one tile per column block
    assert [tiles_per_block(c) for c in (240, 256, 257, 272, 320)] == [1, 1, 1, 1, 1]
    # a remainder of more than 128 rows gets a full tile of its own
    assert tiles_per_block(256 + 129) == 2 and tile_rows(385, 1, 2) == (129, 0)
    assert tiles_per_block(1536) == 6 and tiles_per_block(1600) == 6
