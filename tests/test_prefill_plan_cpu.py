"""The tensor-core prefill's work plan (host logic, no GPU): every query tile
of every (request, head) is computed by exactly one block; blocks hold one
tile or two consecutive tiles; with an odd tile count the lone tile is tile
0; a batch of four waves or more ends with the blocks of each prompt's first
eighth of tiles, longest first; small batches run one tile per block."""
import collections

import pytest

from ring_sliding_window_b200 import rswa

SMS = 148


def _plan(prefill_lens, heads=10, sms=SMS):
    return rswa.rswa_debug_prefill_plan(len(prefill_lens), heads, 128, 128, rswa.RSWA_BF16,
                                        prefill_lens, sms)


def _tiles(p):
    return (p + 127) // 128


def _check_cover(blocks, prefill_lens, heads):
    seen = collections.Counter()
    for b, h, t0, n in blocks:
        assert n in (1, 2)
        assert 0 <= b < len(prefill_lens) and 0 <= h < heads
        assert 0 <= t0 and t0 + n <= _tiles(prefill_lens[b])
        for t in range(t0, t0 + n):
            seen[(b, h, t)] += 1
    want = {(b, h, t) for b, p in enumerate(prefill_lens) for h in range(heads)
            for t in range(_tiles(p))}
    assert set(seen) == want
    assert all(c == 1 for c in seen.values())


@pytest.mark.parametrize("prefill_lens", [[8256] * 8, [32640] * 4, [8192] * 8,
                                          [1024, 16384, 3000, 129, 7777, 12000, 64, 300]])
def test_every_tile_once_and_lone_tile_first(prefill_lens):
    blocks = _plan(prefill_lens)
    _check_cover(blocks, prefill_lens, 10)
    pairs = sum(10 * ((p + 255) // 256) for p in prefill_lens)
    if pairs >= SMS:
        for b, h, t0, n in blocks:
            tiles = _tiles(prefill_lens[b])
            if n == 1:  # the only lone tile of a (b, h) with an odd count is tile 0
                assert tiles % 2 == 1 and t0 == 0, (b, h, t0, tiles)
            else:
                assert t0 % 2 == tiles % 2, (b, h, t0, tiles)


def test_large_batch_ends_with_the_short_blocks():
    lens = [8256] * 8  # 2,640 blocks, 17.8 waves of 148
    blocks = _plan(lens)
    tiles = _tiles(8256)
    short = [blk for blk in blocks if blk[2] < tiles // 8 and blk[3] == 2]
    # the pairs of the first eighth of tiles close the launch, longest first
    assert blocks[-len(short):] == short
    firsts = [blk[2] for blk in short]
    assert firsts == sorted(firsts, reverse=True)
    # the rest: super-groups of about one wave, longest first inside each
    head = blocks[:-len(short)]
    assert all(blk[2] >= tiles // 8 or blk[3] == 1 for blk in head)


def test_small_batch_one_tile_per_block_and_no_deferral():
    lens = [1088]  # 10 heads x 9 tiles: 50 pairs, fewer than the SMs
    blocks = _plan(lens)
    _check_cover(blocks, lens, 10)
    assert len(blocks) == 10 * 9
    assert all(n == 1 for _, _, _, n in blocks)


def test_bad_arguments():
    cfg_lens = [100]
    with pytest.raises(rswa.RswaError):
        rswa.rswa_debug_prefill_plan(1, 10, 128, 128, rswa.RSWA_BF16, cfg_lens, 0)
