"""Token pool (continuous batching): the host-side slot-range allocator and
the pooled state's argument checks.  No GPU needed.

Method: "开源5天Star破万之后：百度Unlimited-OCR的爆火路径复盘" §三 -- serving
with a page size of one token; each request owns prefill_len + W cache slots
for its whole life (§2.1), so the pool hands out contiguous slot ranges.

The allocator is checked against a brute-force model: a bitmap of the pool
where first fit is "the lowest base b such that slots [b, b + n) are all
free", and the statistics are recounted from the bitmap after every call.
"""
import random

import pytest
import torch


@pytest.fixture(scope="module")
def rswa():
    from ring_sliding_window_b200 import build
    build.build()
    from ring_sliding_window_b200 import rswa as mod
    return mod


class BitmapPool:
    def __init__(self, capacity):
        self.free = [True] * capacity
        self.ranges = {}  # base -> length

    def alloc(self, n):
        run = 0
        for i, f in enumerate(self.free):
            run = run + 1 if f else 0
            if run == n:
                b = i - n + 1
                for j in range(b, b + n):
                    self.free[j] = False
                self.ranges[b] = n
                return b
        return None

    def release(self, b):
        n = self.ranges.pop(b)
        for j in range(b, b + n):
            self.free[j] = True

    def stats(self):
        runs, run = [], 0
        for f in self.free + [False]:
            if f:
                run += 1
            elif run:
                runs.append(run)
                run = 0
        return sum(self.free), max(runs, default=0), len(runs), len(self.ranges)


@pytest.mark.parametrize("seed,capacity", [(1, 97), (2, 1000), (3, 4096)])
def test_pool_matches_bitmap_first_fit(rswa, seed, capacity):
    rng = random.Random(seed)
    pool = rswa.rswa_pool_create(capacity)
    model = BitmapPool(capacity)
    try:
        assert rswa.rswa_pool_capacity(pool) == capacity
        for _ in range(1500):
            if model.ranges and rng.random() < 0.45:
                b = rng.choice(sorted(model.ranges))
                rswa.rswa_pool_free(pool, b)
                model.release(b)
            else:
                n = rng.randint(1, max(1, capacity // 6))
                want = model.alloc(n)
                if want is None:
                    with pytest.raises(rswa.RswaError) as e:
                        rswa.rswa_pool_alloc(pool, n)
                    assert e.value.status == rswa.RSWA_ENOMEM
                else:
                    assert rswa.rswa_pool_alloc(pool, n) == want
            assert rswa.rswa_pool_stats(pool) == model.stats()
        # free everything: the free ranges merge back into one
        for b in sorted(model.ranges, key=lambda _: rng.random()):
            rswa.rswa_pool_free(pool, b)
            model.release(b)
        assert rswa.rswa_pool_stats(pool) == (capacity, capacity, 1, 0)
    finally:
        rswa.rswa_pool_destroy(pool)


def test_pool_rejects_bad_calls(rswa):
    for cap in (0, -5, 1 << 40):
        with pytest.raises(rswa.RswaError) as e:
            rswa.rswa_pool_create(cap)
        assert e.value.status == rswa.RSWA_EINVAL
    pool = rswa.rswa_pool_create(100)
    try:
        for n in (0, -1):
            with pytest.raises(rswa.RswaError) as e:
                rswa.rswa_pool_alloc(pool, n)
            assert e.value.status == rswa.RSWA_EINVAL
        a = rswa.rswa_pool_alloc(pool, 30)
        b = rswa.rswa_pool_alloc(pool, 30)
        assert (a, b) == (0, 30)
        for bad in (1, 29, 60, -1):  # not the base of an allocated range
            with pytest.raises(rswa.RswaError) as e:
                rswa.rswa_pool_free(pool, bad)
            assert e.value.status == rswa.RSWA_EINVAL
        rswa.rswa_pool_free(pool, a)
        with pytest.raises(rswa.RswaError):  # double free
            rswa.rswa_pool_free(pool, a)
        with pytest.raises(rswa.RswaError) as e:  # 70 slots free, but at most 40 in a row
            rswa.rswa_pool_alloc(pool, 41)
        assert e.value.status == rswa.RSWA_ENOMEM
        assert rswa.rswa_pool_stats(pool) == (70, 40, 2, 1)
        assert rswa.rswa_pool_alloc(pool, 30) == 0  # first fit reuses the hole
    finally:
        rswa.rswa_pool_destroy(pool)
    assert rswa.lib.rswa_pool_destroy(None) == rswa.RSWA_EINVAL
    assert rswa.lib.rswa_pool_capacity(None) == -1


def test_pool_cache_bytes(rswa):
    cfg = rswa.make_config(3, 12, 10, 128, 128, torch.bfloat16)
    assert rswa.rswa_pool_cache_bytes(cfg, 5000) == 5000 * 10 * 128 * 2
    cfg32 = rswa.make_config(1, 1, 2, 64, 8, torch.float32)
    assert rswa.rswa_pool_cache_bytes(cfg32, 72) == 72 * 2 * 64 * 4
    assert rswa.rswa_pool_cache_bytes(cfg32, 0) == 0
    cfg32.head_dim = 96
    assert rswa.rswa_pool_cache_bytes(cfg32, 72) == 0


@pytest.mark.parametrize("bases,pool_slots", [
    ([0, 50], 200),      # request 0 is [0, 72): overlaps request 1
    ([0, 72], 130),      # request 1 ends at 144 > 130
    ([-1, 100], 300),    # negative base
    ([100, 0], 171),     # request 0 ends at 172 > 171
    ([0, 100], 0),       # no pool
])
def test_pooled_state_rejects_bad_placement(rswa, bases, pool_slots):
    cfg = rswa.make_config(2, 1, 2, 64, 8, torch.float32)
    with pytest.raises(rswa.RswaError) as e:
        rswa.rswa_state_create_pooled(cfg, [64, 64], None, bases, pool_slots, [4096], [4096],
                                      1 << 20, 1 << 20, 0)
    assert e.value.status == rswa.RSWA_EINVAL
