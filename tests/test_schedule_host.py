"""The GEMMs' work schedule (CPU): the library's own schedule code, run on
the host through fp8_selftest_gemm_schedule, for the Qwen3-1.7B shapes, the
GPU tests' shapes and edge cases, with and without the split schedule.

Invariants the kernel relies on:
  * every (tile, slab) unit is computed exactly once;
  * each pair's segments are in increasing unit order;
  * a segment that starts inside a tile is its pair's first segment of the
    split part (so it never waits on another pair before writing), and each
    pair writes at most one partial;
  * the pair holding a tile's first slab, when the tile is split, adds the
    partial sums of exactly the pairs holding the tile's other slabs (its
    loop skips pairs whose split range is empty);
  * without a workspace, with fewer than 32 slabs per tile, or when the last
    wave is at least 95% full, tiles are whole and assigned round-robin.
The invariants are checked with the least-work threshold at 0, so that the
split applies to the small shapes too; the default threshold is checked
separately.
"""
import pytest

import blockwise_fp8_pretraining_b200 as fp8

PAIRS = 74           # 148-SM B200, one CTA pair per two SMs

SHAPES = [
    # (M out rows, N out cols, K contraction): fprop / dgrad / wgrad of the
    # four Qwen3-1.7B linears over 8192 tokens
    (8192, 4096, 2048), (8192, 2048, 2048), (8192, 12288, 2048), (8192, 2048, 6144),
    (8192, 2048, 4096), (8192, 2048, 12288), (8192, 6144, 2048),
    (4096, 2048, 8192), (2048, 2048, 8192), (12288, 2048, 8192), (2048, 6144, 8192),
    # GPU test shapes and edges
    (128, 128, 128), (128, 384, 256), (256, 640, 512), (384, 256, 1152), (1280, 2304, 384),
    (4096, 2560, 256), (256, 256, 32768), (128, 256, 32768), (256, 128, 32768),
    (2048, 2048, 1152), (2560, 4096, 128), (256, 2048, 2048), (2048, 2048, 256),
]


def tiles_of(M, N):
    return ((M + 255) // 256) * ((N + 255) // 256)


@pytest.fixture(scope="module")
def lib():
    from blockwise_fp8_pretraining_b200 import build

    build.build()
    return fp8.load()


@pytest.fixture(autouse=True)
def _split_everywhere(lib):
    fp8.fp8_set_gemm_split_min_work(0)
    yield
    fp8.fp8_set_gemm_split_min_work(fp8.GEMM_SPLIT_MIN_WORK_DEFAULT)


@pytest.mark.parametrize("split", [False, True])
@pytest.mark.parametrize("M,N,K", SHAPES)
def test_schedule_invariants(lib, M, N, K, split):
    segs = fp8.fp8_selftest_gemm_schedule(M, N, K, PAIRS, split)
    T, nkb = tiles_of(M, N), K // 128
    covered = {}
    by_pair = {}
    for pair, tile, kb0, kb1, a0, a1 in segs:
        assert 0 <= tile < T and 0 <= kb0 < kb1 <= nkb and 0 <= pair < PAIRS
        for kb in range(kb0, kb1):
            assert (tile, kb) not in covered, f"unit ({tile}, {kb}) twice"
            covered[(tile, kb)] = pair
        by_pair.setdefault(pair, []).append((tile, kb0, kb1, a0, a1))
    assert len(covered) == T * nkb, "every unit computed"

    partial_writers = {}
    for pair, lst in by_pair.items():
        units = [t * nkb + kb0 for t, kb0, _, _, _ in lst]
        whole = [(t, kb0, kb1) for t, kb0, kb1, _, _ in lst if kb0 == 0 and kb1 == nkb]
        split_part = [x for x in lst if not (x[1] == 0 and x[2] == nkb)]
        # the whole tiles come first, then the split part in unit order
        assert units[len(whole):] == sorted(units[len(whole):])
        writers = [x for x in split_part if x[1] > 0]
        assert len(writers) <= 1
        if writers:
            assert split_part[0] == writers[0], "a partial is its pair's first split segment"
            partial_writers.setdefault(writers[0][0], []).append(pair)

    for pair, lst in by_pair.items():
        for tile, kb0, kb1, a0, a1 in lst:
            holders = sorted(p for (t, _), p in covered.items() if t == tile and p != pair)
            holders = sorted(set(holders))
            if kb0 == 0 and kb1 < nkb:
                # the loop runs over pairs a0 .. a1-1 and skips those whose
                # split range is empty: the rest are exactly the holders
                assert holders == partial_writers.get(tile, [])
                for r in range(a0, a1):
                    has_split_work = any(not (k0 == 0 and k1 == nkb) for _, k0, k1, _, _ in by_pair.get(r, []))
                    assert (r in holders) == has_split_work
                assert set(holders) <= set(range(a0, a1))
            else:
                assert a0 == a1
            if kb0 == 0 and kb1 == nkb:
                assert not holders

    if not split or nkb < 32:
        assert all(kb0 == 0 and kb1 == nkb for _, _, kb0, kb1, _, _ in segs)
        for pair, tile, *_ in segs:
            assert tile % min(T, PAIRS) == pair


@pytest.mark.parametrize("M,N,K", [(8192, 12288, 2048), (8192, 4096, 2048), (8192, 2048, 2048),
                                   (8192, 6144, 2048)])
def test_full_last_waves_keep_whole_tiles(lib, M, N, K):
    """At least 95% of the last wave busy, or fewer than 32 slabs per tile:
    no split even with a workspace."""
    segs = fp8.fp8_selftest_gemm_schedule(M, N, K, PAIRS, True)
    assert all(kb0 == 0 and kb1 == K // 128 for _, _, kb0, kb1, _, _ in segs)


@pytest.mark.parametrize("M,N,K", [(8192, 2048, 4096), (2048, 2048, 8192), (12288, 2048, 8192),
                                   (8192, 2048, 6144), (8192, 2048, 12288)])
def test_partial_last_waves_are_balanced(lib, M, N, K):
    """With the split schedule every pair gets work, and the busiest pair
    has at most one slab more than the split share plus its whole tiles."""
    segs = fp8.fp8_selftest_gemm_schedule(M, N, K, PAIRS, True)
    work = {}
    for pair, _, kb0, kb1, _, _ in segs:
        work[pair] = work.get(pair, 0) + kb1 - kb0
    assert len(work) == PAIRS
    assert max(work.values()) - min(work.values()) <= K // 128 + 1


def test_schedule_rejects_bad_sizes(lib):
    with pytest.raises(fp8.Fp8Error):
        fp8.fp8_selftest_gemm_schedule(100, 128, 128, PAIRS, True)


@pytest.mark.parametrize("M,N,K,splits", [
    (12288, 2048, 8192, True),      # gate_up wgrad: 332 units per pair
    (8192, 2048, 12288, True),      # gate_up dgrad: 332
    (8192, 2048, 6144, True),       # down fprop: 166
    (2048, 6144, 8192, True),       # down wgrad: 166
    (4096, 2048, 8192, False),      # qkv wgrad: 111
    (8192, 2048, 4096, False),      # qkv dgrad: 111
    (2048, 2048, 8192, False),      # o_proj wgrad: 55
    (1280, 2304, 4096, False),
])
def test_default_least_work_keeps_short_gemms_whole(lib, M, N, K, splits):
    fp8.fp8_set_gemm_split_min_work(fp8.GEMM_SPLIT_MIN_WORK_DEFAULT)
    segs = fp8.fp8_selftest_gemm_schedule(M, N, K, PAIRS, True)
    assert any(kb0 > 0 for _, _, kb0, _, _, _ in segs) == splits
    fp8.fp8_set_gemm_split_min_work(tiles_of(M, N) * (K // 128) // PAIRS + 1)
    assert all(kb0 == 0 for _, _, kb0, _, _, _ in fp8.fp8_selftest_gemm_schedule(M, N, K, PAIRS, True))
