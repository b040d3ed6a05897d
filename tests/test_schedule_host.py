"""The tensor-core attention kernel's unit schedule, checked on the host
through infini_attn_schedule_check (the kernel's own map, compiled for the
host): every (segment, query tile) pair is taken by exactly one CTA, and the
key tiles per CTA are balanced."""
import pytest

from compressive_memory_segment_b200 import binding as bd

SEGMENTS = list(range(1, 41)) + [64, 111, 128, 256, 1000, 2048, 4096]


@pytest.mark.parametrize("n_qt", [1, 2, 3, 4, 8, 16])
@pytest.mark.parametrize("grid", [148, 132, 37, 7, 1])
def test_every_unit_taken_once(n_qt, grid):
    for n_seg in SEGMENTS:
        rc, _ = bd.infini_attn_schedule_check(n_seg, n_qt, grid)
        assert rc == 0, (n_seg, n_qt, grid)


@pytest.mark.parametrize("n_seg,n_qt", [
    (4096, 16),   # 1M tokens, 8 heads, N = 2048
    (128, 16),    # one call of 8192 tokens, 32 heads, N = 2048
    (2048, 8),    # 8K tokens, 16 x 16 heads, N = 1024
    (256, 16),    # the 64K profiling case
])
def test_workloads_are_balanced(n_seg, n_qt):
    rc, ratio = bd.infini_attn_schedule_check(n_seg, n_qt, 148)
    assert rc == 0
    assert ratio <= 1.02, ratio


def test_busiest_cta_within_one_unit_of_its_share():
    # Units cannot be split, so the best any schedule can promise is that the
    # busiest CTA exceeds the mean by less than one unit of the largest size
    # (n_qt key tiles); the balanced map keeps that for every shape here,
    # partial groups and odd tile counts included.
    for grid in (148, 132, 37, 7):
        for n_qt in (1, 2, 3, 4, 8, 16):
            for n_seg in list(range(1, 80)) + [100, 300, 1000, 1111, 2048, 4096]:
                rc, ratio = bd.infini_attn_schedule_check(n_seg, n_qt, grid)
                assert rc == 0
                G = min(grid, n_seg * n_qt)
                mean = n_seg * n_qt * (n_qt + 1) / 2 / G
                assert (ratio - 1.0) * mean < n_qt, (grid, n_qt, n_seg, ratio)


def test_bad_arguments():
    assert bd.infini_attn_schedule_check(0, 16, 148)[0] == bd.INFINI_ERR_SHAPE
    assert bd.infini_attn_schedule_check(4, 0, 148)[0] == bd.INFINI_ERR_SHAPE
    assert bd.infini_attn_schedule_check(4, 16, 0)[0] == bd.INFINI_ERR_SHAPE
    assert bd.infini_attn_schedule_check(1 << 21, 16, 148)[0] == bd.INFINI_ERR_SHAPE
