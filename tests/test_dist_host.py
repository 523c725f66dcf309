"""Host logic of the multi-process schemes on CPU: the head chunks of each rank and the HCMS stages."""
import pytest

from sequence_head_attention_b200.dist import rank_chunks, stage_bounds


def test_rank_chunks_cut_at_rank_boundaries():
    # the video-DiT chunks [3, 7, 10, 10, 10] over 4 ranks of 10 heads: rank 0 runs [3, 7], the others [10]
    assert rank_chunks([3, 7, 10, 10, 10], 40, 4) == [[3, 7], [10], [10], [10]]
    # a chunk straddling a boundary is cut there
    assert rank_chunks([6, 2], 8, 2) == [[4], [2, 2]]
    assert rank_chunks([8], 8, 4) == [[2], [2], [2], [2]]
    for chunks, H, P in (([1, 3], 4, 2), ([5, 11, 16], 32, 4), ([40], 40, 8)):
        per = rank_chunks(chunks, H, P)
        assert all(sum(r) == H // P for r in per)
        assert [c for r in per for c in r if c] and sum(sum(r) for r in per) == H


@pytest.mark.parametrize("n,stages,want", [
    (10, 1, [(0, 10)]), (10, 2, [(0, 5), (5, 10)]), (10, 3, [(0, 4), (4, 7), (7, 10)]),
    (5, 8, [(0, 1), (1, 2), (2, 3), (3, 4), (4, 5)]), (1, 3, [(0, 1)]), (7, 0, [(0, 7)]),
])
def test_stage_bounds_cover_the_heads_in_order(n, stages, want):
    assert stage_bounds(n, stages) == want
