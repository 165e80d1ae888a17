"""Host-side arithmetic of bench.py that its JSON line reports."""
import bench


def test_step_launches_match_the_launch_lists():
    # one step on the Wan layer: reorder, pool, score, cut, head scan,
    # finalize, attention, unreorder (profiles/launches_wan.md)
    assert bench.step_launches(1, 40, 308) == 8
    # the Hunyuan layer forms its pooled scores in four chunks of six heads,
    # so score and cut launch four times each (profiles/launches_hunyuan.md)
    assert bench.step_launches(1, 24, 1020) == 14
    # at the block limit (1024 blocks: 8 MiB of scores per head, six heads
    # per 48 MiB chunk) 14 heads take three chunks
    assert bench.step_launches(2, 7, 1024) == 6 + 2 * 3
