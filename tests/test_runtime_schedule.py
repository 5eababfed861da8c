"""Host logic of the step schedules (no GPU).

Step-dLLM (abstract): the mask is rebuilt at anchor steps, every `anchor_every`
steps from step 0, and reused in between.  SparseD (abstract), a prior method
the Step-dLLM abstract compares against: dense attention in the early steps,
then one mask, computed once, reused for every remaining step.
"""
from block_sparse_attention_sdl_b200.runtime import anchor_of, is_anchor, is_dense


def test_step_dllm_anchors_every_interval():
    anchors = [s for s in range(256) if is_anchor(s, 32)]
    assert anchors == list(range(0, 256, 32))
    assert all(not is_dense(s) for s in range(256))
    assert [anchor_of(s, 32) for s in (0, 1, 31, 32, 33, 255)] == [0, 0, 0, 32, 32, 224]


def test_sparsed_dense_warmup_then_one_mask():
    n = 32
    assert [s for s in range(256) if is_dense(s, n)] == list(range(n))
    assert [s for s in range(256) if is_anchor(s, None, n)] == [n]
    assert [anchor_of(s, None, n) for s in (0, 31, 32, 33, 255)] == [None, None, n, n, n]


def test_interval_after_warmup():
    """Periodic refresh after a dense warm-up (both knobs together)."""
    assert [s for s in range(40) if is_anchor(s, 8, 4)] == [4, 12, 20, 28, 36]
    assert anchor_of(11, 8, 4) == 4 and anchor_of(12, 8, 4) == 12
