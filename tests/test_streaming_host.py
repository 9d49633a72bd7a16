"""Host logic of the streaming summary update, against a token-by-token simulation of the
rule "a region is summarised when it holds 8 tokens; a shorter tail waits"
([P2] Step-5-Preview 如何实现1M长上下文 §区域压缩CSA)."""
import random

from sparse_long_context_dsa_b200.pipeline import due_regions
from sparse_long_context_dsa_b200 import workloads as W


def test_due_regions_match_a_simulation():
    rng = random.Random(3)
    lengths = [rng.randrange(1, 200) for _ in range(40)]
    summarised = [set(range(L // 8)) for L in lengths]          # complete regions at the start
    for step in range(30):
        pos = list(lengths)
        due = due_regions(pos)
        for b in range(len(lengths)):
            lengths[b] += 1
            complete = set(range(lengths[b] // 8))
            new = complete - summarised[b]
            assert (b in due) == bool(new)
            if new:
                assert new == {pos[b] // 8}                         # the query's own region
            summarised[b] = complete
            # no incomplete region is ever summarised
            assert all(8 * r + 8 <= lengths[b] for r in summarised[b])


def test_ragged_lengths_recipe():
    L = W.ragged_lengths(32, seed=1239)
    assert len(L) == 32 and min(L) >= 4096 - 8 and max(L) <= (1 << 20) - 8
    tails = {x % 8 for x in L}
    assert len(tails) > 3                                         # tails 0..7 occur
