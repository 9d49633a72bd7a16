"""Host logic of the window layers' ring buffers (pipeline.ring_block_table): each request owns
ring_pages physical pages, and with 64-token pages a token's slot is shared exactly with the
tokens 512 apart, so the newest token overwrites the one that just left its 512-token window
([P2] Step-5-Preview 如何实现1M长上下文 §第一招: the window layers' ring buffer)."""
import numpy as np

from sparse_long_context_dsa_b200 import pipeline

PAGE = 64


def slot(bt, b, t):
    return int(bt[b, t // PAGE]) * PAGE + t % PAGE


def test_each_request_owns_its_ring():
    bt = pipeline.ring_block_table(5, 300, ring_pages=8, device="cpu").numpy()
    assert bt.shape == (5, 300) and bt.dtype == np.int32
    for b in range(5):
        assert set(bt[b].tolist()) == set(range(8 * b, 8 * b + 8))


def test_slots_repeat_every_512_tokens_and_only_then():
    bt = pipeline.ring_block_table(3, 2048, ring_pages=8, device="cpu").numpy()
    rng = np.random.default_rng(0)
    for b in range(3):
        for t in rng.integers(512, 2048 * PAGE, 50):
            t = int(t)
            s = slot(bt, b, t)
            assert s == slot(bt, b, t - 512)
            window = {slot(bt, b, u) for u in range(t - 511, t + 1)}
            assert len(window) == 512                   # the window's tokens all in distinct slots
    # no two requests share a slot
    assert not ({slot(bt, 0, t) for t in range(512)} & {slot(bt, 1, t) for t in range(512)})
