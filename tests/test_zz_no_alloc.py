"""The allocation-free top-k entry point (dsa_topk_regions_noalloc) against the regular one.

Some callers cannot allocate device memory when they select regions (a serving runtime
whose pool already owns the device memory, a plain-C host with no allocator of its own).
For them the library keeps the top-k scratch in one static per-GPU array.  This file runs
last so that a failure here leaves every other result already reported; it must pass
both alone in a fresh process and after the other tests.  The selection is integer work,
so the two entry points must agree exactly, on two calls in a row (the static array keeps
the first call's contents, which the second call must not depend on), and both must equal
the CPU oracle's selection on the same scores.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_long_context_dsa_b200 import dsa

pytestmark = pytest.mark.gpu
G = 4


def indexer_like_scores(seed, nq, ld):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    d = torch.randn((nq, G, 4, ld), generator=g, device="cuda") * 5.6
    z = torch.rand((nq, G, 4, 1), generator=g, device="cuda")
    return ((torch.relu(d) * z).sum(dim=2) / 16).contiguous()


def regular_and_static(scores, q_pos, k):
    nq = scores.shape[0]
    a_idx, a_cnt = dsa.topk_regions(scores, q_pos, k)
    b_idx = torch.full((nq, G, k), 7, dtype=torch.int32, device="cuda")
    b_cnt = torch.full((nq, G), 7, dtype=torch.int32, device="cuda")
    dsa.topk_regions_noalloc(scores, q_pos, k, b_idx, b_cnt)
    dsa.check_device()
    return a_idx.cpu(), a_cnt.cpu(), b_idx.cpu(), b_cnt.cpu()


def oracle_selection(scores, q_pos, k):
    idx, cnt = oracle.topk_regions(scores.cpu().numpy(), q_pos.cpu().numpy(), k)
    return torch.from_numpy(np.ascontiguousarray(idx)), torch.from_numpy(np.ascontiguousarray(cnt))


def test_two_calls_in_a_row_match_the_workspace_entry_point_and_the_oracle():
    # call 1: a 1M-token decode row set (4 groups x 131,071 regions); call 2: a batch of
    # shorter rows with heavy ties, which would expose stale candidates or counters
    s1 = indexer_like_scores(1, 1, 131071)
    p1 = torch.tensor([8 * 131072 - 1], dtype=torch.int32, device="cuda")
    a, ac, b, bc = regular_and_static(s1, p1, 512)
    assert torch.equal(ac, bc) and torch.equal(a, b)
    assert int(bc.min()) == 512
    oi, oc = oracle_selection(s1, p1, 512)
    assert torch.equal(bc, oc) and torch.equal(b, oi)

    s2 = torch.randint(0, 3, (3, G, 20000), device="cuda").float()
    p2 = torch.tensor([8 * 20000, 8 * 9000 + 5, 8 * 300], dtype=torch.int32, device="cuda")
    a, ac, b, bc = regular_and_static(s2, p2, 512)
    assert torch.equal(ac, bc) and torch.equal(a, b)
    oi, oc = oracle_selection(s2, p2, 512)
    assert torch.equal(bc, oc) and torch.equal(b, oi)


def test_oversized_call_is_rejected_with_a_clear_error():
    need = dsa.lib().dsa_topk_workspace_size(8, 131071, 512)
    assert need > (8 << 20)
    s = torch.zeros((8, G, 131071), dtype=torch.float32, device="cuda")
    p = torch.full((8,), 8 * 131072 - 1, dtype=torch.int32, device="cuda")
    idx = torch.empty((8, G, 512), dtype=torch.int32, device="cuda")
    cnt = torch.empty((8, G), dtype=torch.int32, device="cuda")
    with pytest.raises(dsa.DsaError) as e:
        dsa.topk_regions_noalloc(s, p, 512, idx, cnt)
    assert e.value.status == dsa.ERR_UNSUPPORTED
    assert "static buffer" in str(e.value)
