"""dsa_copy (kernel byte copy over unified addressing) and a decode step staged from pinned
host memory with its output written to pinned host memory: the same bytes as the device
path."""
import numpy as np
import pytest
import torch

from sparse_long_context_dsa_b200 import dsa, pipeline
from sparse_long_context_dsa_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n", [1, 15, 16, 4096 + 7, 49664, 1 << 22, (1 << 26) + 37])
def test_copy_between_pinned_host_and_device(n):
    rng = np.random.default_rng(n)
    host = torch.from_numpy(rng.integers(0, 256, n, dtype=np.uint8)).pin_memory()
    dev = torch.zeros(n, dtype=torch.uint8, device="cuda")
    dsa.copy(dev, host)
    back = torch.zeros(n, dtype=torch.uint8).pin_memory()
    dsa.copy(back, dev)
    torch.cuda.synchronize()
    dsa.check_device()
    assert torch.equal(dev.cpu(), host) and torch.equal(back, host)
    # unaligned views (the scalar path)
    if n > 3:
        d2 = torch.zeros(n - 3, dtype=torch.uint8, device="cuda")
        dsa.copy(d2, host[3:])
        torch.cuda.synchronize()
        assert torch.equal(d2.cpu(), host[3:])


def test_copy_rejects_pageable_memory():
    with pytest.raises(ValueError):
        dsa.copy(torch.zeros(8, dtype=torch.uint8, device="cuda"), torch.zeros(8, dtype=torch.uint8))


def test_decode_step_from_pinned_inputs_to_pinned_output():
    dev = torch.device("cuda")
    lengths = [20000, 4099]
    d = W.decode_batch(lengths, seed=71, device=dev, permute=True)
    S = torch.zeros((4, d["n_slots"], 256), dtype=torch.uint8, device=dev)
    C = torch.zeros((4, d["n_slots"]), dtype=torch.float32, device=dev)
    pipeline.compress_all(d["index_k"], d["lengths"], d["tok_base"], d["sum_base"], S, C)
    ld = max(lengths) // 8
    st = pipeline.DecodeStep(S, C, d["sum_base"], d["block_table"], d["k_cache"], d["v_cache"], ld, k=512)
    st.load(d["index_q"], d["gate"], d["q"], d["q_pos"])
    ref = st.run().clone()
    host_arena = st.arena.cpu().pin_memory()
    st.arena.zero_()
    host_out = torch.zeros_like(ref, device="cpu").pin_memory()
    st.stage(host_arena)
    st.run(out=host_out)
    torch.cuda.synchronize()
    dsa.check_device()
    assert torch.equal(host_out, ref.cpu())
