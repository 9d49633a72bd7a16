"""Failure detection on the GPU without a fault, and host-side refusal of memory the GPU
cannot reach.

Every mbarrier wait in the library's kernels is bounded; a wait that runs out sets the
timeout bit of the per-device error word and lets the kernel return, so a stuck pipeline
becomes a status on the host and the context stays usable.  dsa_selftest_wait_timeout runs
one kernel whose barrier nothing completes (no copy, MMA or tensor memory in flight) with a
short bound; the error word must then report the timeout, and the next ordinary call must
work and leave the word clear.

Pageable host memory passed to a call (on a GPU that cannot read pageable memory) must be
refused on the host with DSA_ERR_INVALID_ARG before any kernel is launched: the call goes
through the C symbol directly, as a plain-C caller would, bypassing the Python checks.
"""
import ctypes

import numpy as np
import pytest
import torch

from sparse_long_context_dsa_b200 import dsa

pytestmark = pytest.mark.gpu


def test_a_wait_that_nothing_completes_gives_up_and_reports_it():
    dsa.check_device()                                   # start from a clear error word
    for limit in (100_000, 2_000_000):                   # ~50 us and ~1 ms at 1.9 GHz
        dsa.selftest_wait_timeout(limit)
        with pytest.raises(dsa.DsaError) as e:
            dsa.check_device()
        assert e.value.status == dsa.ERR_DEVICE
        assert "bounded wait timed out" in str(e.value)
        dsa.check_device()                               # the word was cleared by the read
    # the context is still usable: an ordinary call runs and flags nothing
    dev = torch.device("cuda")
    g = torch.Generator(device=dev)
    g.manual_seed(3)
    index_k = torch.randn((16, 4, 256), generator=g, device=dev).to(torch.bfloat16)
    S = torch.zeros((4, 2, 256), dtype=torch.uint8, device=dev)
    C = torch.zeros((4, 2), dtype=torch.float32, device=dev)
    src = torch.tensor([0, 8], dtype=torch.int64, device=dev)
    dst = torch.tensor([0, 1], dtype=torch.int64, device=dev)
    dsa.compress_regions(index_k, src, dst, S, C)
    dsa.check_device()
    assert torch.all(C > 0)


def _attr_pageable():
    from cuda.bindings import runtime as rt
    err, v = rt.cudaDeviceGetAttribute(rt.cudaDeviceAttr.cudaDevAttrPageableMemoryAccess, torch.cuda.current_device())
    assert err == rt.cudaError_t.cudaSuccess
    return bool(v)


def test_pageable_host_memory_is_refused_before_any_launch():
    if _attr_pageable():
        pytest.skip("this GPU reads pageable host memory: such pointers are valid here")
    L = dsa.lib()
    host = np.arange(4096, dtype=np.uint8)                      # plain numpy: pageable memory
    hp = ctypes.c_void_p(host.ctypes.data)
    dev = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert L.dsa_copy(ctypes.c_void_p(dev.data_ptr()), hp, 4096, st) == dsa.ERR_INVALID_ARG
    assert "pageable" in L.dsa_last_error().decode()
    assert L.dsa_copy(hp, ctypes.c_void_p(dev.data_ptr()), 4096, st) == dsa.ERR_INVALID_ARG
    # an attention call whose output is pageable host memory
    nq = 1
    q = torch.zeros((nq, 64, 192), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((1, 4, 64, 192), dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros((1, 1), dtype=torch.int32, device="cuda")
    pos = torch.zeros((1,), dtype=torch.int32, device="cuda")
    sel = torch.zeros((1, 4, 1), dtype=torch.int32, device="cuda")
    cnt = torch.ones((1, 4), dtype=torch.int32, device="cuda")
    out_host = np.zeros(64 * 192 * 2, dtype=np.uint8)
    P = ctypes.c_void_p
    r = L.dsa_sparse_attn_decode(P(q.data_ptr()), P(kc.data_ptr()), P(kc.data_ptr()), 1, P(bt.data_ptr()), 1,
                                 P(pos.data_ptr()), 1, P(sel.data_ptr()), P(cnt.data_ptr()), 1,
                                 P(out_host.ctypes.data), None, None, 0, st)
    assert r == dsa.ERR_INVALID_ARG and "out" in L.dsa_last_error().decode()
    torch.cuda.synchronize()
    dsa.check_device()
    assert torch.all(dev == 0)                                  # nothing was copied
    assert np.all(out_host == 0)


def test_pinned_host_memory_is_accepted():
    host = torch.arange(256, dtype=torch.int32).to(torch.uint8).pin_memory()
    dev = torch.zeros(256, dtype=torch.uint8, device="cuda")
    dsa.copy(dev, host)
    torch.cuda.synchronize()
    dsa.check_device()
    assert torch.equal(dev.cpu(), host)
