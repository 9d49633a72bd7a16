"""GPU region compression (A1) against the oracle: bytes and scales bit-exact."""
import numpy as np
import pytest
import torch

import oracle
from sparse_long_context_dsa_b200 import dsa
from sparse_long_context_dsa_b200 import workloads as W

from _util import bits

pytestmark = pytest.mark.gpu
G, DI = 4, 256


def run_both(index_k, src, dst, n_slots):
    dev = index_k.device
    S = torch.zeros((G, n_slots, DI), dtype=torch.uint8, device=dev)
    C = torch.zeros((G, n_slots), dtype=torch.float32, device=dev)
    dsa.compress_regions(index_k, torch.tensor(src, dtype=torch.int64, device=dev),
                         torch.tensor(dst, dtype=torch.int64, device=dev), S, C)
    dsa.check_device()
    ik = bits(index_k)
    So, Co = oracle.compress_regions(ik.reshape(ik.shape[0], -1), src, dst, n_slots)
    return S.cpu().numpy(), C.cpu().numpy(), So, Co


@pytest.mark.parametrize("n_tokens", [8, 64 * 8 + 5, 40000])
def test_bit_exact_random(n_tokens):
    gen = W.generator(11 + n_tokens, "cuda")
    ik = W.normal_bf16((n_tokens, G, DI), gen, "cuda")
    n = n_tokens // 8
    S, C, So, Co = run_both(ik, [8 * r for r in range(n)], list(range(n)), n)
    assert np.array_equal(C, Co)
    assert np.array_equal(S, So)


def test_bit_exact_special_regions_and_scattered_slots():
    gen = W.generator(3, "cuda")
    ik = W.normal_bf16((96, G, DI), gen, "cuda")
    ik[8:16] = 0                                   # all-zero region -> scale 0
    ik[16:24] = ik[16:17].clone()                  # identical tokens -> mean is the token
    ik[24:32] *= 1e-30                             # tiny values (fp32 subnormal scale range)
    ik[32:40] *= 1e30                              # huge values
    src = [88, 0, 8, 16, 24, 32, 40, 3]            # unaligned region start too
    dst = [0, 9, 2, 7, 5, 1, 11, 4]
    S, C, So, Co = run_both(ik, src, dst, 12)
    assert np.array_equal(C, Co) and np.array_equal(S, So)
    assert np.all(C[:, 2] == 0) and np.all(S[:, 2] == 0)


def test_row_stride_wider_than_a_token():
    gen = W.generator(4, "cuda")
    wide = W.normal_bf16((64, G * DI + 256), gen, "cuda")
    src, dst = [0, 8, 40], [2, 0, 1]
    dev = wide.device
    S = torch.zeros((G, 3, DI), dtype=torch.uint8, device=dev)
    C = torch.zeros((G, 3), dtype=torch.float32, device=dev)
    dsa.compress_regions(wide, torch.tensor(src, device=dev), torch.tensor(dst, device=dev), S, C)
    dsa.check_device()
    So, Co = oracle.compress_regions(bits(wide), src, dst, 3)
    assert np.array_equal(S.cpu().numpy(), So) and np.array_equal(C.cpu().numpy(), Co)


def test_out_of_range_indices_are_flagged_and_skipped():
    gen = W.generator(5, "cuda")
    ik = W.normal_bf16((32, G, DI), gen, "cuda")
    S = torch.full((G, 4, DI), 0x55, dtype=torch.uint8, device="cuda")
    C = torch.zeros((G, 4), dtype=torch.float32, device="cuda")
    dsa.compress_regions(ik, torch.tensor([0, 30], device="cuda"), torch.tensor([1, 2], device="cuda"), S, C)
    with pytest.raises(dsa.DsaError) as e:
        dsa.check_device()
    assert e.value.status == dsa.ERR_DEVICE
    assert np.all(S[:, 2].cpu().numpy() == 0x55)          # the bad region wrote nothing
    So, Co = oracle.compress_regions(bits(ik), [0], [1], 4)
    assert np.array_equal(S[:, 1].cpu().numpy(), So[:, 1])
    dsa.check_device()                                    # the error word was cleared
