"""Small conversions shared by the tests (no method arithmetic)."""
import numpy as np
import torch


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> uint16 numpy array of its bit patterns (any device)."""
    assert t.dtype == torch.bfloat16
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def from_bits(b: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16)


def f64(t_bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float64 values (exact)."""
    u = np.ascontiguousarray(t_bits).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def bf16_from_bits_np(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float32 values."""
    return (np.ascontiguousarray(b).astype(np.uint32) << 16).view(np.float32)


def selection_differs_only_near_threshold(sel_a, cnt_a, sel_b, cnt_b, scores, q_pos, k, rel=1e-3):
    """Checks that two selections (ascending indices, counts) of the same rows agree
    except for regions whose oracle score is within `rel` (relative) of the score of
    the last selected eligible region (the (k-1)-th best).  Returns the number of rows
    that differ."""
    nq = sel_a.shape[0]
    differ = 0
    for i in range(nq):
        own = int(q_pos[i]) // 8
        for g in range(sel_a.shape[1]):
            ca, cb = int(cnt_a[i, g]), int(cnt_b[i, g])
            assert ca == cb == min(k, own + 1), (i, g, ca, cb)
            A = set(sel_a[i, g, :ca].tolist())
            Bs = set(sel_b[i, g, :cb].tolist())
            assert own in A and own in Bs
            if A == Bs:
                continue
            differ += 1
            row = scores[i, g, :own].astype(np.float64)
            order = np.lexsort((np.arange(own), -row))
            thr = row[order[min(k - 1, own) - 1]]
            for r in A ^ Bs:
                assert abs(row[r] - thr) <= rel * abs(thr), (i, g, r, row[r], thr)
    return differ
