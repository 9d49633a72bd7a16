"""The product path has no CPU fallback: host tensors are refused before any work, and a
missing library is an import error, not a silent switch to other code."""
import pytest
import torch

from sparse_long_context_dsa_b200 import dsa


def test_host_tensors_are_refused():
    scores = torch.zeros((2, 4, 100), dtype=torch.float32)
    q_pos = torch.tensor([799, 10], dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        dsa.topk_regions(scores, q_pos, 16)
    q = torch.zeros((2, 64, 192), dtype=torch.bfloat16)
    cache = torch.zeros((4, 4, 64, 192), dtype=torch.bfloat16)
    bt = torch.zeros((1, 4), dtype=torch.int32)
    sel = torch.zeros((2, 4, 16), dtype=torch.int32)
    cnt = torch.ones((2, 4), dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        dsa.sparse_attn_decode(q, cache, cache, bt, q_pos, sel, cnt)


def test_missing_library_is_an_import_error(monkeypatch, tmp_path):
    monkeypatch.setattr(dsa, "_lib", None)
    monkeypatch.setattr(dsa, "LIB_PATH", str(tmp_path / "libdsa.so"))
    with pytest.raises(ImportError, match="missing"):
        dsa.lib()
