"""The oracle's shape constants reproduce every figure the pages print about them.

Fixture: tests/golden/page_figures.txt (each line cites its page and section).
"""
import os

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
FULL_LAYERS, SLIDING_LAYERS, WINDOW = 23, 69, 512      # [P1] §长上下文第一道门: 3:1, 92 layers


def kv_bytes(tokens, elem_bytes=2):
    per_tok_layer = 2 * oracle.G * oracle.D * elem_bytes
    return per_tok_layer * (FULL_LAYERS * tokens + SLIDING_LAYERS * min(tokens, WINDOW))


def rows():
    with open(os.path.join(HERE, "golden", "page_figures.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                parts = line.split()
                yield parts[0], float(parts[1]), (int(parts[2]) if len(parts) > 2 else None)


def printed_precision(v):
    s = repr(v)
    return 10 ** -(len(s.split(".")[1])) / 2 if "." in s and not s.endswith(".0") else 0.5


def test_page_figures():
    seen = set()
    for name, value, arg in rows():
        seen.add(name)
        tol = printed_precision(value)
        if name == "kv_gib_fp16_whole":
            assert abs(kv_bytes(arg) / 2 ** 30 - value) <= tol, (name, arg)
        elif name == "kv_gib_fp16_per_1k":
            assert abs((kv_bytes(8192) - kv_bytes(7168)) / 2 ** 30 - value) <= tol
        elif name == "kv_bytes_per_token_full_layer":
            assert 2 * oracle.G * oracle.D * 2 == value
        elif name == "kv_gib_full_layers_1m":
            assert abs((1 << 20) * 2 * oracle.G * oracle.D * 2 * FULL_LAYERS / 2 ** 30 - value) <= tol
        elif name == "regions_1m":
            assert (1 << 20) // oracle.REGION == value
        elif name == "tokens_512_regions":
            assert 512 * oracle.REGION == value
        else:
            raise AssertionError(f"unknown fixture row {name}")
    assert len(seen) == 6
