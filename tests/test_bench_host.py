"""Host logic of bench.py (CPU): the end-to-end pipeline's chunking."""
import importlib.util
import os

import pytest

_spec = importlib.util.spec_from_file_location(
    "bench_module", os.path.join(os.path.dirname(os.path.dirname(__file__)), "bench.py"))
bench = importlib.util.module_from_spec(_spec)
_spec.loader.exec_module(bench)


@pytest.mark.parametrize("B,H", [(2, 16), (1, 1), (1, 3), (4, 8), (2, 32), (3, 5), (1, 64)])
def test_e2e_chunks_cover_every_head_once_in_order(B, H):
    chunks = bench.e2e_chunks(B, H)
    heads = [(b, h) for b, h0, h1 in chunks for h in range(h0, h1)]
    assert heads == [(b, h) for b in range(B) for h in range(H)]
    for b, h0, h1 in chunks:  # a chunk stays inside one batch item
        assert 0 <= h0 < h1 <= H and 0 <= b < B


def test_e2e_chunks_shrink_towards_the_end():
    # the exposed tail (the last chunk's compute and copy back) is one head; the
    # sizes before it never grow
    for B, H in [(2, 16), (4, 8), (2, 32), (1, 64)]:
        sizes = [h1 - h0 for _, h0, h1 in bench.e2e_chunks(B, H)]
        assert sizes[-1] == 1
        assert len(sizes) <= 2 * (B * H).bit_length() + B
    assert [h1 - h0 for _, h0, h1 in bench.e2e_chunks(2, 16)] == [16, 8, 4, 2, 1, 1]
