"""The chunk plan of gqa_attn_fwd_host, read through gqa_testing_fwd_host_plan (host only, no
GPU): the chunks tile the query rows in order with whole 128-row tiles (at most 8 chunks, at
least 256 rows each unless the suffix is shorter), each chunk reads exactly the keys its last
row sees, so the keys it needs beyond the previous chunk's are the ones the host call copies
next and every key is copied once."""
import ctypes

import pytest


@pytest.fixture(scope="module")
def lib():
    import grouped_query_softmax_b200 as m
    return ctypes.CDLL(m.library_path())


def plan(lib, B, Hq, Hkv, Tq, Tk, D):
    n = ctypes.c_int(-1)
    r0, rows, keys = (ctypes.c_int * 8)(), (ctypes.c_int * 8)(), (ctypes.c_int * 8)()
    assert lib.gqa_testing_fwd_host_plan(B, Hq, Hkv, Tq, Tk, D, ctypes.byref(n), r0, rows, keys) == 0
    return [(r0[c], rows[c], keys[c]) for c in range(n.value)]


SHAPES = [
    (4, 32, 8, 4096, 4096, 128),
    (1, 32, 1, 32768, 32768, 128),
    (8, 16, 16, 512, 8192, 128),
    (2, 8, 2, 1000, 1000, 128),
    (1, 4, 1, 700, 1900, 128),
    (3, 6, 2, 200, 200, 64),
    (1, 4, 2, 1, 513, 64),
    (1, 4, 2, 257, 300, 64),
]


@pytest.mark.parametrize("shape", SHAPES, ids=[str(s) for s in SHAPES])
def test_chunks_tile_the_rows_and_read_each_key_once(lib, shape):
    B, Hq, Hkv, Tq, Tk, D = shape
    chunks = plan(lib, *shape)
    assert 1 <= len(chunks) <= 8
    at = 0
    for c, (r0, rows, keys) in enumerate(chunks):
        assert r0 == at and rows > 0
        if c < len(chunks) - 1:
            assert rows % 128 == 0 and rows >= min(256, Tq)
        assert keys == Tk - Tq + r0 + rows  # the keys the chunk's last row sees
        at += rows
    assert at == Tq
    ks = [k for _, _, k in chunks]
    assert ks == sorted(ks) and ks[-1] == Tk  # keys only grow; every key is copied once in total
    if Tq >= 8 * 256:
        assert len(chunks) == 8


@pytest.mark.parametrize("args", [(0, 4, 2, 8, 8, 64), (1, 3, 2, 8, 8, 64), (1, 4, 2, 9, 8, 64),
                                  (1, 4, 2, 8, 8, 96)])
def test_bad_sizes_are_rejected(lib, args):
    n = ctypes.c_int(0)
    a = (ctypes.c_int * 8)()
    assert lib.gqa_testing_fwd_host_plan(*args, ctypes.byref(n), a, a, a) == 1
