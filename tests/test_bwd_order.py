"""The backward kernel's CTA launch order, read through gqa_testing_bwd_order (host only, no
GPU): every (pair, key block) exactly once, chunks of pairs whose fp32 dQ rows fit the L2
budget, longest key blocks first inside a chunk, and a greedy list schedule over 148 SMs that
comes close to the ideal makespan where the plain pair-major order does not."""
import ctypes
import heapq

import pytest

CHUNK_BUDGET = 72 * 1024 * 1024
N_SM = 148


@pytest.fixture(scope="module")
def lib():
    import grouped_query_softmax_b200 as m
    return ctypes.CDLL(m.library_path())


def order(lib, n_kb, n_bg, G, Tq, D):
    n = n_kb * n_bg
    chunk = ctypes.c_int(-1)
    bg = (ctypes.c_int * n)()
    j = (ctypes.c_int * n)()
    st = lib.gqa_testing_bwd_order(n_kb, n_bg, G, Tq, D, ctypes.byref(chunk), bg, j)
    assert st == 0
    return chunk.value, list(bg), list(j)


SHAPES = [
    # n_kb, n_bg, G, Tq, D
    (32, 32, 4, 4096, 128),    # GQA prefill B4 Hkv8 T4096
    (256, 1, 32, 32768, 128),  # MQA long prefill
    (3, 4, 4, 300, 128),
    (7, 6, 2, 900, 64),
    (1, 1, 1, 1, 64),
    (5, 7, 3, 600, 128),       # a prime number of pairs
]


@pytest.mark.parametrize("shape", SHAPES, ids=[str(s) for s in SHAPES])
def test_order_is_a_chunked_longest_first_permutation(lib, shape):
    n_kb, n_bg, G, Tq, D = shape
    chunk, bg, j = order(lib, n_kb, n_bg, G, Tq, D)
    assert sorted(zip(bg, j)) == [(b, k) for b in range(n_bg) for k in range(n_kb)]
    assert n_bg % chunk == 0
    per_pair = G * Tq * D * 4
    assert chunk == 1 or chunk * per_pair <= CHUNK_BUDGET
    # the largest such divisor
    assert all(n_bg % c or c * per_pair > CHUNK_BUDGET for c in range(chunk + 1, n_bg + 1))
    for L in range(1, len(bg)):
        c_prev, c_cur = bg[L - 1] // chunk, bg[L] // chunk
        assert c_cur >= c_prev
        if c_cur == c_prev:
            assert j[L] >= j[L - 1]


def test_chunk_of_the_gqa_prefill_shape(lib):
    assert order(lib, 32, 32, 4, 4096, 128)[0] == 8


def makespan(work):
    sms = [0] * N_SM
    for w in work:
        heapq.heappush(sms, heapq.heappop(sms) + w)
    return max(sms)


def test_greedy_schedule_of_the_gqa_prefill_shape(lib):
    n_kb, n_bg, G = 32, 32, 4
    _, bg, j = order(lib, n_kb, n_bg, G, 4096, 128)
    steps = lambda k: G * (n_kb - k)  # block k walks the query tiles k .. n_kb - 1 of G heads
    ideal = n_bg * sum(steps(k) for k in range(n_kb)) / N_SM
    ours = makespan([steps(k) for k in j])
    pair_major = makespan([steps(k) for b in range(n_bg) for k in range(n_kb)])
    assert ours <= 1.02 * ideal
    assert pair_major >= 1.1 * ideal


@pytest.mark.parametrize("args", [(0, 1, 1, 1, 64), (1, 0, 1, 1, 64), (1, 1, 0, 1, 64), (1, 1, 1, 0, 64),
                                  (1, 1, 1, 1, 0)])
def test_bad_sizes_are_rejected(lib, args):
    chunk = ctypes.c_int(0)
    a = (ctypes.c_int * 1)()
    assert lib.gqa_testing_bwd_order(*args, ctypes.byref(chunk), a, a) == 1
