"""The split plan of gqa_attn_fwd_split, read through gqa_testing_fwd_split_plan (host only, no
GPU): which launches deal their last wave's key tiles out over the SMs, in how many slices, and
that every split is worth it by the plan's own estimate."""
import ctypes

import pytest


@pytest.fixture(scope="module")
def lib():
    import grouped_query_softmax_b200 as m
    return ctypes.CDLL(m.library_path())


def plan(lib, B, Hq, Hkv, Tq, Tk, D=128, window=0, sms=148):
    slices = ctypes.c_int(-1)
    whole, split, units = ctypes.c_longlong(-1), ctypes.c_longlong(-1), ctypes.c_longlong(-1)
    st = lib.gqa_testing_fwd_split_plan(B, Hq, Hkv, Tq, Tk, D, window, sms, ctypes.byref(slices),
                                        ctypes.byref(whole), ctypes.byref(split), ctypes.byref(units))
    assert st == 0
    return slices.value, whole.value, split.value, units.value


def units_of(B, Hq, Hkv, Tq):
    G = Hq // Hkv
    n_qt = (Tq + 127) // 128
    return B * Hkv * (G // 2) * n_qt if G % 2 == 0 else B * Hq * ((n_qt + 1) // 2)


PIECE_COST = 5.0  # a piece's fixed cost in key tiles, as the plan counts it
GAIN = 0.95       # a split must beat the unsplit estimate by this factor


def estimate(n, full, r, slices):
    """Makespan in key tiles: whole waves, then the busiest slice of the last r units' tiles
    (one piece when slices is a multiple of r, else up to two); slices = 0: no split."""
    if slices == 0:
        return (full + 1) * n
    return full * n + r * n / slices + PIECE_COST * (1 if slices % r == 0 else 2)


def test_small_suffix_launches_split(lib):
    # 12 units of 15 key tiles on 148 SMs: 84 slices, 7 per unit, none crossing a unit
    assert plan(lib, 1, 4, 1, 700, 1900) == (84, 0, 12, 12)
    # B8 H16/16, T_q 512 over T_k 8192: 256 units of 64 tiles on 148 SMs (1.73 waves); the
    # first 148 run whole, the other 108 units' tiles go out in 148 runs of about 47 tiles
    assert plan(lib, 8, 16, 16, 512, 8192) == (148, 148, 108, 256)
    # B2 H32/8, T_q 256 over T_k 32768: 64 units of 256 tiles, all dealt out over 148 SMs
    assert plan(lib, 2, 32, 8, 256, 32768) == (148, 0, 64, 64)


@pytest.mark.parametrize("shape", [
    (4, 32, 8, 4096, 4096),     # T_q = T_k: unequal units, ordered longest first instead
    (1, 32, 1, 32768, 32768),
    (8, 16, 16, 512, 8192, 128, 1024),   # a window: not split
    (2, 16, 16, 900, 1500),     # prefix shorter than the suffix
    (37, 8, 8, 512, 8192),      # 148 units: whole waves only
    (1, 2, 2, 128, 384),        # 3 key tiles: too few to cut
])
def test_launches_that_do_not_split(lib, shape):
    slices, whole, split, units = plan(lib, *shape)
    assert slices == 0 and split == 0 and whole == units


@pytest.mark.parametrize("shape", [
    (8, 16, 16, 512, 8192), (1, 4, 1, 700, 1900), (2, 16, 16, 512, 4096), (1, 8, 8, 1024, 2048), (4, 16, 16, 256, 8192),
    (3, 12, 4, 384, 9000, 64), (5, 32, 8, 1000, 4000), (1, 2, 2, 128, 640), (2, 32, 8, 256, 32768),
])
@pytest.mark.parametrize("sms", [148, 132, 20])
def test_plan_invariants(lib, shape, sms):
    B, Hq, Hkv, Tq, Tk = shape[:5]
    slices, whole, split, units = plan(lib, *shape, sms=sms)
    assert units == units_of(B, Hq, Hkv, Tq)
    assert whole + split == units
    n = (Tk - 1) // 128 + 1
    full, r = divmod(units, sms)
    if slices == 0:
        assert split == 0
        return
    assert split == r and whole == full * sms        # only the last wave is cut
    top = min(sms, r * n // 2, 29 * r)
    assert r <= slices <= top                        # a run crosses at most one unit boundary
    # runs come in lanes of the units of one head when the whole units fill whole heads
    G, n_qt = Hq // Hkv, (Tq + 127) // 128
    group = n_qt if G % 2 == 0 else (n_qt + 1) // 2
    if (full * sms) % group:
        group = 1
    assert slices % group == 0
    costs = {s: estimate(n, full, r, s) for s in range(r, top + 1) if s % group == 0}
    assert estimate(n, full, r, slices) == min(costs.values())   # the best slice count
    assert estimate(n, full, r, slices) <= GAIN * estimate(n, full, r, 0)   # and worth the merge


def test_rejects_bad_arguments(lib):
    k, a, b, c = ctypes.c_int(), ctypes.c_longlong(), ctypes.c_longlong(), ctypes.c_longlong()
    args = (ctypes.byref(k), ctypes.byref(a), ctypes.byref(b), ctypes.byref(c))
    assert lib.gqa_testing_fwd_split_plan(1, 3, 2, 10, 10, 128, 0, 148, *args) == 1   # Hq % Hkv
    assert lib.gqa_testing_fwd_split_plan(1, 2, 2, 10, 10, 128, 0, 0, *args) == 1     # no SMs
    assert lib.gqa_testing_fwd_split_plan(1, 2, 2, 10, 10, 128, -1, 148, *args) == 1  # window < 0
    assert lib.gqa_testing_fwd_split_plan(1, 2, 2, 10, 10, 128, 0, 148, None, *args[1:]) == 1
