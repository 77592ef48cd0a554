"""The split plan of gqa_attn_fwd_split, read through gqa_testing_fwd_split_plan (host only, no
GPU): which launches split their last wave's units along the keys, into how many parts, and
that every split is worth it by the plan's own estimate."""
import ctypes

import pytest


@pytest.fixture(scope="module")
def lib():
    import grouped_query_softmax_b200 as m
    return ctypes.CDLL(m.library_path())


def plan(lib, B, Hq, Hkv, Tq, Tk, D=128, window=0, sms=148):
    k = ctypes.c_int(-1)
    whole, split, units = ctypes.c_longlong(-1), ctypes.c_longlong(-1), ctypes.c_longlong(-1)
    st = lib.gqa_testing_fwd_split_plan(B, Hq, Hkv, Tq, Tk, D, window, sms, ctypes.byref(k), ctypes.byref(whole),
                                        ctypes.byref(split), ctypes.byref(units))
    assert st == 0
    return k.value, whole.value, split.value, units.value


def units_of(B, Hq, Hkv, Tq):
    G = Hq // Hkv
    n_qt = (Tq + 127) // 128
    return B * Hkv * (G // 2) * n_qt if G % 2 == 0 else B * Hq * ((n_qt + 1) // 2)


PART_COST = 5.0  # a part's fixed cost in key tiles, as the plan counts it


def estimate(n, full, r, k, sms):
    """Makespan in key tiles: whole waves, then waves of k-th parts of the last r units."""
    return full * n + -(-r * k // sms) * (n / k + PART_COST) if k > 1 else (full + 1) * n


def test_small_suffix_launches_split(lib):
    # 12 units of 15 key tiles on 148 SMs: all of them cut, into 7 parts
    assert plan(lib, 1, 4, 1, 700, 1900) == (7, 0, 12, 12)
    # B8 H16/16, T_q 512 over T_k 8192: 256 units of 64 tiles on 148 SMs (1.73 waves); cutting
    # the last wave does not pay for the parts' fixed cost
    assert plan(lib, 8, 16, 16, 512, 8192) == (1, 256, 0, 256)


@pytest.mark.parametrize("shape", [
    (4, 32, 8, 4096, 4096),     # T_q = T_k: unequal units, ordered longest first instead
    (1, 32, 1, 32768, 32768),
    (8, 16, 16, 512, 8192, 128, 1024),   # a window: not split
    (2, 16, 16, 900, 1500),     # prefix shorter than the suffix
    (37, 8, 8, 512, 8192),      # 148 units: whole waves only
])
def test_launches_that_do_not_split(lib, shape):
    k, whole, split, units = plan(lib, *shape)
    assert k == 1 and split == 0 and whole == units


@pytest.mark.parametrize("shape", [
    (8, 16, 16, 512, 8192), (1, 4, 1, 700, 1900), (2, 16, 16, 512, 4096), (1, 8, 8, 1024, 2048), (4, 16, 16, 256, 8192),
    (3, 12, 4, 384, 9000, 64), (5, 32, 8, 1000, 4000), (1, 2, 2, 128, 640),
])
@pytest.mark.parametrize("sms", [148, 132, 20])
def test_plan_invariants(lib, shape, sms):
    B, Hq, Hkv, Tq, Tk = shape[:5]
    k, whole, split, units = plan(lib, *shape, sms=sms)
    assert units == units_of(B, Hq, Hkv, Tq)
    assert whole + split == units and 1 <= k <= 8
    n = (Tk - 1) // 128 + 1
    full, r = divmod(units, sms)
    if k == 1:
        assert split == 0
        return
    assert split == r and whole == full * sms        # only the last wave is cut
    assert n // k >= 2                               # parts of at least two key tiles
    costs = {kk: estimate(n, full, r, kk, sms) for kk in range(1, 9) if kk == 1 or n // kk >= 2}
    assert costs[k] == min(costs.values())           # the best part count by the estimate
    assert costs[k] <= 0.9 * costs[1]               # and worth the merge


def test_rejects_bad_arguments(lib):
    k, a, b, c = ctypes.c_int(), ctypes.c_longlong(), ctypes.c_longlong(), ctypes.c_longlong()
    args = (ctypes.byref(k), ctypes.byref(a), ctypes.byref(b), ctypes.byref(c))
    assert lib.gqa_testing_fwd_split_plan(1, 3, 2, 10, 10, 128, 0, 148, *args) == 1   # Hq % Hkv
    assert lib.gqa_testing_fwd_split_plan(1, 2, 2, 10, 10, 128, 0, 0, *args) == 1     # no SMs
    assert lib.gqa_testing_fwd_split_plan(1, 2, 2, 10, 10, 128, -1, 148, *args) == 1  # window < 0
    assert lib.gqa_testing_fwd_split_plan(1, 2, 2, 10, 10, 128, 0, 148, None, *args[1:]) == 1
