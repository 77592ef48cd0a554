"""Host-side check of the split-launch decomposition behind gqa_attn_fwd_split: the plan comes
from the library (gqa_testing_fwd_split_plan), and the piece arithmetic of the forward kernel is
restated here (runs of ticks over lanes of unit groups, ticks mapped to key tiles in proportion,
the merge's walk over the runs that reach a unit). For every plan that splits it checks that the
pieces cover each split unit's key tiles exactly once per sub-tile, that each persistent CTA holds
at most two pieces, and that the merge finds exactly the pieces that wrote each unit. The GPU
parity tests check the kernel itself; this keeps a plan change from breaking the assumptions
the kernel's arithmetic makes."""
import ctypes
import random

import pytest

R = 128  # rows per sub-tile and keys per tile


@pytest.fixture(scope="module")
def lib():
    import grouped_query_softmax_b200 as m
    return ctypes.CDLL(m.library_path())


def plan(lib, B, Hq, Hkv, Tq, Tk, sms):
    slices = ctypes.c_int(-1)
    whole, split, units = ctypes.c_longlong(-1), ctypes.c_longlong(-1), ctypes.c_longlong(-1)
    assert lib.gqa_testing_fwd_split_plan(B, Hq, Hkv, Tq, Tk, 128, 0, sms, ctypes.byref(slices),
                                          ctypes.byref(whole), ctypes.byref(split), ctypes.byref(units)) == 0
    return slices.value, whole.value, split.value, units.value


def unit_tiles(Hq, Hkv, Tq, Tk, u):
    """[j_begin, n_kv) of the two sub-tiles of unit u in a suffix launch (units listed head by
    head, the row levels of one head or head pair together, longest rows first)."""
    G, n_qt, off = Hq // Hkv, (Tq + R - 1) // R, Tk - Tq
    if G % 2 == 0:
        level = u % n_qt
        rows = [(n_qt - 1 - level) * R] * 2
    else:
        n_rb = (n_qt + 1) // 2
        level = u % n_rb
        r0 = (n_rb - 1 - level) * 2 * R
        rows = [r0, r0 + R]
    out = []
    for r0 in rows:
        if r0 >= Tq:
            out.append((0, 0))
        else:
            out.append((0, (off + min(r0 + R - 1, Tq - 1)) // R + 1))
    return out


def group_of(Hq, Hkv, Tq, sms, whole):
    G, n_qt = Hq // Hkv, (Tq + R - 1) // R
    L = n_qt if G % 2 == 0 else (n_qt + 1) // 2
    return L if whole % L == 0 else 1


def piece(slot, S, L, slices, N):
    """(split unit, first tick, end tick) of a slot, or None for an absent piece."""
    m, T = slices // L, (S // L) * N
    j, lane = divmod(slot >> 1, L)
    lo, hi = T * j // m, T * (j + 1) // m
    g0 = lo // N
    if slot & 1:
        start = (g0 + 1) * N
        return None if hi <= start else ((g0 + 1) * L + lane, 0, hi - start)
    return None if hi <= lo else (g0 * L + lane, lo - g0 * N, min(hi, (g0 + 1) * N) - g0 * N)


def clamp(tiles, a, b, N):
    n_max = max(e for _, e in tiles)
    j0, j1 = n_max * a // N, n_max * b // N
    out = []
    for jb, ne in tiles:
        if ne == 0:
            out.append((0, 0))
            continue
        jb, ne = max(jb, j0), min(ne, j1)
        out.append((jb, ne) if jb < ne else (0, 0))
    return out


def check(lib, B, Hq, Hkv, Tq, Tk, sms):
    slices, whole, S, units = plan(lib, B, Hq, Hkv, Tq, Tk, sms)
    if slices == 0:
        return False
    N = (Tk - 1) // R + 1
    L = group_of(Hq, Hkv, Tq, sms, whole)
    assert whole % sms == 0 and S % L == 0 and slices % L == 0 and S // L <= slices // L <= sms
    covered = {}
    writers = {}
    for cta in range(slices):
        pieces = 0
        for i in range(2):
            pc = piece(2 * cta + i, S, L, slices, N)
            if pc is None:
                continue
            su, a, b = pc
            assert 0 <= su < S and 0 <= a < b <= N
            tiles = clamp(unit_tiles(Hq, Hkv, Tq, Tk, whole + su), a, b, N)
            if all(ne == 0 for _, ne in tiles):
                continue
            pieces += 1
            for s, (jb, ne) in enumerate(tiles):
                if ne:
                    covered.setdefault((su, s), []).extend(range(jb, ne))
                    writers.setdefault((su, s), []).append(2 * cta + i)
        assert pieces <= 2
    m, T = slices // L, (S // L) * N
    for su in range(S):
        for s, (jb, ne) in enumerate(unit_tiles(Hq, Hkv, Tq, Tk, whole + su)):
            if ne == 0:
                assert (su, s) not in covered
                continue
            assert sorted(covered[(su, s)]) == list(range(jb, ne))       # each tile exactly once
            gr, ln = divmod(su, L)
            x0, x1 = gr * N, gr * N + N
            c0 = ((x0 + 1) * m - 1) // T
            c1 = min(m, (x1 * m + T - 1) // T)
            assert c1 - c0 <= 32
            cand = [2 * (c * L + ln) + (1 if T * c // m < x0 else 0) for c in range(c0, c1)]
            assert set(writers[(su, s)]) <= set(cand)                  # the merge reads every piece
            for slot in cand:                                          # and only pieces of this unit
                pc = piece(slot, S, L, slices, N)
                assert pc is None or pc[0] == su
    return True


@pytest.mark.parametrize("shape", [
    (8, 16, 16, 512, 8192),     # the MHA suffix workload: a whole wave, then runs crossing units
    (2, 32, 8, 256, 32768),     # 64 head-pair units of 256 tiles over 148 SMs
    (1, 4, 1, 700, 1900),       # 12 short units, 84 runs
    (7, 16, 16, 384, 4096),     # whole wave, units whose second sub-tile is absent
    (7, 32, 32, 128, 4096),     # one-sub-tile units
    (6, 32, 8, 512, 16384),     # two whole waves, lanes of 4 levels
])
def test_split_pieces_cover_each_unit_once(lib, shape):
    assert check(lib, *shape, sms=148)


def test_split_pieces_random_shapes(lib):
    rng = random.Random(7)
    n_split = 0
    for _ in range(150):
        Hkv = rng.choice([1, 2, 4, 8])
        Hq = Hkv * rng.choice([1, 2, 3, 4, 8])
        Tq = rng.randint(1, 1100)
        Tk = 2 * Tq + rng.randint(0, 30000)
        n_split += check(lib, rng.randint(1, 6), Hq, Hkv, Tq, Tk, rng.choice([148, 132, 20, 7]))
    assert n_split >= 50
