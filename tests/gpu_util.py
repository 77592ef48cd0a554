"""Helpers shared by the GPU parity tests: device transfer of bf16 bit arrays and
the parity bar (max-abs <= 2e-2, mean-abs <= 2e-3 of the bf16 GPU output against
the fp64 oracle, both on the same seeded inputs)."""
import numpy as np

import gqa_inputs as gi

MAX_ABS = 2e-2
MEAN_ABS = 2e-3


def torch_mod():
    import torch
    if not torch.cuda.is_available():
        raise RuntimeError("GPU test needs CUDA; none visible")
    return torch


def to_dev(u16: np.ndarray):
    torch = torch_mod()
    return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).cuda().view(torch.bfloat16)


def from_dev(t) -> np.ndarray:
    """bf16 CUDA tensor -> float32 numpy (exact)."""
    torch = torch_mod()
    u = t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    return gi.bf16_bits_to_f32(u).reshape(tuple(t.shape))


def bits_of(t) -> np.ndarray:
    torch = torch_mod()
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def assert_parity(got: np.ndarray, ref: np.ndarray, what: str, max_abs=MAX_ABS, mean_abs=MEAN_ABS):
    got = np.asarray(got, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - ref)
    mx, mean = float(err.max()), float(err.mean())
    assert mx <= max_abs and mean <= mean_abs, f"{what}: max-abs {mx:.3e}, mean-abs {mean:.3e}"
    return mx, mean


def rand_qkv(B, Hq, Hkv, Tq, Tk, D, seed=0, q_pow2=0):
    w = gi.Workload("test", B, Hq, Hkv, Tq, Tk, D, q_pow2=q_pow2, seed=seed)
    return w.make()


def sample_rows(B, Hq, Tq, n, seed=0, tile=128):
    """A seeded row sample plus the special rows: i = 0, tile boundaries +-1, the
    last row, and every (b, a) represented. Returns sorted flat row ids."""
    rng = np.random.default_rng(seed)
    total = B * Hq * Tq
    rows = set(rng.integers(0, total, size=min(n, total)).tolist())
    special_i = {0, Tq - 1}
    for t in range(tile, Tq, tile):
        special_i.update({t - 1, t, t + 1})
    special_i = [i for i in special_i if 0 <= i < Tq]
    for b in range(B):
        for a in range(Hq):
            base = (b * Hq + a) * Tq
            rows.add(base + int(rng.integers(0, Tq)))
            if (b * Hq + a) % 7 == 0:
                rows.update(base + i for i in special_i)
    return np.array(sorted(rows), dtype=np.int64)
