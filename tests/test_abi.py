"""The C ABI without a GPU: the library loads, exports every declared symbol, and
rejects bad arguments on the host before any CUDA call."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def gqa():
    import grouped_query_softmax_b200 as m
    return m


def declared_functions():
    names = []
    for h in ("gqa.h", "gqa_testing.h"):
        src = open(os.path.join(ROOT, "include", h)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names += re.findall(r"\b(gqa_[a-z_0-9]+)\s*\(", src)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(gqa):
    lib = ctypes.CDLL(gqa.library_path())
    names = declared_functions()
    assert {"gqa_attn_fwd", "gqa_attn_decode", "gqa_attn_decode_workspace_bytes",
            "gqa_status_string", "gqa_get_device_error"} <= set(names)
    for n in names:
        assert hasattr(lib, n), f"{n} declared but not exported"


def test_only_declared_symbols_are_exported(gqa):
    out = os.popen(f"nm -D --defined-only {gqa.library_path()}").read()
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l and l.split()[-1].startswith("gqa")}
    assert exported == set(declared_functions())


def test_status_strings(gqa):
    assert gqa.gqa_status_string(gqa.GQA_OK) == "GQA_OK"
    assert gqa.gqa_status_string(gqa.GQA_ERR_TIMEOUT) == "GQA_ERR_TIMEOUT"
    assert gqa.gqa_status_string(99) == "GQA_ERR_UNKNOWN"


P = 1 << 20  # a 16-byte-aligned fake device address; never dereferenced on these paths


def fwd(gqa, **kw):
    a = dict(q=P, k=P, v=P, o=P, lse=None, B=1, Hq=4, Hkv=2, Tq=8, Tk=8, D=64,
             k_sb=2 * 8 * 64, k_sh=8 * 64, v_sb=2 * 8 * 64, v_sh=8 * 64, softmax_scale=0.0, stream=None)
    a.update(kw)
    return gqa.gqa_attn_fwd(**a)


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), 1), (dict(o=None), 1), (dict(k=P + 8), 1),       # null / misaligned
    (dict(Hq=3), 1),                                                   # Hq % Hkv != 0
    (dict(Tq=9), 1),                                                   # Tq > Tk
    (dict(B=0), 1), (dict(Tk=0, Tq=0), 1), (dict(Hkv=0), 1),
    (dict(D=96), 2), (dict(D=256), 2),                                # unsupported head dim
    (dict(k_sh=8 * 64 + 4), 1), (dict(B=2, v_sb=-512), 1),            # bad strides (a batch stride of B=1 is unused)
    (dict(softmax_scale=float("nan")), 1),
    (dict(lse=P + 2), 1),
])
def test_fwd_rejects_bad_arguments(gqa, kw, status):
    assert fwd(gqa, **kw) == status


def dec(gqa, **kw):
    a = dict(q=P, k_cache=P, v_cache=P, o=P, B=1, Hq=4, Hkv=2, Tk=1024, D=128,
             k_sb=2 * 1024 * 128, k_sh=1024 * 128, v_sb=2 * 1024 * 128, v_sh=1024 * 128,
             softmax_scale=0.0, num_splits=4, workspace=None, workspace_bytes=0, stream=None)
    a.update(kw)
    return gqa.gqa_attn_decode(**a)


def test_decode_rejects_bad_arguments_and_small_workspace(gqa):
    assert dec(gqa, Hq=6, Hkv=4) == gqa.GQA_ERR_INVALID_ARGUMENT
    assert dec(gqa, D=80) == gqa.GQA_ERR_UNSUPPORTED
    assert dec(gqa, q=None) == gqa.GQA_ERR_INVALID_ARGUMENT
    need = gqa.gqa_attn_decode_workspace_bytes(1, 4, 2, 1024, 128, 4)
    assert need > 0
    assert dec(gqa) == gqa.GQA_ERR_WORKSPACE                          # none given
    assert dec(gqa, workspace=P, workspace_bytes=need - 4) == gqa.GQA_ERR_WORKSPACE
    assert dec(gqa, workspace=P + 16, workspace_bytes=need) == gqa.GQA_ERR_WORKSPACE  # not 256-aligned


def test_decode_split_planning(gqa):
    # explicit requests are clamped to [1, ceil(Tk/128)] and never leave a split empty
    assert gqa.gqa_attn_decode_num_splits(1, 4, 2, 1024, 128, 4) == 4
    assert gqa.gqa_attn_decode_num_splits(1, 4, 2, 1024, 128, 100) == 8
    assert gqa.gqa_attn_decode_num_splits(1, 4, 2, 1100, 128, 4) == 3   # 9 tiles -> 3 per split
    assert gqa.gqa_attn_decode_num_splits(1, 4, 2, 100, 128, 0) == 1
    assert gqa.gqa_attn_decode_workspace_bytes(1, 4, 2, 1024, 128, 1) == 0
    s = 4
    o_bytes = s * 1 * 4 * 128 * 4
    assert gqa.gqa_attn_decode_workspace_bytes(1, 4, 2, 1024, 128, s) == ((o_bytes + 255) // 256) * 256 + s * 4 * 4


def test_selftest_rejects_out_of_range_timeouts(gqa):
    assert gqa.gqa_selftest_bounded_wait(10) == gqa.GQA_ERR_INVALID_ARGUMENT
    assert gqa.gqa_selftest_bounded_wait(10 ** 11) == gqa.GQA_ERR_INVALID_ARGUMENT


def test_product_does_not_reference_the_oracle():
    pkg = os.path.join(ROOT, "grouped_query_softmax_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".cpp", ".h")):
                txt = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert "import oracle" not in txt and "gqa_oracle" not in txt, f


def varlen_fwd(gqa, **kw):
    rows = 64
    lay = (0, 64, 4 * 64)  # token-major [rows, 4, 64]
    lay_k = (0, 64, 2 * 64)
    a = dict(q=P, k=P, v=P, o=P, lse=None, cu_seqlens_q=P, cu_seqlens_k=P, seqlens_q=None,
             seqlens_k=None, S=2, Hq=4, Hkv=2, D=64, rows_q=rows, rows_k=rows, max_seqlen_q=40,
             q_layout=lay, k_layout=lay_k, v_layout=lay_k, o_layout=lay, softmax_scale=0.0, window=0,
             workspace=P, workspace_bytes=1 << 20, stream=None)
    a.update(kw)
    return gqa.gqa_attn_fwd_varlen(**a)


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), 1), (dict(k=P + 8), 1), (dict(lse=P + 2), 1),
    (dict(S=0), 1), (dict(Hq=3), 1), (dict(rows_q=0), 1), (dict(max_seqlen_q=0), 1),
    (dict(D=96), 2), (dict(window=-1), 1),
    (dict(seqlens_q=P), 1),                                   # packed and padded on one side
    (dict(q_layout=(0, 64, 100)), 1),                         # row stride not a multiple of 8
    (dict(k_layout=(0, 64, 32)), 1),                          # rows closer than D
    (dict(o_layout=(0, 0, 256)), 1),                          # zero head stride with 4 heads
    (dict(cu_seqlens_q=None, q_layout=(0, 64, 256)), 1),      # padded, 2 batches, zero batch stride
    (dict(workspace=None), 3), (dict(workspace_bytes=64), 3), (dict(workspace=P + 16), 3),
])
def test_varlen_fwd_rejects_bad_arguments(gqa, kw, status):
    assert varlen_fwd(gqa, **kw) == status


def test_varlen_workspace_sizes(gqa):
    # 4 heads over 2 KV heads (G = 2, head pairs): S * ceil(max_q/128) * Hq/2 units + a header
    assert gqa.gqa_attn_fwd_varlen_workspace_bytes(2, 4, 2, 300) == 256 + 4 * 2 * 3 * 2
    # G = 3 (row pairs): S * ceil(ceil(max_q/128)/2) * Hq
    assert gqa.gqa_attn_fwd_varlen_workspace_bytes(2, 6, 2, 300) == 256 + 4 * 2 * 2 * 6
    assert gqa.gqa_attn_fwd_varlen_workspace_bytes(0, 4, 2, 300) == 0
    assert gqa.gqa_attn_fwd_varlen_workspace_bytes(2, 5, 2, 300) == 0


def varlen_dec(gqa, **kw):
    a = dict(q=P, k_cache=P, v_cache=P, o=P, seqlens_k=P, block_table=P, page_size=64, num_pages=100,
             max_pages=16, B=2, Hq=4, Hkv=2, Tq=1, max_seqlen_k=1024, D=128,
             k_layout=(64 * 2 * 128, 128, 2 * 128), v_layout=(64 * 2 * 128, 128, 2 * 128),
             softmax_scale=0.0, window=0, num_splits=1, workspace=None, workspace_bytes=0, stream=None)
    a.update(kw)
    return gqa.gqa_attn_decode_varlen(**a)


@pytest.mark.parametrize("kw,status", [
    (dict(seqlens_k=None), 1), (dict(q=None), 1), (dict(Tq=17), 2), (dict(D=96), 2),
    (dict(page_size=48), 1), (dict(page_size=8), 1), (dict(page_size=200), 1),
    (dict(num_pages=0), 1), (dict(max_pages=0), 1),
    (dict(k_layout=(64 * 2 * 128, 128, 100)), 1),
    (dict(num_splits=4), 3),                                  # splits need a workspace
    (dict(block_table=None, k_layout=(0, 1024 * 128, 128)), 1),  # contiguous: 2 sequences, no batch stride
])
def test_varlen_decode_rejects_bad_arguments(gqa, kw, status):
    assert varlen_dec(gqa, **kw) == status


def test_varlen_decode_split_planning(gqa):
    # the automatic plan aims at twice the CTAs of the dense plan; explicit requests agree
    assert gqa.gqa_attn_decode_varlen_num_splits(64, 32, 8, 1, 32768, 128, 0, 0) == 3
    assert gqa.gqa_attn_decode_ex_num_splits(64, 32, 8, 1, 32768, 128, 0, 0) == 2
    for s in (1, 4, 7):
        assert gqa.gqa_attn_decode_varlen_num_splits(4, 8, 2, 1, 4096, 128, 0, s) == \
            gqa.gqa_attn_decode_ex_num_splits(4, 8, 2, 1, 4096, 128, 0, s)
    assert gqa.gqa_attn_decode_varlen_workspace_bytes(64, 32, 8, 1, 32768, 128, 0, 1) == 0
    assert gqa.gqa_attn_decode_varlen_workspace_bytes(64, 32, 8, 17, 32768, 128, 0, 0) == 0  # Tq > 16


def bwd(gqa, **kw):
    a = dict(q=P, k=P, v=P, o=P, dout=P, lse=P, dq=P, dk=P, dv=P, B=1, Hq=4, Hkv=2, Tq=8, Tk=8, D=64,
             k_sb=2 * 8 * 64, k_sh=8 * 64, v_sb=2 * 8 * 64, v_sh=8 * 64, softmax_scale=0.0, window=0,
             workspace=P, workspace_bytes=1 << 20, stream=None)
    a.update(kw)
    return gqa.gqa_attn_bwd(**a)


@pytest.mark.parametrize("kw,status", [
    (dict(Hq=3), 1), (dict(Tq=9), 1), (dict(dk=None), 1), (dict(lse=P + 4), 1), (dict(D=96), 2),
    (dict(k_sh=8 * 64 + 4), 1), (dict(workspace=None), 3), (dict(workspace_bytes=16), 3),
    (dict(workspace=P + 64), 3), (dict(window=-1), 1),
])
def test_bwd_rejects_bad_arguments(gqa, kw, status):
    assert bwd(gqa, **kw) == status


def test_bwd_workspace_size(gqa):
    # fp32 dQ [B,Hq,Tq,D] + two fp32 values per row padded to 128-row tiles, each 256-aligned
    assert gqa.gqa_attn_bwd_workspace_bytes(1, 4, 2, 8, 8, 64) == 8192 + 2 * 2048
    assert gqa.gqa_attn_bwd_workspace_bytes(1, 4, 2, 9, 8, 64) == 0


def paged_fwd(gqa, **kw):
    lay_q = (0, 64, 4 * 64)
    lay_kv = (64 * 2 * 64, 64, 2 * 64)   # pool [pages, 64, 2, 64] (NHD)
    a = dict(q=P, k_pool=P, v_pool=P, o=P, lse=None, cu_seqlens_q=P, seqlens_q=None, seqlens_k=P,
             block_table=P, page_size=64, num_pages=10, max_pages=4, S=2, Hq=4, Hkv=2, D=64, rows_q=64,
             max_seqlen_q=40, q_layout=lay_q, k_layout=lay_kv, v_layout=lay_kv, o_layout=lay_q,
             softmax_scale=0.0, window=0, workspace=P, workspace_bytes=1 << 20, stream=None)
    a.update(kw)
    return gqa.gqa_attn_fwd_varlen_paged(**a)


@pytest.mark.parametrize("kw,status", [
    (dict(seqlens_k=None), 1), (dict(block_table=None), 1), (dict(page_size=48), 1), (dict(page_size=8), 1),
    (dict(num_pages=0), 1), (dict(max_pages=0), 1), (dict(k_layout=(64 * 2 * 64, 64, 100)), 1),
    (dict(workspace=None), 3), (dict(seqlens_q=P), 1),
])
def test_paged_fwd_rejects_bad_arguments(gqa, kw, status):
    assert paged_fwd(gqa, **kw) == status


H = 1 << 22  # a fake host address; these calls fail before touching memory or the GPU


def fwd_host(gqa, **kw):
    a = dict(q=H, k=H, v=H, o=H, lse=None, B=1, Hq=4, Hkv=2, Tq=300, Tk=300, D=64, softmax_scale=0.0, window=0,
             workspace=P, workspace_bytes=1 << 30, stream=None)
    a.update(kw)
    return gqa.gqa_attn_fwd_host(**a)


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), 1), (dict(v=None), 1), (dict(o=None), 1),
    (dict(Hq=3), 1), (dict(Tq=301), 1), (dict(window=-1), 1), (dict(softmax_scale=float("nan")), 1),
    (dict(lse=H + 2), 1), (dict(D=96), 2),
    (dict(workspace=None), 3), (dict(workspace=P + 128), 3), (dict(workspace_bytes=1024), 3),
])
def test_fwd_host_rejects_bad_arguments(gqa, kw, status):
    assert fwd_host(gqa, **kw) == status


def test_fwd_host_workspace_size(gqa):
    # K and V whole, plus two slots of query rows, outputs and LSE; chunks of whole 128-row
    # tiles, at most 8 of them and at least 256 rows each
    def rnd(x):
        return (x + 255) // 256 * 256
    for B, Hq, Hkv, Tq, Tk, D in [(4, 32, 8, 4096, 4096, 128), (1, 4, 2, 300, 700, 64), (2, 8, 8, 100, 100, 128),
                                  (1, 32, 1, 32768, 32768, 128)]:
        rows = max(256, -(-(-(-Tq // 8)) // 128) * 128)
        rows = min(rows, Tq)
        want = 2 * rnd(B * Hkv * Tk * D * 2) + 2 * (2 * rnd(B * Hq * rows * D * 2) + rnd(B * Hq * rows * 4))
        assert gqa.gqa_attn_fwd_host_workspace_bytes(B, Hq, Hkv, Tq, Tk, D) == want
    assert gqa.gqa_attn_fwd_host_workspace_bytes(1, 3, 2, 8, 8, 64) == 0
    assert gqa.gqa_attn_fwd_host_workspace_bytes(1, 4, 2, 8, 8, 80) == 0
