"""The C-ABI library loads, exports every symbol include/w4a16.h declares, and rejects bad
arguments on the host before touching the GPU (CPU only: no compute call is made)."""
import ctypes
import os
import re

import pytest

from weight_only_int4_06_b200 import w4a16 as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "w4a16.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(B.LIB_PATH):
        from weight_only_int4_06_b200 import build_lib
        build_lib.build()
    return B.lib()


def test_header_declares_expected_api():
    names = declared_functions()
    for n in ("w4_quantize_pack", "w4_gemm", "w4_gemm_ex", "w4_gemm_host", "w4_gemm_workspace_size",
              "awq_scale_search", "awq_workspace_size", "awq_clip_search", "awq_clip_workspace_size",
              "awq_scale_search_gram", "awq_gram_workspace_size", "gptq_quantize", "gptq_workspace_size",
              "gptq_quantize_ex", "w4_quantize_pack_bits", "wb_gemm", "wb_gemm_workspace_size", "w4_act_prepare",
              "awq_colsum", "awq_scales_from_colsum", "awq_sse", "awq_sse_workspace_size", "awq_select",
              "w4_check_device_status", "w4_status_string"):
        assert n in names, n


def test_every_declared_symbol_is_exported(L):
    for n in declared_functions():
        assert hasattr(L, n), n
        assert n in B.SIGNATURES, n


def test_status_strings(L):
    for code in range(9):
        s = B.w4_status_string(code)
        assert isinstance(s, str) and s
    assert B.w4_status_string(99) == "unknown status"


P = ctypes.c_void_p
GOOD = P(1 << 20)        # never dereferenced: every call below is rejected on the host
BAD_ALIGN = P((1 << 20) + 2)


def test_quantize_pack_rejects(L):
    q = L.w4_quantize_pack
    assert q(GOOD, 8, 256, 64, None, GOOD, GOOD, GOOD, None) == 4        # group != 128
    assert q(GOOD, 8, 200, 128, None, GOOD, GOOD, GOOD, None) == 2       # K % 128
    assert q(GOOD, 12, 256, 128, None, GOOD, GOOD, GOOD, None) == 2      # N % 8
    assert q(GOOD, -8, 256, 128, None, GOOD, GOOD, GOOD, None) == 2      # negative
    assert q(None, 8, 256, 128, None, GOOD, GOOD, GOOD, None) == 1       # null W
    assert q(GOOD, 8, 256, 128, None, None, GOOD, GOOD, None) == 1       # null packed
    assert q(BAD_ALIGN, 8, 256, 128, None, GOOD, GOOD, GOOD, None) == 3  # misaligned W
    assert q(GOOD, 8, 256, 128, BAD_ALIGN, GOOD, GOOD, GOOD, None) == 3  # misaligned act_scale
    assert q(GOOD, 0, 256, 128, None, None, None, None, None) == 0       # empty: no-op
    assert q(GOOD, 1 << 31, 256, 128, None, GOOD, GOOD, GOOD, None) == 2 # too large


def test_gemm_rejects(L):
    g = L.w4_gemm_ex
    args = lambda **kw: [kw.get("X", GOOD), kw.get("M", 4), kw.get("N", 16), kw.get("K", 256),
                         kw.get("p", GOOD), GOOD, GOOD, kw.get("group", 128), kw.get("Y", GOOD),
                         None, 0, kw.get("variant", 0), None]
    assert g(*args(group=32)) == 4
    assert g(*args(variant=7)) == 4
    assert g(*args(K=100)) == 2
    assert g(*args(N=12)) == 2
    assert g(*args(M=-1)) == 2
    assert g(*args(X=None)) == 1
    assert g(*args(p=None)) == 1
    assert g(*args(Y=None)) == 1
    assert g(*args(X=BAD_ALIGN)) == 3
    assert g(*args(Y=BAD_ALIGN)) == 3
    assert g(*args(M=0)) == 0
    assert g(*args(N=0)) == 0
    # a shape whose GEMV cuts K: no workspace, a short one, a misaligned one
    need = 7 * 8 * 8192 * 4
    big = [GOOD, 8, 8192, 28672, GOOD, GOOD, GOOD, 128, GOOD]
    assert g(*big, None, 0, 0, None) == 5
    assert g(*big, GOOD, need - 1, 0, None) == 5
    assert g(*big, BAD_ALIGN, need, 0, None) == 3


def test_workspace_queries(L):
    n = ctypes.c_size_t(123)
    assert L.w4_gemm_workspace_size(1, 4096, 4096, 128, ctypes.byref(n)) == 0
    assert L.w4_gemm_workspace_size(1, 4096, 4000, 128, ctypes.byref(n)) == 2
    assert L.w4_gemm_workspace_size(1, 4096, 4096, 64, ctypes.byref(n)) == 4
    assert L.w4_gemm_workspace_size(1, 4096, 4096, 128, None) == 1
    # decode shapes need none; the GEMV's K slices (K = 28672: 7 slices of 4096) need fp32 partials
    assert L.w4_gemm_workspace_size(1, 4096, 11008, 128, ctypes.byref(n)) == 0 and n.value == 0
    assert L.w4_gemm_workspace_size(4, 8192, 8192, 128, ctypes.byref(n)) == 0 and n.value == 0
    assert L.w4_gemm_workspace_size(8, 8192, 28672, 128, ctypes.byref(n)) == 0
    assert n.value == 7 * 8 * 8192 * 4
    assert L.w4_gemm_workspace_size(16, 8192, 28672, 128, ctypes.byref(n)) == 0
    assert n.value == 7 * 8 * 8192 * 4  # 8-row launches (7 slices of 4096) reuse it in turn
    assert L.w4_gemm_workspace_size(16, 8192, 8192, 128, ctypes.byref(n)) == 0
    assert n.value == 4 * 16 * 8192 * 4  # one 16-row launch (4 slices of 2048) at K = 8192
    assert L.w4_gemm_workspace_size(32, 8192, 8192, 128, ctypes.byref(n)) == 0
    assert n.value == 4 * 32 * 8192 * 4  # the tensor cores' 4 K slices
    assert L.w4_gemm_workspace_size(12, 4096, 11008, 128, ctypes.byref(n)) == 0 and n.value == 0
    assert L.awq_workspace_size(256, 64, 512, 128, 0, ctypes.byref(n)) == 4
    assert L.awq_workspace_size(256, 64, 500, 128, 20, ctypes.byref(n)) == 2
    assert L.awq_clip_workspace_size(256, 64, 512, 128, 10, ctypes.byref(n)) == 0 and n.value > 0
    assert L.awq_clip_workspace_size(256, 64, 512, 128, 11, ctypes.byref(n)) == 4
    assert L.awq_clip_workspace_size(256, 64, 512, 128, 0, ctypes.byref(n)) == 4
    assert L.awq_clip_workspace_size(256, 64, 500, 128, 10, ctypes.byref(n)) == 2
    assert L.awq_clip_workspace_size(0, 64, 512, 128, 10, ctypes.byref(n)) == 2
    assert L.awq_gram_workspace_size(300, 64, 512, 128, 20, ctypes.byref(n)) == 0
    assert n.value >= 512 * 320 * 2 + 512 * 512 * 14 + 64 * 512 * 2  # X^T padded to 320 rows, G (fp32, fp64), G', E'
    assert L.awq_gram_workspace_size(256, 64, 512, 128, 0, ctypes.byref(n)) == 4
    assert L.awq_gram_workspace_size(256, 60, 512, 128, 20, ctypes.byref(n)) == 2


def test_gram_search_rejects(L):
    P = ctypes.c_void_p
    buf = ctypes.create_string_buffer(1 << 12)
    d = P(ctypes.addressof(buf) + (-ctypes.addressof(buf) % 16))
    args = lambda **kw: [kw.get("X", d), 64, kw.get("W", d), 64, 512, kw.get("group", 128), kw.get("A", 20), d, d,
                         d, kw.get("ws", d), kw.get("ws_bytes", 1 << 30), None]
    assert L.awq_scale_search_gram(*args(A=65)) == 4
    assert L.awq_scale_search_gram(*args(group=64)) == 4
    assert L.awq_scale_search_gram(*args(ws_bytes=16)) == 5
    assert L.awq_scale_search_gram(*args(X=None)) == 1
    assert L.awq_scale_search_gram(*args(W=P(d.value + 2))) == 3


def test_clip_search_rejects(L):
    P = ctypes.c_void_p
    buf = ctypes.create_string_buffer(1 << 12)
    d = P(ctypes.addressof(buf) + (-ctypes.addressof(buf) % 16))
    args = lambda **kw: [kw.get("X", d), 64, kw.get("W", d), 64, 512, kw.get("group", 128), kw.get("R", 10), None,
                         kw.get("best", d), None, d, d, d, kw.get("ws", d), kw.get("ws_bytes", 1 << 30), None]
    assert L.awq_clip_search(*args(R=0)) == 4
    assert L.awq_clip_search(*args(group=64)) == 4
    assert L.awq_clip_search(*args(ws_bytes=16)) == 5
    assert L.awq_clip_search(*args(X=None)) == 1
    assert L.awq_clip_search(*args(best=None)) == 1
    assert L.awq_clip_search(*args(W=P(d.value + 2))) == 3


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(B, "_lib", None)
    monkeypatch.setattr(B, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError):
        B.lib()


def test_gemm_host_rejects(L):
    P = ctypes.c_void_p
    buf = ctypes.create_string_buffer(1 << 12)
    d = P(ctypes.addressof(buf) + (-ctypes.addressof(buf) % 16))
    args = lambda **kw: [kw.get("X", d), kw.get("M", 1), 64, kw.get("K", 128), d, d, d, kw.get("group", 128),
                         kw.get("Y", d), kw.get("xd", d), kw.get("yd", d), None, 0, 0, None]
    assert L.w4_gemm_host(*args(group=64)) == 4
    assert L.w4_gemm_host(*args(K=100)) == 2
    assert L.w4_gemm_host(*args(Y=None)) == 1
    assert L.w4_gemm_host(*args(xd=None)) == 1
    assert L.w4_gemm_host(*args(yd=None)) == 1
    assert L.w4_gemm_host(*args(M=0)) == 0  # empty: nothing enqueued


def test_gptq_rejects(L):
    P = ctypes.c_void_p
    buf = ctypes.create_string_buffer(1 << 12)
    d = P(ctypes.addressof(buf) + (-ctypes.addressof(buf) % 16))
    n = ctypes.c_size_t(0)
    assert L.gptq_workspace_size(100, 64, 512, 128, ctypes.byref(n)) == 0
    assert n.value >= 512 * 512 * 16 + 64 * 512 * 8  # H and its factors in fp64, W in fp64
    assert L.gptq_workspace_size(100, 64, 512, 32, ctypes.byref(n)) == 4
    assert L.gptq_workspace_size(100, 64, 576, 64, ctypes.byref(n)) == 0  # group 64 (quantize_ex)
    assert L.gptq_workspace_size(100, 60, 512, 128, ctypes.byref(n)) == 2
    assert L.gptq_workspace_size(100, 64, 65536, 128, ctypes.byref(n)) == 2  # K above 32768
    args = lambda **kw: [kw.get("X", d), 100, kw.get("W", d), 64, 512, kw.get("group", 128),
                         kw.get("damp", 0.01), kw.get("p", d), d, d, kw.get("ws", d), kw.get("ws_bytes", 1 << 40),
                         None]
    assert L.gptq_quantize(*args(group=64)) == 4
    assert L.gptq_quantize(*args(damp=-1.0)) == 4
    assert L.gptq_quantize(*args(damp=float("nan"))) == 4
    assert L.gptq_quantize(*args(ws_bytes=16)) == 5
    assert L.gptq_quantize(*args(X=None)) == 1
    assert L.gptq_quantize(*args(p=P(d.value + 4))) == 3


def test_width_calls_reject(L):
    P = ctypes.c_void_p
    buf = ctypes.create_string_buffer(1 << 12)
    d = P(ctypes.addressof(buf) + (-ctypes.addressof(buf) % 16))
    q = lambda **kw: [kw.get("W", d), 64, kw.get("K", 512), kw.get("bits", 3), kw.get("group", 128), None, d, d, d,
                      None]
    assert L.w4_quantize_pack_bits(*q(bits=5)) == 4
    assert L.w4_quantize_pack_bits(*q(group=32)) == 4
    assert L.w4_quantize_pack_bits(*q(K=500)) == 2
    assert L.w4_quantize_pack_bits(*q(W=None)) == 1
    assert L.w4_quantize_pack_bits(*q(W=P(d.value + 2))) == 3
    n = ctypes.c_size_t(0)
    assert L.wb_gemm_workspace_size(4, 64, 512, 3, 128, ctypes.byref(n)) == 0 and n.value == 64 * 512 * 2
    assert L.wb_gemm_workspace_size(4, 64, 512, 6, 128, ctypes.byref(n)) == 4
    g = lambda **kw: [d, 4, 64, 512, d, d, d, kw.get("bits", 2), kw.get("group", 64), kw.get("Y", d), d,
                      kw.get("ws_bytes", 1 << 30), None]
    assert L.wb_gemm(*g(bits=1)) == 4
    assert L.wb_gemm(*g(ws_bytes=100)) == 5
    assert L.wb_gemm(*g(Y=None)) == 1
    e = lambda **kw: [d, 100, d, 64, 512, kw.get("bits", 3), kw.get("group", 128), kw.get("damp", 0.01),
                      kw.get("ao", 0), None, d, d, d, kw.get("perm", None), d, kw.get("ws_bytes", 1 << 40), None]
    assert L.gptq_quantize_ex(*e(bits=7)) == 4
    assert L.gptq_quantize_ex(*e(group=256)) == 4
    assert L.gptq_quantize_ex(*e(ao=1)) == 1  # act-order needs perm
    assert L.gptq_quantize_ex(*e(ws_bytes=8)) == 5
    assert L.w4_act_prepare(None, 2, 128, None, None, d, None) == 1
    assert L.w4_act_prepare(d, 0, 128, None, None, d, None) == 0


def test_row_split_calls_reject(L):
    P = ctypes.c_void_p
    buf = ctypes.create_string_buffer(1 << 12)
    d = P(ctypes.addressof(buf) + (-ctypes.addressof(buf) % 16))
    assert L.awq_colsum(d, 10, 500, d, None) == 2
    assert L.awq_colsum(None, 10, 512, d, None) == 1
    assert L.awq_colsum(P(d.value + 2), 10, 512, d, None) == 3
    assert L.awq_scales_from_colsum(d, 0, 512, 20, d, None) == 2
    assert L.awq_scales_from_colsum(d, 10, 512, 65, d, None) == 4
    n = ctypes.c_size_t(0)
    assert L.awq_sse_workspace_size(100, 64, 512, 128, 20, ctypes.byref(n)) == 0 and n.value > 64 * 512 * 2
    assert L.awq_sse(d, 100, d, 64, 512, 128, 20, d, d, d, 16, None) == 5
    assert L.awq_sse(d, 100, d, 64, 512, 128, 20, None, d, d, 1 << 30, None) == 1
    assert L.awq_select(d, 0, 20, 100, 64, d, 512, d, d, d, None) == 2
    assert L.awq_select(d, 2, 0, 100, 64, d, 512, d, d, d, None) == 4


def _layers(specs):
    arr = (B.GemmLayer * max(1, len(specs)))()
    for i, (M, N, K, xo, yo) in enumerate(specs):
        arr[i] = B.GemmLayer(M, N, K, GOOD.value, GOOD.value, GOOD.value, xo, yo)
    return ctypes.cast(arr, P), arr


def test_host_batch_rejects_before_enqueuing(L):
    """w4_gemm_host_batch validates every layer first (CPU only: the pointers are never used)."""
    f = L.w4_gemm_host_batch
    ok = [(1, 4096, 4096, 0, 0), (1, 12288, 4096, 8192, 8192)]
    xb, yb = 8192 * 2, 8192 + 2 * 12288

    def call(specs, n=None, x_bytes=xb, y_bytes=yb, xdev=GOOD, ydev=GOOD, group=128, variant=0):
        p, keep = _layers(specs)
        return f(p, len(specs) if n is None else n, group, GOOD, xdev, x_bytes, GOOD, ydev, y_bytes, None, 0,
                 variant, None)

    assert call(ok, n=0) == 2                                        # no layer: W4_ERR_SHAPE
    assert call(ok, group=64) == 4                                   # W4_ERR_UNSUPPORTED
    assert call(ok, variant=77) == 4
    assert call([(1, 4096, 4096, 8, 0)]) == 3                        # x_offset not a multiple of 16
    assert call([(1, 4096, 4096, 0, 0), (1, 12288, 4096, 8208, 8192)]) == 2  # second X beyond x_bytes
    assert call(ok, x_bytes=xb - 16) == 2                            # X region outside the buffer
    assert call(ok, y_bytes=yb - 16) == 2                            # Y region outside the buffer
    assert call([(1, 4100, 4096, 0, 0)]) == 2                        # N % 8 != 0
    assert call(ok, xdev=BAD_ALIGN) == 3
    assert call(ok, ydev=P(0)) == 1                                  # W4_ERR_NULL
    assert f(None, 1, 128, GOOD, GOOD, xb, GOOD, GOOD, yb, None, 0, 0, None) == 1


def test_gemm_plan_query(L):
    """The dispatch query (CPU: no device work) agrees with the documented rule."""
    assert B.w4_gemm_plan(1, 4096, 4096) == (B.VARIANT_GEMV, 1)
    # 8 rows of K = 8192 leave 2 ring stages whole: K is cut in two, + 1 reducing launch; 9-16 rows
    # run as one 16-row launch over slices of 2048 (+ 1 reducing launch); above 16 rows the tensor
    # cores, their 32 tiles cut along K into 4 slices (+ 1 reducing launch)
    assert B.w4_gemm_plan(4, 8192, 8192) == (B.VARIANT_GEMV, 1)
    assert B.w4_gemm_plan(8, 8192, 8192) == (B.VARIANT_GEMV, 2)
    assert B.w4_gemm_plan(16, 8192, 8192) == (B.VARIANT_GEMV, 2)
    assert B.w4_gemm_plan(32, 8192, 8192) == (B.VARIANT_TC, 2)
    assert B.w4_gemm_plan(16, 520, 2048) == (B.VARIANT_GEMV, 1)  # one slice: no reducing launch
    assert B.w4_gemm_plan(12, 136, 1536) == (B.VARIANT_GEMV, 2)  # K/128 = 12: two 8-row launches
    # K = 28672 is cut into slices (4 rows of it do not fit whole): the GEMV, then the slice sum
    assert B.w4_gemm_plan(4, 8192, 28672) == (B.VARIANT_GEMV, 2)
    assert B.w4_gemm_plan(16, 8192, 28672) == (B.VARIANT_GEMV, 4)  # 8-row launches at K = 28672
    assert B.w4_gemm_plan(32, 8192, 28672) == (B.VARIANT_TC, 2)
    assert B.w4_gemm_plan(4, 8192, 28800) == (B.VARIANT_SKINNY, 1)  # K/128 = 225: no slices, no fit
    assert B.w4_gemm_plan(33, 4096, 4096) == (B.VARIANT_TC, 2)  # 16 tiles: K in 8 slices + their sum
    assert B.w4_gemm_plan(2048, 11008, 4096) == (B.VARIANT_TC, 3)  # 344 tiles: full waves + tail slices + sum
    assert B.w4_gemm_plan(0, 4096, 4096) == (B.VARIANT_AUTO, 0)
    assert B.w4_gemm_plan(64, 4096, 4096, variant=B.VARIANT_SKINNY) == (B.VARIANT_SKINNY, 2)
    fam, n = ctypes.c_int(0), ctypes.c_int(0)
    assert L.w4_gemm_plan(1, 4096, 4096, 128, B.VARIANT_GEMV, BAD_ALIGN, GOOD, ctypes.byref(fam),
                          ctypes.byref(n)) == 3  # explicit GEMV with misaligned scales: W4_ERR_ALIGN
    assert L.w4_gemm_plan(1, 4096, 4096, 128, 0, BAD_ALIGN, GOOD, ctypes.byref(fam), ctypes.byref(n)) == 0
    assert (fam.value, n.value) == (B.VARIANT_SKINNY, 1)  # AUTO falls back to the skinny kernel


def test_plan_and_workspace_agree():
    """Every shape whose plan sums K slices in a further launch (the GEMV in split mode, the
    tensor-core K split or tail split) gets a non-zero workspace from w4_gemm_workspace_size, for
    AUTO and for each explicit family."""
    shapes = [(M, N, K) for M in (1, 4, 8, 9, 16, 17, 32, 33, 64, 130, 512, 2048)
              for (N, K) in ((8192, 8192), (8192, 28672), (28672, 8192), (4096, 4096), (11008, 4096),
                             (4096, 11008), (520, 2048), (5000, 2048))]
    n = ctypes.c_size_t(0)
    for (M, N, K) in shapes:
        assert B.lib().w4_gemm_workspace_size(M, N, K, 128, ctypes.byref(n)) == 0
        need = n.value
        for variant in (B.VARIANT_AUTO, B.VARIANT_GEMV, B.VARIANT_TC):
            try:
                fam, launches = B.w4_gemm_plan(M, N, K, variant=variant)
            except B.W4Error:
                continue  # the explicit family cannot serve this shape
            if fam == B.VARIANT_TC and launches > 1:  # K slices or a tail split: fp32 partials
                assert need > 0, (M, N, K, variant)
            if fam == B.VARIANT_GEMV and M <= 8 and launches > 1:  # one GEMV launch + its slice sum
                assert need > 0, (M, N, K, variant)
