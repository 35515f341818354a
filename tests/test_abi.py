"""The C ABI without a GPU: the library loads, exports what include/lisa.h
declares, and rejects bad arguments on the host before launching anything."""

import ctypes
import os
import re

import pytest

from conftest import ROOT

L = pytest.importorskip("hybrid_linear_top_b200.lisa")

HEADER = os.path.join(ROOT, "include", "lisa.h")


def declared_symbols():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"LISA_API\s+[\w\s\*]*?\b(lisa_\w+)\s*\(", src)))


def test_header_declares_the_four_calls():
    names = declared_symbols()
    for n in ["lisa_prefill", "lisa_decode_step", "lisa_indexer_topk", "lisa_append_cache",
              "lisa_workspace_bytes", "lisa_status_str", "lisa_last_error_msg"]:
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(L.LIB_PATH)
    for n in declared_symbols():
        assert hasattr(lib, n), n
    assert sorted(L.EXPORTED) == sorted(declared_symbols())


def _layer(**kw):
    f = dict(B=1, Hq=12, Hkv=2, d=128, HI=4, dI=64, M=256, L_max=16384, dtype=L.LISA_BF16)
    f.update(kw)
    c = L.LisaLayerC(f["B"], f["Hq"], f["Hkv"], f["d"], f["HI"], f["dI"], f["M"], f["L_max"], f["dtype"])
    fake = 0x10000  # aligned, never dereferenced: every call below fails validation first
    for name in ["k_cache", "v_cache", "kidx_cache", "state", "pos", "err_word"]:
        setattr(c, name, kw.get(name, fake))
    for name in ["decode_split", "independent", "debug_flags"]:
        setattr(c, name, kw.get(name, 0))
    return c


FAKE = ctypes.c_void_p(0x20000)


def _decode(c, ws=FAKE, ws_bytes=1 << 40, **ptrs):
    args = {n: ptrs.get(n, FAKE) for n in ["q", "k", "v", "kidx", "qidx", "w", "gate", "out"]}
    lib = L.lib()
    return lib.lisa_decode_step(ctypes.byref(c), args["q"], args["k"], args["v"], args["kidx"], args["qidx"],
                                args["w"], args["gate"], 1, args["out"], None, ws, ws_bytes, None)


def test_status_strings():
    assert L.status_str(L.LISA_OK) == "LISA_OK"
    assert L.status_str(L.LISA_ERR_UNSUPPORTED) == "LISA_ERR_UNSUPPORTED"
    assert L.status_str(99) == "LISA_ERR_UNKNOWN"


@pytest.mark.parametrize("kw,status", [
    (dict(d=96), L.LISA_ERR_UNSUPPORTED),
    (dict(dI=48), L.LISA_ERR_UNSUPPORTED),
    (dict(Hq=13), L.LISA_ERR_UNSUPPORTED),
    (dict(HI=3), L.LISA_ERR_UNSUPPORTED),
    (dict(M=48), L.LISA_ERR_UNSUPPORTED),
    (dict(M=2048), L.LISA_ERR_UNSUPPORTED),
    (dict(Hq=34, Hkv=2, HI=2), L.LISA_ERR_UNSUPPORTED),     # G = 17 > 16
    (dict(HI=18, Hkv=2, Hq=2), L.LISA_ERR_UNSUPPORTED),     # R = 9 > 8
    (dict(L_max=0), L.LISA_ERR_INVALID_ARG),
    (dict(B=-1), L.LISA_ERR_INVALID_ARG),
    (dict(dtype=7), L.LISA_ERR_INVALID_ARG),
    (dict(k_cache=0), L.LISA_ERR_INVALID_ARG),
    (dict(pos=0), L.LISA_ERR_INVALID_ARG),
    (dict(state=0), L.LISA_ERR_INVALID_ARG),
    (dict(v_cache=0x10008), L.LISA_ERR_INVALID_ARG),        # misaligned
])
def test_decode_rejects_bad_layer(kw, status):
    assert _decode(_layer(**kw)) == status
    assert L.last_error_msg() != ""


def test_decode_rejects_null_and_misaligned_inputs():
    c = _layer()
    assert _decode(c, q=None) == L.LISA_ERR_INVALID_ARG
    assert "q" in L.last_error_msg()
    assert _decode(c, out=ctypes.c_void_p(0x20004)) == L.LISA_ERR_INVALID_ARG


def test_decode_workspace_is_the_wide_forms_and_context_is_bounded():
    """The decode workspace holds the wide form's pieces, each rounded to 256
    bytes and sized for 64 CTAs per (sequence, KV head): arrival counters,
    per-CTA partial readouts of two heads, and the order keys of every cached
    position."""
    r256 = lambda x: (x + 255) // 256 * 256
    c = _layer(B=3, L_max=1000)
    pairs, d = 3 * 2, 128
    want = r256(pairs * 4) + r256(pairs * 64 * 2 * d * 4) + r256(pairs * 1000 * 4)
    assert L.lisa_workspace_bytes(c, 1, L.LISA_OP_DECODE) == want
    assert L.lisa_workspace_bytes(_layer(dtype=L.LISA_FP32), 1, L.LISA_OP_DECODE) == 0
    # the wide form asked for explicitly needs bf16 storage and the workspace
    assert _decode(_layer(decode_split=64), ws=None, ws_bytes=0) == L.LISA_ERR_WORKSPACE
    assert _decode(_layer(decode_split=32), ws_bytes=16) == L.LISA_ERR_WORKSPACE
    assert _decode(_layer(decode_split=64, dtype=L.LISA_FP32)) == L.LISA_ERR_UNSUPPORTED
    assert _decode(_layer(decode_split=24)) == L.LISA_ERR_INVALID_ARG
    # keys of one (sequence, KV head) must fit in a cluster's shared memory
    assert _decode(_layer(L_max=1 << 22)) == L.LISA_ERR_UNSUPPORTED


def test_empty_inputs_are_noops():
    c = _layer(B=0)
    assert _decode(c) == L.LISA_OK
    lib = L.lib()
    c1 = _layer()
    assert lib.lisa_append_cache(ctypes.byref(c1), FAKE, FAKE, FAKE, 0, None) == L.LISA_OK
    assert lib.lisa_prefill(ctypes.byref(c1), 0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 0,
                            None) == L.LISA_OK
    assert lib.lisa_indexer_topk(ctypes.byref(c1), FAKE, FAKE, 0, FAKE, FAKE, 0, None) == L.LISA_OK


def test_row_calls_validate():
    lib = L.lib()
    c = _layer(L_max=100)
    assert lib.lisa_append_cache(ctypes.byref(c), FAKE, FAKE, FAKE, -1, None) == L.LISA_ERR_INVALID_ARG
    assert lib.lisa_append_cache(ctypes.byref(c), FAKE, FAKE, FAKE, 101, None) == L.LISA_ERR_INVALID_ARG
    assert lib.lisa_append_cache(ctypes.byref(c), None, FAKE, FAKE, 5, None) == L.LISA_ERR_INVALID_ARG
    assert lib.lisa_indexer_topk(ctypes.byref(c), FAKE, FAKE, 5, None, FAKE, 1 << 40, None) == L.LISA_ERR_INVALID_ARG
    assert lib.lisa_indexer_topk(ctypes.byref(c), FAKE, FAKE, 5, FAKE, FAKE, 16, None) == L.LISA_ERR_WORKSPACE
    assert lib.lisa_prefill(ctypes.byref(c), 5, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 16,
                            None) == L.LISA_ERR_WORKSPACE
    assert lib.lisa_prefill(ctypes.byref(c), 5, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, None, FAKE, 1 << 40,
                            None) == L.LISA_ERR_INVALID_ARG


def test_workspace_sizes():
    c = _layer()
    pre = L.lisa_workspace_bytes(c, 16384, L.LISA_OP_PREFILL)
    assert pre >= 16384 * 12 * 128 * 4          # per-token linear outputs
    assert L.lisa_workspace_bytes(c, 4, L.LISA_OP_INDEXER_TOPK) > 0
    assert L.lisa_workspace_bytes(_layer(d=96), 1, L.LISA_OP_DECODE) == 0
    assert L.lisa_workspace_bytes(c, 1, 42) == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    lib = L.lib()
    # 2 KV heads x 4M positions x 4 bytes = 32 MiB per query row > the fixed scratch
    c = _layer(L_max=1 << 22)
    st = lib.lisa_indexer_topk_noalloc(ctypes.byref(c), FAKE, FAKE, 1, FAKE, None)
    assert st == L.LISA_ERR_UNSUPPORTED
    assert "scratch" in L.last_error_msg()
    assert lib.lisa_indexer_topk_noalloc(ctypes.byref(c), FAKE, FAKE, 0, FAKE, None) == L.LISA_OK
    assert lib.lisa_indexer_topk_noalloc(ctypes.byref(_layer()), FAKE, None, 1, FAKE, None) == L.LISA_ERR_INVALID_ARG


def _decode_variant(c, variant, ws=FAKE, ws_bytes=1 << 40, **ptrs):
    args = {n: ptrs.get(n, FAKE) for n in ["q", "k", "v", "kidx", "qidx", "w", "gate", "k_lin", "v_lin", "out"]}
    return L.lib().lisa_decode_step_variant(ctypes.byref(c), variant, args["q"], args["k"], args["v"], args["kidx"],
                                            args["qidx"], args["w"], args["gate"], args["k_lin"], args["v_lin"], 1,
                                            args["out"], None, ws, ws_bytes, None)


def test_variant_flags_are_validated():
    c = _layer()
    assert _decode_variant(c, 8) == L.LISA_ERR_INVALID_ARG
    assert "variant" in L.last_error_msg()
    # the linear branch's own keys / values are required by that variant only
    assert _decode_variant(c, L.LISA_VAR_LINEAR_KV_PER_QUERY_HEAD, k_lin=None) == L.LISA_ERR_INVALID_ARG
    assert "k_lin" in L.last_error_msg()
    assert _decode_variant(_layer(B=0), L.LISA_VAR_LINEAR_KV_PER_QUERY_HEAD, k_lin=None) == L.LISA_OK
    # a shared set sums all indexer heads in one group: at most 8 without per-head keys
    big = _layer(Hq=16, Hkv=4, HI=16)
    assert _decode_variant(big, L.LISA_VAR_SHARED_SET) == L.LISA_ERR_UNSUPPORTED
    assert L.lisa_workspace_bytes_variant(big, L.LISA_VAR_SHARED_SET, 1, L.LISA_OP_DECODE) == 0
    assert L.lisa_workspace_bytes_variant(
        big, L.LISA_VAR_SHARED_SET | L.LISA_VAR_KEY_PER_INDEXER_HEAD, 1, L.LISA_OP_DECODE) > 0


def test_variant_workspace_sizes():
    c = _layer()
    V1, V2, V3 = L.LISA_VAR_KEY_PER_INDEXER_HEAD, L.LISA_VAR_SHARED_SET, L.LISA_VAR_LINEAR_KV_PER_QUERY_HEAD
    ws = lambda v, T, op: L.lisa_workspace_bytes_variant(c, v, T, op)
    # variant 0 needs what the default calls need
    assert ws(0, 1, L.LISA_OP_DECODE) == L.lisa_workspace_bytes(c, 1, L.LISA_OP_DECODE)
    assert ws(0, 300, L.LISA_OP_PREFILL) == L.lisa_workspace_bytes(c, 300, L.LISA_OP_PREFILL)
    assert ws(0, 7, L.LISA_OP_INDEXER_TOPK) == L.lisa_workspace_bytes(c, 7, L.LISA_OP_INDEXER_TOPK)
    # the linear branch's own k / v alone keeps the fused decode kernel
    assert ws(V3, 1, L.LISA_OP_DECODE) == 0
    assert ws(V3, 300, L.LISA_OP_PREFILL) > ws(0, 300, L.LISA_OP_PREFILL)   # per-query-head increments
    # the other two run the indexer through the row path: order keys of every cached position
    for v in (V1, V2, V1 | V2):
        assert ws(v, 1, L.LISA_OP_DECODE) >= 16384 * 4
    # per-head keys: the per-head scores are kept beside the group sums
    assert ws(V1, 7, L.LISA_OP_INDEXER_TOPK) > ws(0, 7, L.LISA_OP_INDEXER_TOPK)
    assert ws(V2, 7, L.LISA_OP_INDEXER_TOPK) < ws(0, 7, L.LISA_OP_INDEXER_TOPK)    # one group instead of two
    assert ws(8, 7, L.LISA_OP_INDEXER_TOPK) == 0


def test_variant_calls_validate():
    lib = L.lib()
    c = _layer(L_max=100)
    V1 = L.LISA_VAR_KEY_PER_INDEXER_HEAD
    assert _decode_variant(c, V1, ws_bytes=16) == L.LISA_ERR_WORKSPACE
    assert lib.lisa_append_cache_variant(ctypes.byref(c), V1, FAKE, FAKE, None, 5, None) == L.LISA_ERR_INVALID_ARG
    assert lib.lisa_indexer_topk_variant(ctypes.byref(c), V1, FAKE, FAKE, 5, FAKE, FAKE, 16,
                                         None) == L.LISA_ERR_WORKSPACE
    assert lib.lisa_prefill_variant(ctypes.byref(c), V1, 101, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None,
                                    FAKE, None, FAKE, 1 << 40, None) == L.LISA_ERR_INVALID_ARG
    assert lib.lisa_prefill_variant(ctypes.byref(c), 0, 0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None,
                                    FAKE, None, FAKE, 0, None) == L.LISA_OK


def test_projection_calls_validate():
    lib = L.lib()
    c = _layer()
    pj = L.LisaProjC(1536, 0x30000, 0x30000)
    args = [FAKE] * 8
    assert lib.lisa_project_in(ctypes.byref(c), 0, None, 4, FAKE, *args[:7], None) == L.LISA_ERR_INVALID_ARG
    assert lib.lisa_project_in(ctypes.byref(c), 0, ctypes.byref(pj), 4, FAKE, *args[:6], None,
                               None) == L.LISA_ERR_INVALID_ARG
    bad = L.LisaProjC(1537, 0x30000, 0x30000)
    assert lib.lisa_project_in(ctypes.byref(c), 0, ctypes.byref(bad), 4, FAKE, *args[:7],
                               None) == L.LISA_ERR_UNSUPPORTED
    assert lib.lisa_project_out(ctypes.byref(_layer(dtype=L.LISA_FP32)), ctypes.byref(pj), 4, FAKE, FAKE,
                                None) == L.LISA_ERR_UNSUPPORTED
    assert lib.lisa_project_out(ctypes.byref(c), ctypes.byref(pj), 0, FAKE, FAKE, None) == L.LISA_OK
    assert lib.lisa_project_in(ctypes.byref(c), 16, ctypes.byref(pj), 4, FAKE, *args[:7],
                               None) == L.LISA_ERR_INVALID_ARG


def test_variant_workspace_formula():
    """Variant workspace = the documented pieces, each rounded to 256 bytes:
    order keys per selection group (and per indexer head with one key per
    head), the index lists, and for the prefill o_lin and the chunk
    increments of the linear branch (per query head with its own k, v)."""
    r256 = lambda x: (x + 255) // 256 * 256
    c = _layer(L_max=1000)
    B, Hq, Hkv, d, HI, M, T = 1, 12, 2, 128, 4, 256, 300
    V1, V2, V3 = L.LISA_VAR_KEY_PER_INDEXER_HEAD, L.LISA_VAR_SHARED_SET, L.LISA_VAR_LINEAR_KV_PER_QUERY_HEAD
    # decode (one row, every cached position): keys [Gs][L_keys] (+ [HI][L_keys]) + idx [Gs][M]
    Lk = 1000
    assert L.lisa_workspace_bytes_variant(c, V2, 1, L.LISA_OP_DECODE) == r256(Lk * 4) + r256(M * 4)
    assert L.lisa_workspace_bytes_variant(c, V1, 1, L.LISA_OP_DECODE) == (
        r256(Hkv * Lk * 4) + r256(HI * Lk * 4) + r256(Hkv * M * 4))
    # prefill: keys [Gs][T][T] + idx [T][Gs][M] + o_lin [T][Hq][d] + dS [LH][chunks][d][d] + total [LH][d][d]
    nc = (T + 63) // 64
    for v, Gs, LH, per_head in [(V2, 1, Hkv, False), (V3, Hkv, Hq, False), (V1 | V2, 1, Hkv, True)]:
        want = (r256(Gs * T * T * 4) + (r256(HI * T * T * 4) if per_head else 0) + r256(T * Gs * M * 4) +
                r256(T * Hq * d * 4) + r256(LH * nc * d * d * 4) + r256(LH * d * d * 4))
        assert L.lisa_workspace_bytes_variant(c, v, T, L.LISA_OP_PREFILL) == want, v
    # variant 0 runs the default calls: their workspace
    assert L.lisa_workspace_bytes_variant(c, 0, T, L.LISA_OP_PREFILL) == L.lisa_workspace_bytes(c, T, L.LISA_OP_PREFILL)
    assert B == 1
