"""The C-ABI library: it loads, exports every symbol ``include/*.h`` declares,
and rejects bad arguments on the host with the documented status codes.
No compute call is made here (every case below fails its host-side checks
before anything is enqueued)."""
import ctypes
import glob
import os
import re

import pytest

import serving_block_union_b200 as ca
from serving_block_union_b200 import build as ca_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    ca_build.build()
    return ca.load_library()


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w\s\*]*?\b(ca_\w+)\s*\(", text, flags=re.M):
            names.add(m.group(1))
    return names


def test_exports_every_declared_symbol(lib):
    declared = _declared_functions()
    assert {"ca_build_block_tables", "ca_chunk_attention", "ca_dense_chunk_attention"} <= declared
    for name in sorted(declared):
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"
    assert set(ca.EXPORTED_SYMBOLS) <= declared


def test_status_strings(lib):
    for code, name in [(0, "CA_OK"), (1, "CA_ERR_INVALID_ARG"), (2, "CA_ERR_SHAPE"),
                       (3, "CA_ERR_ALIGN"), (4, "CA_ERR_UNSUPPORTED"), (5, "CA_ERR_WORKSPACE"),
                       (6, "CA_ERR_TABLE"), (7, "CA_ERR_TIMEOUT"), (8, "CA_ERR_CUDA")]:
        assert ca.status_string(code) == name
    assert ca.status_string(99) == "CA_ERR_UNKNOWN"
    assert lib.ca_version() >= 100


def test_workspace_bytes(lib):
    n = lib.ca_workspace_bytes(1, 32, 8, 2048, 128)
    assert n >= 16 and n % 256 == 0
    assert lib.ca_workspace_bytes(0, 32, 8, 2048, 128) == 0
    # 128K headline shape on 148 SMs (the count used where no device can be
    # read, and B200's): 256 work items, 148 whole, 108 cut into 4 segments;
    # 256-byte header, one uint32 counter per split item (padded to 256 B),
    # fp32 partial LSE and bf16 partial O per segment row (256 rows, D = 128)
    rows = 108 * 4 * 256
    assert n == 256 + 512 + 4 * rows + 2 * rows * 128


# Fake device addresses: never dereferenced because every call below fails
# its host-side checks first.
A16 = ctypes.c_void_p(1 << 20)
A_MIS = ctypes.c_void_p((1 << 20) + 2)


def _attn(lib, **kw):
    a = dict(Q=A16, K=A16, V=A16, tables=A16, counts=A16, B=1, H_q=32, H_kv=8, C=2048,
             L_max=34816, D=128, blk=128, scale=0.088, O=A16, LSE=A16, ws=A16, ws_bytes=256,
             cs=[32768])
    a.update(kw)
    cs = (ctypes.c_int32 * len(a["cs"]))(*a["cs"])
    return lib.ca_chunk_attention(a["Q"], a["K"], a["V"], a["tables"], a["counts"], cs, a["B"],
                                  a["H_q"], a["H_kv"], a["C"], a["L_max"], a["D"], a["blk"],
                                  a["scale"], a["O"], a["LSE"], a["ws"], a["ws_bytes"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(Q=None), ca.CA_ERR_INVALID_ARG),
    (dict(tables=None), ca.CA_ERR_INVALID_ARG),
    (dict(ws=None), ca.CA_ERR_INVALID_ARG),
    (dict(C=0), ca.CA_ERR_INVALID_ARG),
    (dict(scale=0.0), ca.CA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), ca.CA_ERR_INVALID_ARG),
    (dict(H_kv=6), ca.CA_ERR_SHAPE),
    (dict(L_max=34800), ca.CA_ERR_SHAPE),
    (dict(cs=[33000]), ca.CA_ERR_SHAPE),
    (dict(cs=[-1]), ca.CA_ERR_SHAPE),
    (dict(D=96), ca.CA_ERR_UNSUPPORTED),
    (dict(blk=32, L_max=34816), ca.CA_ERR_UNSUPPORTED),
    (dict(H_q=96, H_kv=3), ca.CA_ERR_UNSUPPORTED),
    (dict(Q=A_MIS), ca.CA_ERR_ALIGN),
    (dict(O=A_MIS), ca.CA_ERR_ALIGN),
    (dict(ws_bytes=16), ca.CA_ERR_WORKSPACE),
    (dict(ws=ctypes.c_void_p((1 << 20) + 16)), ca.CA_ERR_WORKSPACE),
])
def test_attention_host_checks(lib, kw, code):
    assert _attn(lib, **kw) == code


@pytest.mark.parametrize("kw,code", [
    (dict(Q=None), ca.CA_ERR_INVALID_ARG),
    (dict(counts=None), ca.CA_ERR_INVALID_ARG),
    (dict(C=0), ca.CA_ERR_INVALID_ARG),
    (dict(scale=-1.0), ca.CA_ERR_INVALID_ARG),
    (dict(H_kv=6), ca.CA_ERR_SHAPE),          # H_q % H_kv != 0: the same code as above
    (dict(L_max=34800), ca.CA_ERR_SHAPE),
    (dict(cs=[33000]), ca.CA_ERR_SHAPE),
    (dict(D=96), ca.CA_ERR_UNSUPPORTED),
    (dict(H_q=96, H_kv=3), ca.CA_ERR_UNSUPPORTED),
    (dict(V=A_MIS), ca.CA_ERR_ALIGN),
    (dict(LSE=ctypes.c_void_p((1 << 20) + 2)), ca.CA_ERR_ALIGN),
])
def test_noalloc_host_checks_match_workspace_entry_point(lib, kw, code):
    """The allocation-free entry point reports the same host-side error codes
    as ca_chunk_attention, before it touches the GPU (no device needed)."""
    a = dict(Q=A16, K=A16, V=A16, tables=A16, counts=A16, B=1, H_q=32, H_kv=8, C=2048,
             L_max=34816, D=128, blk=128, scale=0.088, O=A16, LSE=A16, cs=[32768])
    a.update(kw)
    cs = (ctypes.c_int32 * len(a["cs"]))(*a["cs"])
    st = lib.ca_chunk_attention_noalloc(a["Q"], a["K"], a["V"], a["tables"], a["counts"], cs,
                                        a["B"], a["H_q"], a["H_kv"], a["C"], a["L_max"], a["D"],
                                        a["blk"], a["scale"], a["O"], a["LSE"], None, None)
    assert st == code
    assert _attn(lib, **{k: v for k, v in kw.items()}) == code


def test_dense_host_checks(lib):
    cs = (ctypes.c_int32 * 1)(32768)
    st = lib.ca_dense_chunk_attention(A16, A16, A16, cs, 1, 32, 8, 2048, 34816, 96, 128, 0.1,
                                      A16, A16, A16, 256, None)
    assert st == ca.CA_ERR_UNSUPPORTED
    st = lib.ca_dense_chunk_attention(A16, A16, A16, None, 1, 32, 8, 2048, 34816, 128, 128, 0.1,
                                      A16, A16, A16, 256, None)
    assert st == ca.CA_ERR_INVALID_ARG


def test_build_tables_host_checks(lib):
    f = lib.ca_build_block_tables
    assert f(None, 1, 32, 16, 272, 4, A16, A16, None, None, None) == ca.CA_ERR_INVALID_ARG
    assert f(A16, 1, 32, 16, 272, 5, A16, A16, None, None, None) == ca.CA_ERR_SHAPE
    assert f(A16, 1, 32, 16, 272, 4, A_MIS, A16, None, None, None) == ca.CA_ERR_ALIGN
    assert f(A16, 1, 32, 16, 272, 4, A16, A16, None, A16, None) == ca.CA_ERR_INVALID_ARG
    assert f(A16, 0, 32, 16, 272, 4, A16, A16, None, None, None) == ca.CA_ERR_INVALID_ARG


def test_tile_path_host_checks(lib):
    assert lib.ca_tile_span(128) == 2 and lib.ca_tile_span(64) == 4
    assert lib.ca_tile_span(32) == 0
    f = lib.ca_build_tile_tables
    assert f(None, 1, 32, 16, 272, 128, A16, A16, None) == ca.CA_ERR_INVALID_ARG
    assert f(A16, 1, 32, 16, 272, 32, A16, A16, None) == ca.CA_ERR_UNSUPPORTED
    assert f(A16, 1, 32, 16, 1 << 24, 128, A16, A16, None) == ca.CA_ERR_SHAPE
    assert f(A16, 1, 32, 16, 272, 128, A_MIS, A16, None) == ca.CA_ERR_ALIGN
    cs = (ctypes.c_int32 * 1)(32768)
    g = lib.ca_tile_chunk_attention
    assert g(A16, A16, A16, None, A16, cs, 1, 32, 8, 2048, 34816, 128, 128, 0.1, A16, A16, A16,
             256, None) == ca.CA_ERR_INVALID_ARG
    assert g(A16, A16, A16, A16, A16, cs, 1, 32, 8, 2048, 34800, 128, 128, 0.1, A16, A16, A16,
             256, None) == ca.CA_ERR_SHAPE
    assert g(A16, A16, A16, A16, A16, cs, 1, 32, 8, 2048, 34816, 96, 128, 0.1, A16, A16, A16,
             256, None) == ca.CA_ERR_UNSUPPORTED


def test_bits_build_host_checks(lib):
    f = lib.ca_build_block_tables_bits
    assert f(None, 1, 32, 16, 272, 4, A16, A16, None, None, None) == ca.CA_ERR_INVALID_ARG
    assert f(A16, 1, 32, 16, 272, 3, A16, A16, None, None, None) == ca.CA_ERR_SHAPE
    assert f(ctypes.c_void_p((1 << 20) + 2), 1, 32, 16, 272, 4, A16, A16, None, None,
             None) == ca.CA_ERR_ALIGN
    assert f(A16, 1, 32, 16, 272, 4, A16, A16, None, A16, None) == ca.CA_ERR_INVALID_ARG


def test_paged_path_host_checks(lib):
    f = lib.ca_build_kv_pages
    assert f(A16, 1, 32, 16, 272, 4, A16, A16, None, A16, None) == ca.CA_ERR_INVALID_ARG
    assert f(A16, 1, 32, 16, 272, 5, A16, A16, A16, A16, None) == ca.CA_ERR_SHAPE
    assert f(A16, 1, 32, 16, 272, 4, A16, A16, A_MIS, A16, None) == ca.CA_ERR_ALIGN
    g = lib.ca_paged_chunk_attention
    cs = (ctypes.c_int32 * 2)(32768, 1024)

    def call(indptr=A16, nnz=100, lens=(2048, 100), L_max=34816):
        cl = None if lens is None else (ctypes.c_int32 * 2)(*lens)
        return g(A16, A16, A16, indptr, A16, nnz, cs, cl, 2, 32, 8, 2048, L_max, 128, 128, 0.1,
                 A16, A16, A16, 256, None)
    assert call(indptr=None) == ca.CA_ERR_INVALID_ARG
    assert call(nnz=-1) == ca.CA_ERR_INVALID_ARG
    assert call(lens=(2049, 100)) == ca.CA_ERR_SHAPE      # longer than C
    assert call(lens=(-1, 100)) == ca.CA_ERR_SHAPE
    # a short chunk may sit where a full one would not fit
    cs2 = (ctypes.c_int32 * 2)(34000, 0)
    cl2 = (ctypes.c_int32 * 2)(816, 2048)
    assert g(A16, A16, A16, A16, A16, 10, cs2, cl2, 2, 32, 8, 2048, 34816, 96, 128, 0.1, A16,
             A16, A16, 256, None) == ca.CA_ERR_UNSUPPORTED   # passes the shape checks, D = 96
    cl3 = (ctypes.c_int32 * 2)(817, 2048)
    assert g(A16, A16, A16, A16, A16, 10, cs2, cl3, 2, 32, 8, 2048, 34816, 128, 128, 0.1, A16,
             A16, A16, 256, None) == ca.CA_ERR_SHAPE


def test_merge_states_host_checks(lib):
    f = lib.ca_merge_attention_states
    assert f(None, A16, A16, A16, 10, 128, A16, A16, None) == ca.CA_ERR_INVALID_ARG
    assert f(A16, None, A16, A16, 10, 128, A16, A16, None) == ca.CA_ERR_INVALID_ARG
    assert f(A16, A16, A16, A16, 10, 128, None, A16, None) == ca.CA_ERR_INVALID_ARG
    assert f(A16, A16, A16, A16, -1, 128, A16, A16, None) == ca.CA_ERR_INVALID_ARG
    assert f(A16, A16, A16, A16, 10, 0, A16, A16, None) == ca.CA_ERR_INVALID_ARG
    assert f(A16, A16, A16, A16, 10, 100, A16, A16, None) == ca.CA_ERR_SHAPE
    assert f(A16, A16, A16, A16, 10, 4096, A16, A16, None) == ca.CA_ERR_UNSUPPORTED
    assert f(A_MIS, A16, A16, A16, 10, 128, A16, A16, None) == ca.CA_ERR_ALIGN
    assert f(A16, A16, A16, A16, 10, 128, A_MIS, A16, None) == ca.CA_ERR_ALIGN
    assert f(A16, ctypes.c_void_p((1 << 20) + 2), A16, A16, 10, 128, A16, A16,
             None) == ca.CA_ERR_ALIGN
    assert f(A16, A16, A16, A16, 0, 128, A16, None, None) == ca.CA_OK   # empty: no launch
    g = lib.ca_merge_attention_states_n
    arr = (ctypes.c_void_p * 9)(*([A16.value] * 9))
    assert g(arr, arr, 1, 10, 128, A16, A16, None) == ca.CA_ERR_INVALID_ARG
    assert g(arr, arr, 9, 10, 128, A16, A16, None) == ca.CA_ERR_UNSUPPORTED
    assert g(None, arr, 2, 10, 128, A16, A16, None) == ca.CA_ERR_INVALID_ARG
    holey = (ctypes.c_void_p * 3)(A16.value, None, A16.value)
    assert g(holey, arr, 3, 10, 128, A16, A16, None) == ca.CA_ERR_INVALID_ARG
    assert g(arr, arr, 8, 0, 64, A16, A16, None) == ca.CA_OK


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    import importlib
    monkeypatch.setattr(ca, "_lib", None)
    monkeypatch.setattr(ca, "_LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError):
        ca.load_library()
