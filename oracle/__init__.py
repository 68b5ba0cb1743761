"""CPU oracle for the Block-Union chunked-prefill path (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` use this package. The CUDA library never imports it and shares
no code with it. The arithmetic lives in ``ca_oracle.c`` (plain C, fp64);
this file only compiles it with gcc and marshals numpy / torch CPU arrays.

What each function computes, and the passages it follows, is documented in
``ca_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ca_oracle.c")
_LIB = os.path.join(_HERE, "libcaoracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``ca_oracle.c`` into ``libcaoracle.so`` (gcc, -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                               "-fno-fast-math", "-ffp-contract=off",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            I = ctypes.c_int
            lib.oracle_block_tables.argtypes = [P, I, I, I, I, I, P, P, P, P]
            lib.oracle_block_tables.restype = I
            lib.oracle_attention_rows.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I,
                                                  ctypes.c_double, P, ctypes.c_int64, P, P, I]
            lib.oracle_attention_rows.restype = I
            lib.oracle_attention_tile_rows.argtypes = [P, P, P, P, I, P, I, I, I, I, I, I, I,
                                                       ctypes.c_double, P, ctypes.c_int64, P, P,
                                                       I]
            lib.oracle_attention_tile_rows.restype = I
            lib.oracle_attention_rows_e4m3.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I,
                                                       ctypes.c_double, P, ctypes.c_int64, P, P,
                                                       I]
            lib.oracle_attention_rows_e4m3.restype = I
            lib.oracle_e4m3_decode.argtypes = [I]
            lib.oracle_e4m3_decode.restype = ctypes.c_double
            lib.oracle_merge_states.argtypes = [P, P, P, P, ctypes.c_int64, I, P, P]
            lib.oracle_merge_states.restype = I
            lib.oracle_tile_span_tables.argtypes = [P, I, I, I, I, I, P, P]
            lib.oracle_tile_span_tables.restype = I
            lib.oracle_visible_pairs.argtypes = [P, P, P, I, I, I, I, I, I]
            lib.oracle_visible_pairs.restype = ctypes.c_int64
            _lib = lib
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _bf16_bits(t) -> np.ndarray:
    """torch bf16 CPU tensor -> contiguous uint16 numpy view of its bits."""
    import torch
    if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16:
        raise TypeError("expected a torch.bfloat16 tensor")
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def block_tables(mask: np.ndarray, group: int, csr: bool = True):
    """Block-Union tables of a uint8 mask [B, H_q, nQ, nKVmax].

    Returns ``(tables [B, H_kv, nKVmax] int32, counts [B, H_kv] int32,
    indptr [B*H_kv + 1] int32 | None, indices [sum counts] int32 | None)``."""
    mask = np.ascontiguousarray(mask, dtype=np.uint8)
    if mask.ndim != 4:
        raise ValueError("mask must be [B, H_q, nQ, nKVmax]")
    B, H_q, nQ, nK = mask.shape
    if group <= 0 or H_q % group:
        raise ValueError("group must divide H_q")
    H_kv = H_q // group
    tables = np.empty((B, H_kv, nK), np.int32)
    counts = np.empty((B, H_kv), np.int32)
    indptr = np.empty(B * H_kv + 1, np.int32) if csr else None
    indices = np.empty(max(1, B * H_kv * nK), np.int32) if csr else None
    st = _load().oracle_block_tables(_ptr(mask), B, H_q, nQ, nK, group, _ptr(tables),
                                     _ptr(counts), _ptr(indptr), _ptr(indices))
    if st != 0:
        raise ValueError(f"oracle_block_tables failed ({st})")
    if csr:
        indices = indices[: int(indptr[-1])].copy()
    return tables, counts, indptr, indices


def attention(Q, K, V, chunk_start: Sequence[int], blk: int, tables=None, counts=None,
              scale: Optional[float] = None, rows: Optional[np.ndarray] = None,
              threads: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """fp64 chunk attention over the selected blocks (``tables is None``: dense).

    Q bf16 [B, H_q, C, D]; K, V bf16 [B, H_kv, L_max, D] (torch CPU tensors).
    ``rows``: optional int64 flat row ids ``(b*H_q + h)*C + r``; then the result
    is ``O [n, D], LSE [n]``, else ``O [B, H_q, C, D], LSE [B, H_q, C]``."""
    B, H_q, C, D = Q.shape
    Bk, H_kv, L_max, Dk = K.shape
    if Bk != B or Dk != D or tuple(V.shape) != tuple(K.shape):
        raise ValueError("shape mismatch")
    if scale is None:
        scale = 1.0 / float(np.sqrt(D))
    q, k, v = _bf16_bits(Q), _bf16_bits(K), _bf16_bits(V)
    cs = np.ascontiguousarray(chunk_start, dtype=np.int32)
    if cs.shape != (B,):
        raise ValueError("chunk_start must have B entries")
    t = c = None
    if tables is not None:
        t = np.ascontiguousarray(tables, dtype=np.int32)
        c = np.ascontiguousarray(counts, dtype=np.int32)
        if t.shape != (B, H_kv, L_max // blk) or c.shape != (B, H_kv):
            raise ValueError("tables must be [B, H_kv, L_max/blk], counts [B, H_kv]")
    r = None
    n = B * H_q * C
    if rows is not None:
        r = np.ascontiguousarray(rows, dtype=np.int64)
        n = r.size
    O = np.empty((n, D), np.float64)
    LSE = np.empty(n, np.float64)
    st = _load().oracle_attention_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(t), _ptr(c), _ptr(cs),
                                       B, H_q, H_kv, C, L_max, D, blk, float(scale), _ptr(r),
                                       n, _ptr(O), _ptr(LSE), int(threads))
    if st != 0:
        raise ValueError(f"oracle_attention_rows failed ({st})")
    if rows is None:
        return O.reshape(B, H_q, C, D), LSE.reshape(B, H_q, C)
    return O, LSE


def _u8(t) -> np.ndarray:
    """uint8 codes of a torch uint8 / float8_e4m3fn tensor or a numpy array."""
    if hasattr(t, "detach"):
        import torch
        t = t.detach().cpu().contiguous()
        if t.dtype != torch.uint8:
            t = t.view(torch.uint8)
        return t.numpy()
    return np.ascontiguousarray(t, dtype=np.uint8)


def e4m3_decode(code: int) -> float:
    """The real value of one FP8 E4M3 code (0..255)."""
    return float(_load().oracle_e4m3_decode(int(code)))


def attention_e4m3(Q8, K8, V8, descale: Sequence[float], chunk_start: Sequence[int], blk: int,
                   tables=None, counts=None, scale: Optional[float] = None,
                   rows: Optional[np.ndarray] = None,
                   threads: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """fp64 chunk attention on FP8 inputs: the real Q, K, V are
    ``descale[0] * Q8``, ``descale[1] * K8``, ``descale[2] * V8`` with the
    E4M3 codes decoded exactly. Shapes and results as :func:`attention`."""
    q, k, v = _u8(Q8), _u8(K8), _u8(V8)
    B, H_q, C, D = q.shape
    Bk, H_kv, L_max, Dk = k.shape
    if Bk != B or Dk != D or v.shape != k.shape:
        raise ValueError("shape mismatch")
    if scale is None:
        scale = 1.0 / float(np.sqrt(D))
    ds = np.ascontiguousarray(descale, dtype=np.float64)
    if ds.shape != (3,):
        raise ValueError("descale must hold the Q, K and V factors")
    cs = np.ascontiguousarray(chunk_start, dtype=np.int32)
    t = c = None
    if tables is not None:
        t = np.ascontiguousarray(tables, dtype=np.int32)
        c = np.ascontiguousarray(counts, dtype=np.int32)
    r = None
    n = B * H_q * C
    if rows is not None:
        r = np.ascontiguousarray(rows, dtype=np.int64)
        n = r.size
    O = np.empty((n, D), np.float64)
    LSE = np.empty(n, np.float64)
    st = _load().oracle_attention_rows_e4m3(_ptr(q), _ptr(k), _ptr(v), _ptr(ds), _ptr(t), _ptr(c),
                                            _ptr(cs), B, H_q, H_kv, C, L_max, D, blk,
                                            float(scale), _ptr(r), n, _ptr(O), _ptr(LSE),
                                            int(threads))
    if st != 0:
        raise ValueError(f"oracle_attention_rows_e4m3 failed ({st})")
    if rows is None:
        return O.reshape(B, H_q, C, D), LSE.reshape(B, H_q, C)
    return O, LSE


def attention_tile(Q, K, V, chunk_start: Sequence[int], blk: int, mask,
                   scale: Optional[float] = None, rows: Optional[np.ndarray] = None,
                   threads: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """fp64 per-tile block-sparse chunk attention: row r of head h attends to
    the keys k <= chunk_start[b] + r of the blocks its own Q-block selects,
    ``mask[b, h, r // blk, k // blk] != 0`` (no Q-block or head union).

    ``mask`` uint8 [B, H_q, nQ, L_max/blk]; the rest as in :func:`attention`."""
    B, H_q, C, D = Q.shape
    Bk, H_kv, L_max, Dk = K.shape
    if Bk != B or Dk != D or tuple(V.shape) != tuple(K.shape):
        raise ValueError("shape mismatch")
    if scale is None:
        scale = 1.0 / float(np.sqrt(D))
    m = np.ascontiguousarray(mask, dtype=np.uint8)
    if m.ndim != 4 or m.shape[:2] != (B, H_q) or m.shape[3] != L_max // blk:
        raise ValueError("mask must be [B, H_q, nQ, L_max/blk]")
    q, k, v = _bf16_bits(Q), _bf16_bits(K), _bf16_bits(V)
    cs = np.ascontiguousarray(chunk_start, dtype=np.int32)
    if cs.shape != (B,):
        raise ValueError("chunk_start must have B entries")
    r = None
    n = B * H_q * C
    if rows is not None:
        r = np.ascontiguousarray(rows, dtype=np.int64)
        n = r.size
    O = np.empty((n, D), np.float64)
    LSE = np.empty(n, np.float64)
    st = _load().oracle_attention_tile_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(m), m.shape[2],
                                            _ptr(cs), B, H_q, H_kv, C, L_max, D, blk,
                                            float(scale), _ptr(r), n, _ptr(O), _ptr(LSE),
                                            int(threads))
    if st != 0:
        raise ValueError(f"oracle_attention_tile_rows failed ({st})")
    if rows is None:
        return O.reshape(B, H_q, C, D), LSE.reshape(B, H_q, C)
    return O, LSE


def merge_states(O_a, LSE_a, O_b, LSE_b) -> Tuple[np.ndarray, np.ndarray]:
    """Merge of two attention results over disjoint key sets (fp64): returns
    ``O, LSE`` with ``LSE = ln(e^LSE_a + e^LSE_b)`` and ``O`` the
    ``e^(LSE_x - LSE)``-weighted sum. Shapes ``[..., D]`` and ``[...]``."""
    oa = np.ascontiguousarray(O_a, dtype=np.float64)
    ob = np.ascontiguousarray(O_b, dtype=np.float64)
    la = np.ascontiguousarray(LSE_a, dtype=np.float64)
    lb = np.ascontiguousarray(LSE_b, dtype=np.float64)
    if oa.shape != ob.shape or la.shape != lb.shape or oa.shape[:-1] != la.shape:
        raise ValueError("shape mismatch")
    D = oa.shape[-1]
    rows = la.size
    O = np.empty_like(oa)
    LSE = np.empty_like(la)
    st = _load().oracle_merge_states(_ptr(oa), _ptr(la), _ptr(ob), _ptr(lb), rows, D, _ptr(O),
                                     _ptr(LSE))
    if st != 0:
        raise ValueError(f"oracle_merge_states failed ({st})")
    return O, LSE


def tile_span_tables(mask, span: int) -> Tuple[np.ndarray, np.ndarray]:
    """Span tables of the per-tile path: per (b, h, span of ``span`` Q-blocks)
    the ascending KV blocks any Q-block of the span selects, each entry
    ``j | bits << 24`` with bit u set iff Q-block ``span*s + u`` selects j;
    padded with -1. Returns tables int32 [B, H_q, nS, nKVmax], counts int32
    [B, H_q, nS], nS = ceil(nQ / span)."""
    m = np.ascontiguousarray(mask, dtype=np.uint8)
    B, H_q, nQ, nKVmax = m.shape
    nS = -(-nQ // span)
    T = np.empty((B, H_q, nS, nKVmax), np.int32)
    c = np.empty((B, H_q, nS), np.int32)
    st = _load().oracle_tile_span_tables(_ptr(m), B, H_q, nQ, nKVmax, span, _ptr(T), _ptr(c))
    if st != 0:
        raise ValueError(f"oracle_tile_span_tables failed ({st})")
    return T, c


def visible_pairs(chunk_start: Sequence[int], B: int, H_q: int, H_kv: int, C: int, L_max: int,
                  blk: int, tables=None, counts=None) -> int:
    """Number of (query row, key) pairs the attention touches (4*D flops each)."""
    cs = np.ascontiguousarray(chunk_start, dtype=np.int32)
    t = None if tables is None else np.ascontiguousarray(tables, dtype=np.int32)
    c = None if counts is None else np.ascontiguousarray(counts, dtype=np.int32)
    return int(_load().oracle_visible_pairs(_ptr(t), _ptr(c), _ptr(cs), B, H_q, H_kv, C,
                                            L_max, blk))
