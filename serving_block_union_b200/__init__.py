"""serving_block_union_b200 — B200 (sm_100a) CompactAttention chunked-prefill hot path.

Python binding of ``libcompactattn.so`` (C ABI declared in
``include/compactattn.h``). This module only marshals arguments: it checks
dtypes, devices and contiguity, allocates outputs with torch when the caller
did not pass them, and hands raw pointers plus the current CUDA stream to the
library. Every step of the path runs in the library's kernels; there is no
fallback. If the library is missing or fails to load, every call raises.

Entry points (same names as the C ABI, minus the ``ca_`` prefix):

* ``build_block_tables(mask, group)`` — Block-Union tables (selection stage).
* ``chunk_attention(Q, K, V, tables, counts, chunk_start)`` — zero-copy paged
  attention over the tables (execution stage).
* ``dense_chunk_attention(Q, K, V, chunk_start, blk)`` — the dense paged path.
"""
from __future__ import annotations

import ctypes
import math
import os
import threading
from typing import Optional, Sequence, Tuple

import torch

__all__ = [
    "CAError",
    "library_path",
    "load_library",
    "status_string",
    "build_block_tables",
    "workspace_bytes",
    "new_workspace",
    "chunk_attention",
    "dense_chunk_attention",
    "read_device_status",
    "chunk_attention_noalloc",
    "compact_kv_blocks",
    "compacted_chunk_attention",
    "build_block_tables_bits",
    "build_kv_pages",
    "selftest_bounded_wait",
    "tile_span",
    "build_tile_tables",
    "tile_chunk_attention",
    "paged_chunk_attention",
    "chunk_attention_fp8",
    "merge_attention_states",
    "EXPORTED_SYMBOLS",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libcompactattn.so")
_lock = threading.Lock()
_lib = None

CA_OK = 0
CA_ERR_INVALID_ARG = 1
CA_ERR_SHAPE = 2
CA_ERR_ALIGN = 3
CA_ERR_UNSUPPORTED = 4
CA_ERR_WORKSPACE = 5
CA_ERR_TABLE = 6
CA_ERR_TIMEOUT = 7
CA_ERR_CUDA = 8

EXPORTED_SYMBOLS = (
    "ca_status_string",
    "ca_version",
    "ca_build_block_tables",
    "ca_workspace_bytes",
    "ca_chunk_attention",
    "ca_dense_chunk_attention",
    "ca_read_device_status",
    "ca_chunk_attention_noalloc",
    "ca_selftest_bounded_wait",
    "ca_compact_kv_blocks",
    "ca_compacted_chunk_attention",
    "ca_tile_span",
    "ca_build_kv_pages",
    "ca_build_block_tables_bits",
    "ca_chunk_attention_fp8",
    "ca_paged_chunk_attention",
    "ca_build_tile_tables",
    "ca_tile_chunk_attention",
    "ca_merge_attention_states",
    "ca_merge_attention_states_n",
)


class CAError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {status_string(status)} ({status})")
        self.status = status


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load ``libcompactattn.so`` (raises if it is absent: build it with
    ``python -m serving_block_union_b200.build``)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is missing; run `python -m serving_block_union_b200.build`")
        lib = ctypes.CDLL(_LIB_PATH)
        P, I, F, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        lib.ca_status_string.argtypes = [I]
        lib.ca_status_string.restype = ctypes.c_char_p
        lib.ca_version.argtypes = []
        lib.ca_version.restype = I
        lib.ca_build_block_tables.argtypes = [P, I, I, I, I, I, P, P, P, P, P]
        lib.ca_build_block_tables.restype = I
        lib.ca_workspace_bytes.argtypes = [I, I, I, I, I]
        lib.ca_workspace_bytes.restype = S
        lib.ca_chunk_attention.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, F, P, P, P, S, P]
        lib.ca_chunk_attention.restype = I
        lib.ca_dense_chunk_attention.argtypes = [P, P, P, P, I, I, I, I, I, I, I, F, P, P, P, S, P]
        lib.ca_dense_chunk_attention.restype = I
        lib.ca_read_device_status.argtypes = [P, P]
        lib.ca_read_device_status.restype = I
        lib.ca_chunk_attention_noalloc.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, F, P, P,
                                                   P, P]
        lib.ca_chunk_attention_noalloc.restype = I
        lib.ca_selftest_bounded_wait.argtypes = [P, ctypes.c_longlong, P]
        lib.ca_selftest_bounded_wait.restype = I
        lib.ca_compact_kv_blocks.argtypes = [P, P, P, P, I, I, I, I, I, P, P, P]
        lib.ca_compact_kv_blocks.restype = I
        lib.ca_compacted_chunk_attention.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, F, P,
                                                     P, P, S, P]
        lib.ca_compacted_chunk_attention.restype = I
        lib.ca_chunk_attention_fp8.argtypes = [P, P, P, F, F, F, P, P, P, I, I, I, I, I, I, I, F,
                                               P, P, P, S, P]
        lib.ca_chunk_attention_fp8.restype = I
        lib.ca_build_block_tables_bits.argtypes = [P, I, I, I, I, I, P, P, P, P, P]
        lib.ca_build_block_tables_bits.restype = I
        lib.ca_build_kv_pages.argtypes = [P, I, I, I, I, I, P, P, P, P, P]
        lib.ca_build_kv_pages.restype = I
        lib.ca_paged_chunk_attention.argtypes = [P, P, P, P, P, ctypes.c_longlong, P, P, I, I, I,
                                                 I, I, I, I, F, P, P, P, S, P]
        lib.ca_paged_chunk_attention.restype = I
        lib.ca_tile_span.argtypes = [I]
        lib.ca_tile_span.restype = I
        lib.ca_build_tile_tables.argtypes = [P, I, I, I, I, I, P, P, P]
        lib.ca_build_tile_tables.restype = I
        lib.ca_tile_chunk_attention.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, F, P, P, P,
                                                S, P]
        lib.ca_tile_chunk_attention.restype = I
        lib.ca_merge_attention_states.argtypes = [P, P, P, P, ctypes.c_longlong, I, P, P, P]
        lib.ca_merge_attention_states.restype = I
        lib.ca_merge_attention_states_n.argtypes = [P, P, I, ctypes.c_longlong, I, P, P, P]
        lib.ca_merge_attention_states_n.restype = I
        _lib = lib
        return lib


def status_string(status: int) -> str:
    return load_library().ca_status_string(int(status)).decode()


# ----------------------------------------------------------------- helpers

def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream: Optional[torch.cuda.Stream], device: torch.device):
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, ndim: int):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got shape {tuple(t.shape)}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _chunk_start_host(chunk_start, B: int) -> ctypes.Array:
    if isinstance(chunk_start, torch.Tensor):
        vals = [int(x) for x in chunk_start.detach().cpu().reshape(-1).tolist()]
    else:
        vals = [int(x) for x in chunk_start]
    if len(vals) != B:
        raise ValueError(f"chunk_start must have B={B} entries, got {len(vals)}")
    return (ctypes.c_int32 * B)(*vals)


def _check(fn: str, status: int):
    if status != CA_OK:
        raise CAError(fn, status)


# ----------------------------------------------------------------- tables

def build_block_tables(mask: torch.Tensor, group: int, csr: bool = False,
                       tables: Optional[torch.Tensor] = None,
                       counts: Optional[torch.Tensor] = None,
                       stream: Optional[torch.cuda.Stream] = None):
    """Block-Union tables of a uint8 / bool mask ``[B, H_q, nQ, nKVmax]``.

    Returns ``(tables int32 [B, H_kv, nKVmax], counts int32 [B, H_kv],
    indptr int32 [B*H_kv+1] | None, indices int32 [B*H_kv*nKVmax] | None)``;
    the valid part of ``indices`` is ``indices[:indptr[-1]]``."""
    if mask.dtype == torch.bool:
        mask = mask.view(torch.uint8)
    _need(mask, "mask", torch.uint8, 4)
    lib = load_library()
    B, H_q, nQ, nK = mask.shape
    if group <= 0 or H_q % group:
        raise ValueError("group must divide H_q")
    H_kv = H_q // group
    dev = mask.device
    if tables is None:
        tables = torch.empty((B, H_kv, nK), dtype=torch.int32, device=dev)
    if counts is None:
        counts = torch.empty((B, H_kv), dtype=torch.int32, device=dev)
    _need(tables, "tables", torch.int32, 3)
    _need(counts, "counts", torch.int32, 2)
    indptr = indices = None
    if csr:
        indptr = torch.empty(B * H_kv + 1, dtype=torch.int32, device=dev)
        indices = torch.empty(B * H_kv * nK, dtype=torch.int32, device=dev)
    st = lib.ca_build_block_tables(_ptr(mask), B, H_q, nQ, nK, int(group), _ptr(tables),
                                   _ptr(counts), _ptr(indptr), _ptr(indices),
                                   _stream_handle(stream, dev))
    _check("ca_build_block_tables", st)
    return tables, counts, indptr, indices


def build_block_tables_bits(mask_bits: torch.Tensor, nKVmax: int, group: int, csr: bool = False,
                            tables: Optional[torch.Tensor] = None,
                            counts: Optional[torch.Tensor] = None,
                            stream: Optional[torch.cuda.Stream] = None):
    """Block-Union tables from a bit-packed mask ``int32/uint32 [B, H_q, nQ,
    ceil(nKVmax/32)]`` (bit k of word w selects block 32*w + k); the same
    outputs as :func:`build_block_tables`."""
    if mask_bits.dtype not in (torch.int32, torch.uint32):
        raise TypeError("mask_bits must be int32 or uint32")
    if mask_bits.dim() != 4 or not mask_bits.is_cuda or not mask_bits.is_contiguous():
        raise ValueError("mask_bits must be a contiguous 4-D CUDA tensor")
    B, H_q, nQ, nW = mask_bits.shape
    if nW != -(-nKVmax // 32):
        raise ValueError("last dim must be ceil(nKVmax / 32)")
    if group <= 0 or H_q % group:
        raise ValueError("group must divide H_q")
    H_kv = H_q // group
    dev = mask_bits.device
    if tables is None:
        tables = torch.empty((B, H_kv, nKVmax), dtype=torch.int32, device=dev)
    if counts is None:
        counts = torch.empty((B, H_kv), dtype=torch.int32, device=dev)
    _need(tables, "tables", torch.int32, 3)
    _need(counts, "counts", torch.int32, 2)
    if tuple(tables.shape) != (B, H_kv, nKVmax) or tuple(counts.shape) != (B, H_kv):
        raise ValueError(f"tables must be {(B, H_kv, nKVmax)}, counts {(B, H_kv)}")
    indptr = indices = None
    if csr:
        indptr = torch.empty(B * H_kv + 1, dtype=torch.int32, device=dev)
        indices = torch.empty(B * H_kv * nKVmax, dtype=torch.int32, device=dev)
    st = load_library().ca_build_block_tables_bits(_ptr(mask_bits), B, H_q, nQ, int(nKVmax),
                                                   int(group), _ptr(tables), _ptr(counts),
                                                   _ptr(indptr), _ptr(indices),
                                                   _stream_handle(stream, dev))
    _check("ca_build_block_tables_bits", st)
    return tables, counts, indptr, indices


def build_kv_pages(mask: torch.Tensor, group: int, stream: Optional[torch.cuda.Stream] = None):
    """Block-Union tables in the paged metadata form: ``(kv_indptr int32
    [B*H_kv+1], kv_indices int32 [B*H_kv*nKVmax])`` with global page ids
    ``(b*H_kv + g)*nKVmax + j``; the valid part of ``kv_indices`` is
    ``kv_indices[:kv_indptr[-1]]``. Also returns the dense ``tables, counts``."""
    if mask.dtype == torch.bool:
        mask = mask.view(torch.uint8)
    _need(mask, "mask", torch.uint8, 4)
    B, H_q, nQ, nK = mask.shape
    if group <= 0 or H_q % group:
        raise ValueError("group must divide H_q")
    H_kv = H_q // group
    dev = mask.device
    tables = torch.empty((B, H_kv, nK), dtype=torch.int32, device=dev)
    counts = torch.empty((B, H_kv), dtype=torch.int32, device=dev)
    indptr = torch.empty(B * H_kv + 1, dtype=torch.int32, device=dev)
    indices = torch.empty(B * H_kv * nK, dtype=torch.int32, device=dev)
    st = load_library().ca_build_kv_pages(_ptr(mask), B, H_q, nQ, nK, int(group), _ptr(tables),
                                          _ptr(counts), _ptr(indptr), _ptr(indices),
                                          _stream_handle(stream, dev))
    _check("ca_build_kv_pages", st)
    return indptr, indices, tables, counts


# ----------------------------------------------------------------- attention

def workspace_bytes(B: int, H_q: int, H_kv: int, C: int, blk: int) -> int:
    return int(load_library().ca_workspace_bytes(B, H_q, H_kv, C, blk))


def new_workspace(B: int, H_q: int, H_kv: int, C: int, blk: int,
                  device="cuda") -> torch.Tensor:
    """Zero-filled device workspace for the attention calls (reusable)."""
    n = workspace_bytes(B, H_q, H_kv, C, blk)
    if n == 0:
        raise ValueError("invalid sizes for the workspace")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def _attn_common(Q, K, V, O, LSE, workspace, blk):
    _need(Q, "Q", torch.bfloat16, 4)
    _need(K, "K", torch.bfloat16, 4)
    _need(V, "V", torch.bfloat16, 4)
    B, H_q, C, D = Q.shape
    Bk, H_kv, L_max, Dk = K.shape
    if Bk != B or Dk != D or tuple(V.shape) != tuple(K.shape):
        raise ValueError(f"shape mismatch: Q {tuple(Q.shape)}, K {tuple(K.shape)}, V {tuple(V.shape)}")
    dev = Q.device
    if O is None:
        O = torch.empty_like(Q)
    _need(O, "O", torch.bfloat16, 4)
    if tuple(O.shape) != tuple(Q.shape):
        raise ValueError("O must have Q's shape")
    if LSE is None:
        LSE = torch.empty((B, H_q, C), dtype=torch.float32, device=dev)
    _need(LSE, "LSE", torch.float32, 3)
    if workspace is None:
        workspace = new_workspace(B, H_q, H_kv, C, blk, device=dev)
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    return B, H_q, H_kv, C, L_max, D, O, LSE, workspace


def chunk_attention(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, tables: torch.Tensor,
                    counts: torch.Tensor, chunk_start: Sequence[int], scale: Optional[float] = None,
                    O: Optional[torch.Tensor] = None, LSE: Optional[torch.Tensor] = None,
                    workspace: Optional[torch.Tensor] = None,
                    stream: Optional[torch.cuda.Stream] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Causal chunk attention over the selected KV blocks, read in place.

    Q bf16 [B, H_q, C, D]; K, V bf16 [B, H_kv, L_max, D]; tables int32
    [B, H_kv, nKVmax] (blk = L_max / nKVmax); counts int32 [B, H_kv];
    chunk_start: B host ints. Returns (O bf16 [B, H_q, C, D], LSE fp32 [B, H_q, C])."""
    _need(tables, "tables", torch.int32, 3)
    _need(counts, "counts", torch.int32, 2)
    nK = tables.shape[-1]
    L_max = K.shape[2]
    if nK <= 0 or L_max % nK:
        raise ValueError("tables' last dim must divide L_max (it is L_max / blk)")
    blk = L_max // nK
    B, H_q, H_kv, C, L_max, D, O, LSE, workspace = _attn_common(Q, K, V, O, LSE, workspace, blk)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    cs = _chunk_start_host(chunk_start, B)
    lib = load_library()
    st = lib.ca_chunk_attention(_ptr(Q), _ptr(K), _ptr(V), _ptr(tables), _ptr(counts), cs, B, H_q,
                                H_kv, C, L_max, D, blk, float(scale), _ptr(O), _ptr(LSE),
                                _ptr(workspace), workspace.numel(), _stream_handle(stream, Q.device))
    _check("ca_chunk_attention", st)
    return O, LSE


def dense_chunk_attention(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor,
                          chunk_start: Sequence[int], blk: int, scale: Optional[float] = None,
                          O: Optional[torch.Tensor] = None, LSE: Optional[torch.Tensor] = None,
                          workspace: Optional[torch.Tensor] = None,
                          stream: Optional[torch.cuda.Stream] = None
                          ) -> Tuple[torch.Tensor, torch.Tensor]:
    """The dense paged path: every block of each sequence's visible length."""
    B, H_q, H_kv, C, L_max, D, O, LSE, workspace = _attn_common(Q, K, V, O, LSE, workspace, blk)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    cs = _chunk_start_host(chunk_start, B)
    lib = load_library()
    st = lib.ca_dense_chunk_attention(_ptr(Q), _ptr(K), _ptr(V), cs, B, H_q, H_kv, C, L_max, D,
                                      int(blk), float(scale), _ptr(O), _ptr(LSE), _ptr(workspace),
                                      workspace.numel(), _stream_handle(stream, Q.device))
    _check("ca_dense_chunk_attention", st)
    return O, LSE


def selftest_bounded_wait(workspace: torch.Tensor, limit_cycles: int = 20_000_000,
                          stream: Optional[torch.cuda.Stream] = None) -> None:
    """Runs the bounded-wait self-test kernel (a wait that nothing completes
    gives up after ``limit_cycles`` and records a timeout in ``workspace``)."""
    st = load_library().ca_selftest_bounded_wait(_ptr(workspace), int(limit_cycles),
                                                 _stream_handle(stream, workspace.device))
    _check("ca_selftest_bounded_wait", st)


def read_device_status(workspace: torch.Tensor, stream: Optional[torch.cuda.Stream] = None) -> int:
    """Synchronise and return the sticky device status (CA_OK / CA_ERR_TABLE /
    CA_ERR_TIMEOUT)."""
    return int(load_library().ca_read_device_status(_ptr(workspace),
                                                      _stream_handle(stream, workspace.device)))


def chunk_attention_noalloc(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor,
                            tables: torch.Tensor, counts: torch.Tensor,
                            chunk_start: Sequence[int], O: torch.Tensor, LSE: torch.Tensor,
                            scale: Optional[float] = None,
                            device_status: Optional[torch.Tensor] = None,
                            stream: Optional[torch.cuda.Stream] = None
                            ) -> Tuple[torch.Tensor, torch.Tensor]:
    """chunk_attention for callers that cannot allocate device memory: no
    workspace, and the caller passes the outputs O and LSE (this wrapper
    allocates nothing either). The library's fixed scratch array stands in for
    the workspace; calls that overlap on the GPU share it and race.
    ``device_status``: optional int32 CUDA tensor of one element that receives
    the call's device status word (0 = OK)."""
    _need(tables, "tables", torch.int32, 3)
    _need(counts, "counts", torch.int32, 2)
    _need(Q, "Q", torch.bfloat16, 4)
    _need(K, "K", torch.bfloat16, 4)
    _need(V, "V", torch.bfloat16, 4)
    _need(O, "O", torch.bfloat16, 4)
    _need(LSE, "LSE", torch.float32, 3)
    B, H_q, C, D = Q.shape
    _, H_kv, L_max, _ = K.shape
    nK = tables.shape[-1]
    if nK <= 0 or L_max % nK:
        raise ValueError("tables' last dim must divide L_max (it is L_max / blk)")
    if tuple(O.shape) != tuple(Q.shape) or tuple(LSE.shape) != (B, H_q, C):
        raise ValueError("O must have Q's shape and LSE [B, H_q, C]")
    if device_status is not None:
        if (device_status.dtype != torch.int32 or not device_status.is_cuda
                or device_status.numel() < 1):
            raise ValueError("device_status must be an int32 CUDA tensor of one element")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    cs = _chunk_start_host(chunk_start, B)
    # the C side uses the scratch array of the current device: make Q's
    # device current for the call, so scratch and stream belong together
    with torch.cuda.device(Q.device):
        st = load_library().ca_chunk_attention_noalloc(
            _ptr(Q), _ptr(K), _ptr(V), _ptr(tables), _ptr(counts), cs, B, H_q, H_kv, C, L_max,
            D, L_max // nK, float(scale), _ptr(O), _ptr(LSE), _ptr(device_status),
            _stream_handle(stream, Q.device))
    _check("ca_chunk_attention_noalloc", st)
    return O, LSE


# ----------------------------------------------------------------- ablation

def compact_kv_blocks(K: torch.Tensor, V: torch.Tensor, tables: torch.Tensor,
                      counts: torch.Tensor, Kc: Optional[torch.Tensor] = None,
                      Vc: Optional[torch.Tensor] = None,
                      stream: Optional[torch.cuda.Stream] = None
                      ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Explicit-compaction ablation: gathers the blocks each table selects into
    compact K / V buffers (block t of table (b, g) at rows [t*blk, (t+1)*blk))."""
    _need(K, "K", torch.bfloat16, 4)
    _need(V, "V", torch.bfloat16, 4)
    _need(tables, "tables", torch.int32, 3)
    _need(counts, "counts", torch.int32, 2)
    B, H_kv, L_max, D = K.shape
    nK = tables.shape[-1]
    if nK <= 0 or L_max % nK:
        raise ValueError("tables' last dim must divide L_max (it is L_max / blk)")
    if Kc is None:
        Kc = torch.zeros_like(K)
    if Vc is None:
        Vc = torch.zeros_like(V)
    _need(Kc, "Kc", torch.bfloat16, 4)
    _need(Vc, "Vc", torch.bfloat16, 4)
    st = load_library().ca_compact_kv_blocks(_ptr(K), _ptr(V), _ptr(tables), _ptr(counts), B,
                                             H_kv, L_max, D, L_max // nK, _ptr(Kc), _ptr(Vc),
                                             _stream_handle(stream, K.device))
    _check("ca_compact_kv_blocks", st)
    return Kc, Vc


def compacted_chunk_attention(Q: torch.Tensor, Kc: torch.Tensor, Vc: torch.Tensor,
                              tables: torch.Tensor, counts: torch.Tensor,
                              chunk_start: Sequence[int], scale: Optional[float] = None,
                              O: Optional[torch.Tensor] = None, LSE: Optional[torch.Tensor] = None,
                              workspace: Optional[torch.Tensor] = None,
                              stream: Optional[torch.cuda.Stream] = None
                              ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Explicit-compaction ablation: chunk_attention over compact_kv_blocks'
    buffers (same results as chunk_attention on the original cache)."""
    _need(tables, "tables", torch.int32, 3)
    _need(counts, "counts", torch.int32, 2)
    nK = tables.shape[-1]
    L_max = Kc.shape[2]
    if nK <= 0 or L_max % nK:
        raise ValueError("tables' last dim must divide L_max (it is L_max / blk)")
    blk = L_max // nK
    B, H_q, H_kv, C, L_max, D, O, LSE, workspace = _attn_common(Q, Kc, Vc, O, LSE, workspace, blk)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    cs = _chunk_start_host(chunk_start, B)
    st = load_library().ca_compacted_chunk_attention(
        _ptr(Q), _ptr(Kc), _ptr(Vc), _ptr(tables), _ptr(counts), cs, B, H_q, H_kv, C, L_max, D,
        blk, float(scale), _ptr(O), _ptr(LSE), _ptr(workspace), workspace.numel(),
        _stream_handle(stream, Q.device))
    _check("ca_compacted_chunk_attention", st)
    return O, LSE


# ------------------------------------------- per-tile block-sparse ablation

def tile_span(blk: int) -> int:
    """Q-blocks per span of the per-tile path's tables (256 chunk rows)."""
    n = int(load_library().ca_tile_span(int(blk)))
    if n == 0:
        raise ValueError(f"unsupported block size {blk}")
    return n


def build_tile_tables(mask: torch.Tensor, blk: int, tables: Optional[torch.Tensor] = None,
                      counts: Optional[torch.Tensor] = None,
                      stream: Optional[torch.cuda.Stream] = None):
    """Span tables of the per-tile block-sparse path from a uint8 / bool mask
    ``[B, H_q, nQ, nKVmax]``: per (b, h, span of ``tile_span(blk)`` Q-blocks)
    the ascending KV blocks any Q-block of the span selects, each entry
    ``j | bits << 24`` (bit u: Q-block ``span*s + u`` selects j), tail -1.
    Returns ``(tables int32 [B, H_q, nS, nKVmax], counts int32 [B, H_q, nS])``."""
    if mask.dtype == torch.bool:
        mask = mask.view(torch.uint8)
    _need(mask, "mask", torch.uint8, 4)
    B, H_q, nQ, nK = mask.shape
    span = tile_span(blk)
    nS = -(-nQ // span)
    dev = mask.device
    if tables is None:
        tables = torch.empty((B, H_q, nS, nK), dtype=torch.int32, device=dev)
    if counts is None:
        counts = torch.empty((B, H_q, nS), dtype=torch.int32, device=dev)
    _need(tables, "tables", torch.int32, 4)
    _need(counts, "counts", torch.int32, 3)
    if tuple(tables.shape) != (B, H_q, nS, nK) or tuple(counts.shape) != (B, H_q, nS):
        raise ValueError(f"tables must be {(B, H_q, nS, nK)}, counts {(B, H_q, nS)}")
    st = load_library().ca_build_tile_tables(_ptr(mask), B, H_q, nQ, nK, int(blk), _ptr(tables),
                                             _ptr(counts), _stream_handle(stream, dev))
    _check("ca_build_tile_tables", st)
    return tables, counts


def tile_chunk_attention(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, tables: torch.Tensor,
                         counts: torch.Tensor, chunk_start: Sequence[int],
                         scale: Optional[float] = None, O: Optional[torch.Tensor] = None,
                         LSE: Optional[torch.Tensor] = None,
                         workspace: Optional[torch.Tensor] = None,
                         stream: Optional[torch.cuda.Stream] = None
                         ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Per-tile block-sparse chunk attention over build_tile_tables' span
    tables: row r of head h attends to the keys k <= chunk_start[b] + r of the
    blocks its own Q-block selected (no union), read in place from the cache."""
    _need(tables, "tables", torch.int32, 4)
    _need(counts, "counts", torch.int32, 3)
    nK = tables.shape[-1]
    L_max = K.shape[2]
    if nK <= 0 or L_max % nK:
        raise ValueError("tables' last dim must divide L_max (it is L_max / blk)")
    blk = L_max // nK
    B, H_q, H_kv, C, L_max, D, O, LSE, workspace = _attn_common(Q, K, V, O, LSE, workspace, blk)
    nS = -(-C // 256)
    if tuple(tables.shape[:3]) != (B, H_q, nS) or tuple(counts.shape) != (B, H_q, nS):
        raise ValueError(f"tables must be {(B, H_q, nS, nK)}, counts {(B, H_q, nS)}")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    cs = _chunk_start_host(chunk_start, B)
    st = load_library().ca_tile_chunk_attention(
        _ptr(Q), _ptr(K), _ptr(V), _ptr(tables), _ptr(counts), cs, B, H_q, H_kv, C, L_max, D,
        blk, float(scale), _ptr(O), _ptr(LSE), _ptr(workspace), workspace.numel(),
        _stream_handle(stream, Q.device))
    _check("ca_tile_chunk_attention", st)
    return O, LSE


# -------------------------------------------- paged metadata, ragged chunks

def paged_chunk_attention(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor,
                          kv_indptr: torch.Tensor, kv_indices: torch.Tensor,
                          chunk_start: Sequence[int], blk: int,
                          chunk_len: Optional[Sequence[int]] = None,
                          scale: Optional[float] = None, O: Optional[torch.Tensor] = None,
                          LSE: Optional[torch.Tensor] = None,
                          workspace: Optional[torch.Tensor] = None,
                          stream: Optional[torch.cuda.Stream] = None
                          ) -> Tuple[torch.Tensor, torch.Tensor]:
    """chunk_attention over the ``kv_indptr`` / ``kv_indices`` (global page)
    form, with per-sequence chunk lengths ``chunk_len`` (rows past a
    sequence's length are left untouched in ``O`` / ``LSE``)."""
    _need(kv_indptr, "kv_indptr", torch.int32, 1)
    _need(kv_indices, "kv_indices", torch.int32, 1)
    B, H_q, H_kv, C, L_max, D, O, LSE, workspace = _attn_common(Q, K, V, O, LSE, workspace, blk)
    if kv_indptr.numel() != B * H_kv + 1:
        raise ValueError("kv_indptr must have B*H_kv + 1 entries")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    cs = _chunk_start_host(chunk_start, B)
    cl = None if chunk_len is None else _chunk_start_host(chunk_len, B)
    st = load_library().ca_paged_chunk_attention(
        _ptr(Q), _ptr(K), _ptr(V), _ptr(kv_indptr), _ptr(kv_indices), kv_indices.numel(), cs, cl,
        B, H_q, H_kv, C, L_max, D, int(blk), float(scale), _ptr(O), _ptr(LSE), _ptr(workspace),
        workspace.numel(), _stream_handle(stream, Q.device))
    _check("ca_paged_chunk_attention", st)
    return O, LSE


# ------------------------------------------------------------- FP8 (E4M3) cache

def chunk_attention_fp8(Q8: torch.Tensor, K8: torch.Tensor, V8: torch.Tensor,
                        descale: Sequence[float], chunk_start: Sequence[int], blk: int,
                        tables: Optional[torch.Tensor] = None,
                        counts: Optional[torch.Tensor] = None, scale: Optional[float] = None,
                        O: Optional[torch.Tensor] = None, LSE: Optional[torch.Tensor] = None,
                        workspace: Optional[torch.Tensor] = None,
                        stream: Optional[torch.cuda.Stream] = None
                        ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Chunk attention on E4M3 inputs (uint8 or float8_e4m3fn tensors with the
    bf16 layouts; the real inputs are ``descale[i]`` times the codes). Tables
    as in :func:`chunk_attention`, or none for the dense path. O is bf16."""
    def codes(t, name, ndim):
        if t.dtype == torch.float8_e4m3fn:
            t = t.view(torch.uint8)
        _need(t, name, torch.uint8, ndim)
        return t
    Q8, K8, V8 = codes(Q8, "Q8", 4), codes(K8, "K8", 4), codes(V8, "V8", 4)
    B, H_q, C, D = Q8.shape
    Bk, H_kv, L_max, Dk = K8.shape
    if Bk != B or Dk != D or tuple(V8.shape) != tuple(K8.shape):
        raise ValueError("shape mismatch")
    if (tables is None) != (counts is None):
        raise ValueError("give both tables and counts, or neither (dense path)")
    if tables is not None:
        _need(tables, "tables", torch.int32, 3)
        _need(counts, "counts", torch.int32, 2)
    dev = Q8.device
    if O is None:
        O = torch.empty((B, H_q, C, D), dtype=torch.bfloat16, device=dev)
    _need(O, "O", torch.bfloat16, 4)
    if LSE is None:
        LSE = torch.empty((B, H_q, C), dtype=torch.float32, device=dev)
    _need(LSE, "LSE", torch.float32, 3)
    if workspace is None:
        workspace = new_workspace(B, H_q, H_kv, C, blk, device=dev)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    qd, kd, vd = (float(x) for x in descale)
    cs = _chunk_start_host(chunk_start, B)
    st = load_library().ca_chunk_attention_fp8(
        _ptr(Q8), _ptr(K8), _ptr(V8), qd, kd, vd, _ptr(tables), _ptr(counts), cs, B, H_q, H_kv,
        C, L_max, D, int(blk), float(scale), _ptr(O), _ptr(LSE), _ptr(workspace),
        workspace.numel(), _stream_handle(stream, dev))
    _check("ca_chunk_attention_fp8", st)
    return O, LSE


# ----------------------------------------------------------------- merge

def merge_attention_states(parts: Sequence[Tuple[torch.Tensor, torch.Tensor]],
                           O: Optional[torch.Tensor] = None, LSE: Optional[torch.Tensor] = None,
                           want_lse: bool = True, stream: Optional[torch.cuda.Stream] = None
                           ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Merges attention results over disjoint key sets of the same query rows:
    ``parts`` = [(O_i bf16 [..., D], LSE_i fp32 [...]), ...] (2 to 8 parts, as
    ``chunk_attention`` returns them) -> attention over the union of the key
    sets, ``LSE = ln sum exp(LSE_i)``, ``O = sum exp(LSE_i - LSE) O_i``. ``O`` /
    ``LSE`` may be given (also one of the parts' own tensors, for in place);
    with ``want_lse=False`` and no ``LSE`` the merged LSE is not written."""
    parts = list(parts)
    if len(parts) < 2:
        raise ValueError("merge_attention_states needs at least two parts")
    O0, L0 = parts[0]
    shape = tuple(O0.shape)
    for i, (Oi, Li) in enumerate(parts):
        _need(Oi, f"O_{i}", torch.bfloat16, len(shape))
        _need(Li, f"LSE_{i}", torch.float32, len(shape) - 1)
        if tuple(Oi.shape) != shape or tuple(Li.shape) != shape[:-1]:
            raise ValueError(f"part {i}: shapes {tuple(Oi.shape)} / {tuple(Li.shape)} "
                             f"do not match {shape} / {shape[:-1]}")
    D = shape[-1]
    rows = O0.numel() // D if D else 0
    if O is None:
        O = torch.empty_like(O0)
    _need(O, "O", torch.bfloat16, len(shape))
    if tuple(O.shape) != shape:
        raise ValueError(f"O must have shape {shape}")
    if LSE is None and want_lse:
        LSE = torch.empty_like(L0)
    if LSE is not None:
        _need(LSE, "LSE", torch.float32, len(shape) - 1)
        if tuple(LSE.shape) != shape[:-1]:
            raise ValueError(f"LSE must have shape {shape[:-1]}")
    n = len(parts)
    o_arr = (ctypes.c_void_p * n)(*[Oi.data_ptr() for Oi, _ in parts])
    l_arr = (ctypes.c_void_p * n)(*[Li.data_ptr() for _, Li in parts])
    st = load_library().ca_merge_attention_states_n(o_arr, l_arr, n, rows, D, _ptr(O), _ptr(LSE),
                                                    _stream_handle(stream, O0.device))
    _check("ca_merge_attention_states_n", st)
    return O, LSE
