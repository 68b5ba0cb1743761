"""Seeded synthetic inputs for the chunked-prefill Block-Union attention path.

This module only draws random numbers and lays them out in the shapes the
path consumes. It holds none of the method's arithmetic: no union, no table,
no attention. Both the CPU oracle (``oracle/``) and the CUDA library
(``serving_block_union_b200``) are fed from here, so that the two sides see
bit-identical inputs.

Shapes follow the KV-head-major layout of the CompactAttention pages
("Execution stage: zero-copy paged attention", the ``[B, H_kv, L, D]`` cache):

* ``mask``  uint8 ``[B, H_q, nQ, nKVmax]``; nonzero = tile selected. KV block
  ``j`` is absolute from sequence position 0 (cached blocks, then the chunk).
* ``Q``     bf16 ``[B, H_q, C, D]`` (the chunk's queries).
* ``K, V``  bf16 ``[B, H_kv, L_max, D]`` (the accumulated cache; rows
  ``[cs_b, cs_b + C)`` hold the chunk's own keys/values).

The pages evaluate on RULER / LongBench V2 prompts with LLaMA-3.1-8B-Instruct
at 128K context ("Experimental results"); neither weights nor datasets are
available here, so these draws stand in for them: Q, V ~ N(0, 1); K = N(0, 1)
plus a per-(b, g, block) bias vector with entries N(0, 2), shared by the
block's keys, which makes per-block logit offsets peaky the way trained
attention is. Masks are sink + local window + vertical stripes (+ noise),
the structure pattern-search methods such as SeerAttention / FlashPrefill emit.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence, Tuple

import numpy as np
import torch

__all__ = [
    "Workload",
    "tiny",
    "llama8b_32k",
    "llama8b_128k",
    "batched",
    "llama8b_1m",
    "full_prefill_chunk",
    "qwen3_30b_128k",
    "by_name",
    "make_mask",
    "make_qkv",
    "make_q",
    "make_kv",
    "poison_beyond_kv_len",
    "pack_mask_bits",
    "quantize_e4m3",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    """One chunked-prefill step: B sequences, each with ``chunk_start[b]`` cached
    tokens, processing a chunk of ``C`` new tokens against a cache of ``L_max``
    allocated rows. ``blk`` is both the Q-block and the KV-block (page) size."""

    name: str
    B: int
    H_q: int
    H_kv: int
    D: int
    blk: int
    C: int
    L_max: int
    chunk_start: Tuple[int, ...]
    seed: int
    mask_kind: str                 # "bernoulli" | "stripes" | "batched"
    density: float = 0.0           # per-head target density ("stripes")
    noise: float = 0.0             # i.i.d. Bernoulli noise on causal tiles
    n_stripes: int = -1            # fixed stripe count (-1: derive from density)
    kv_seed: Optional[int] = None  # seed for Q/K/V if it differs from ``seed``
    stripe_base: str = "cached"    # stripe count from density x ("cached" | "visible") blocks
    kv_kind: str = "normal"        # "normal" | "pooled" (long caches; see make_kv)

    @property
    def group(self) -> int:
        return self.H_q // self.H_kv

    @property
    def nQ(self) -> int:
        return self.C // self.blk

    @property
    def nKVmax(self) -> int:
        return self.L_max // self.blk

    def kv_len(self, b: int) -> int:
        return self.chunk_start[b] + self.C

    def nC(self, b: int) -> int:
        return self.chunk_start[b] // self.blk

    def nKV(self, b: int) -> int:
        return self.nC(b) + self.nQ

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, stream])))


# --------------------------------------------------------------------------
# Configurations. Sizes are the LLaMA-3.1-8B attention shape (32 query heads,
# 8 KV heads, head dim 128) the pages evaluate on, with 128-token blocks.
# --------------------------------------------------------------------------

def tiny() -> Workload:
    """B=1, 4/1 heads, D=64, block 64, 768 cached + 256-token chunk
    (4 Q-blocks x 16 KV-blocks); Bernoulli(0.3) mask on every tile, future
    tiles included, with block 0 and each Q-block's diagonal block forced on."""
    return Workload("tiny", B=1, H_q=4, H_kv=1, D=64, blk=64, C=256, L_max=1024,
                    chunk_start=(768,), seed=0, mask_kind="bernoulli", density=0.3)


def llama8b_32k() -> Workload:
    """32K cached + 2048-token chunk; sink + local window of 4 + 6 stripes +
    Bernoulli(0.05) noise per head (about 10% density)."""
    return Workload("llama8b_32k", B=1, H_q=32, H_kv=8, D=128, blk=128, C=2048,
                    L_max=32768 + 2048, chunk_start=(32768,), seed=1,
                    mask_kind="stripes", n_stripes=6, noise=0.05)


def llama8b_128k(density: float = 0.10, noise: bool = False) -> Workload:
    """128K cached (1024 KV blocks) + 2048-token chunk. Per head: sink + local
    window of 4 + round(density * 1024) - 5 stripes drawn independently per
    head, so that the intra-group union grows. ``noise=True`` gives the
    32K config's mask style (6 stripes + Bernoulli(0.05)) at 128K."""
    pct = int(round(density * 100))
    if noise:
        return Workload("llama8b_128k_noise", B=1, H_q=32, H_kv=8, D=128, blk=128,
                        C=2048, L_max=131072 + 2048, chunk_start=(131072,), seed=299,
                        mask_kind="stripes", n_stripes=6, noise=0.05)
    return Workload(f"llama8b_128k_d{pct}", B=1, H_q=32, H_kv=8, D=128, blk=128,
                    C=2048, L_max=131072 + 2048, chunk_start=(131072,),
                    seed=200 + pct, mask_kind="stripes", density=density)


def qwen3_30b_128k(density: float = 0.10) -> Workload:
    """The 128K sweep's mask and sizes with a GQA group of 8: 32 query heads
    over 4 KV heads, head dim 128 (the attention shape of the pages' second
    model, Qwen3-30B-A3B; the pages do not print it). Eight heads' independent
    stripes make the group union larger than at G = 4."""
    pct = int(round(density * 100))
    return Workload(f"qwen3_30b_128k_d{pct}", B=1, H_q=32, H_kv=4, D=128, blk=128,
                    C=2048, L_max=131072 + 2048, chunk_start=(131072,),
                    seed=300 + pct, mask_kind="stripes", density=density)


def llama8b_1m(density: float = 0.02) -> Workload:
    """1M-token context: 1,046,528 cached tokens + a 2048-token chunk (8192
    KV blocks), the 128K sweep's per-head mask recipe (sink + local window of
    4 + round(density * 8176) - 5 independent stripes per head). The cache is
    drawn with the pooled recipe of ``make_kv`` (8 GB of independent normals
    would take minutes on the host)."""
    pct = int(round(density * 100))
    L = 1 << 20
    return Workload(f"llama8b_1m_d{pct}", B=1, H_q=32, H_kv=8, D=128, blk=128, C=2048,
                    L_max=L, chunk_start=(L - 2048,), seed=500 + pct, mask_kind="stripes",
                    density=density, kv_kind="pooled")


def batched() -> Workload:
    """B=4 sequences with 16K/32K/64K/96K cached tokens and a 4096-token chunk;
    per-head density U(2%, 15%); heads of a group share only half of their
    stripes (a per-(b, g) shared draw plus a head-private draw)."""
    return Workload("batched", B=4, H_q=32, H_kv=8, D=128, blk=128, C=4096,
                    L_max=102400, chunk_start=(16384, 32768, 65536, 98304), seed=3,
                    mask_kind="batched")


def full_prefill_chunk(k: int, n_chunks: int = 64) -> Workload:
    """Chunk ``k`` of a 128K-token prompt processed as ``n_chunks`` chunks of
    2048 tokens; the cache holds the whole prompt (drawn once, seed 4), the
    mask is fresh per chunk (5% density, seed 4000 + k)."""
    C = 2048
    return Workload(f"full_prefill_c{k}", B=1, H_q=32, H_kv=8, D=128, blk=128, C=C,
                    L_max=C * n_chunks, chunk_start=(C * k,), seed=4000 + k,
                    mask_kind="stripes", density=0.05, kv_seed=4, stripe_base="visible")


def by_name(name: str) -> Workload:
    if name == "tiny":
        return tiny()
    if name == "llama8b_32k":
        return llama8b_32k()
    if name.startswith("llama8b_128k_d"):
        return llama8b_128k(int(name[len("llama8b_128k_d"):]) / 100.0)
    if name == "llama8b_128k_noise":
        return llama8b_128k(noise=True)
    if name == "batched":
        return batched()
    if name.startswith("llama8b_1m_d"):
        return llama8b_1m(int(name[len("llama8b_1m_d"):]) / 100.0)
    if name.startswith("qwen3_30b_128k_d"):
        return qwen3_30b_128k(int(name[len("qwen3_30b_128k_d"):]) / 100.0)
    if name.startswith("full_prefill_c"):
        return full_prefill_chunk(int(name[len("full_prefill_c"):]))
    raise KeyError(name)


# --------------------------------------------------------------------------
# Masks
# --------------------------------------------------------------------------

def _stripe_count(density: float, nKV: int) -> int:
    return max(0, int(round(density * nKV)) - 5)


def make_mask(wl: Workload) -> np.ndarray:
    """uint8 [B, H_q, nQ, nKVmax] block mask for ``wl`` (seeded)."""
    B, H, nQ, nK = wl.B, wl.H_q, wl.nQ, wl.nKVmax
    m = np.zeros((B, H, nQ, nK), dtype=np.uint8)
    rng = _rng(wl.seed, 0)
    if wl.mask_kind == "bernoulli":
        for b in range(B):
            nC = wl.nC(b)
            for h in range(H):
                m[b, h] = (rng.random((nQ, nK)) < wl.density).astype(np.uint8)
                m[b, h, :, 0] = 1
                for i in range(nQ):
                    m[b, h, i, nC + i] = 1
        return m

    if wl.mask_kind == "stripes":
        for b in range(B):
            nC, nKV = wl.nC(b), wl.nKV(b)
            if wl.n_stripes >= 0:
                s = wl.n_stripes
            else:
                # full prefill sizes the stripe count by the whole visible
                # length; the 128K sweep by the cached part ("1024 KV blocks")
                base = nKV if wl.stripe_base == "visible" else nC
                s = _stripe_count(wl.density, base)
            for h in range(H):
                if nC > 1 and s > 0:
                    stripes = rng.choice(np.arange(1, nC), size=min(s, nC - 1), replace=False)
                else:
                    stripes = np.zeros(0, dtype=np.int64)
                for i in range(nQ):
                    diag = nC + i
                    m[b, h, i, 0] = 1
                    m[b, h, i, max(0, diag - 3): diag + 1] = 1
                    if stripes.size:
                        m[b, h, i, stripes] = 1
                if wl.noise > 0:
                    noise = rng.random((nQ, nK)) < wl.noise
                    causal = np.arange(nK)[None, :] <= (nC + np.arange(nQ))[:, None]
                    m[b, h] |= (noise & causal).astype(np.uint8)
        return m

    if wl.mask_kind == "batched":
        G = wl.group
        for b in range(B):
            nC = wl.nC(b)
            for g in range(wl.H_kv):
                shared = rng.permutation(np.arange(1, nC)) if nC > 1 else np.zeros(0, np.int64)
                for hl in range(G):
                    h = g * G + hl
                    d_h = rng.uniform(0.02, 0.15)
                    s = _stripe_count(d_h, nC)
                    s_shared = (s + 1) // 2
                    s_priv = s - s_shared
                    priv = (rng.choice(np.arange(1, nC), size=min(s_priv, nC - 1), replace=False)
                            if nC > 1 and s_priv > 0 else np.zeros(0, np.int64))
                    stripes = np.concatenate([shared[:s_shared], priv]).astype(np.int64)
                    for i in range(nQ):
                        diag = nC + i
                        m[b, h, i, 0] = 1
                        m[b, h, i, max(0, diag - 3): diag + 1] = 1
                        if stripes.size:
                            m[b, h, i, stripes] = 1
        return m

    raise ValueError(wl.mask_kind)


# --------------------------------------------------------------------------
# Q / K / V
# --------------------------------------------------------------------------

def _normal_bf16(rng: np.random.Generator, shape: Sequence[int]) -> torch.Tensor:
    x = rng.standard_normal(size=tuple(shape), dtype=np.float32)
    return torch.from_numpy(x).to(torch.bfloat16)


def make_q(wl: Workload) -> torch.Tensor:
    """bf16 [B, H_q, C, D], N(0, 1)."""
    return _normal_bf16(_rng(wl.seed, 1), (wl.B, wl.H_q, wl.C, wl.D))


def _make_kv_pooled(wl: Workload, seed: int) -> Tuple[torch.Tensor, torch.Tensor]:
    """Long caches: every (b, g, block) takes one of 64 N(0, 1) blocks of a
    pool (a uniform index per block, separately for K and V) plus its own
    bias vector, N(0, 2) for K and N(0, 1) for V, shared by the block's rows;
    a read of the wrong block still sees different values."""
    B, H, nK, blk, D = wl.B, wl.H_kv, wl.nKVmax, wl.blk, wl.D
    n_pool = 64
    out = []
    for stream, bias_sd in ((2, math.sqrt(2.0)), (4, 1.0)):
        rng = _rng(seed, stream)
        pool = torch.from_numpy(rng.standard_normal(size=(n_pool, blk, D), dtype=np.float32))
        idx = torch.from_numpy(rng.integers(0, n_pool, size=(B, H, nK)))
        bias = torch.from_numpy(
            rng.standard_normal(size=(B, H, nK, 1, D), dtype=np.float32) * np.float32(bias_sd))
        X = torch.empty((B, H, wl.L_max, D), dtype=torch.bfloat16)
        for b in range(B):
            for g in range(H):
                X[b, g] = (pool[idx[b, g]] + bias[b, g]).reshape(nK * blk, D).to(torch.bfloat16)
        out.append(X)
    return out[0], out[1]


def make_kv(wl: Workload) -> Tuple[torch.Tensor, torch.Tensor]:
    """bf16 K, V [B, H_kv, L_max, D]. K = N(0,1) + per-(b, g, block) bias
    vector with entries N(0, 2); V = N(0, 1). (Long caches: the pooled recipe
    of ``_make_kv_pooled``.)"""
    seed = wl.seed if wl.kv_seed is None else wl.kv_seed
    if wl.kv_kind == "pooled":
        return _make_kv_pooled(wl, seed)
    shape = (wl.B, wl.H_kv, wl.L_max, wl.D)
    rk = _rng(seed, 2)
    k = rk.standard_normal(size=shape, dtype=np.float32)
    bias = (_rng(seed, 3).standard_normal(
        size=(wl.B, wl.H_kv, wl.nKVmax, 1, wl.D), dtype=np.float32) * np.float32(math.sqrt(2.0)))
    k = (k.reshape(wl.B, wl.H_kv, wl.nKVmax, wl.blk, wl.D) + bias).reshape(shape)
    K = torch.from_numpy(k).to(torch.bfloat16)
    del k
    V = _normal_bf16(_rng(seed, 4), shape)
    return K, V


def make_qkv(wl: Workload) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    Q = make_q(wl)
    K, V = make_kv(wl)
    return Q, K, V


def poison_beyond_kv_len(wl: Workload, K: torch.Tensor, V: torch.Tensor) -> None:
    """Fill cache rows at positions >= kv_len(b) with NaN, in place: any read of
    memory past a sequence's end then shows up in the output."""
    for b in range(wl.B):
        n = wl.kv_len(b)
        if n < wl.L_max:
            K[b, :, n:, :] = float("nan")
            V[b, :, n:, :] = float("nan")


def chunk_starts(wl: Workload) -> List[int]:
    return list(wl.chunk_start)


def pack_mask_bits(mask: np.ndarray) -> np.ndarray:
    """Bit-packed form of a block mask (an input encoding, no method
    arithmetic): uint32 ``[B, H_q, nQ, ceil(nKVmax / 32)]``, bit k (value
    ``1 << k``) of word w set iff ``mask[..., 32 * w + k] != 0``; bits past
    nKVmax are zero."""
    B, H, nQ, nK = mask.shape
    nW = -(-nK // 32)
    padded = np.zeros((B, H, nQ, nW * 32), dtype=bool)
    padded[..., :nK] = mask != 0
    bytes_ = np.packbits(padded.reshape(B, H, nQ, nW, 4, 8), axis=-1, bitorder="little")
    return bytes_.reshape(B, H, nQ, nW, 4).copy().view("<u4").reshape(B, H, nQ, nW)


def quantize_e4m3(x: torch.Tensor) -> Tuple[torch.Tensor, float]:
    """FP8 E4M3 form of an input tensor for the FP8 path (an input encoding,
    no method arithmetic): a per-tensor descale factor amax / 448 and the
    codes of x / descale rounded to nearest by torch's float8_e4m3fn cast.
    Returns (uint8 codes, descale)."""
    xf = x.float()
    amax = float(xf.abs().max())
    descale = amax / 448.0 if amax > 0 else 1.0
    codes = (xf / descale).clamp(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.contiguous(), descale
