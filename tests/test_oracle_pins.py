"""Pins for the CPU oracle: checks against what the CompactAttention pages and
the mathematics fix, never against the oracle itself.

Tables ("Methodology", selection stage): a hand-worked example, brute-force
set unions, coverage, minimality, permutation invariance, monotonicity,
idempotence, the G=1 / nQ=1 reductions and the CSR (kv_indptr / kv_indices)
form. Attention ("Methodology", execution stage): torch's fp64
scaled_dot_product_attention with a lower-right causal mask (all-ones mask
and dense path), per-tile masked softmax on union-closed masks, closed forms
(K = 0, V = const), a hand-worked example, the LSE merge identity and NaN
poison outside the visible keys.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- helpers

def _rand_mask(rng, B, H_q, nQ, nK, p):
    return (rng.random((B, H_q, nQ, nK)) < p).astype(np.uint8)


def _brute_tables(mask, G):
    """Python sets: for each (b, g) the set of j with some M[b, h, i, j] != 0."""
    B, H_q, nQ, nK = mask.shape
    H_kv = H_q // G
    T = np.full((B, H_kv, nK), -1, np.int32)
    cnt = np.zeros((B, H_kv), np.int32)
    for b in range(B):
        for g in range(H_kv):
            sel = set()
            for hl in range(G):
                for i in range(nQ):
                    for j in range(nK):
                        if mask[b, g * G + hl, i, j]:
                            sel.add(j)
            s = sorted(sel)
            T[b, g, :len(s)] = s
            cnt[b, g] = len(s)
    return T, cnt


def _bf16(x):
    return torch.as_tensor(x, dtype=torch.float32).to(torch.bfloat16)


def _rand_qkv(seed, B, H_q, H_kv, C, L, D):
    g = torch.Generator().manual_seed(seed)
    Q = torch.randn(B, H_q, C, D, generator=g).to(torch.bfloat16)
    K = torch.randn(B, H_kv, L, D, generator=g).to(torch.bfloat16)
    V = torch.randn(B, H_kv, L, D, generator=g).to(torch.bfloat16)
    return Q, K, V


def _sdpa_masked(Q, K, V, allowed, scale):
    """torch fp64 SDPA with GQA expansion and an explicit boolean mask
    allowed[b, h, r, k] (True = attend). Rows with no allowed key return
    O = 0, LSE = -inf."""
    B, H_q, C, D = Q.shape
    H_kv = K.shape[1]
    G = H_q // H_kv
    q = Q.double()
    k = K.double().repeat_interleave(G, dim=1)
    v = V.double().repeat_interleave(G, dim=1)
    empty = ~allowed.any(dim=-1)
    safe = allowed.clone()
    safe[..., 0] |= empty  # keep softmax finite; overwritten below
    O = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=safe, scale=scale)
    # LSE in numpy: torch's CPU logsumexp was seen to return a value off by
    # ~2e-10 (relative) on rare first calls in a process.
    logits = np.einsum("bhrd,bhkd->bhrk", q.numpy(), k.numpy()) * scale
    logits = np.where(safe.numpy(), logits, -np.inf)
    mx = logits.max(axis=-1, keepdims=True)
    LSE = (mx + np.log(np.exp(logits - mx).sum(axis=-1, keepdims=True)))[..., 0]
    O = O.numpy()
    e = empty.numpy()
    O[e] = 0.0
    LSE[e] = -np.inf
    return O, LSE


def _causal_allowed(B, H_q, C, L, chunk_start):
    r = torch.arange(C)[:, None]
    k = torch.arange(L)[None, :]
    out = torch.zeros(B, H_q, C, L, dtype=torch.bool)
    for b in range(B):
        out[b] = (k <= chunk_start[b] + r)[None]
    return out


# ---------------------------------------------------------------- tables

def _read_union_golden():
    path = os.path.join(GOLDEN, "union_worked_example.txt")
    mask = np.zeros((2, 4, 2, 6), np.uint8)
    tables = np.zeros((2, 2, 6), np.int32)
    out = {}
    for line in open(path):
        line = line.split("#")[0].strip()
        if not line:
            continue
        key, vals = line.split(":")
        vals = [int(x) for x in vals.split()]
        key = key.split()
        if key[0] == "mask":
            b, h, i = map(int, key[1:])
            mask[b, h, i] = vals
        elif key[0] == "table":
            b, g = map(int, key[1:])
            tables[b, g] = vals
        else:
            out[key[0]] = np.array(vals, np.int32)
    return mask, tables, out


def test_union_worked_example():
    mask, T_exp, rest = _read_union_golden()
    T, cnt, indptr, indices = oracle.block_tables(mask, group=2)
    np.testing.assert_array_equal(T, T_exp)
    np.testing.assert_array_equal(cnt.reshape(-1), rest["counts"])
    np.testing.assert_array_equal(indptr, rest["indptr"])
    np.testing.assert_array_equal(indices, rest["indices"])


@pytest.mark.parametrize("shape", [(1, 4, 4, 16, 4), (2, 8, 3, 37, 2), (3, 6, 5, 50, 3),
                                   (1, 8, 1, 9, 8), (2, 4, 2, 7, 1)])
@pytest.mark.parametrize("p", [0.0, 0.03, 0.2, 1.0])
def test_tables_brute_force(shape, p):
    B, H_q, nQ, nK, G = shape
    rng = np.random.default_rng(hash((shape, p)) % 2**32)
    mask = _rand_mask(rng, B, H_q, nQ, nK, p)
    mask[mask == 1] = rng.integers(1, 256, size=int(mask.sum()), dtype=np.uint8)  # any nonzero selects
    T, cnt, indptr, indices = oracle.block_tables(mask, G)
    T_b, cnt_b = _brute_tables(mask, G)
    np.testing.assert_array_equal(T, T_b)
    np.testing.assert_array_equal(cnt, cnt_b)
    np.testing.assert_array_equal(indptr, np.concatenate([[0], np.cumsum(cnt_b.reshape(-1))]))
    np.testing.assert_array_equal(indices, np.concatenate(
        [T_b.reshape(-1, nK)[i, :c] for i, c in enumerate(cnt_b.reshape(-1))] + [np.zeros(0, np.int32)]))


def test_tables_coverage_minimality_order():
    rng = np.random.default_rng(7)
    B, H_q, nQ, nK, G = 2, 32, 16, 272, 4
    mask = _rand_mask(rng, B, H_q, nQ, nK, 0.004)
    T, cnt, _, _ = oracle.block_tables(mask, G)
    for b in range(B):
        for g in range(H_q // G):
            grp = mask[b, g * G:(g + 1) * G]           # [G, nQ, nK]
            chosen = set(T[b, g, :cnt[b, g]].tolist())
            # coverage: every selected tile's block is in the table
            for hl, i, j in zip(*np.nonzero(grp)):
                assert j in chosen
            # minimality: every table entry was selected somewhere in the group
            for j in chosen:
                assert grp[:, :, j].any()
            row = T[b, g, :cnt[b, g]]
            assert np.all(np.diff(row) > 0)
            assert np.all(T[b, g, cnt[b, g]:] == -1)


def test_tables_invariances():
    rng = np.random.default_rng(11)
    B, H_q, nQ, nK, G = 2, 8, 6, 40, 4
    mask = _rand_mask(rng, B, H_q, nQ, nK, 0.05)
    T, cnt, _, _ = oracle.block_tables(mask, G)
    # permuting heads inside each group and permuting Q-blocks leaves tables unchanged
    perm_h = np.concatenate([g * G + rng.permutation(G) for g in range(H_q // G)])
    T2, cnt2, _, _ = oracle.block_tables(mask[:, perm_h][:, :, rng.permutation(nQ)], G)
    np.testing.assert_array_equal(T, T2)
    np.testing.assert_array_equal(cnt, cnt2)
    # monotone: setting one more tile can only add that tile's block
    m3 = mask.copy()
    m3[1, 5, 2, 17] = 1
    T3, cnt3, _, _ = oracle.block_tables(m3, G)
    s_old = set(T[1, 1, :cnt[1, 1]].tolist())
    s_new = set(T3[1, 1, :cnt3[1, 1]].tolist())
    assert s_old <= s_new and s_new - s_old <= {17}
    # idempotent on the union-closed mask of its own output
    closed = np.zeros_like(mask)
    for b in range(B):
        for g in range(H_q // G):
            closed[b, g * G:(g + 1) * G, :, T[b, g, :cnt[b, g]]] = 1
    T4, cnt4, _, _ = oracle.block_tables(closed, G)
    np.testing.assert_array_equal(T, T4)
    np.testing.assert_array_equal(cnt, cnt4)


def test_tables_reductions():
    rng = np.random.default_rng(3)
    # G = 1 and nQ = 1: the table is the single mask row's support
    mask = _rand_mask(rng, 2, 3, 1, 33, 0.3)
    T, cnt, _, _ = oracle.block_tables(mask, 1)
    for b in range(2):
        for h in range(3):
            nz = np.nonzero(mask[b, h, 0])[0]
            assert cnt[b, h] == nz.size
            np.testing.assert_array_equal(T[b, h, :nz.size], nz)
    # all-zero mask: count 0, all padding
    T, cnt, indptr, indices = oracle.block_tables(np.zeros((2, 4, 3, 10), np.uint8), 2)
    assert (cnt == 0).all() and (T == -1).all() and (indptr == 0).all() and indices.size == 0
    # all-ones mask: every block
    T, cnt, _, _ = oracle.block_tables(np.ones((1, 4, 2, 10), np.uint8), 4)
    np.testing.assert_array_equal(T[0, 0], np.arange(10))


def test_tables_reject_bad_group():
    with pytest.raises(ValueError):
        oracle.block_tables(np.zeros((1, 6, 2, 8), np.uint8), 4)


# ---------------------------------------------------------------- attention

def _read_attn_golden():
    vals = {}
    for line in open(os.path.join(GOLDEN, "attention_worked_example.txt")):
        line = line.split("#")[0].strip()
        if not line:
            continue
        k, v = line.split(":")
        toks = []
        for t in v.split():
            toks.append({"ln3": math.log(3.0), "ln4": math.log(4.0)}.get(t, None)
                        if t.startswith("ln") else float(t))
        vals[k.strip()] = toks
    return vals


def test_attention_worked_example():
    g = _read_attn_golden()
    Q = _bf16(np.array(g["q"]).reshape(1, 1, 2, 1))
    K = _bf16(np.array(g["k"]).reshape(1, 1, 2, 1))
    V = _bf16(np.array(g["v"]).reshape(1, 1, 2, 1))
    T = np.array([[[int(g["table"][0])]]], np.int32)
    c = np.array([[int(g["count"][0])]], np.int32)
    O, LSE = oracle.attention(Q, K, V, [0], blk=2, tables=T, counts=c, scale=g["scale"][0])
    np.testing.assert_allclose(O.reshape(-1), g["O"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(LSE.reshape(-1), g["LSE"], rtol=0, atol=1e-12)


@pytest.mark.parametrize("cfg", [
    # B, H_q, H_kv, D, blk, C, L_max, chunk_start
    (1, 4, 1, 16, 8, 24, 64, (16,)),
    (2, 6, 2, 8, 4, 12, 40, (0, 20)),
    (1, 8, 8, 4, 16, 32, 64, (32,)),
    (2, 4, 2, 32, 8, 16, 48, (32, 8)),
])
def test_all_ones_mask_equals_dense_causal_sdpa(cfg):
    B, H_q, H_kv, D, blk, C, L, cs = cfg
    Q, K, V = _rand_qkv(sum(cfg[:7]), B, H_q, H_kv, C, L, D)
    mask = np.ones((B, H_q, C // blk, L // blk), np.uint8)
    T, cnt, _, _ = oracle.block_tables(mask, H_q // H_kv)
    scale = 0.7 / math.sqrt(D)
    O, LSE = oracle.attention(Q, K, V, cs, blk, T, cnt, scale=scale)
    Od, LSEd = oracle.attention(Q, K, V, cs, blk, None, None, scale=scale)
    Oref, LSEref = _sdpa_masked(Q, K, V, _causal_allowed(B, H_q, C, L, cs), scale)
    np.testing.assert_allclose(O, Oref, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(LSE, LSEref, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(Od, Oref, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(LSEd, LSEref, rtol=1e-10, atol=1e-10)


@pytest.mark.parametrize("cfg", [
    # B, H_q, H_kv, D, blk, C, L_max, chunk_start: starts that are not block
    # multiples and chunk lengths that are not either
    (2, 4, 1, 16, 8, 20, 64, (5, 37)),
    (1, 6, 2, 8, 8, 13, 48, (27,)),
    (3, 2, 2, 4, 4, 7, 24, (0, 1, 15)),
])
def test_unaligned_chunk_start_equals_causal_sdpa(cfg):
    """Chunk starts off the block grid: the dense path covers the blocks up to
    ceil((chunk_start + C) / blk) and the table path the selected blocks, both
    with key k visible to row r iff k <= chunk_start + r (the bottom-right
    causal reading). Pinned against torch's fp64 SDPA with an explicit
    token-level mask built from the mask's blocks, not from the tables."""
    B, H_q, H_kv, D, blk, C, L, cs = cfg
    G = H_q // H_kv
    nQ, nK = -(-C // blk), L // blk
    Q, K, V = _rand_qkv(sum(cfg[:7]), B, H_q, H_kv, C, L, D)
    scale = 1.0 / math.sqrt(D)
    # dense: every key up to the row's own position
    Od, LSEd = oracle.attention(Q, K, V, cs, blk, None, None, scale=scale)
    Oref, LSEref = _sdpa_masked(Q, K, V, _causal_allowed(B, H_q, C, L, cs), scale)
    np.testing.assert_allclose(Od, Oref, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(LSEd, LSEref, rtol=1e-10, atol=1e-10)
    # tables from a random mask; the reference key set is the union of the
    # group's mask rows, expanded to tokens, intersected with causality
    rng = np.random.default_rng(sum(cfg[:7]))
    mask = _rand_mask(rng, B, H_q, nQ, nK, 0.4)
    mask[..., 0] = 1
    T, cnt, _, _ = oracle.block_tables(mask, G)
    O, LSE = oracle.attention(Q, K, V, cs, blk, T, cnt, scale=scale)
    sel = torch.from_numpy(mask.reshape(B, H_kv, G * nQ, nK).any(axis=2))  # [B, H_kv, nK]
    tok = sel.repeat_interleave(blk, dim=2)[:, :, :L]                    # [B, H_kv, L]
    allowed = _causal_allowed(B, H_q, C, L, cs) & tok.repeat_interleave(G, dim=1)[:, :, None, :]
    Oref, LSEref = _sdpa_masked(Q, K, V, allowed, scale)
    np.testing.assert_allclose(O, Oref, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(LSE, LSEref, rtol=1e-10, atol=1e-10)
    # with a dropped term (a key past the row's position), the pin fails
    bad = _causal_allowed(B, H_q, C, L, [s + 1 for s in cs]) & \
        tok.repeat_interleave(G, dim=1)[:, :, None, :]
    Obad, _ = _sdpa_masked(Q, K, V, bad, scale)
    assert np.abs(Obad - O).max() > 1e-3


def test_dense_equals_sdpa_on_tiny_workload():
    wl = workloads.tiny()
    Q, K, V = workloads.make_qkv(wl)
    O, LSE = oracle.attention(Q, K, V, wl.chunk_start, wl.blk, scale=wl.scale)
    Oref, LSEref = _sdpa_masked(Q, K, V, _causal_allowed(wl.B, wl.H_q, wl.C, wl.L_max, wl.chunk_start),
                                wl.scale)
    np.testing.assert_allclose(O, Oref, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(LSE, LSEref, rtol=1e-10, atol=1e-10)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_union_closed_mask_equals_per_tile_masked_attention(seed):
    """When every head of a group already selects the group's union on every
    causal tile, executing the table is exactly per-tile masked attention."""
    rng = np.random.default_rng(seed)
    B, H_q, H_kv, D, blk, C, L = 2, 4, 2, 16, 8, 32, 96
    cs = (40, 16)
    G = H_q // H_kv
    nQ, nK = C // blk, L // blk
    U = (rng.random((B, H_kv, nK)) < 0.4)
    mask = np.zeros((B, H_q, nQ, nK), np.uint8)
    for b in range(B):
        for h in range(H_q):
            for i in range(nQ):
                for j in range(nK):
                    if U[b, h // G, j] and j <= cs[b] // blk + i:
                        mask[b, h, i, j] = 1
    T, cnt, _, _ = oracle.block_tables(mask, G)
    Q, K, V = _rand_qkv(100 + seed, B, H_q, H_kv, C, L, D)
    O, LSE = oracle.attention(Q, K, V, cs, blk, T, cnt)
    allowed = torch.zeros(B, H_q, C, L, dtype=torch.bool)
    for b in range(B):
        for h in range(H_q):
            for r in range(C):
                for k in range(L):
                    allowed[b, h, r, k] = bool(mask[b, h, r // blk, k // blk]) and k <= cs[b] + r
    Oref, LSEref = _sdpa_masked(Q, K, V, allowed, 1.0 / math.sqrt(D))
    np.testing.assert_allclose(O, Oref, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(LSE, LSEref, rtol=1e-10, atol=1e-10)


def test_closed_forms():
    B, H_q, H_kv, D, blk, C, L = 1, 4, 2, 8, 4, 8, 32
    cs = (12,)
    rng = np.random.default_rng(5)
    mask = _rand_mask(rng, B, H_q, C // blk, L // blk, 0.5)
    mask[..., 0] = 1
    T, cnt, _, _ = oracle.block_tables(mask, H_q // H_kv)
    Q, K, V = _rand_qkv(9, B, H_q, H_kv, C, L, D)
    # K = 0: uniform weights -> O = mean of visible V rows, LSE = ln(#visible)
    Kz = torch.zeros_like(K)
    O, LSE = oracle.attention(Q, Kz, V, cs, blk, T, cnt)
    for h in range(H_q):
        g = h // (H_q // H_kv)
        blocks = T[0, g, :cnt[0, g]]
        for r in range(C):
            keys = [j * blk + c for j in blocks for c in range(blk) if j * blk + c <= cs[0] + r]
            np.testing.assert_allclose(O[0, h, r], V[0, g, keys].double().mean(0).numpy(),
                                       rtol=1e-12, atol=1e-12)
            assert abs(LSE[0, h, r] - math.log(len(keys))) < 1e-12
    # V = const per dim: O = that constant, whatever the weights
    cvec = _bf16(rng.standard_normal(D))
    Vc = cvec.expand(B, H_kv, L, D).contiguous()
    O, _ = oracle.attention(Q, K, Vc, cs, blk, T, cnt)
    np.testing.assert_allclose(O, np.broadcast_to(cvec.double().numpy(), O.shape), rtol=1e-12, atol=1e-12)


def test_lse_merge_identity():
    """Attention over disjoint block sets, merged with softmax(LSE) weights,
    equals attention over their union; pins the natural-log LSE convention."""
    B, H_q, H_kv, D, blk, C, L = 1, 2, 1, 16, 8, 16, 64
    cs = (48,)
    Q, K, V = _rand_qkv(21, B, H_q, H_kv, C, L, D)
    nK = L // blk
    full = np.array([[[0, 1, 3, 4, 6, 7] + [-1] * (nK - 6)]], np.int32)
    a = np.array([[[0, 3, 6] + [-1] * (nK - 3)]], np.int32)
    bb = np.array([[[1, 4, 7] + [-1] * (nK - 3)]], np.int32)
    n6, n3 = np.array([[6]], np.int32), np.array([[3]], np.int32)
    O, L_ = oracle.attention(Q, K, V, cs, blk, full, n6)
    O1, L1 = oracle.attention(Q, K, V, cs, blk, a, n3)
    O2, L2 = oracle.attention(Q, K, V, cs, blk, bb, n3)
    Lm = np.logaddexp(L1, L2)
    Om = np.exp(L1 - Lm)[..., None] * O1 + np.exp(L2 - Lm)[..., None] * O2
    np.testing.assert_allclose(Om, O, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(Lm, L_, rtol=1e-12, atol=1e-12)


def test_merge_states_pins():
    """The oracle's state merge: disjoint halves merged equal attention over
    the union; the special cases (one side empty, equal LSEs, both empty,
    LSEs far beyond exp's range) have closed forms."""
    B, H_q, H_kv, D, blk, C, L = 1, 2, 1, 16, 8, 16, 64
    cs = (48,)
    Q, K, V = _rand_qkv(22, B, H_q, H_kv, C, L, D)
    nK = L // blk
    full = np.array([[[0, 2, 3, 5, 6, 7] + [-1] * (nK - 6)]], np.int32)
    a = np.array([[[2, 5, 7] + [-1] * (nK - 3)]], np.int32)
    bb = np.array([[[0, 3, 6] + [-1] * (nK - 3)]], np.int32)
    n6, n3 = np.array([[6]], np.int32), np.array([[3]], np.int32)
    O, L_ = oracle.attention(Q, K, V, cs, blk, full, n6)
    O1, L1 = oracle.attention(Q, K, V, cs, blk, a, n3)
    O2, L2 = oracle.attention(Q, K, V, cs, blk, bb, n3)
    Om, Lm = oracle.merge_states(O1, L1, O2, L2)
    np.testing.assert_allclose(Om, O, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(Lm, L_, rtol=1e-12, atol=1e-12)
    Os, Ls = oracle.merge_states(O2, L2, O1, L1)  # symmetric
    np.testing.assert_allclose(Os, Om, rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(Ls, Lm, rtol=1e-14, atol=1e-14)

    rng = np.random.default_rng(5)
    Oa, Ob = rng.standard_normal((2, 6, 4))
    la = np.array([0.0, -3.0, 2.5, 1000.0, -1000.0, -np.inf])
    inf = np.full(6, -np.inf)
    O, Lz = oracle.merge_states(Oa, la, Ob, inf)       # other side empty
    np.testing.assert_array_equal(O[:5], Oa[:5])
    np.testing.assert_array_equal(Lz[:5], la[:5])
    assert np.all(O[5] == 0.0) and Lz[5] == -np.inf   # both empty
    O, Le = oracle.merge_states(Oa[:5], la[:5], Ob[:5], la[:5].copy())
    np.testing.assert_allclose(O, (Oa[:5] + Ob[:5]) / 2, rtol=1e-15, atol=1e-15)
    np.testing.assert_allclose(Le, la[:5] + math.log(2.0), rtol=1e-15, atol=1e-12)
    # weights e/(1+e) and 1/(1+e) at an LSE gap of 1, far from exp's range
    O, Lg = oracle.merge_states(Oa[3:5], la[3:5] + 1.0, Ob[3:5], la[3:5])
    w = math.e / (1.0 + math.e)
    np.testing.assert_allclose(O, w * Oa[3:5] + (1 - w) * Ob[3:5], rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(Lg, la[3:5] + 1.0 + math.log1p(math.exp(-1.0)), rtol=1e-15)
    with pytest.raises(ValueError):
        oracle.merge_states(Oa, la, Ob[:5], la[:5])


def test_nan_poison_outside_visible_keys_is_never_read():
    B, H_q, H_kv, D, blk, C, L = 2, 4, 1, 8, 4, 8, 48
    cs = (16, 32)
    rng = np.random.default_rng(2)
    mask = _rand_mask(rng, B, H_q, C // blk, L // blk, 0.3)
    T, cnt, _, _ = oracle.block_tables(mask, 4)
    Q, K, V = _rand_qkv(4, B, H_q, H_kv, C, L, D)
    O, LSE = oracle.attention(Q, K, V, cs, blk, T, cnt)
    Kp, Vp = K.clone(), V.clone()
    for b in range(B):
        sel = set(T[b, 0, :cnt[b, 0]].tolist())
        for j in range(L // blk):
            if j not in sel:
                Kp[b, :, j * blk:(j + 1) * blk] = float("nan")
                Vp[b, :, j * blk:(j + 1) * blk] = float("nan")
        Kp[b, :, cs[b] + C:] = float("nan")
        Vp[b, :, cs[b] + C:] = float("nan")
    O2, LSE2 = oracle.attention(Q, Kp, Vp, cs, blk, T, cnt)
    np.testing.assert_array_equal(O, O2)
    np.testing.assert_array_equal(LSE, LSE2)


def test_empty_table_rows():
    B, H_q, H_kv, D, blk, C, L = 1, 2, 1, 8, 4, 8, 32
    Q, K, V = _rand_qkv(1, B, H_q, H_kv, C, L, D)
    T = np.full((1, 1, 8), -1, np.int32)
    # one selected block entirely in the future of the first chunk rows
    T[0, 0, 0] = 5
    cnt = np.array([[1]], np.int32)
    O, LSE = oracle.attention(Q, K, V, (16,), blk, T, cnt)
    # rows r < 4 (positions 16..19) see no key; rows r >= 4 see block 5 up to p
    assert np.all(O[0, :, :4] == 0.0) and np.all(np.isneginf(LSE[0, :, :4]))
    assert np.all(np.isfinite(LSE[0, :, 4:]))
    cnt0 = np.array([[0]], np.int32)
    O, LSE = oracle.attention(Q, K, V, (16,), blk, T, cnt0)
    assert np.all(O == 0.0) and np.all(np.isneginf(LSE))


def test_row_sampling_matches_full():
    wl = workloads.tiny()
    Q, K, V = workloads.make_qkv(wl)
    T, cnt, _, _ = oracle.block_tables(workloads.make_mask(wl), wl.group)
    O, LSE = oracle.attention(Q, K, V, wl.chunk_start, wl.blk, T, cnt)
    rows = np.array([0, 5, 255, 256, 700, 1023], np.int64)
    Os, LSEs = oracle.attention(Q, K, V, wl.chunk_start, wl.blk, T, cnt, rows=rows)
    np.testing.assert_array_equal(Os, O.reshape(-1, wl.D)[rows])
    np.testing.assert_array_equal(LSEs, LSE.reshape(-1)[rows])


def test_rejects_out_of_range_table_entries():
    Q, K, V = _rand_qkv(1, 1, 2, 1, 8, 32, 8)
    T = np.full((1, 1, 8), -1, np.int32)
    T[0, 0, 0] = 9  # beyond nKVmax = 8
    with pytest.raises(ValueError):
        oracle.attention(Q, K, V, (16,), 4, T, np.array([[1]], np.int32))


def test_visible_pair_count():
    # dense, one head: pairs = C*cs + C*(C+1)/2
    C, cs, blk = 16, 32, 8
    n = oracle.visible_pairs([cs], 1, 1, 1, C, 64, blk)
    assert n == C * cs + C * (C + 1) // 2
    # the 128K / 2048 chunk dense count quoted for the LLaMA-8B shape
    assert 2048 * 131072 + 2048 * 2049 // 2 == 270_533_632


# ------------------------------------------------ per-tile block-sparse path

def _tile_allowed(mask, B, H_q, C, L, blk, cs):
    """allowed[b, h, r, k]: block (r // blk, k // blk) selected by head h and
    key k causally visible from position cs[b] + r (token-level expansion of
    the block mask, built with plain indexing)."""
    m = torch.as_tensor(mask).bool()
    rows = torch.arange(C) // blk
    keys = torch.arange(L) // blk
    tile = m[:, :, rows][:, :, :, keys]  # [B, H_q, C, L]
    return tile & _causal_allowed(B, H_q, C, L, cs)


@pytest.mark.parametrize("cfg", [
    # B, H_q, H_kv, D, blk, C, L_max, chunk_start, density
    (1, 4, 1, 16, 8, 24, 64, (16,), 0.3),
    (2, 6, 2, 8, 4, 12, 40, (0, 20), 0.5),
    (2, 4, 2, 32, 8, 32, 96, (40, 8), 0.2),
])
def test_tile_attention_equals_sdpa_with_expanded_block_mask(cfg):
    """Per-tile block-sparse attention is SDPA with the token-level mask that
    the per-head per-Q-block block mask expands to (causal on top)."""
    B, H_q, H_kv, D, blk, C, L, cs, dens = cfg
    rng = np.random.default_rng(sum(cfg[:7]))
    nQ, nK = C // blk, L // blk
    mask = _rand_mask(rng, B, H_q, nQ, nK, dens)
    Q, K, V = _rand_qkv(7 + B, B, H_q, H_kv, C, L, D)
    scale = 0.9 / math.sqrt(D)
    O, LSE = oracle.attention_tile(Q, K, V, cs, blk, mask, scale=scale)
    Oref, LSEref = _sdpa_masked(Q, K, V, _tile_allowed(mask, B, H_q, C, L, blk, cs), scale)
    np.testing.assert_allclose(O, Oref, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(LSE, LSEref, rtol=1e-10, atol=1e-10)
    # some rows see no key at these densities: the convention O = 0, LSE = -inf
    empty = ~_tile_allowed(mask, B, H_q, C, L, blk, cs).any(dim=-1).numpy()
    assert np.all(O[empty] == 0.0) and np.all(np.isneginf(LSE[empty]))


def test_tile_attention_on_union_closed_mask_equals_block_union_attention():
    """When every head and Q-block of a group selects exactly the group's
    union, the per-tile path and the Block-Union path attend to the same keys."""
    rng = np.random.default_rng(11)
    B, H_q, H_kv, D, blk, C, L = 2, 4, 2, 16, 8, 32, 96
    cs = (48, 16)
    G = H_q // H_kv
    U = (rng.random((B, H_kv, L // blk)) < 0.4).astype(np.uint8)
    mask = np.repeat(U, G, axis=1)[:, :, None, :].repeat(C // blk, axis=2)
    T, cnt, _, _ = oracle.block_tables(mask, G)
    Q, K, V = _rand_qkv(5, B, H_q, H_kv, C, L, D)
    O1, L1 = oracle.attention_tile(Q, K, V, cs, blk, mask)
    O2, L2 = oracle.attention(Q, K, V, cs, blk, T, cnt)
    np.testing.assert_array_equal(np.isneginf(L1), np.isneginf(L2))
    fin = ~np.isneginf(L2)
    np.testing.assert_allclose(O1, O2, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(L1[fin], L2[fin], rtol=1e-12, atol=1e-12)


def test_tile_attention_all_ones_is_dense_causal():
    B, H_q, H_kv, D, blk, C, L, cs = 1, 4, 2, 16, 8, 24, 64, (24,)
    Q, K, V = _rand_qkv(3, B, H_q, H_kv, C, L, D)
    mask = np.ones((B, H_q, C // blk, L // blk), np.uint8)
    O, LSE = oracle.attention_tile(Q, K, V, cs, blk, mask)
    Oref, LSEref = _sdpa_masked(Q, K, V, _causal_allowed(B, H_q, C, L, cs), 1 / math.sqrt(D))
    np.testing.assert_allclose(O, Oref, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(LSE, LSEref, rtol=1e-10, atol=1e-10)


@pytest.mark.parametrize("span", [1, 2, 3, 4])
def test_tile_span_tables_round_trip_and_order(span):
    """The span tables encode the mask losslessly: decoding every entry's
    bits gives back exactly the nonzero pattern of every mask row; entries are
    strictly ascending, each has at least one bit, the tail is -1."""
    rng = np.random.default_rng(100 + span)
    B, H_q, nQ, nK = 2, 3, 7, 40
    mask = (rng.random((B, H_q, nQ, nK)) < 0.25).astype(np.uint8) * rng.integers(1, 255, (B, H_q, nQ, nK), dtype=np.uint8)
    T, cnt = oracle.tile_span_tables(mask, span)
    nS = -(-nQ // span)
    assert T.shape == (B, H_q, nS, nK) and cnt.shape == (B, H_q, nS)
    rebuilt = np.zeros((B, H_q, nS * span, nK), bool)
    for b in range(B):
        for h in range(H_q):
            for s in range(nS):
                n = cnt[b, h, s]
                e = T[b, h, s, :n].astype(np.int64)
                j, bits = e & ((1 << 24) - 1), e >> 24
                assert np.all(np.diff(j) > 0) and np.all(bits > 0)
                assert np.all(bits < (1 << span))
                assert np.all(T[b, h, s, n:] == -1)
                for u in range(span):
                    rebuilt[b, h, s * span + u, j[(bits >> u) & 1 == 1]] = True
    np.testing.assert_array_equal(rebuilt[:, :, :nQ], mask != 0)
    assert not rebuilt[:, :, nQ:].any()


# ------------------------------------------------------------ FP8 (E4M3) inputs

def test_e4m3_decode_matches_torch_on_every_code():
    """The oracle's E4M3 decoder, written from the format's definition, against
    torch's float8_e4m3fn conversion on all 256 codes (NaN codes included)."""
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = np.array([oracle.e4m3_decode(i) for i in range(256)])
    assert np.array_equal(np.isnan(ref), np.isnan(mine))
    np.testing.assert_array_equal(mine[~np.isnan(mine)], ref[~np.isnan(ref)])
    assert mine[0x7E] == 448.0 and mine[0x01] == 2.0 ** -9 and mine[0x08] == 2.0 ** -6


@pytest.mark.parametrize("cfg", [
    # B, H_q, H_kv, D, blk, C, L_max, chunk_start
    (1, 4, 1, 16, 8, 24, 64, (16,)),
    (2, 4, 2, 32, 8, 16, 48, (32, 8)),
])
def test_e4m3_attention_equals_sdpa_on_dequantized_inputs(cfg):
    """FP8 attention is the bf16 definition on the dequantized tensors: fp64
    SDPA on descale * decode(codes) (decoded by torch), under the tables."""
    B, H_q, H_kv, D, blk, C, L, cs = cfg
    Q, K, V = _rand_qkv(sum(cfg[:7]) + 1, B, H_q, H_kv, C, L, D)
    (q8, qd), (k8, kd), (v8, vd) = (workloads.quantize_e4m3(t) for t in (Q, K, V))
    rng = np.random.default_rng(5)
    mask = (rng.random((B, H_q, C // blk, L // blk)) < 0.5).astype(np.uint8)
    mask[..., 0] = 1
    T, cnt, _, _ = oracle.block_tables(mask, H_q // H_kv)
    scale = 0.8 / math.sqrt(D)
    O, LSE = oracle.attention_e4m3(q8, k8, v8, (qd, kd, vd), cs, blk, T, cnt, scale=scale)
    deq = lambda c, d: (c.view(torch.float8_e4m3fn).to(torch.float64) * d)
    Qd, Kd, Vd = deq(q8, qd), deq(k8, kd), deq(v8, vd)
    # the union's key set, expanded to tokens, causal on top
    allowed = torch.zeros(B, H_q, C, L, dtype=torch.bool)
    for b in range(B):
        for h in range(H_q):
            sel = torch.zeros(L, dtype=torch.bool)
            for j in T[b, h // (H_q // H_kv), :cnt[b, h // (H_q // H_kv)]]:
                sel[j * blk:(j + 1) * blk] = True
            allowed[b, h] = sel[None, :]
    allowed &= _causal_allowed(B, H_q, C, L, cs)
    Oref, LSEref = _sdpa_masked(Qd, Kd, Vd, allowed, scale)
    np.testing.assert_allclose(O, Oref, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(LSE, LSEref, rtol=1e-10, atol=1e-10)


def test_quantize_e4m3_round_trip_bound():
    """The FP8 input encoding: |x - descale * decode(code)| is within half an
    E4M3 step of x / descale (relative 2^-4 for normal codes, 2^-10 absolute
    below 2^-6), and amax maps to 448."""
    x = torch.randn(4096, generator=torch.Generator().manual_seed(3)) * 3
    codes, d = workloads.quantize_e4m3(x)
    dec = np.array([oracle.e4m3_decode(int(c)) for c in codes.numpy()])
    y = x.double().numpy() / d
    err = np.abs(dec - y)
    bound = np.maximum(np.abs(y) * 2.0 ** -4, 2.0 ** -10)
    assert np.all(err <= bound * (1 + 1e-12))
    assert np.isclose(np.abs(dec).max(), 448.0)
