"""Merge of attention states over disjoint key sets on the GPU vs the fp64
oracle: random states (every D class, ragged row counts, -inf rows, LSEs far
outside exp's range), 2 to 8 parts, in place, without an LSE output, the
two-part C entry, and end to end: chunk attention over disjoint halves (and
thirds) of the Block-Union tables, merged, against the oracle's attention over
the whole tables."""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle
import serving_block_union_b200 as ca
from parity_util import compare

pytestmark = pytest.mark.gpu

# bf16 output of an fp32 merge: half an ulp of bf16 relative to the value,
# plus fp32 rounding relative to the largest input it sums.
O_REL = 2.0 ** -8
O_ABS_OF_MAX = 1e-5


def _states(n, lead, D, seed, spread=4.0):
    g = torch.Generator().manual_seed(seed)
    Os = [torch.randn(*lead, D, generator=g).to(torch.bfloat16) for _ in range(n)]
    Ls = [(torch.rand(*lead, generator=g) * 2 - 1) * spread for _ in range(n)]
    flat = [L.view(-1) for L in Ls]
    rows = flat[0].numel()
    rng = np.random.default_rng(seed)
    for i in range(n):
        # some rows empty in one part, some rows empty in every part
        flat[i][torch.from_numpy(rng.random(rows) < 0.1)] = -math.inf
    if rows >= 4:
        for i in range(n):
            flat[i][3] = -math.inf
        flat[0][1] = 1000.0      # exp() of it alone would overflow fp32
        flat[-1][2] = -1000.0
    return Os, Ls


def _oracle_fold(Os, Ls):
    O = Os[0].double().numpy()
    L = Ls[0].double().numpy()
    for Oi, Li in zip(Os[1:], Ls[1:]):
        O, L = oracle.merge_states(O, L, Oi.double().numpy(), Li.double().numpy())
    return O, L


def _check(O, L, O_ref, L_ref, Os):
    D = O.shape[-1]
    o = O.float().cpu().numpy().reshape(-1, D)
    ref = O_ref.reshape(-1, D)
    big = max(float(x.float().abs().max()) for x in Os)
    err = np.abs(o - ref)
    assert (err <= O_REL * np.abs(ref) + O_ABS_OF_MAX * big).all(), f"O err {err.max():.3e}"
    l = L.cpu().numpy().reshape(-1)
    lr = L_ref.reshape(-1)
    inf = np.isneginf(lr)
    assert np.array_equal(np.isneginf(l), inf)
    assert (o[inf] == 0).all()
    fin = ~inf
    lerr = np.abs(l[fin] - lr[fin])
    assert (lerr <= 2e-7 * np.abs(lr[fin]) + 2e-6).all(), f"LSE err {lerr.max():.3e}"


@pytest.mark.parametrize("lead,D", [((1, 32, 2048), 128), ((7,), 64), ((3, 1001), 256),
                                    ((5, 333), 96), ((2, 37), 8), ((11,), 2048),
                                    ((100003,), 128), ((1,), 128)])
def test_two_parts_random(cuda_ok, lead, D):
    Os, Ls = _states(2, lead, D, seed=D + sum(lead))
    O, L = ca.merge_attention_states([(o.cuda(), l.cuda()) for o, l in zip(Os, Ls)])
    torch.cuda.synchronize()
    O_ref, L_ref = _oracle_fold(Os, Ls)
    _check(O, L, O_ref, L_ref, Os)


@pytest.mark.parametrize("n", [3, 5, 8])
def test_n_parts_random(cuda_ok, n):
    Os, Ls = _states(n, (4, 8, 300), 128, seed=40 + n)
    O, L = ca.merge_attention_states([(o.cuda(), l.cuda()) for o, l in zip(Os, Ls)])
    torch.cuda.synchronize()
    O_ref, L_ref = _oracle_fold(Os, Ls)
    _check(O, L, O_ref, L_ref, Os)


def test_in_place_and_without_lse(cuda_ok):
    Os, Ls = _states(3, (2, 4, 500), 128, seed=77)
    parts = [(o.cuda(), l.cuda()) for o, l in zip(Os, Ls)]
    O, L = ca.merge_attention_states(parts)
    O2, L2 = ca.merge_attention_states(parts, want_lse=False)
    assert L2 is None
    assert torch.equal(O2, O)
    # in place into part 1 (output O and LSE both alias that part)
    ca.merge_attention_states(parts, O=parts[1][0], LSE=parts[1][1])
    torch.cuda.synchronize()
    assert torch.equal(parts[1][0], O)
    assert torch.equal(parts[1][1], L)


def test_two_part_c_entry_matches(cuda_ok):
    Os, Ls = _states(2, (3, 1000), 64, seed=5)
    a, b = [(o.cuda(), l.cuda()) for o, l in zip(Os, Ls)]
    O, L = ca.merge_attention_states([a, b])
    O2, L2 = torch.empty_like(O), torch.empty_like(L)
    lib = ca.load_library()
    st = lib.ca_merge_attention_states(
        ctypes.c_void_p(a[0].data_ptr()), ctypes.c_void_p(a[1].data_ptr()),
        ctypes.c_void_p(b[0].data_ptr()), ctypes.c_void_p(b[1].data_ptr()), 3000, 64,
        ctypes.c_void_p(O2.data_ptr()), ctypes.c_void_p(L2.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == ca.CA_OK
    torch.cuda.synchronize()
    assert torch.equal(O2, O) and torch.equal(L2, L)


def _split_tables(T, c, k):
    """k disjoint sub-tables: entry t of each (b, g) table goes to part t % k
    (ascending order kept)."""
    B, H_kv, nK = T.shape
    parts = []
    for i in range(k):
        Ti = np.full_like(T, -1)
        ci = np.zeros_like(c)
        for b in range(B):
            for g in range(H_kv):
                sel = T[b, g, :c[b, g]][i::k]
                Ti[b, g, :len(sel)] = sel
                ci[b, g] = len(sel)
        parts.append((Ti, ci))
    return parts


@pytest.mark.parametrize("k", [2, 3])
def test_split_tables_merged_equals_union(cuda_ok, k):
    B, H_q, H_kv, D, blk, C, L_max = 2, 16, 4, 128, 128, 512, 2560
    cs = (2048, 1024)
    nQ, nK = C // blk, L_max // blk
    rng = np.random.default_rng(11 + k)
    mask = (rng.random((B, H_q, nQ, nK)) < 0.2).astype(np.uint8)
    g = torch.Generator().manual_seed(12)
    Q = torch.randn(B, H_q, C, D, generator=g).to(torch.bfloat16)
    K = torch.randn(B, H_kv, L_max, D, generator=g).to(torch.bfloat16)
    V = torch.randn(B, H_kv, L_max, D, generator=g).to(torch.bfloat16)
    T, c, _, _ = oracle.block_tables(mask, H_q // H_kv)
    # (b=1, g=0) has a single table entry, so with k parts some are empty
    assert c[1, 0] >= 1
    T[1, 0, 1:] = -1
    c[1, 0] = 1
    Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
    results = []
    for Ti, ci in _split_tables(T, c, k):
        results.append(ca.chunk_attention(Qd, Kd, Vd, torch.from_numpy(Ti).cuda(),
                                          torch.from_numpy(ci).cuda(), cs))
    O, L = ca.merge_attention_states(results)
    torch.cuda.synchronize()
    O_ref, L_ref = oracle.attention(Q, K, V, cs, blk, T, c)
    compare(O, L, O_ref, L_ref)


def test_rejects_bad_tensors(cuda_ok):
    a = (torch.zeros(4, 128, dtype=torch.bfloat16, device="cuda"),
         torch.zeros(4, device="cuda"))
    with pytest.raises(ValueError):
        ca.merge_attention_states([a])
    with pytest.raises(ValueError):
        ca.merge_attention_states([a, (a[0][:2], a[1][:2])])
    with pytest.raises(TypeError):
        ca.merge_attention_states([a, (a[0].float(), a[1])])
    with pytest.raises(ca.CAError):
        b = (torch.zeros(4, 100, dtype=torch.bfloat16, device="cuda"), a[1])
        ca.merge_attention_states([b, b])
