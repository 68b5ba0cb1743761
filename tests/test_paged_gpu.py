"""The paged metadata form (kv_indptr / kv_indices with global page ids) and
ragged chunk lengths, on the GPU, against the fp64 CPU oracle.

The builder's CSR output must be the oracle's CSR with every entry offset to
its (b, g)'s first page, bit for bit. The paged attention must match the
oracle element by element on every row inside each sequence's chunk, leave
rows past a shorter chunk untouched, and report (not fault on) metadata that
points outside its own (b, g) or outside kv_indices."""
import numpy as np
import pytest
import torch

import oracle
import serving_block_union_b200 as ca
import workloads
from parity_util import compare, sample_rows

pytestmark = pytest.mark.gpu

SENTINEL = 7.0


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g).to(torch.bfloat16)


def _global_indices(indptr, indices, H_kv, nKVmax):
    out = indices[: indptr[-1]].astype(np.int64).copy()
    for bg in range(len(indptr) - 1):
        out[indptr[bg]:indptr[bg + 1]] += bg * nKVmax
    return out


@pytest.mark.parametrize("name", ["tiny", "llama8b_32k", "llama8b_128k_d10", "batched",
                                  "qwen3_30b_128k_d10"])
def test_kv_pages_bit_exact(cuda_ok, name):
    wl = workloads.by_name(name)
    mask = workloads.make_mask(wl)
    ip, ix, T, c = ca.build_kv_pages(torch.from_numpy(mask).cuda(), wl.group)
    T_ref, c_ref, ip_ref, ix_ref = oracle.block_tables(mask, wl.group)
    np.testing.assert_array_equal(T.cpu().numpy(), T_ref)
    np.testing.assert_array_equal(c.cpu().numpy(), c_ref)
    np.testing.assert_array_equal(ip.cpu().numpy(), ip_ref)
    nnz = int(ip_ref[-1])
    np.testing.assert_array_equal(ix.cpu().numpy()[:nnz],
                                  _global_indices(ip_ref, ix_ref, wl.H_kv, wl.nKVmax))


def _ragged_case(B, H_q, H_kv, D, blk, C, L_max, cs, lens, p, seed):
    nQ = -(-C // blk)
    nK = L_max // blk
    rng = np.random.default_rng(seed)
    mask = (rng.random((B, H_q, nQ, nK)) < p).astype(np.uint8)
    for b in range(B):  # Q-blocks wholly past a sequence's chunk select nothing
        mask[b, :, -(-lens[b] // blk):] = 0
    Q = _rand((B, H_q, C, D), seed + 1)
    K = _rand((B, H_kv, L_max, D), seed + 2)
    V = _rand((B, H_kv, L_max, D), seed + 3)
    return mask, Q, K, V


def _valid_rows(B, H_q, C, lens):
    rows = []
    for b in range(B):
        for h in range(H_q):
            base = (b * H_q + h) * C
            rows.extend(range(base, base + lens[b]))
    return np.asarray(rows, dtype=np.int64)


def _check_ragged(O, L, O_ref, L_ref, B, H_q, C, lens):
    O, L = O.float().cpu(), L.cpu()
    for b in range(B):
        n = lens[b]
        if n > 0:
            compare(O[b:b + 1, :, :n], L[b:b + 1, :, :n], O_ref[b:b + 1, :, :n],
                    L_ref[b:b + 1, :, :n])
        assert (O[b, :, n:] == SENTINEL).all() and (L[b, :, n:] == SENTINEL).all()


RAGGED = [
    # B, H_q, H_kv, D, blk, C, L_max, chunk_start, chunk_len
    (3, 8, 2, 128, 128, 512, 2048, (1024, 256, 1536), (512, 200, 129)),
    (2, 4, 1, 64, 64, 256, 1024, (700, 64), (256, 37)),
    (4, 16, 2, 128, 64, 384, 1536, (0, 512, 1100, 64), (384, 1, 300, 0)),   # G = 8, empty chunk
    (2, 32, 8, 128, 128, 1024, 128 * 70, (128 * 60, 128 * 8), (1024, 513)),
]


@pytest.mark.parametrize("case", RAGGED)
def test_ragged_paged_attention_full_compare(cuda_ok, case):
    B, H_q, H_kv, D, blk, C, L_max, cs, lens = case
    mask, Q, K, V = _ragged_case(B, H_q, H_kv, D, blk, C, L_max, cs, lens, 0.3,
                                 seed=sum(case[:7]))
    ip, ix, _, _ = ca.build_kv_pages(torch.from_numpy(mask).cuda(), H_q // H_kv)
    O = torch.full((B, H_q, C, D), SENTINEL, dtype=torch.bfloat16, device="cuda")
    L = torch.full((B, H_q, C), SENTINEL, dtype=torch.float32, device="cuda")
    ws = ca.new_workspace(B, H_q, H_kv, C, blk)
    ca.paged_chunk_attention(Q.cuda(), K.cuda(), V.cuda(), ip, ix, cs, blk, chunk_len=lens,
                             O=O, LSE=L, workspace=ws)
    assert ca.read_device_status(ws) == ca.CA_OK
    T, c, _, _ = oracle.block_tables(mask, H_q // H_kv)
    O_ref, L_ref = oracle.attention(Q, K, V, cs, blk, T, c)
    _check_ragged(O, L, O_ref, L_ref, B, H_q, C, lens)


def test_full_size_paged_equals_oracle(cuda_ok):
    """128K / 10% through the paged form (chunk_len = C): sampled rows."""
    wl = workloads.llama8b_128k(0.10)
    mask = workloads.make_mask(wl)
    Q, K, V = workloads.make_qkv(wl)
    ip, ix, _, _ = ca.build_kv_pages(torch.from_numpy(mask).cuda(), wl.group)
    ws = ca.new_workspace(wl.B, wl.H_q, wl.H_kv, wl.C, wl.blk)
    O, L = ca.paged_chunk_attention(Q.cuda(), K.cuda(), V.cuda(), ip, ix, wl.chunk_start,
                                    wl.blk, workspace=ws)
    assert ca.read_device_status(ws) == ca.CA_OK
    T, c, _, _ = oracle.block_tables(mask, wl.group)
    rows = sample_rows(wl, n_random=256)
    O_ref, L_ref = oracle.attention(Q, K, V, wl.chunk_start, wl.blk, T, c, rows=rows)
    compare(O, L, O_ref, L_ref, rows=rows)


def test_full_size_batched_ragged(cuda_ok):
    """The batched workload (B4, 16K-96K cached, chunk 4096) with chunks of
    4096 / 2048 / 3000 / 1000 rows: sampled rows inside each chunk."""
    wl = workloads.batched()
    lens = (4096, 2048, 3000, 1000)
    mask = workloads.make_mask(wl)
    for b in range(wl.B):
        mask[b, :, -(-lens[b] // wl.blk):] = 0
    Q, K, V = workloads.make_qkv(wl)
    ip, ix, _, _ = ca.build_kv_pages(torch.from_numpy(mask).cuda(), wl.group)
    O = torch.full((wl.B, wl.H_q, wl.C, wl.D), SENTINEL, dtype=torch.bfloat16, device="cuda")
    L = torch.full((wl.B, wl.H_q, wl.C), SENTINEL, dtype=torch.float32, device="cuda")
    ws = ca.new_workspace(wl.B, wl.H_q, wl.H_kv, wl.C, wl.blk)
    ca.paged_chunk_attention(Q.cuda(), K.cuda(), V.cuda(), ip, ix, wl.chunk_start, wl.blk,
                             chunk_len=lens, O=O, LSE=L, workspace=ws)
    assert ca.read_device_status(ws) == ca.CA_OK
    T, c, _, _ = oracle.block_tables(mask, wl.group)
    rows = sample_rows(wl, n_random=512)
    r, b = rows % wl.C, rows // (wl.H_q * wl.C)
    rows = rows[r < np.asarray(lens)[b]]
    O_ref, L_ref = oracle.attention(Q, K, V, wl.chunk_start, wl.blk, T, c, rows=rows)
    compare(O, L, O_ref, L_ref, rows=rows)
    Oc, Lc = O.float().cpu(), L.cpu()
    for b in range(wl.B):
        assert (Oc[b, :, lens[b]:] == SENTINEL).all() and (Lc[b, :, lens[b]:] == SENTINEL).all()


@pytest.mark.parametrize("corrupt", ["foreign_page", "indptr_past_nnz", "decreasing_indptr"])
def test_invalid_paged_metadata_is_reported(cuda_ok, corrupt):
    B, H_q, H_kv, D, blk, C, L_max, cs, lens = RAGGED[0]
    mask, Q, K, V = _ragged_case(B, H_q, H_kv, D, blk, C, L_max, cs, lens, 0.5, seed=9)
    ip, ix, _, _ = ca.build_kv_pages(torch.from_numpy(mask).cuda(), H_q // H_kv)
    ip, ix = ip.clone(), ix.clone()
    nnz = ix.numel()
    if corrupt == "foreign_page":
        ix[int(ip[1].item())] = 0            # (b=0, g=1) gets a page of (0, 0)
    elif corrupt == "indptr_past_nnz":
        ip[-1] = nnz + 5
        nnz = int(ip[-2].item()) + 2         # and the array is declared shorter
    else:
        ip[2] = ip[1] - 1
    ws = ca.new_workspace(B, H_q, H_kv, C, blk)
    ca.paged_chunk_attention(Q.cuda(), K.cuda(), V.cuda(), ip, ix[:nnz], cs, blk,
                             chunk_len=lens, workspace=ws)
    assert ca.read_device_status(ws) == ca.CA_ERR_TABLE
