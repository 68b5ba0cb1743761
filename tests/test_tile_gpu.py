"""Per-tile block-sparse ablation path on the GPU vs the fp64 CPU oracle.

The span-table builder must match the oracle bit for bit (padding included);
the per-tile attention (every head and Q-block with its own blocks, no union)
must match ``oracle.attention_tile`` element by element on small shapes and on
sampled rows at the full workload sizes, including rows that see no key."""
import numpy as np
import pytest
import torch

import oracle
import serving_block_union_b200 as ca
import workloads
from parity_util import compare, sample_rows

pytestmark = pytest.mark.gpu


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g).to(torch.bfloat16)


def _small_case(B, H_q, H_kv, D, blk, C, L_max, p, seed):
    nQ = -(-C // blk)
    nK = L_max // blk
    rng = np.random.default_rng(seed)
    mask = (rng.random((B, H_q, nQ, nK)) < p).astype(np.uint8)
    Q = _rand((B, H_q, C, D), seed + 1)
    K = _rand((B, H_kv, L_max, D), seed + 2)
    V = _rand((B, H_kv, L_max, D), seed + 3)
    return mask, Q, K, V


def _gpu_tile(mask, Q, K, V, cs, blk, ws=None):
    Td, cd = ca.build_tile_tables(torch.from_numpy(mask).cuda(), blk)
    O, L = ca.tile_chunk_attention(Q.cuda(), K.cuda(), V.cuda(), Td, cd, cs, workspace=ws)
    torch.cuda.synchronize()
    return Td, cd, O, L


SMALL = [
    # B, H_q, H_kv, D, blk, C, L_max, chunk_start
    (1, 4, 1, 64, 64, 256, 1024, (768,)),
    (2, 8, 2, 128, 128, 384, 1152, (256, 640)),
    (1, 32, 8, 128, 128, 512, 2048, (1536,)),
    (2, 8, 8, 64, 128, 256, 768, (512, 128)),          # G = 1
    (1, 16, 2, 64, 64, 320, 1024, (192,)),             # G = 8, odd number of tiles
    (2, 8, 2, 128, 128, 200, 640, (128, 0)),           # ragged chunk length
    (2, 4, 1, 64, 64, 150, 512, (100, 37)),            # unaligned chunk starts
    (1, 8, 2, 128, 64, 96, 64 * 6, (0,)),              # first chunk, no cache
]


@pytest.mark.parametrize("case", SMALL)
@pytest.mark.parametrize("p", [0.2, 1.0])
def test_small_shapes_tables_and_attention(cuda_ok, case, p):
    B, H_q, H_kv, D, blk, C, L_max, cs = case
    mask, Q, K, V = _small_case(B, H_q, H_kv, D, blk, C, L_max, p, seed=sum(case[:7]))
    Td, cd, O, L = _gpu_tile(mask, Q, K, V, cs, blk)
    T, c = oracle.tile_span_tables(mask, ca.tile_span(blk))
    np.testing.assert_array_equal(Td.cpu().numpy(), T)
    np.testing.assert_array_equal(cd.cpu().numpy(), c)
    O_ref, L_ref = oracle.attention_tile(Q, K, V, cs, blk, mask)
    compare(O, L, O_ref, L_ref)


def test_split_last_wave(cuda_ok):
    """Few per-head items over a long cache: segments merged through the
    workspace, checked against the oracle in full."""
    B, H_q, H_kv, D, blk, C, L_max, cs = 1, 4, 2, 128, 128, 512, 128 * 400, (128 * 396,)
    # dense enough that every item's table (about 400 entries) makes
    # segments of at least 24 entries
    mask, Q, K, V = _small_case(B, H_q, H_kv, D, blk, C, L_max, 0.9, seed=41)
    ws = ca.new_workspace(B, H_q, H_kv, C, blk)
    _, _, O, L = _gpu_tile(mask, Q, K, V, cs, blk, ws=ws)
    assert ca.read_device_status(ws) == ca.CA_OK
    items = B * H_q * (-(-C // 256))  # per-head items, one merge counter each
    assert int(ws[256:256 + 4 * items].count_nonzero()) == 0
    O_ref, L_ref = oracle.attention_tile(Q, K, V, cs, blk, mask)
    compare(O, L, O_ref, L_ref)


def test_rows_without_keys(cuda_ok):
    """A Q-block that selects nothing (or only future blocks) gives O = 0 and
    LSE = -inf on its rows, whatever its span partner selects."""
    B, H_q, H_kv, D, blk, C, L_max, cs = 1, 8, 2, 128, 128, 512, 1536, (512,)
    mask, Q, K, V = _small_case(B, H_q, H_kv, D, blk, C, L_max, 0.4, seed=21)
    mask[0, 0, 0] = 0          # head 0, Q-block 0: nothing
    mask[0, 3, 2] = 0
    mask[0, 3, 2, 7] = 1       # head 3, Q-block 2 (positions 768..895): only block 7 (future)
    _, _, O, L = _gpu_tile(mask, Q, K, V, cs, blk)
    O_ref, L_ref = oracle.attention_tile(Q, K, V, cs, blk, mask)
    compare(O, L, O_ref, L_ref)
    Oc, Lc = O.float().cpu(), L.cpu()
    assert (Oc[0, 0, :128] == 0).all() and torch.isneginf(Lc[0, 0, :128]).all()
    assert (Oc[0, 3, 256:384] == 0).all() and torch.isneginf(Lc[0, 3, 256:384]).all()


FULL = ["llama8b_32k", "llama8b_128k_d10", "batched", "full_prefill_c63"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled_rows(cuda_ok, name):
    wl = workloads.by_name(name)
    mask = workloads.make_mask(wl)
    Q, K, V = workloads.make_qkv(wl)
    # NaN past kv_len and in every block no head of the group selected
    Kp, Vp = K.clone(), V.clone()
    workloads.poison_beyond_kv_len(wl, Kp, Vp)
    U, cU, _, _ = oracle.block_tables(mask, wl.group)
    for b in range(wl.B):
        for g in range(wl.H_kv):
            sel = np.zeros(wl.nKVmax, bool)
            sel[U[b, g, :cU[b, g]]] = True
            for j in np.nonzero(~sel)[0]:
                Kp[b, g, j * wl.blk:(j + 1) * wl.blk] = float("nan")
                Vp[b, g, j * wl.blk:(j + 1) * wl.blk] = float("nan")
    ws = ca.new_workspace(wl.B, wl.H_q, wl.H_kv, wl.C, wl.blk)
    Td, cd, O, L = _gpu_tile(mask, Q, Kp, Vp, wl.chunk_start, wl.blk, ws=ws)
    assert ca.read_device_status(ws) == ca.CA_OK
    T, c = oracle.tile_span_tables(mask, ca.tile_span(wl.blk))
    np.testing.assert_array_equal(Td.cpu().numpy(), T)
    np.testing.assert_array_equal(cd.cpu().numpy(), c)
    rows = sample_rows(wl, n_random=512)
    O_ref, L_ref = oracle.attention_tile(Q, K, V, wl.chunk_start, wl.blk, mask, rows=rows)
    compare(O, L, O_ref, L_ref, rows=rows)
    assert torch.isfinite(O.float()).all()


def test_invalid_span_table_is_reported(cuda_ok):
    B, H_q, H_kv, D, blk, C, L_max, cs = 1, 8, 2, 128, 128, 256, 1024, (512,)
    mask, Q, K, V = _small_case(B, H_q, H_kv, D, blk, C, L_max, 0.5, seed=8)
    T, c = oracle.tile_span_tables(mask, ca.tile_span(blk))
    T, c = T.copy(), c.copy()
    c[0, 2, 0] = L_max // blk + 5
    ws = ca.new_workspace(B, H_q, H_kv, C, blk)
    ca.tile_chunk_attention(Q.cuda(), K.cuda(), V.cuda(), torch.from_numpy(T).cuda(),
                            torch.from_numpy(c).cuda(), cs, workspace=ws)
    assert ca.read_device_status(ws) == ca.CA_ERR_TABLE
