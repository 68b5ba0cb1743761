"""Explicit-compaction ablation on the GPU (the copy path the CompactAttention
pages' efficiency ablation compares zero-copy execution against): the gather
copies exactly the selected blocks (checked against torch indexing on the
CPU); attention over the compact buffers matches the fp64 oracle's attention
over the same tables element by element (every row on the small workload,
sampled rows at the full sizes), and gives the same bits as the zero-copy
attention over the cache (same blocks, same order, same arithmetic)."""
import numpy as np
import pytest
import torch

import oracle
import serving_block_union_b200 as ca
import workloads
from parity_util import compare, sample_rows

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["tiny", "llama8b_32k", "batched"])
def test_compaction_matches_oracle_and_zero_copy(cuda_ok, name):
    wl = workloads.by_name(name)
    mask = workloads.make_mask(wl)
    Q, K, V = workloads.make_qkv(wl)
    T, c, _, _ = oracle.block_tables(mask, wl.group)
    dev = torch.device("cuda")
    Qd, Kd, Vd = Q.to(dev), K.to(dev), V.to(dev)
    Td, cd = torch.from_numpy(T).to(dev), torch.from_numpy(c).to(dev)
    Kc, Vc = ca.compact_kv_blocks(Kd, Vd, Td, cd)
    ws = ca.new_workspace(wl.B, wl.H_q, wl.H_kv, wl.C, wl.blk)
    O2, L2 = ca.compacted_chunk_attention(Qd, Kc, Vc, Td, cd, wl.chunk_start, workspace=ws)
    assert ca.read_device_status(ws) == ca.CA_OK
    # against the oracle: all rows on the small workload, sampled rows otherwise
    if name == "tiny":
        O_ref, L_ref = oracle.attention(Q, K, V, wl.chunk_start, wl.blk, T, c)
        compare(O2, L2, O_ref, L_ref)
    else:
        rows = sample_rows(wl, n_random=512)
        O_ref, L_ref = oracle.attention(Q, K, V, wl.chunk_start, wl.blk, T, c, rows=rows)
        compare(O2, L2, O_ref, L_ref, rows=rows)
    assert torch.isfinite(O2.float()).all()
    # against the zero-copy walk over the cache: the same bits
    O1, L1 = ca.chunk_attention(Qd, Kd, Vd, Td, cd, wl.chunk_start)
    torch.cuda.synchronize()
    assert torch.equal(O1, O2) and torch.equal(L1, L2)
    # the gather itself, for a few (b, g): rows t*blk.. of Kc are block T[t] of K
    Kc_h, Vc_h = Kc.cpu(), Vc.cpu()
    rng = np.random.default_rng(0)
    for _ in range(4):
        b = int(rng.integers(wl.B)); g = int(rng.integers(wl.H_kv))
        n = int(c[b, g])
        idx = np.concatenate([np.arange(j * wl.blk, (j + 1) * wl.blk) for j in T[b, g, :n]])
        assert torch.equal(Kc_h[b, g, :n * wl.blk], K[b, g, torch.from_numpy(idx)])
        assert torch.equal(Vc_h[b, g, :n * wl.blk], V[b, g, torch.from_numpy(idx)])
