"""The allocation-free attention entry point (ca_chunk_attention_noalloc),
called through the C ABI. Some callers cannot allocate device memory when
they run attention (an engine that sizes its memory once at start-up, code
inside a fixed pool); this entry point takes no workspace and uses the
library's fixed scratch array instead. Checked here:

- its results match the fp64 oracle and ca_chunk_attention's (workspace)
  results on the same inputs, on two calls in a row (the second call runs on
  the scratch the first one left behind);
- the device status word it reports: a call whose table count is invalid
  (flagged and clamped by the kernel) sets bit 0, and the next valid call
  reports 0, so each call clears the status it inherits;
- a launch shape the workspace path would split over several CTAs per item
  runs unsplit on the small scratch and still matches the oracle.

This file is collected last on purpose (test_zz_...): if it fails, a run that
stops at the first failure has already run every other test."""
import numpy as np
import pytest
import torch

import oracle
import serving_block_union_b200 as ca
import workloads
from parity_util import O_MAX_ABS, O_MEAN_ABS, LSE_ABS, compare

pytestmark = pytest.mark.gpu


def _inputs():
    wl = workloads.Workload("noalloc", B=2, H_q=16, H_kv=4, D=128, blk=128, C=512, L_max=4096,
                            chunk_start=(2048, 3584), seed=23, mask_kind="stripes",
                            n_stripes=3, noise=0.1)
    mask = workloads.make_mask(wl)
    Q, K, V = workloads.make_qkv(wl)
    T, c, _, _ = oracle.block_tables(mask, wl.group)
    return wl, Q, K, V, T, c


def _close(O_a, L_a, O_b, L_b):
    err = (O_a.float() - O_b.float()).abs()
    assert err.max().item() <= O_MAX_ABS and err.mean().item() <= O_MEAN_ABS
    la, lb = L_a.cpu().numpy(), L_b.cpu().numpy()
    assert np.array_equal(np.isneginf(la), np.isneginf(lb))
    fin = ~np.isneginf(la)
    assert np.abs(la[fin] - lb[fin]).max() <= LSE_ABS


def _outputs(B, H_q, C, D):
    O = torch.full((B, H_q, C, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    L = torch.full((B, H_q, C), float("nan"), dtype=torch.float32, device="cuda")
    return O, L


def test_noalloc_matches_oracle_and_workspace_entry_point_twice(cuda_ok):
    wl, Q, K, V, T, c = _inputs()
    O_or, L_or = oracle.attention(Q, K, V, wl.chunk_start, wl.blk, T, c)
    Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
    Td, cd = torch.from_numpy(T).cuda(), torch.from_numpy(c).cuda()
    O_ref, L_ref = ca.chunk_attention(Qd, Kd, Vd, Td, cd, wl.chunk_start)
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for _ in range(2):
        O, L = _outputs(wl.B, wl.H_q, wl.C, wl.D)
        ca.chunk_attention_noalloc(Qd, Kd, Vd, Td, cd, wl.chunk_start, O, L,
                                   device_status=status)
        torch.cuda.synchronize()
        _close(O, L, O_ref, L_ref)
        compare(O, L, O_or, L_or)
        assert int(status.item()) == 0


def test_noalloc_status_set_by_bad_count_then_cleared(cuda_ok):
    wl, Q, K, V, T, c = _inputs()
    Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    bad = c.copy()
    bad[0, 0] = wl.nKVmax + 3  # the kernel flags it and runs the item with no blocks
    O, L = _outputs(wl.B, wl.H_q, wl.C, wl.D)
    ca.chunk_attention_noalloc(Qd, Kd, Vd, torch.from_numpy(T).cuda(),
                               torch.from_numpy(bad).cuda(), wl.chunk_start, O, L,
                               device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & 1 == 1
    # the next valid call starts from a cleared status word and is correct
    O, L = _outputs(wl.B, wl.H_q, wl.C, wl.D)
    ca.chunk_attention_noalloc(Qd, Kd, Vd, torch.from_numpy(T).cuda(),
                               torch.from_numpy(c).cuda(), wl.chunk_start, O, L,
                               device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    O_or, L_or = oracle.attention(Q, K, V, wl.chunk_start, wl.blk, T, c)
    compare(O, L, O_or, L_or)


def test_noalloc_runs_a_split_shape_unsplit(cuda_ok):
    # one sequence, 400 KV blocks, 4 work items: the workspace path cuts each
    # item into 8 segments; the 4 KB scratch has no room for that
    B, H_q, H_kv, D, blk, C, L_max, cs = 1, 4, 1, 128, 64, 256, 64 * 400, (64 * 396,)
    rng = np.random.default_rng(41)
    mask = (rng.random((B, H_q, C // blk, L_max // blk)) < 0.3).astype(np.uint8)
    g = torch.Generator().manual_seed(41)
    Q = torch.randn(B, H_q, C, D, generator=g).to(torch.bfloat16)
    K = torch.randn(B, H_kv, L_max, D, generator=g).to(torch.bfloat16)
    V = torch.randn(B, H_kv, L_max, D, generator=g).to(torch.bfloat16)
    T, c, _, _ = oracle.block_tables(mask, H_q // H_kv)
    assert ca.workspace_bytes(B, H_q, H_kv, C, blk) > 4096  # the workspace path would split
    Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
    Td, cd = torch.from_numpy(T).cuda(), torch.from_numpy(c).cuda()
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    O, L = _outputs(B, H_q, C, D)
    ca.chunk_attention_noalloc(Qd, Kd, Vd, Td, cd, cs, O, L, device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    O_or, L_or = oracle.attention(Q, K, V, cs, blk, T, c)
    compare(O, L, O_or, L_or)
    O_ws, L_ws = ca.chunk_attention(Qd, Kd, Vd, Td, cd, cs)
    torch.cuda.synchronize()
    _close(O, L, O_ws, L_ws)
