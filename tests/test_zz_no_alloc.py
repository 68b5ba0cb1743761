"""The allocation-free attention entry point (ca_chunk_attention_noalloc),
called through the C ABI: its results match ca_chunk_attention's on the same
inputs, on two calls in a row (the second call runs on the scratch the first
one left behind), and the device status it reports is clean.

This file is collected last on purpose (test_zz_...): if it fails, a run that
stops at the first failure has already run every other test."""
import numpy as np
import pytest
import torch

import oracle
import serving_block_union_b200 as ca
import workloads
from parity_util import O_MAX_ABS, O_MEAN_ABS, LSE_ABS

pytestmark = pytest.mark.gpu


def _inputs():
    wl = workloads.Workload("noalloc", B=2, H_q=16, H_kv=4, D=128, blk=128, C=512, L_max=4096,
                            chunk_start=(2048, 3584), seed=23, mask_kind="stripes",
                            n_stripes=3, noise=0.1)
    mask = workloads.make_mask(wl)
    Q, K, V = workloads.make_qkv(wl)
    T, c, _, _ = oracle.block_tables(mask, wl.group)
    dev = torch.device("cuda")
    return wl, Q.to(dev), K.to(dev), V.to(dev), torch.from_numpy(T).to(dev), torch.from_numpy(c).to(dev)


def _close(O_a, L_a, O_b, L_b):
    err = (O_a.float() - O_b.float()).abs()
    assert err.max().item() <= O_MAX_ABS and err.mean().item() <= O_MEAN_ABS
    la, lb = L_a.cpu().numpy(), L_b.cpu().numpy()
    assert np.array_equal(np.isneginf(la), np.isneginf(lb))
    fin = ~np.isneginf(la)
    assert np.abs(la[fin] - lb[fin]).max() <= LSE_ABS


def test_noalloc_matches_workspace_entry_point_twice(cuda_ok):
    wl, Q, K, V, T, c = _inputs()
    O_ref, L_ref = ca.chunk_attention(Q, K, V, T, c, wl.chunk_start)
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for _ in range(2):
        O = torch.full_like(Q, float("nan"))
        L = torch.full((wl.B, wl.H_q, wl.C), float("nan"), dtype=torch.float32, device="cuda")
        ca.chunk_attention_noalloc(Q, K, V, T, c, wl.chunk_start, O, L, device_status=status)
        torch.cuda.synchronize()
        _close(O, L, O_ref, L_ref)
        assert int(status.item()) == 0
