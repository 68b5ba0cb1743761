"""The hot path under CUDA graph capture: table build + attention (with the
last-wave split) captured once and replayed gives bit-identical results to
the eager calls, and the oracle's; the split's merge counters are back at
zero after every replay."""
import numpy as np
import pytest
import torch

import oracle
import serving_block_union_b200 as ca
import workloads
from parity_util import compare

pytestmark = pytest.mark.gpu


def test_captured_step_matches_eager_and_oracle(cuda_ok):
    # 8 items over a 400-block cache, tables ~99% full: every item is split
    wl = workloads.Workload("graph", B=1, H_q=8, H_kv=2, D=128, blk=128, C=256,
                            L_max=128 * 400, chunk_start=(128 * 396,), seed=12,
                            mask_kind="bernoulli", density=0.5)
    mask = torch.from_numpy(workloads.make_mask(wl)).cuda()
    Q, K, V = (t.cuda() for t in workloads.make_qkv(wl))
    ws = ca.new_workspace(wl.B, wl.H_q, wl.H_kv, wl.C, wl.blk)
    T = torch.empty((wl.B, wl.H_kv, wl.nKVmax), dtype=torch.int32, device="cuda")
    c = torch.empty((wl.B, wl.H_kv), dtype=torch.int32, device="cuda")
    O = torch.empty_like(Q)
    L = torch.empty((wl.B, wl.H_q, wl.C), dtype=torch.float32, device="cuda")

    def step():
        ca.build_block_tables(mask, wl.group, tables=T, counts=c)
        ca.chunk_attention(Q, K, V, T, c, wl.chunk_start, O=O, LSE=L, workspace=ws)

    step()  # eager first call: one-time host set-up (attributes, SM count)
    torch.cuda.synchronize()
    O_eager, L_eager = O.clone(), L.clone()
    O.zero_()
    L.zero_()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            step()
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(3):
        O.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(O, O_eager) and torch.equal(L, L_eager)
        assert int(ws[256:512].count_nonzero()) == 0
    assert ca.read_device_status(ws) == ca.CA_OK
    T_ref, c_ref, _, _ = oracle.block_tables(mask.cpu().numpy(), wl.group)
    O_ref, L_ref = oracle.attention(Q.cpu(), K.cpu(), V.cpu(), wl.chunk_start, wl.blk, T_ref,
                                    c_ref)
    compare(O, L, O_ref, L_ref)
