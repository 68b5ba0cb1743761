"""FP8 (E4M3) cache path on the GPU vs the fp64 CPU oracle on the same
codes (decoded exactly, times the per-tensor descales).

Tolerance, from the arithmetic. Q.K^T of E4M3 codes is exact in each product
and accumulated in fp32 (error ~1e-6 relative on S). P is rounded to E4M3:
relative error at most 2^-4 for P >= 2^-6 (P is 2^(x + 4) with x at most 4.5
above the running reference, and the row's largest P is at least 2^4, so that
covers every key within 2^-10 of the reference), at most 2^-10 absolute below,
i.e. at most 2^-14 of the row's largest P, with independent signs. O is
normalised by the fp32 sum of the unrounded P (as the bf16 path is), so
O = sum_k w_k (1 + e_k) v_k with the exact weights w_k, and
|O - O_exact| <= 2^-4 * sum_k w_k |v_k| (+ 2^-9 |O| for the bf16 output).
For these inputs (V ~ N(0, 1), |v| averaging about 0.8 under the weights)
that is about 5e-2 per element in the worst case, with the rounding errors of
different keys independent and of either sign, so the mean error is an order
of magnitude lower: O max-abs 6e-2, mean-abs 6e-3. (Measured on sampled rows
of the 32K, 128K and batched workloads: max-abs at most 1.2e-2, mean-abs at
most 7.6e-4, the same as when O was normalised by the sum of the rounded P.)
The LSE uses the same fp32 sum and keeps the bf16 path's bound, 1e-3. A
quarter of the exponentials come from a polynomial on the FMA pipe with
relative error at most 1.02e-4, far below the E4M3 rounding of P.
"""
import numpy as np
import pytest
import torch

import oracle
import serving_block_union_b200 as ca
import workloads
from parity_util import compare, sample_rows

pytestmark = pytest.mark.gpu

O_MAX_FP8 = 6e-2
O_MEAN_FP8 = 6e-3
LSE_FP8 = 1e-3


def _quant(Q, K, V):
    (q8, qd), (k8, kd), (v8, vd) = (workloads.quantize_e4m3(t) for t in (Q, K, V))
    return q8, k8, v8, (qd, kd, vd)


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g)


SMALL = [
    # B, H_q, H_kv, blk, C, L_max, chunk_start
    (1, 4, 1, 128, 256, 1024, (768,)),
    (2, 8, 2, 64, 320, 1280, (448, 64)),
    (1, 32, 8, 128, 512, 2048, (1536,)),
    (2, 8, 8, 128, 200, 768, (512, 128)),     # G = 1, ragged chunk
    (1, 16, 2, 64, 128, 64 * 400, (64 * 390,)),  # G = 8, long cache: the last wave is split
]


@pytest.mark.parametrize("case", SMALL)
@pytest.mark.parametrize("dense", [False, True])
def test_small_shapes_full_compare(cuda_ok, case, dense):
    B, H_q, H_kv, blk, C, L_max, cs = case
    D = 128
    seed = sum(case[:6])
    Q, K, V = _rand((B, H_q, C, D), seed), _rand((B, H_kv, L_max, D), seed + 1), \
        _rand((B, H_kv, L_max, D), seed + 2)
    q8, k8, v8, ds = _quant(Q, K, V)
    T = c = None
    if not dense:
        rng = np.random.default_rng(seed)
        mask = (rng.random((B, H_q, -(-C // blk), L_max // blk)) < 0.3).astype(np.uint8)
        T, c, _, _ = oracle.block_tables(mask, H_q // H_kv)
    O, L = ca.chunk_attention_fp8(q8.cuda(), k8.cuda(), v8.cuda(), ds, cs, blk,
                                  None if dense else torch.from_numpy(T).cuda(),
                                  None if dense else torch.from_numpy(c).cuda())
    torch.cuda.synchronize()
    O_ref, L_ref = oracle.attention_e4m3(q8, k8, v8, ds, cs, blk, T, c)
    compare(O, L, O_ref, L_ref, o_max=O_MAX_FP8, o_mean=O_MEAN_FP8, lse_abs=LSE_FP8)


@pytest.mark.parametrize("name", ["llama8b_128k_d10", "llama8b_32k"])
def test_full_size_sampled_rows(cuda_ok, name):
    wl = workloads.by_name(name)
    mask = workloads.make_mask(wl)
    Q, K, V = workloads.make_qkv(wl)
    q8, k8, v8, ds = _quant(Q, K, V)
    Td, cd, _, _ = ca.build_block_tables(torch.from_numpy(mask).cuda(), wl.group)
    ws = ca.new_workspace(wl.B, wl.H_q, wl.H_kv, wl.C, wl.blk)
    O, L = ca.chunk_attention_fp8(q8.cuda(), k8.cuda(), v8.cuda(), ds, wl.chunk_start, wl.blk,
                                  Td, cd, workspace=ws)
    assert ca.read_device_status(ws) == ca.CA_OK
    T, c, _, _ = oracle.block_tables(mask, wl.group)
    rows = sample_rows(wl, n_random=256)
    O_ref, L_ref = oracle.attention_e4m3(q8, k8, v8, ds, wl.chunk_start, wl.blk, T, c, rows=rows)
    compare(O, L, O_ref, L_ref, rows=rows, o_max=O_MAX_FP8, o_mean=O_MEAN_FP8, lse_abs=LSE_FP8)


def test_dominant_key_is_exact(cuda_ok):
    """One key far above the rest in every row: its P is 2^4, exact in E4M3,
    and the other keys carry about 1e-4 of the weight, so O is that key's
    value row (up to bf16)."""
    B, H_q, H_kv, D, blk, C, L_max, cs = 1, 4, 1, 128, 128, 128, 512, (384,)
    Q = torch.ones(B, H_q, C, D) * 0.5
    K = _rand((B, H_kv, L_max, D), 4) * 0.05
    K[0, 0, 7] = 3.0          # key 7: logit ~ 0.5 * 3 * 128 / sqrt(128) = 17 above the rest
    V = _rand((B, H_kv, L_max, D), 5)
    q8, k8, v8, ds = _quant(Q, K, V)
    O, L = ca.chunk_attention_fp8(q8.cuda(), k8.cuda(), v8.cuda(), ds, cs, blk)
    torch.cuda.synchronize()
    O_ref, L_ref = oracle.attention_e4m3(q8, k8, v8, ds, cs, blk)
    v7 = float(ds[2]) * np.array([oracle.e4m3_decode(int(x)) for x in v8[0, 0, 7]])
    # the other 511 keys keep about 1e-4 of the weight
    np.testing.assert_allclose(O_ref[0, :, :], np.broadcast_to(v7, O_ref.shape[1:]), atol=1e-3)
    compare(O, L, O_ref, L_ref, o_max=1e-2, o_mean=2e-3, lse_abs=LSE_FP8)


def test_fp8_rejects_bad_arguments(cuda_ok):
    Q8 = torch.zeros(1, 4, 128, 64, dtype=torch.uint8, device="cuda")
    K8 = torch.zeros(1, 1, 512, 64, dtype=torch.uint8, device="cuda")
    with pytest.raises(ca.CAError):      # D = 64 is not compiled for FP8
        ca.chunk_attention_fp8(Q8, K8, K8, (1.0, 1.0, 1.0), [256], 128)
    Q8 = torch.zeros(1, 4, 128, 128, dtype=torch.uint8, device="cuda")
    K8 = torch.zeros(1, 1, 512, 128, dtype=torch.uint8, device="cuda")
    with pytest.raises(ca.CAError):
        ca.chunk_attention_fp8(Q8, K8, K8, (1.0, 0.0, 1.0), [256], 128)
