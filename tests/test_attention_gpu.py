"""Zero-copy paged chunk attention on the GPU (tcgen05 kernel) vs the fp64
CPU oracle, element by element: full comparison on small shapes (every
supported D / blk / G, ragged chunk lengths, unaligned chunk starts, several
sequences), sampled rows at the full workload sizes with the launch
configuration the benchmark times, and the edge cases (empty tables, blocks
wholly in the future, NaN poison outside the visible keys, invalid tables
reported through the device status word)."""
import math

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


def _small_case(B, H_q, H_kv, D, blk, C, L_max, cs, p, seed):
    nQ = -(-C // blk)
    nK = L_max // blk
    rng = np.random.default_rng(seed)
    mask = (rng.random((B, H_q, nQ, nK)) < p).astype(np.uint8)
    Q = _rand((B, H_q, C, D), seed + 1)
    K = _rand((B, H_kv, L_max, D), seed + 2) + _rand((B, H_kv, nK, 1, D), seed + 3).repeat_interleave(
        blk, dim=3).reshape(B, H_kv, L_max, D) * 1.4
    K = K.to(torch.bfloat16)
    V = _rand((B, H_kv, L_max, D), seed + 4)
    return mask, Q, K, V


def _run_gpu(Q, K, V, T, c, cs, scale=None, dense=False, blk=None):
    Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
    if dense:
        O, L = ca.dense_chunk_attention(Qd, Kd, Vd, cs, blk, scale=scale)
    else:
        O, L = ca.chunk_attention(Qd, Kd, Vd, torch.from_numpy(T).cuda(),
                                  torch.from_numpy(c).cuda(), cs, scale=scale)
    torch.cuda.synchronize()
    return O, L


SMALL = [
    # B, H_q, H_kv, D, blk, C, L_max, chunk_start
    (1, 4, 1, 64, 64, 256, 1024, (768,)),
    (2, 8, 2, 128, 128, 384, 1152, (256, 640)),
    (1, 32, 8, 128, 128, 512, 2048, (1536,)),
    (2, 8, 8, 64, 128, 256, 768, (512, 128)),          # G = 1
    (1, 16, 8, 128, 64, 192, 512, (256,)),             # G = 2
    (1, 16, 2, 64, 64, 128, 384, (192,)),              # G = 8
    (1, 16, 1, 128, 128, 256, 512, (128,)),            # G = 16
    (2, 8, 2, 128, 128, 200, 640, (128, 0)),           # ragged chunk length
    (2, 4, 1, 64, 64, 150, 512, (100, 37)),            # unaligned chunk starts
    (1, 8, 2, 128, 64, 96, 64 * 6, (0,)),              # first chunk, no cache
]


@pytest.mark.parametrize("case", SMALL)
@pytest.mark.parametrize("p", [0.15, 1.0])
def test_small_shapes_full_compare(cuda_ok, case, p):
    B, H_q, H_kv, D, blk, C, L_max, cs = case
    mask, Q, K, V = _small_case(B, H_q, H_kv, D, blk, C, L_max, cs, p, seed=sum(case[:7]))
    T, c, _, _ = oracle.block_tables(mask, H_q // H_kv)
    O, L = _run_gpu(Q, K, V, T, c, cs)
    O_ref, L_ref = oracle.attention(Q, K, V, cs, blk, T, c)
    compare(O, L, O_ref, L_ref)


@pytest.mark.parametrize("case", SMALL[:4] + SMALL[7:])
def test_small_shapes_dense_full_compare(cuda_ok, case):
    B, H_q, H_kv, D, blk, C, L_max, cs = case
    _, Q, K, V = _small_case(B, H_q, H_kv, D, blk, C, L_max, cs, 0.0, seed=7 + sum(case[:7]))
    O, L = _run_gpu(Q, K, V, None, None, cs, dense=True, blk=blk)
    O_ref, L_ref = oracle.attention(Q, K, V, cs, blk)
    compare(O, L, O_ref, L_ref)


def test_explicit_scale(cuda_ok):
    B, H_q, H_kv, D, blk, C, L_max, cs = SMALL[1]
    mask, Q, K, V = _small_case(B, H_q, H_kv, D, blk, C, L_max, cs, 0.3, seed=3)
    T, c, _, _ = oracle.block_tables(mask, H_q // H_kv)
    O, L = _run_gpu(Q, K, V, T, c, cs, scale=0.05)
    O_ref, L_ref = oracle.attention(Q, K, V, cs, blk, T, c, scale=0.05)
    compare(O, L, O_ref, L_ref)


def test_max_batch(cuda_ok):
    B, H_q, H_kv, D, blk, C, L_max = 128, 4, 1, 64, 64, 64, 256
    cs = tuple(int(x) for x in np.random.default_rng(1).integers(0, 3, size=B) * 64)
    mask, Q, K, V = _small_case(B, H_q, H_kv, D, blk, C, L_max, cs, 0.5, seed=11)
    T, c, _, _ = oracle.block_tables(mask, 4)
    O, L = _run_gpu(Q, K, V, T, c, cs)
    O_ref, L_ref = oracle.attention(Q, K, V, cs, blk, T, c)
    compare(O, L, O_ref, L_ref)


def test_tiny_workload_tables_from_gpu_builder(cuda_ok):
    """The end-to-end path: GPU-built tables feed the GPU attention."""
    wl = workloads.tiny()
    mask = workloads.make_mask(wl)
    Q, K, V = workloads.make_qkv(wl)
    Td, cd, _, _ = ca.build_block_tables(torch.from_numpy(mask).cuda(), wl.group)
    O, L = ca.chunk_attention(Q.cuda(), K.cuda(), V.cuda(), Td, cd, wl.chunk_start)
    torch.cuda.synchronize()
    T, c, _, _ = oracle.block_tables(mask, wl.group)
    O_ref, L_ref = oracle.attention(Q, K, V, wl.chunk_start, wl.blk, T, c)
    compare(O, L, O_ref, L_ref)


# ------------------------------------------------------- split of the last wave

SPLIT = [
    # B, H_q, H_kv, D, blk, C, L_max, chunk_start, density: few items over
    # long caches, so the launch cuts every item into segments merged through
    # the workspace (each segment at least 24 table entries long)
    (1, 4, 1, 128, 64, 256, 64 * 400, (64 * 396,), 0.3),      # 4 items -> 8 segments each
    (2, 8, 2, 64, 128, 384, 128 * 300, (128 * 292, 128 * 292), 0.3),  # 24 items -> 6 each
    (1, 32, 8, 128, 128, 128, 128 * 380, (128 * 379,), 0.6),  # G = 4, 16 items -> 8 each
]

# entries a split item's segments must each walk, else the kernel keeps the
# item whole (the library's kMinSegEntries)
MIN_SEG_ENTRIES = 24


def _split_layout(n_items, n_sms):
    """(n_first, split, byte offset of the partial-LSE slots) of a launch: the
    full waves stay whole, the split makes the remaining segment waves
    shortest (the library's plan for one cache length)."""
    n_first = (n_items // n_sms) * n_sms
    n_rest = n_items - n_first
    best, best_frac = 1, 1.0
    for s in range(2, 9):
        frac = -(-n_rest * s // n_sms) / s
        if frac < best_frac:
            best, best_frac = s, frac
    return n_first, best, 256 + -(-4 * n_rest // 256) * 256


def _run_split_case(B, H_q, H_kv, D, blk, C, L_max, cs, mask, Q, K, V):
    """Runs the case on a full workspace whose partial-LSE slots start as NaN;
    returns O, LSE, the tables, and for every split item (rest item order) the
    segments that wrote their slots."""
    T, c, _, _ = oracle.block_tables(mask, H_q // H_kv)
    Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
    Td, cd = torch.from_numpy(T).cuda(), torch.from_numpy(c).cuda()
    ws = ca.new_workspace(B, H_q, H_kv, C, blk)
    G = H_q // H_kv
    n_pairs = (-(-C // (128 // G)) + 1) // 2
    items = B * H_kv * n_pairs
    n_first, split, lse_off = _split_layout(items, torch.cuda.get_device_properties(0).multi_processor_count)
    assert n_first == 0 and split > 1  # every item is a split item
    n_slot = items * split * 256
    ws[lse_off:lse_off + 4 * n_slot] = 255  # NaN in every partial LSE slot
    O, L = ca.chunk_attention(Qd, Kd, Vd, Td, cd, cs, workspace=ws)
    assert ca.read_device_status(ws) == ca.CA_OK
    # every merge counter (one uint32 per split item, after the 256-byte
    # header) is back at zero, ready for the next call
    assert int(ws[256:256 + 4 * items].count_nonzero()) == 0
    slots = ws[lse_off:lse_off + 4 * n_slot].view(torch.float32).view(items, split, 256)
    wrote = ~torch.isnan(slots).all(dim=2)  # [item, segment]
    return O, L, T, c, wrote.cpu().numpy(), ws, (Qd, Kd, Vd, Td, cd)


@pytest.mark.parametrize("case", SPLIT)
def test_split_last_wave_full_compare(cuda_ok, case):
    B, H_q, H_kv, D, blk, C, L_max, cs, p = case
    mask, Q, K, V = _small_case(B, H_q, H_kv, D, blk, C, L_max, cs, p, seed=sum(case[:7]))
    O, L, T, c, wrote, ws, dev = _run_split_case(B, H_q, H_kv, D, blk, C, L_max, cs, mask, Q, K, V)
    assert wrote.all()  # every segment of every item ran and wrote its partial
    O_ref, L_ref = oracle.attention(Q, K, V, cs, blk, T, c)
    compare(O, L, O_ref, L_ref)
    Qd, Kd, Vd, Td, cd = dev
    # the same call on a minimal workspace runs unsplit: same result within rounding
    ws_min = torch.zeros(256, dtype=torch.uint8, device="cuda")
    O1, L1 = ca.chunk_attention(Qd, Kd, Vd, Td, cd, cs, workspace=ws_min)
    compare(O1, L1, O_ref, L_ref)
    # reusing the workspace gives the identical result
    O2, L2 = ca.chunk_attention(Qd, Kd, Vd, Td, cd, cs, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(O, O2) and torch.equal(L, L2)


def test_split_only_long_items(cuda_ok):
    """Groups 0-3 select most of a 380-block cache, groups 4-7 about a third:
    the long groups' items run as 8 segments merged in the kernel, the short
    ones (fewer than 24 entries per segment) stay whole on their first
    segment's CTA while the other segments leave at once; all rows match the
    oracle and no merge counter is left set."""
    B, H_q, H_kv, D, blk, C, L_max, cs = 1, 32, 8, 128, 128, 128, 128 * 380, (128 * 379,)
    mask, Q, K, V = _small_case(B, H_q, H_kv, D, blk, C, L_max, cs, 0.6, seed=77)
    thin = np.random.default_rng(78).random(mask[:, 16:].shape) < 0.15
    mask[:, 16:] &= thin.astype(np.uint8)  # heads 16-31 (groups 4-7): density 0.09
    O, L, T, c, wrote, ws, _ = _run_split_case(B, H_q, H_kv, D, blk, C, L_max, cs, mask, Q, K, V)
    split = wrote.shape[1]
    n_pairs = wrote.shape[0] // H_kv
    for item in range(wrote.shape[0]):
        g = item // n_pairs  # one sequence: items run group by group
        # every item walks its group's whole table (the cache ends at the chunk)
        if c[0, g] >= MIN_SEG_ENTRIES * split:
            assert wrote[item].all(), (item, int(c[0, g]))
        else:
            assert not wrote[item].any(), (item, int(c[0, g]))
    assert c[0, :4].min() >= MIN_SEG_ENTRIES * split and c[0, 4:].max() < MIN_SEG_ENTRIES * split
    O_ref, L_ref = oracle.attention(Q, K, V, cs, blk, T, c)
    compare(O, L, O_ref, L_ref)


def test_split_dense_full_compare(cuda_ok):
    B, H_q, H_kv, D, blk, C, L_max, cs, _ = SPLIT[0]
    _, Q, K, V = _small_case(B, H_q, H_kv, D, blk, C, L_max, cs, 0.0, seed=31)
    O, L = _run_gpu(Q, K, V, None, None, cs, dense=True, blk=blk)
    O_ref, L_ref = oracle.attention(Q, K, V, cs, blk)
    compare(O, L, O_ref, L_ref)


# ------------------------------------------------------------------ full sizes

FULL = ["llama8b_32k", "llama8b_128k_d2", "llama8b_128k_d5", "llama8b_128k_d10",
        "llama8b_128k_d20", "llama8b_128k_noise", "batched", "full_prefill_c0",
        "full_prefill_c1", "full_prefill_c31", "full_prefill_c63", "qwen3_30b_128k_d10"]


def _poison_unselected(wl, K, V, T, c):
    """NaN in every cache block a group did not select and past kv_len."""
    workloads.poison_beyond_kv_len(wl, K, V)
    for b in range(wl.B):
        for g in range(wl.H_kv):
            sel = np.zeros(wl.nKVmax, bool)
            sel[T[b, g, :c[b, g]]] = True
            for j in np.nonzero(~sel)[0]:
                K[b, g, j * wl.blk:(j + 1) * wl.blk] = float("nan")
                V[b, g, j * wl.blk:(j + 1) * wl.blk] = float("nan")


@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled_rows(cuda_ok, name):
    wl = workloads.by_name(name)
    mask = workloads.make_mask(wl)
    Q, K, V = workloads.make_qkv(wl)
    T, c, _, _ = oracle.block_tables(mask, wl.group)
    Kp, Vp = K.clone(), V.clone()
    _poison_unselected(wl, Kp, Vp, T, c)
    Td, cd, _, _ = ca.build_block_tables(torch.from_numpy(mask).cuda(), wl.group)
    ws = ca.new_workspace(wl.B, wl.H_q, wl.H_kv, wl.C, wl.blk)
    O, L = ca.chunk_attention(Q.cuda(), Kp.cuda(), Vp.cuda(), Td, cd, wl.chunk_start,
                              workspace=ws)
    assert ca.read_device_status(ws) == ca.CA_OK
    np.testing.assert_array_equal(Td.cpu().numpy(), T)
    rows = sample_rows(wl, n_random=512)
    O_ref, L_ref = oracle.attention(Q, K, V, wl.chunk_start, wl.blk, T, c, rows=rows)
    compare(O, L, O_ref, L_ref, rows=rows)
    # every output row is finite: no poisoned (unselected / future) memory was read
    assert torch.isfinite(O.float()).all()


def test_long_context_1m_sampled_rows(cuda_ok):
    """1M-token context (8192 KV blocks, 2% per-head density): GPU tables
    bit-exact; the dense path on sampled rows; then, with NaN in every
    unselected block, the table path and the paged (kv_indptr / kv_indices)
    path on sampled rows, the poison never reaching O."""
    wl = workloads.by_name("llama8b_1m_d2")
    mask = workloads.make_mask(wl)
    Q, K, V = workloads.make_qkv(wl)
    T, c, _, _ = oracle.block_tables(mask, wl.group)
    maskd = torch.from_numpy(mask).cuda()
    Td, cd, _, _ = ca.build_block_tables(maskd, wl.group)
    np.testing.assert_array_equal(Td.cpu().numpy(), T)
    np.testing.assert_array_equal(cd.cpu().numpy(), c)
    Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
    ws = ca.new_workspace(wl.B, wl.H_q, wl.H_kv, wl.C, wl.blk)
    # dense: every block of the 1M cache, a few rows per group
    Od, Ld = ca.dense_chunk_attention(Qd, Kd, Vd, wl.chunk_start, wl.blk, workspace=ws)
    assert ca.read_device_status(ws) == ca.CA_OK
    rng = np.random.default_rng(9)
    rows_d = np.unique(np.concatenate([
        [(g * wl.group * wl.C) + r for g in range(wl.H_kv) for r in (0, wl.C - 1)],
        rng.integers(0, wl.B * wl.H_q * wl.C, size=16)]).astype(np.int64))
    Od_ref, Ld_ref = oracle.attention(Q, K, V, wl.chunk_start, wl.blk, rows=rows_d)
    compare(Od, Ld, Od_ref, Ld_ref, rows=rows_d)
    # poison every block no group selected
    sel = torch.zeros((wl.B, wl.H_kv, wl.nKVmax), dtype=torch.bool)
    for b in range(wl.B):
        for g in range(wl.H_kv):
            sel[b, g, torch.from_numpy(T[b, g, :c[b, g]].astype(np.int64))] = True
    shape5 = (wl.B, wl.H_kv, wl.nKVmax, wl.blk, wl.D)
    Kd.view(shape5)[~sel.cuda()] = float("nan")
    Vd.view(shape5)[~sel.cuda()] = float("nan")
    rows = sample_rows(wl, n_random=256)
    O_ref, L_ref = oracle.attention(Q, K, V, wl.chunk_start, wl.blk, T, c, rows=rows)
    O, L = ca.chunk_attention(Qd, Kd, Vd, Td, cd, wl.chunk_start, workspace=ws)
    assert ca.read_device_status(ws) == ca.CA_OK
    compare(O, L, O_ref, L_ref, rows=rows)
    assert torch.isfinite(O.float()).all()
    ip, ix, _, _ = ca.build_kv_pages(maskd, wl.group)
    Op, Lp = ca.paged_chunk_attention(Qd, Kd, Vd, ip, ix, wl.chunk_start, wl.blk, workspace=ws)
    assert ca.read_device_status(ws) == ca.CA_OK
    compare(Op, Lp, O_ref, L_ref, rows=rows)
    assert torch.isfinite(Op.float()).all()


@pytest.mark.parametrize("name", ["llama8b_32k", "llama8b_128k_d10", "batched"])
def test_full_size_dense_sampled_rows(cuda_ok, name):
    wl = workloads.by_name(name)
    Q, K, V = workloads.make_qkv(wl)
    Kp, Vp = K.clone(), V.clone()
    workloads.poison_beyond_kv_len(wl, Kp, Vp)
    O, L = ca.dense_chunk_attention(Q.cuda(), Kp.cuda(), Vp.cuda(), wl.chunk_start, wl.blk)
    torch.cuda.synchronize()
    rng = np.random.default_rng(3)
    rows = np.unique(np.concatenate([
        sample_rows(wl, n_random=0)[:: max(1, wl.blk // 8)],
        rng.integers(0, wl.B * wl.H_q * wl.C, size=64)]).astype(np.int64))
    O_ref, L_ref = oracle.attention(Q, K, V, wl.chunk_start, wl.blk, rows=rows)
    compare(O, L, O_ref, L_ref, rows=rows)
    assert torch.isfinite(O.float()).all()


# ------------------------------------------------------------------ edge cases

def test_empty_and_future_only_tables(cuda_ok):
    B, H_q, H_kv, D, blk, C, L_max, cs = 1, 8, 2, 128, 128, 256, 1024, (512,)
    _, Q, K, V = _small_case(B, H_q, H_kv, D, blk, C, L_max, cs, 0.0, seed=5)
    nK = L_max // blk
    T = np.full((B, H_kv, nK), -1, np.int32)
    c = np.zeros((B, H_kv), np.int32)
    T[0, 1, 0] = 5          # group 1: only the chunk's second block (positions 640..767)
    c[0, 1] = 1
    O, L = _run_gpu(Q, K, V, T, c, cs)
    O_ref, L_ref = oracle.attention(Q, K, V, cs, blk, T, c)
    compare(O, L, O_ref, L_ref)
    Oc = O.float().cpu()
    assert (Oc[0, :4] == 0).all() and torch.isneginf(L.cpu()[0, :4]).all()   # group 0 empty
    assert (Oc[0, 4:, :128] == 0).all() and torch.isneginf(L.cpu()[0, 4:, :128]).all()


def test_deterministic(cuda_ok):
    wl = workloads.llama8b_32k()
    mask = workloads.make_mask(wl)
    Q, K, V = (t.cuda() for t in workloads.make_qkv(wl))
    Td, cd, _, _ = ca.build_block_tables(torch.from_numpy(mask).cuda(), wl.group)
    O1, L1 = ca.chunk_attention(Q, K, V, Td, cd, wl.chunk_start)
    O2, L2 = ca.chunk_attention(Q, K, V, Td, cd, wl.chunk_start)
    torch.cuda.synchronize()
    assert torch.equal(O1, O2) and torch.equal(L1, L2)


@pytest.mark.parametrize("corrupt", ["count_too_big", "entry_out_of_range", "negative_entry",
                                     "not_ascending"])
def test_invalid_tables_are_reported_not_faulted(cuda_ok, corrupt):
    B, H_q, H_kv, D, blk, C, L_max, cs = 1, 8, 2, 128, 128, 256, 1024, (512,)
    mask, Q, K, V = _small_case(B, H_q, H_kv, D, blk, C, L_max, cs, 0.5, seed=8)
    T, c, _, _ = oracle.block_tables(mask, H_q // H_kv)
    T, c = T.copy(), c.copy()
    if corrupt == "count_too_big":
        c[0, 0] = L_max // blk + 3
    elif corrupt == "entry_out_of_range":
        T[0, 0, 0] = 10 ** 6
    elif corrupt == "negative_entry":
        T[0, 1, 0] = -7
    else:
        assert c[0, 0] >= 2
        T[0, 0, 0], T[0, 0, 1] = T[0, 0, 1], T[0, 0, 0]
    ws = ca.new_workspace(B, H_q, H_kv, C, blk)
    O, L = ca.chunk_attention(Q.cuda(), K.cuda(), V.cuda(), torch.from_numpy(T).cuda(),
                              torch.from_numpy(c).cuda(), cs, workspace=ws)
    assert ca.read_device_status(ws) == ca.CA_ERR_TABLE
    # the context is still usable: a clean call afterwards succeeds
    ws2 = ca.new_workspace(B, H_q, H_kv, C, blk)
    T0, c0, _, _ = oracle.block_tables(mask, H_q // H_kv)
    O, L = ca.chunk_attention(Q.cuda(), K.cuda(), V.cuda(), torch.from_numpy(T0).cuda(),
                              torch.from_numpy(c0).cuda(), cs, workspace=ws2)
    assert ca.read_device_status(ws2) == ca.CA_OK
    O_ref, L_ref = oracle.attention(Q, K, V, cs, blk, T0, c0)
    compare(O, L, O_ref, L_ref)


def test_python_binding_rejects_bad_tensors(cuda_ok):
    Q = torch.zeros(1, 4, 64, 64, dtype=torch.float16, device="cuda")
    K = torch.zeros(1, 1, 256, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(TypeError):
        ca.dense_chunk_attention(Q, K, K, [0], 64)
    with pytest.raises(ca.CAError):
        ca.dense_chunk_attention(Q.to(torch.bfloat16), K, K, [250], 64)  # cs + C > L_max


# ------------------------------------------------------- running-max rescales

@pytest.mark.parametrize("dense", [False, True])
def test_large_logit_jumps_between_blocks(cuda_ok, dense):
    """Logits that jump by tens of nats from block to block (up and down, a
    later block's maximum far above everything before it), so the online
    softmax has to raise its running maximum and rescale O in tensor memory
    many times, including jumps larger than its lazy threshold: every query
    has a unit component along one direction and each KV block's keys a
    block-constant component a_j along it, so the row's logits in block j sit
    near a_j / sqrt(D)."""
    B, H_q, H_kv, D, blk, C, L_max, cs = 1, 8, 2, 128, 128, 256, 1280, (1024,)
    nK = L_max // blk
    g = torch.Generator().manual_seed(77)
    Q = torch.randn(B, H_q, C, D, generator=g) * 0.3
    Q[..., 0] = 1.0
    K = torch.randn(B, H_kv, L_max, D, generator=g) * 0.3
    V = torch.randn(B, H_kv, L_max, D, generator=g)
    a = torch.tensor([0.0, 200.0, -300.0, 700.0, 100.0, 1000.0, -800.0, 500.0, 1100.0, 40.0])
    K[..., 0] = a.repeat_interleave(blk)[None, None, :]
    Q, K, V = Q.to(torch.bfloat16), K.to(torch.bfloat16), V.to(torch.bfloat16)
    mask = np.ones((B, H_q, C // blk, nK), np.uint8)
    T, c, _, _ = oracle.block_tables(mask, H_q // H_kv)
    O, L = _run_gpu(Q, K, V, T, c, cs, dense=dense, blk=blk)
    O_ref, L_ref = oracle.attention(Q, K, V, cs, blk, None if dense else T, None if dense else c)
    compare(O, L, O_ref, L_ref)
