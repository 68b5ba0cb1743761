"""Block-Union table construction on the GPU vs the CPU oracle: bit-exact
tables (padding included), counts and CSR on every workload and on edge
cases (odd widths that take the scalar path, misaligned masks, empty and full
masks, nonzero values other than 1, every supported group size)."""
import numpy as np
import pytest
import torch

import oracle
import serving_block_union_b200 as ca
import workloads

pytestmark = pytest.mark.gpu

WORKLOADS = ["tiny", "llama8b_32k", "llama8b_128k_d2", "llama8b_128k_d5", "llama8b_128k_d10",
             "llama8b_128k_d20", "llama8b_128k_noise", "batched", "full_prefill_c0",
             "full_prefill_c1", "full_prefill_c31", "full_prefill_c63", "qwen3_30b_128k_d10"]


def _check(mask_np, group, mask_dev=None):
    T_ref, c_ref, ip_ref, ix_ref = oracle.block_tables(mask_np, group)
    m = mask_dev if mask_dev is not None else torch.from_numpy(mask_np).cuda()
    T, c, ip, ix = ca.build_block_tables(m, group, csr=True)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(T.cpu().numpy(), T_ref)
    np.testing.assert_array_equal(c.cpu().numpy(), c_ref)
    np.testing.assert_array_equal(ip.cpu().numpy(), ip_ref)
    n = int(ip_ref[-1])
    np.testing.assert_array_equal(ix.cpu().numpy()[:n], ix_ref)


@pytest.mark.parametrize("name", WORKLOADS)
def test_tables_bit_exact_on_workloads(cuda_ok, name):
    wl = workloads.by_name(name)
    _check(workloads.make_mask(wl), wl.group)


@pytest.mark.parametrize("shape", [
    # B, H_q, nQ, nKVmax, G
    (1, 4, 4, 16, 4), (2, 8, 3, 37, 2), (3, 6, 5, 50, 3), (1, 8, 1, 9, 8),
    (2, 4, 2, 7, 1), (1, 32, 16, 16400, 4), (1, 2, 64, 3000, 2), (5, 16, 2, 1, 16),
    # many (b, g): one CTA each instead of a cluster, the bulk-copy form
    # (one piece; three pieces, a batch of 64 sequences at 128K; 2, 3, 4 and
    # 13 pieces through the two-stage ring, with 1, 2 and 4 units per thread);
    # an odd width (the register form); a KV range too long for the bulk form
    # and the cluster's shared memory
    (24, 32, 4, 160, 4), (64, 32, 16, 1040, 4), (40, 8, 2, 8192, 8), (40, 4, 1, 16384, 4),
    (45, 8, 5, 4096, 4), (40, 1, 37, 9600, 1), (40, 8, 3, 1000, 4), (1, 2, 1, 131088, 2),
])
@pytest.mark.parametrize("p", [0.0, 0.01, 0.3, 1.0])
def test_tables_random_shapes(cuda_ok, shape, p):
    B, H_q, nQ, nK, G = shape
    rng = np.random.default_rng(abs(hash((shape, p))) % 2**32)
    mask = (rng.random((B, H_q, nQ, nK)) < p).astype(np.uint8)
    mask[mask == 1] = rng.integers(1, 256, size=int(mask.sum()), dtype=np.uint8)
    _check(mask, G)


def test_tables_misaligned_mask_pointer(cuda_ok):
    rng = np.random.default_rng(5)
    B, H_q, nQ, nK, G = 2, 8, 4, 64, 4
    mask = (rng.random((B, H_q, nQ, nK)) < 0.05).astype(np.uint8)
    flat = torch.zeros(mask.size + 1, dtype=torch.uint8, device="cuda")
    view = flat[1:].view(B, H_q, nQ, nK)
    view.copy_(torch.from_numpy(mask))
    _check(mask, G, mask_dev=view)


def test_tables_bool_mask(cuda_ok):
    rng = np.random.default_rng(9)
    mask = rng.random((1, 8, 4, 48)) < 0.1
    T_ref, c_ref, _, _ = oracle.block_tables(mask.astype(np.uint8), 2)
    T, c, _, _ = ca.build_block_tables(torch.from_numpy(mask).cuda(), 2)
    np.testing.assert_array_equal(T.cpu().numpy(), T_ref)
    np.testing.assert_array_equal(c.cpu().numpy(), c_ref)


def test_tables_stream_ordering(cuda_ok):
    """Launch on a side stream; results visible after that stream syncs."""
    wl = workloads.llama8b_32k()
    mask = workloads.make_mask(wl)
    s = torch.cuda.Stream()
    m = torch.from_numpy(mask).cuda()
    torch.cuda.current_stream().synchronize()
    with torch.cuda.stream(s):
        T, c, _, _ = ca.build_block_tables(m, wl.group, stream=s)
    s.synchronize()
    T_ref, c_ref, _, _ = oracle.block_tables(mask, wl.group)
    np.testing.assert_array_equal(T.cpu().numpy(), T_ref)
    np.testing.assert_array_equal(c.cpu().numpy(), c_ref)



@pytest.mark.parametrize("name", WORKLOADS)
def test_bit_packed_mask_gives_the_same_tables(cuda_ok, name):
    """The bit-packed input (uint32 words) yields the byte mask's tables and
    CSR, bit for bit."""
    wl = workloads.by_name(name)
    mask = workloads.make_mask(wl)
    words = torch.from_numpy(workloads.pack_mask_bits(mask).view(np.int32)).cuda()
    T, c, ip, ix = ca.build_block_tables_bits(words, wl.nKVmax, wl.group, csr=True)
    T_ref, c_ref, ip_ref, ix_ref = oracle.block_tables(mask, wl.group)
    np.testing.assert_array_equal(T.cpu().numpy(), T_ref)
    np.testing.assert_array_equal(c.cpu().numpy(), c_ref)
    np.testing.assert_array_equal(ip.cpu().numpy(), ip_ref)
    n = int(ip_ref[-1])
    np.testing.assert_array_equal(ix.cpu().numpy()[:n], ix_ref[:n])


@pytest.mark.parametrize("shape", [(1, 4, 3, 33, 1), (2, 8, 5, 64, 4), (1, 16, 2, 1, 8),
                                   (3, 6, 7, 100, 2), (20, 16, 2, 100, 4), (64, 32, 16, 1040, 4),
                                   # bulk form over 4 and 2 pieces (rows a multiple
                                   # of four per piece); rows * words not a multiple
                                   # of four (the register form)
                                   (40, 16, 16, 4096, 16), (40, 1, 37, 9600, 1),
                                   (40, 8, 7, 96, 2), (1, 2, 1, 262200, 2)])
def test_bit_packed_random_masks(cuda_ok, shape):
    B, H_q, nQ, nK, G = shape
    rng = np.random.default_rng(sum(shape))
    mask = (rng.random((B, H_q, nQ, nK)) < 0.1).astype(np.uint8)
    words = workloads.pack_mask_bits(mask)
    # garbage in the bits past nKVmax must be ignored
    tail = (-nK) % 32
    if tail:
        words[..., -1] |= np.uint32(((1 << tail) - 1) << (32 - tail))
    T, c, _, _ = ca.build_block_tables_bits(torch.from_numpy(words.view(np.int32)).cuda(), nK, G)
    T_ref, c_ref, _, _ = oracle.block_tables(mask, G)
    np.testing.assert_array_equal(T.cpu().numpy(), T_ref)
    np.testing.assert_array_equal(c.cpu().numpy(), c_ref)
