"""Host-side logic without a GPU: the benchmark's work count against the
oracle's, and the benchmark's profile bookkeeping (the roofline traffic field
is taken only from a profile of the current kernel source)."""
import os

import numpy as np

import bench
import oracle
import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_bench_visible_pairs_matches_oracle():
    for wl in (workloads.tiny(),
               workloads.Workload("t", B=2, H_q=8, H_kv=2, D=64, blk=64, C=192, L_max=1024,
                                  chunk_start=(320, 64), seed=5, mask_kind="stripes",
                                  n_stripes=2, noise=0.1)):
        mask = workloads.make_mask(wl)
        T, c, _, _ = oracle.block_tables(mask, wl.group)
        ours = bench.visible_pairs(T, c, wl.chunk_start, wl.C, wl.blk, wl.group)
        ref = oracle.visible_pairs(wl.chunk_start, wl.B, wl.H_q, wl.H_kv, wl.C, wl.L_max, wl.blk,
                                   T, c)
        assert ours == ref
        nkv = [-(-(cs + wl.C) // wl.blk) for cs in wl.chunk_start]
        dense = bench.visible_pairs(T, c, wl.chunk_start, wl.C, wl.blk, wl.group, dense_nkv=nkv)
        assert dense == oracle.visible_pairs(wl.chunk_start, wl.B, wl.H_q, wl.H_kv, wl.C,
                                             wl.L_max, wl.blk)


def test_bench_tile_visible_pairs_matches_token_count():
    """Per-tile work count: the token-level expansion of the block mask, causal
    on top, counted pair by pair."""
    rng = np.random.default_rng(4)
    B, H_q, blk, C, L = 2, 3, 8, 40, 128
    cs = (56, 8)
    nQ, nK = -(-C // blk), L // blk
    mask = (rng.random((B, H_q, nQ, nK)) < 0.3).astype(np.uint8)
    tok = np.repeat(np.repeat(mask != 0, blk, axis=2)[:, :, :C], blk, axis=3)
    total = 0
    for b in range(B):
        causal = np.arange(L)[None, :] <= cs[b] + np.arange(C)[:, None]
        total += int((tok[b] & causal[None]).sum())
    assert bench.tile_visible_pairs(mask, cs, C, blk) == total


def test_bench_executed_pairs_brute_force():
    """Executed (whole-tile) work: every packed row of an item's two tiles
    against every key of each table block starting at or before the item's
    last position; never below the visible pairs; equal to them when nothing
    is causally cut (blocks wholly in the past, rows filling every tile)."""
    rng = np.random.default_rng(6)
    for G, C, cs in ((4, 128, (256, 64)), (8, 96, (128, 0)), (2, 256, (512, 384))):
        B, H_kv, blk, L = 2, 2, 64, 1024
        H_q = G * H_kv
        nQ, nK = -(-C // blk), L // blk
        mask = (rng.random((B, H_q, nQ, nK)) < 0.3).astype(np.uint8)
        T, c, _, _ = oracle.block_tables(mask, G)
        R = 128 // G
        brute = 0
        for b in range(B):
            for g in range(H_kv):
                for r0 in range(0, C, 2 * R):
                    last = cs[b] + min(r0 + 2 * R, C) - 1
                    for t in range(c[b, g]):
                        if T[b, g, t] * blk <= last:
                            brute += 2 * 128 * blk
        ex = bench.executed_pairs(T, c, cs, C, blk, G)
        assert ex == brute
        assert ex >= bench.visible_pairs(T, c, cs, C, blk, G)
    # past-only tables and full tiles: executed == visible
    B, H_kv, G, blk, C = 1, 1, 4, 128, 256
    T = np.array([[[0, 2, 5, -1, -1, -1, -1, -1]]], np.int32)
    c = np.array([[3]], np.int32)
    assert bench.executed_pairs(T, c, (768,), C, blk, G) == \
        bench.visible_pairs(T, c, (768,), C, blk, G) == 3 * blk * C * G


def test_pack_mask_bits_round_trip():
    """The bit-packed mask input: bit k of word w is block 32*w + k, any
    nonzero byte selects, bits past nKVmax stay clear (checked bit by bit
    with Python integers, independent of numpy's packing)."""
    rng = np.random.default_rng(9)
    for nK in (1, 31, 32, 33, 95):
        m = (rng.random((2, 2, 3, nK)) < 0.4).astype(np.uint8) * 3
        w = workloads.pack_mask_bits(m)
        assert w.dtype == np.uint32 and w.shape == (2, 2, 3, -(-nK // 32))
        for idx in np.ndindex(m.shape[:3]):
            value = sum(1 << j for j in range(nK) if m[idx + (j,)])
            words = [int(x) for x in w[idx]]
            assert sum(x << (32 * i) for i, x in enumerate(words)) == value


def test_profiled_traffic_needs_matching_kernel_hash(tmp_path, monkeypatch):
    """The roofline traffic field comes from a committed ncu summary only when
    that summary was captured from the current kernel code; comment-only edits
    of the kernel keep the hash."""
    monkeypatch.setattr(bench, "PROFILES", str(tmp_path))
    h = bench.kernel_source_hash()
    (tmp_path / "chunk_attn_kernel_w.md").write_text(
        f"text\n```\ndram_bytes_per_launch: 1234\nsource_sha256_16: {h}\n```\n")
    assert bench.profiled_traffic("w") == 1234
    (tmp_path / "chunk_attn_kernel_w.md").write_text(
        "dram_bytes_per_launch: 1234\nsource_sha256_16: 0000000000000000\n")
    assert bench.profiled_traffic("w") is None
    assert bench.profiled_traffic("missing") is None
    # comments and whitespace do not change the hash
    src = tmp_path / "k.cu"
    src.write_text("int a; // one\n/* two */ int  b;\n")
    monkeypatch.setattr(bench, "KERNEL_SOURCES", [str(src)])
    h1 = bench.kernel_source_hash()
    src.write_text("int a;   // changed comment\nint b;\n")
    assert bench.kernel_source_hash() == h1
    src.write_text("int a; int c;\n")
    assert bench.kernel_source_hash() != h1


def _poly_constants():
    """The FMA-pipe exponential's coefficients, read from the kernel header
    (so the test checks the constants the kernel compiles)."""
    import re
    src = open(os.path.join(os.path.dirname(__file__), "..", "serving_block_union_b200", "csrc",
                            "sm100_ptx.cuh")).read()
    body = src[src.index("exp2_poly2(uint64_t x2)"):]
    body = body[:body.index("\n}\n")]
    vals = [float(v) for v in re.findall(r"f2_pack\(([0-9.]+)f, \1f\)", body)]
    # 1.5 * 2^23 (round shift), then c3, c2, c1, 1 in Horner order
    return vals


def test_fma_pipe_exp2_meets_its_stated_bound():
    """exp2_poly2 (FP8 softmax, every 4th pair): the same float32 steps as
    the device code; relative error at most 1.02e-4 against 2^x over the
    softmax's range, +0 at the -127 clamp, positive and finite above it."""
    vals = _poly_constants()
    assert vals[0] == 12582912.0
    c3, c2, c1, one = (np.float32(v) for v in vals[1:5])
    assert one == 1.0
    f32 = np.float32
    x = np.concatenate([np.linspace(-127, 8.5, 2_000_001), [-127.0, -126.5, -0.5, 0.5, 8.5]])
    x = np.maximum(x.astype(f32), f32(-127))
    t = (x + f32(12582912.0)).astype(f32)
    r = (t - f32(12582912.0)).astype(f32)
    f = (x - r).astype(f32)

    def fma(a, b, c):  # one rounding, as the device's fused multiply-add
        return (a.astype(np.float64) * np.float64(b) + np.float64(c)).astype(f32)

    p = fma(fma(fma(np.full_like(f, c3), f, c2), f, c1), f, one)
    bits = (t.view(np.uint32).astype(np.uint64) * 8388608 + p.view(np.uint32)) % (1 << 32)
    y = bits.astype(np.uint32).view(np.float32).astype(np.float64)
    assert y[x == -127].max() == 0.0
    ok = x > -126  # normal results
    rel = np.abs(y[ok] / np.exp2(x[ok].astype(np.float64)) - 1)
    assert rel.max() <= 1.02e-4
    assert np.all(np.isfinite(y)) and np.all(y >= 0)
