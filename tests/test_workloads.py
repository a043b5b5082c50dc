"""Structure of the seeded synthetic workloads (CPU only)."""
import numpy as np

import workloads as W


def test_values_are_seeded_and_reproducible():
    a = W.normal_bits((3, 5, 7), "bf16", 9, "x", 1)
    b = W.normal_bits((3, 5, 7), "bf16", 9, "x", 1)
    c = W.normal_bits((3, 5, 7), "bf16", 9, "x", 2)
    assert np.array_equal(a, b) and not np.array_equal(a, c)


def test_normal_statistics():
    x = W.normal_bits((1 << 20,), "fp16", 1, "stat")
    v = x.view(np.float16).astype(np.float64)
    assert abs(v.mean()) < 0.01 and abs(v.std() - 1.0) < 0.01
    y = W.normal_bits((1 << 20,), "bf16", 1, "stat", std=0.5)
    vy = (y.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert abs(vy.std() - 0.5) < 0.005


def test_bf16_rounding_is_nearest_even():
    import torch
    x = np.random.default_rng(3).standard_normal(100000).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(W.f32_to_bf16_bits(x), ref)


def test_paged_gqa_structure():
    c = W.paged_gqa()
    assert c.B == 64 and c.page_size == 16 and c.max_pages == 513
    L = c.seq_lens
    assert L.min() >= 128 and L.max() <= 8192
    sh = c.shared_requests
    assert len(sh) == 16 and np.all(L[sh] >= 1024)
    bt = c.block_table
    # shared prefix: the same 64 physical pages, in the same order
    for b in sh:
        assert np.array_equal(bt[b, :64], bt[sh[0], :64])
    used = []
    for b in range(c.B):
        n = -(-(int(L[b]) + c.T_new) // 16)
        assert np.all(bt[b, :n] >= 0) and np.all(bt[b, n:] == -1)
        used.append(bt[b, 64:n] if b in sh else bt[b, :n])
    used = np.concatenate(used + [bt[sh[0], :64]])
    # every pool page used exactly once (private pages never alias)
    assert np.array_equal(np.sort(used), np.arange(c.num_pages))
    # appended row falls in a private page for the sharers
    assert np.all(L[sh] // 16 >= 64)


def test_spec_verify_structure():
    for g in (2, 4, 8):
        for hkv in (8, 1):
            c = W.spec_verify(g, hkv)
            assert c.B == 32 and c.T_new == g and c.rows == 32 // hkv * g
            assert c.seq_lens.min() >= 8192 and c.seq_lens.max() <= 32768
            assert c.max_pages == -(-(32768 + g) // 16)


def test_kv_bytes_accounting():
    c = W.gqa_32layer()
    # one layer: 16 requests x 4097 positions x K and V x 8 heads x 128 x 2 bytes
    assert c.kv_read_bytes() == 16 * 4097 * 2 * 8 * 128 * 2
    p = W.paged_gqa()
    assert p.kv_read_bytes(True) == p.kv_read_bytes(False) - 15 * 1024 * 2 * 8 * 128 * 2
