"""Host-side checks of the seeded input recipe (no method arithmetic here)."""
import torch

import workloads


def test_configs_match_recipe():
    W = workloads.WORKLOADS
    assert (W["tiny"].batch, W["tiny"].prefix, W["tiny"].window, W["tiny"].seed) == (1, 64, 6, 0)
    assert (W["single_image"].layers, W["single_image"].prefix) == (36, 1024)
    assert (W["max_context"].layers, W["max_context"].prefix) == (36, 4096)
    assert W["max_context_w1"].window == 1 and W["max_context_w1"].seed == 2
    assert (W["ragged"].batch, W["ragged"].prefix) == (64, None)
    assert (W["long"].batch, W["long"].prefix, W["long"].k_seq_offset_std) == (8, 32768, 0.5)
    for wl in W.values():
        assert (wl.num_q_heads, wl.num_kv_heads, wl.head_dim) == (16, 2, 128)


def test_deterministic_and_bf16():
    a = workloads.generate(workloads.WORKLOADS["tiny"])
    b = workloads.generate(workloads.WORKLOADS["tiny"])
    la, lb = a.layers[0], b.layers[0]
    for x, y in [(la.q, lb.q), (la.k_cache, lb.k_cache), (la.v_new, lb.v_new)]:
        assert x.dtype == torch.bfloat16 and torch.equal(x, y)
    assert la.q.shape == (1, 6, 16, 128)
    assert la.k_cache.shape == (1, 2, a.max_seq, 128) and a.max_seq >= 70


def test_ragged_lengths():
    wi = workloads.generate(workloads.WORKLOADS["ragged"], layers=0)
    P = wi.seq_lens
    assert P.shape == (64,) and P.dtype == torch.int32
    assert int(P.min()) >= 513 and int(P.max()) <= 4101
    assert wi.max_seq >= int(P.max()) + 6


def test_window1_shares_caches():
    a = workloads.generate(workloads.WORKLOADS["max_context"], layers=1)
    b = workloads.generate(workloads.WORKLOADS["max_context_w1"], layers=1)
    assert a.max_seq == b.max_seq
    assert torch.equal(a.layers[0].k_cache, b.layers[0].k_cache)
    assert torch.equal(a.layers[0].v_cache, b.layers[0].v_cache)


def test_outlier_channels():
    wl = workloads.WORKLOADS["single_image"]
    plain = workloads.dataclasses.replace(wl, k_outlier_frac=0.0)
    a = workloads.generate(wl, layers=1).layers[0].k_cache.float()
    # Same seed without outliers differs from the randperm draw, so compare scale:
    rms = a.pow(2).mean(dim=(0, 2)).sqrt()            # [Hkv, D]
    big = (rms > 4.0).sum().item()
    assert big == 3, rms
    assert plain.k_outlier_frac == 0.0


def test_algorithmic_bytes():
    # tiny: 2 (K,V) * 2 heads * 70 tokens * 128 * 2 B + Q and out 2 * 6 * 16 * 128 * 2 B
    assert workloads.algorithmic_bytes([64], 6) == 2 * 2 * 70 * 128 * 2 + 2 * 6 * 16 * 128 * 2
