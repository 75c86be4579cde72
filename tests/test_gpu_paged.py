"""GPU parity of the paged KV cache (la_pbd_step_paged / la_pbd_attn_paged) against the fp64
oracle.

The pool is built from a contiguous cache by a seeded page permutation (pages of different
sequences interleaved, spare pages filled with NaN); after the step the pool is gathered back
to the contiguous layout and compared with the oracle's append bit for bit, and the output is
compared with the oracle on the logical cache. Table entries past each sequence's pages are
set to an invalid page index: they must never be read.
"""
import numpy as np
import pytest
import torch

import block_masked_window_b200 as bmw
import oracle
import workloads
from gpu_util import assert_parity, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_lib):
    return cuda_lib


def paginate(cache, seq_lens, W, page_size, pages_per_seq, spare, seed):
    """cache [B, Hkv, S, D] -> pool [num_pages, Hkv, page_size, D] and block table [B, pps]."""
    B, Hkv, S, D = cache.shape
    used = [-(-(int(P) + W) // page_size) for P in seq_lens]
    num_pages = sum(used) + spare
    g = torch.Generator().manual_seed(seed)
    perm = torch.randperm(num_pages, generator=g).tolist()
    pool = torch.full((num_pages, Hkv, page_size, D), float("nan"), dtype=cache.dtype)
    table = torch.full((B, pages_per_seq), 1 << 30, dtype=torch.int32)   # never a valid page
    k = 0
    for b in range(B):
        for i in range(used[b]):
            pg = perm[k]
            k += 1
            table[b, i] = pg
            rows = cache[b, :, i * page_size:(i + 1) * page_size]
            pool[pg, :, :rows.shape[1]] = rows
    return pool, table


def gather(pool, table, seq_lens, W, S):
    B = table.shape[0]
    Hkv, ps, D = pool.shape[1], pool.shape[2], pool.shape[3]
    out = torch.zeros(B, Hkv, S, D, dtype=pool.dtype)
    for b in range(B):
        n = int(seq_lens[b]) + W
        for i in range(-(-n // ps)):
            seg = pool[int(table[b, i])]
            j1 = min(S, (i + 1) * ps)
            out[b, :, i * ps:j1] = seg[:, :j1 - i * ps]
    return out


@pytest.mark.parametrize("W", [6, 10])
@pytest.mark.parametrize("page_size", [64, 128, 256])
@pytest.mark.parametrize("mask_mode", [bmw.LA_MASK_PBD, bmw.LA_MASK_CAUSAL_WINDOW], ids=["pbd", "causal"])
def test_paged_step(page_size, mask_mode, W):
    prefixes = (0, 5, 121, 122, 1000, 2041, 300)
    wi = workloads.random_case(len(prefixes), prefixes, W, seed=73)
    li = wi.layers[0]
    B, S = len(prefixes), wi.max_seq
    pps = -(-S // page_size) + 1
    kp, table = paginate(li.k_cache, wi.seq_lens, W, page_size, pps, spare=3, seed=77)
    vp, _ = paginate(li.v_cache, wi.seq_lens, W, page_size, pps, spare=3, seed=77)
    cfg = bmw.Config.make(B, 16, 2, S, mask_mode=mask_mode)
    kp_d, vp_d = to_dev(kp), to_dev(vp)
    out = torch.empty_like(to_dev(li.q))
    ws = bmw.Workspace(cfg, W)
    bmw.la_pbd_step_paged(cfg, to_dev(li.q), to_dev(li.k_new), to_dev(li.v_new), kp_d, vp_d,
                          to_dev(table), to_dev(wi.seq_lens), W, out, ws)
    torch.cuda.synchronize()
    assert bmw.la_pbd_check(ws) == 0
    k_ref, v_ref = oracle.kv_append(li.k_cache, li.v_cache, li.k_new, li.v_new, wi.seq_lens)
    kg = gather(kp_d.cpu(), table, wi.seq_lens, W, S)
    vg = gather(vp_d.cpu(), table, wi.seq_lens, W, S)
    for b, P in enumerate(prefixes):
        n = P + W
        assert np.array_equal(kg[b, :, :n].double().numpy(), k_ref[b, :, :n])
        assert np.array_equal(vg[b, :, :n].double().numpy(), v_ref[b, :, :n])
    mode = "causal" if mask_mode == bmw.LA_MASK_CAUSAL_WINDOW else "pbd"
    ref = oracle.window_attention(li.q, k_ref, v_ref, wi.seq_lens, wi.workload.scale, mask=mode)
    assert_parity(out.cpu(), ref, f"paged page_size={page_size} {mode} W={W}")


def test_paged_attn_matches_contiguous():
    """la_pbd_attn_paged on a paged copy of an appended cache gives the same bits as
    la_pbd_attn on the contiguous cache (same tiles, same arithmetic)."""
    prefixes, W, page_size = (700, 64, 1500), 6, 128
    wi = workloads.random_case(len(prefixes), prefixes, W, seed=79)
    li = wi.layers[0]
    B, S = len(prefixes), wi.max_seq
    k_ref, v_ref = oracle.kv_append(li.k_cache, li.v_cache, li.k_new, li.v_new, wi.seq_lens)
    kc = torch.from_numpy(k_ref).to(torch.bfloat16)
    vc = torch.from_numpy(v_ref).to(torch.bfloat16)
    pps = -(-S // page_size)
    kp, table = paginate(kc, wi.seq_lens, W, page_size, pps, spare=0, seed=81)
    vp, _ = paginate(vc, wi.seq_lens, W, page_size, pps, spare=0, seed=81)
    cfg = bmw.Config.make(B, 16, 2, S, algo=bmw.LA_ALGO_TCGEN05)
    ws = bmw.Workspace(cfg, W)
    out1 = torch.empty_like(to_dev(li.q))
    out2 = torch.empty_like(out1)
    bmw.la_pbd_attn_paged(cfg, to_dev(li.q), to_dev(kp), to_dev(vp), to_dev(table),
                          to_dev(wi.seq_lens), W, out1, ws)
    bmw.la_pbd_attn(cfg, to_dev(li.q), to_dev(kc), to_dev(vc), to_dev(wi.seq_lens), W, out2, ws)
    torch.cuda.synchronize()
    assert torch.equal(out1, out2)
