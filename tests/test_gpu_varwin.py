"""GPU parity of per-sequence window lengths (la_pbd_step_varwin / la_pbd_attn_varwin) against
the fp64 oracle, through the C ABI.

The RKLLM engine's step sends each sequence's accepted tokens plus 5 <text_mask> tokens, so the
window length W_b differs within a batch. Padding rows (i >= W_b) of q, k_new and v_new are
filled with NaN here: they must neither reach any output nor be appended, and the padding rows
of the output must be exactly zero.
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


def _case(prefixes, wlens, W_max, seed, Hq=16, Hkv=2):
    wi = workloads.random_case(len(prefixes), prefixes, W_max, num_q_heads=Hq,
                               num_kv_heads=Hkv, seed=seed)
    li = wi.layers[0]
    q, kn, vn = li.q.clone(), li.k_new.clone(), li.v_new.clone()
    for b, w in enumerate(wlens):
        q[b, w:] = float("nan")
        kn[b, w:] = float("nan")
        vn[b, w:] = float("nan")
    return wi, li, q, kn, vn, torch.tensor(wlens, dtype=torch.int32)


CASES = {
    # (prefixes, window lengths, W_max); the pages' engine sends the accepted tokens (1..5)
    # plus 5 masks, so W_b in [6, 10]; the tcgen05 kernel takes W_max * 8 <= 80
    "w8": ((0, 5, 121, 1000, 2047, 300, 64, 250), (1, 8, 6, 7, 2, 8, 5, 3), 8),
    "w10": ((0, 5, 121, 1000, 2047, 300, 64, 250), (1, 10, 6, 7, 2, 9, 5, 10), 10),
    "w16": ((0, 5, 121, 1000), (16, 9, 3, 12), 16),
}


@pytest.mark.parametrize("mask_mode", [bmw.LA_MASK_PBD, bmw.LA_MASK_CAUSAL_WINDOW],
                         ids=["pbd", "causal"])
@pytest.mark.parametrize("algo,key", [(bmw.LA_ALGO_TCGEN05, "w8"), (bmw.LA_ALGO_TCGEN05, "w10"),
                                      (bmw.LA_ALGO_SIMT, "w10"), (bmw.LA_ALGO_SIMT, "w16")],
                         ids=["tcgen05-w8", "tcgen05-w10", "simt-w10", "simt-w16"])
def test_variable_windows(algo, key, mask_mode):
    prefixes, wlens, W_max = CASES[key]
    wi, li, q, kn, vn, wl = _case(prefixes, wlens, W_max, seed=51)
    B = len(prefixes)
    cfg = bmw.Config.make(B, 16, 2, wi.max_seq, mask_mode=mask_mode, algo=algo)
    kc, vc = to_dev(li.k_cache), to_dev(li.v_cache)
    out = torch.full_like(to_dev(q), 7.0)
    ws = bmw.Workspace(cfg, W_max)
    bmw.la_pbd_step_varwin(cfg, to_dev(q), to_dev(kn), to_dev(vn), kc, vc, to_dev(wi.seq_lens),
                           to_dev(wl), W_max, out, ws)
    torch.cuda.synchronize()
    assert bmw.la_pbd_check(ws) == 0
    k_ref, v_ref = oracle.kv_append_varwin(li.k_cache, li.v_cache, kn, vn, wi.seq_lens, wl)
    assert np.array_equal(kc.cpu().double().numpy(), k_ref)
    assert np.array_equal(vc.cpu().double().numpy(), v_ref)
    mode = "causal" if mask_mode == bmw.LA_MASK_CAUSAL_WINDOW else "pbd"
    ref = oracle.window_attention_varwin(q, k_ref, v_ref, wi.seq_lens, wl, wi.workload.scale,
                                         mask=mode)
    o = out.cpu()
    for b, w in enumerate(wlens):
        assert torch.equal(o[b, w:], torch.zeros_like(o[b, w:])), f"padding rows of {b}"
        assert_parity(o[b, :w], ref[b, :w], f"varwin {key} {mode} b={b} W_b={w}")


@pytest.mark.parametrize("key", ["w8", "w10"])
def test_variable_windows_fused_matches_separate(key):
    """The tcgen05 step (append fused into the attention launch) against the CUDA-core step
    (append kernel, then attention): same caches bit for bit, outputs within rounding."""
    prefixes, wlens, W_max = CASES[key]
    wi, li, q, kn, vn, wl = _case(prefixes, wlens, W_max, seed=53)
    B = len(prefixes)
    outs, caches = [], []
    for algo in (bmw.LA_ALGO_TCGEN05, bmw.LA_ALGO_SIMT):
        cfg = bmw.Config.make(B, 16, 2, wi.max_seq, algo=algo)
        kc, vc = to_dev(li.k_cache), to_dev(li.v_cache)
        out = torch.empty_like(to_dev(q))
        ws = bmw.Workspace(cfg, W_max)
        bmw.la_pbd_step_varwin(cfg, to_dev(q), to_dev(kn), to_dev(vn), kc, vc,
                               to_dev(wi.seq_lens), to_dev(wl), W_max, out, ws)
        torch.cuda.synchronize()
        outs.append(out.cpu().double())
        caches.append((kc.cpu(), vc.cpu()))
    assert torch.equal(caches[0][0], caches[1][0]) and torch.equal(caches[0][1], caches[1][1])
    rel = float((outs[0] - outs[1]).norm() / outs[1].norm())
    assert rel < 2e-3, rel


@pytest.mark.parametrize("algo", [bmw.LA_ALGO_TCGEN05, bmw.LA_ALGO_SIMT], ids=["tcgen05", "simt"])
def test_invalid_window_lengths_flagged(algo):
    """W_b = 0 or W_b > W_max: zero output rows, untouched cache, sticky status; the other
    sequences are unaffected."""
    prefixes, W_max = (10, 20, 30, 40), 4
    wlens = (2, 0, 5, 4)
    wi, li, q, kn, vn, wl = _case(prefixes, (2, 0, 4, 4), W_max, seed=57)
    wl = torch.tensor(wlens, dtype=torch.int32)
    cfg = bmw.Config.make(4, 16, 2, wi.max_seq, algo=algo)
    kc, vc = to_dev(li.k_cache), to_dev(li.v_cache)
    out = torch.full_like(to_dev(q), 7.0)
    ws = bmw.Workspace(cfg, W_max)
    bmw.la_pbd_step_varwin(cfg, to_dev(q), to_dev(kn), to_dev(vn), kc, vc, to_dev(wi.seq_lens),
                           to_dev(wl), W_max, out, ws)
    torch.cuda.synchronize()
    assert bmw.la_pbd_check(ws) == 5
    o = out.cpu()
    for b in (1, 2):
        assert torch.equal(o[b], torch.zeros_like(o[b]))
        assert torch.equal(kc[b].cpu(), li.k_cache[b]) and torch.equal(vc[b].cpu(), li.v_cache[b])
    good = [0, 3]
    ref = oracle.pbd_step_varwin(q[good], li.k_cache[good], li.v_cache[good], kn[good], vn[good],
                                 wi.seq_lens[good], wl[good], wi.workload.scale)
    for j, b in enumerate(good):
        w = wlens[b]
        assert_parity(o[b, :w], ref[j, :w], f"valid sequence {b} beside invalid ones")
