"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

Each pin is a plain function of the oracle module so that the planted-mistake
test at the end can run all pins against a deliberately broken oracle and show
that every plausible mistake is caught by at least one pin.

Pins and their anchors:
* golden masks typed by hand from the RK3588 card, "How it differs from the
  original", item 1 (bidirectional window, causal to the prefix);
* a worked step derived by hand (append, mask, scale, softmax, PV);
* W = 1 equals ordinary causal decode, computed by torch's SDPA in float64
  (SKILL.md page: ``slow`` mode is next-token prediction);
* the whole window equals SDPA in float64 with the brute-force block mask over
  the full sequence, last W rows;
* GQA equals SDPA's own grouped-query mode (``enable_gqa``), i.e. the ONNX
  card's [1, 2, seq, 128] K/V shared by 16 query heads;
* invariants: probabilities sum to 1, uniform V gives V, a constant added to
  every K element changes nothing, all-zero K gives the mean of visible V,
  permuting the window tokens permutes the outputs (bidirectionality).
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import pbd as opbd
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
F = torch.nn.functional


def _read_sections(path):
    sections, cur = {}, None
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.startswith("["):
                cur = line.strip("[]")
                sections[cur] = []
                continue
            sections[cur].append([float(x) for x in line.split()])
    return {k: np.array(v) for k, v in sections.items()}


def _case(B=2, prefix=(5, 9), W=3, Hq=4, Hkv=2, D=8, seed=7):
    wi = workloads.random_case(B, prefix, W, Hq, Hkv, D, seed=seed)
    li = wi.layers[0]
    return wi, li


# ----------------------------------------------------------------- pins ---
def pin_golden_mask(o):
    g = _read_sections(os.path.join(GOLDEN, "pbd_mask_P3_W2.txt"))
    full = o.block_mask_bruteforce(o.pbd_block_ids(3, 2))
    assert np.array_equal(full.astype(int), g["pbd"].astype(int))
    assert np.array_equal(o.pbd_window_mask(3, 2, 5).astype(int), g["pbd"][3:].astype(int))
    fullc = o.block_mask_bruteforce(o.pbd_block_ids(3, 2, causal_window=True))
    assert np.array_equal(fullc.astype(int), g["causal_window"].astype(int))
    assert np.array_equal(o.causal_window_mask(3, 2, 5).astype(int),
                          g["causal_window"][3:].astype(int))


def pin_mask_bruteforce(o):
    for P in range(0, 13):
        for W in range(1, 9):
            T = P + W
            S = T + 3  # capacity beyond the visible range must stay masked
            bf = o.block_mask_bruteforce(o.pbd_block_ids(P, W))[P:, :]
            m = o.pbd_window_mask(P, W, S)
            assert np.array_equal(m[:, :T], bf), (P, W)
            assert not m[:, T:].any(), (P, W)
            bfc = o.block_mask_bruteforce(o.pbd_block_ids(P, W, causal_window=True))[P:, :]
            mc = o.causal_window_mask(P, W, S)
            assert np.array_equal(mc[:, :T], bfc), (P, W)
            assert not mc[:, T:].any(), (P, W)


def pin_worked_example(o):
    g = _read_sections(os.path.join(GOLDEN, "worked_example_P1_W2.txt"))
    l3, l4 = math.log(3.0), math.log(4.0)
    kc = np.array([[[[0, 0], [9, 9], [9, 9], [100, 100]]]], dtype=np.float64)
    vc = np.array([[[[1, 0], [7, 7], [7, 7], [1000, 1000]]]], dtype=np.float64)
    kn = np.array([[[[2 * l3, 0]], [[0, 2 * l4]]]], dtype=np.float64)   # [1, 2, 1, 2]
    vn = np.array([[[[0, 1]], [[6, 12]]]], dtype=np.float64)
    q = np.array([[[[1, 0]], [[0, 1]]]], dtype=np.float64)              # [1, 2, 1, 2]
    P = np.array([1])
    out = o.pbd_step(q, kc, vc, kn, vn, P, 0.5)
    np.testing.assert_allclose(out[0, :, 0, :], g["pbd"], rtol=1e-14, atol=1e-14)
    outc = o.pbd_step(q, kc, vc, kn, vn, P, 0.5, mask="causal")
    np.testing.assert_allclose(outc[0, :, 0, :], g["causal_window"], rtol=1e-14, atol=1e-14)


def _full_sequence(li, seq_lens, o):
    k, v = o.kv_append(li.k_cache, li.v_cache, li.k_new, li.v_new, seq_lens)
    return k, v


def pin_w1_is_causal_decode(o):
    wi, li = _case(B=2, prefix=(0, 11), W=1, Hq=4, Hkv=4, D=16, seed=11)
    out = o.pbd_step(li.q, li.k_cache, li.v_cache, li.k_new, li.v_new, wi.seq_lens,
                     wi.workload.scale)
    k, v = _full_sequence(li, wi.seq_lens, o)
    for b in range(2):
        T = int(wi.seq_lens[b]) + 1
        # Full causal self-attention over T tokens whose last query is the window row.
        qf = torch.zeros(1, 4, T, 16, dtype=torch.float64)
        qf[0, :, T - 1, :] = li.q[b, 0].double()
        kk = torch.from_numpy(k[b, :, :T, :])[None]
        vv = torch.from_numpy(v[b, :, :T, :])[None]
        ref = F.scaled_dot_product_attention(qf, kk, vv, is_causal=True,
                                             scale=wi.workload.scale)
        np.testing.assert_allclose(out[b, 0], ref[0, :, T - 1, :].numpy(), rtol=1e-12, atol=1e-12)


def pin_window_is_sdpa_blockmask(o):
    for causal in (False, True):
        wi, li = _case(B=2, prefix=(3, 8), W=4, Hq=2, Hkv=2, D=8, seed=13)
        out = o.pbd_step(li.q, li.k_cache, li.v_cache, li.k_new, li.v_new, wi.seq_lens,
                         wi.workload.scale, mask="causal" if causal else "pbd")
        k, v = _full_sequence(li, wi.seq_lens, o)
        for b in range(2):
            P = int(wi.seq_lens[b])
            T = P + 4
            mask = torch.from_numpy(o.block_mask_bruteforce(o.pbd_block_ids(P, 4, causal)))
            qf = torch.zeros(1, 2, T, 8, dtype=torch.float64)
            qf[0, :, P:, :] = li.q[b].double().permute(1, 0, 2)
            ref = F.scaled_dot_product_attention(
                qf, torch.from_numpy(k[b, :, :T])[None], torch.from_numpy(v[b, :, :T])[None],
                attn_mask=mask, scale=wi.workload.scale)
            np.testing.assert_allclose(out[b].transpose(1, 0, 2), ref[0, :, P:, :].numpy(),
                                       rtol=1e-12, atol=1e-12)


def pin_gqa_is_sdpa_gqa(o):
    wi, li = _case(B=1, prefix=(10,), W=3, Hq=16, Hkv=2, D=16, seed=17)
    out = o.pbd_step(li.q, li.k_cache, li.v_cache, li.k_new, li.v_new, wi.seq_lens,
                     wi.workload.scale)
    k, v = _full_sequence(li, wi.seq_lens, o)
    T = 13
    qq = li.q[0].double().permute(1, 0, 2)[None]                 # [1, Hq, W, D]
    ref = F.scaled_dot_product_attention(
        qq, torch.from_numpy(k[0, :, :T])[None], torch.from_numpy(v[0, :, :T])[None],
        enable_gqa=True, scale=wi.workload.scale)
    np.testing.assert_allclose(out[0].transpose(1, 0, 2), ref[0].numpy(), rtol=1e-12, atol=1e-12)


def pin_invariants(o):
    wi, li = _case(B=2, prefix=(0, 21), W=6, Hq=8, Hkv=2, D=32, seed=19)
    sc = wi.workload.scale
    out, p = o.pbd_step(li.q, li.k_cache, li.v_cache, li.k_new, li.v_new, wi.seq_lens, sc,
                        return_probs=True)
    # row sums
    np.testing.assert_allclose(p.sum(axis=-1), 1.0, rtol=0, atol=1e-12)
    # nothing outside [0, P+W)
    for b in range(2):
        T = int(wi.seq_lens[b]) + 6
        assert not p[b, :, :, T:].any()
        assert (p[b, :, :, :T] > 0).all()
    # uniform V -> same vector on every row
    vec = np.linspace(-1.0, 2.0, 32)
    vc = np.broadcast_to(vec, li.v_cache.shape).copy()
    vn = np.broadcast_to(vec, li.v_new.shape).copy()
    outu = o.pbd_step(li.q, li.k_cache, vc, li.k_new, vn, wi.seq_lens, sc)
    np.testing.assert_allclose(outu, np.broadcast_to(vec, outu.shape), rtol=0, atol=1e-12)
    # constant K offset: score shift per row is constant -> output unchanged
    kc = li.k_cache.double() + 0.75
    kn = li.k_new.double() + 0.75
    outo = o.pbd_step(li.q, kc, li.v_cache, kn, li.v_new, wi.seq_lens, sc)
    np.testing.assert_allclose(outo, out, rtol=1e-10, atol=1e-10)
    # all-zero K -> uniform weights -> mean of the visible V rows
    k0c = np.zeros(li.k_cache.shape)
    k0n = np.zeros(li.k_new.shape)
    outz = o.pbd_step(li.q, k0c, li.v_cache, k0n, li.v_new, wi.seq_lens, sc)
    _, v = o.kv_append(li.k_cache, li.v_cache, li.k_new, li.v_new, wi.seq_lens)
    for b in range(2):
        T = int(wi.seq_lens[b]) + 6
        for h in range(8):
            mean = v[b, h // 4, :T, :].mean(axis=0)
            np.testing.assert_allclose(outz[b, :, h, :], np.broadcast_to(mean, (6, 32)),
                                       rtol=0, atol=1e-12)


def pin_window_permutation(o):
    wi, li = _case(B=1, prefix=(7,), W=5, Hq=4, Hkv=2, D=16, seed=23)
    sc = wi.workload.scale
    perm = np.array([3, 0, 4, 1, 2])
    out = o.pbd_step(li.q, li.k_cache, li.v_cache, li.k_new, li.v_new, wi.seq_lens, sc)
    outp = o.pbd_step(li.q[:, perm], li.k_cache, li.v_cache, li.k_new[:, perm],
                      li.v_new[:, perm], wi.seq_lens, sc)
    np.testing.assert_allclose(outp, out[:, perm], rtol=1e-12, atol=1e-12)
    # identical window queries -> identical output rows (every row sees the same keys)
    qs = li.q.clone()
    qs[:, :] = li.q[:, 2:3]
    outs = o.pbd_step(qs, li.k_cache, li.v_cache, li.k_new, li.v_new, wi.seq_lens, sc)
    for i in range(5):
        np.testing.assert_allclose(outs[:, i], outs[:, 0], rtol=0, atol=1e-13)


def pin_causal_window_breaks_permutation(o):
    """The same permutation test must fail under the causal-window mask."""
    wi, li = _case(B=1, prefix=(7,), W=5, Hq=4, Hkv=2, D=16, seed=23)
    sc = wi.workload.scale
    perm = np.array([3, 0, 4, 1, 2])
    out = o.pbd_step(li.q, li.k_cache, li.v_cache, li.k_new, li.v_new, wi.seq_lens, sc,
                     mask="causal")
    outp = o.pbd_step(li.q[:, perm], li.k_cache, li.v_cache, li.k_new[:, perm],
                      li.v_new[:, perm], wi.seq_lens, sc, mask="causal")
    assert np.abs(outp - out[:, perm]).max() > 1e-3


def pin_append(o):
    wi, li = _case(B=3, prefix=(0, 4, 9), W=2, Hq=2, Hkv=2, D=4, seed=29)
    k, v = o.kv_append(li.k_cache, li.v_cache, li.k_new, li.v_new, wi.seq_lens)
    kc = li.k_cache.double().numpy()
    for b, P in enumerate([0, 4, 9]):
        for h in range(2):
            for j in range(k.shape[2]):
                if P <= j < P + 2:
                    assert np.array_equal(k[b, h, j], li.k_new[b, j - P, h].double().numpy())
                    assert np.array_equal(v[b, h, j], li.v_new[b, j - P, h].double().numpy())
                else:
                    assert np.array_equal(k[b, h, j], kc[b, h, j])


def pin_block_prefill(o):
    """Prefill block mask vs SDPA with the brute-force mask (blocks of 3)."""
    T, Hq, Hkv, D = 11, 4, 2, 8
    g = torch.Generator().manual_seed(31)
    q = torch.randn(T, Hq, D, generator=g, dtype=torch.float64)
    k = torch.randn(T, Hkv, D, generator=g, dtype=torch.float64)
    v = torch.randn(T, Hkv, D, generator=g, dtype=torch.float64)
    ids = [0, 1, 2, 3, 4, 5, 5, 5, 6, 6, 6]
    out = o.block_prefill_attention(q, k, v, ids, 0.3)
    mask = torch.from_numpy(o.block_mask_bruteforce(ids))
    ref = F.scaled_dot_product_attention(q.permute(1, 0, 2)[None], k.permute(1, 0, 2)[None],
                                         v.permute(1, 0, 2)[None], attn_mask=mask, scale=0.3,
                                         enable_gqa=True)
    np.testing.assert_allclose(out, ref[0].permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-12)
    # the single-row form, row by row, against the same SDPA reference
    for i in range(T):
        row = o.block_prefill_row(q[i], k, v, i, ids, 0.3)
        np.testing.assert_allclose(row, ref[0, :, i, :].numpy(), rtol=1e-12, atol=1e-12)


def pin_varwin_is_sdpa_blockmask(o):
    """Per-sequence windows (W_b = accepted tokens + masks, RKLLM engine's step): each
    sequence's rows i < W_b equal fp64 SDPA over its own full sequence with the brute-force
    block mask of a W_b-row window; padding rows are zero; the append writes exactly the
    W_b rows of each sequence at P_b.. and nothing else."""
    W_max, Hq, Hkv, D = 5, 4, 2, 8
    prefix, wlens = (4, 0, 9), (1, 5, 3)
    wi, li = _case(B=3, prefix=prefix, W=W_max, Hq=Hq, Hkv=Hkv, D=D, seed=29)
    wl = torch.tensor(wlens, dtype=torch.int32)
    sc = wi.workload.scale
    k, v = o.kv_append_varwin(li.k_cache, li.v_cache, li.k_new, li.v_new, wi.seq_lens, wl)
    for mode in ("pbd", "causal"):
        out = o.pbd_step_varwin(li.q, li.k_cache, li.v_cache, li.k_new, li.v_new, wi.seq_lens,
                                wl, sc, mask=mode)
        for b in range(3):
            P, w = prefix[b], wlens[b]
            T = P + w
            # the append, written out
            kk = li.k_cache[b].double().clone()
            vv = li.v_cache[b].double().clone()
            kk[:, P:T] = li.k_new[b, :w].double().permute(1, 0, 2)
            vv[:, P:T] = li.v_new[b, :w].double().permute(1, 0, 2)
            assert np.array_equal(k[b], kk.numpy()) and np.array_equal(v[b], vv.numpy())
            mask = torch.from_numpy(o.block_mask_bruteforce(o.pbd_block_ids(P, w, mode == "causal")))
            qf = torch.zeros(1, Hq, T, D, dtype=torch.float64)
            qf[0, :, P:, :] = li.q[b, :w].double().permute(1, 0, 2)
            ref = F.scaled_dot_product_attention(qf, kk[None, :, :T], vv[None, :, :T],
                                                 attn_mask=mask, scale=sc, enable_gqa=True)
            np.testing.assert_allclose(out[b, :w].transpose(1, 0, 2), ref[0, :, P:, :].numpy(),
                                       rtol=1e-12, atol=1e-12)
            assert not out[b, w:].any()


PINS = [pin_golden_mask, pin_mask_bruteforce, pin_worked_example, pin_w1_is_causal_decode,
        pin_window_is_sdpa_blockmask, pin_gqa_is_sdpa_gqa, pin_invariants,
        pin_window_permutation, pin_causal_window_breaks_permutation, pin_append,
        pin_block_prefill, pin_varwin_is_sdpa_blockmask]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin(oracle)


# ------------------------------------------------ planted mistakes (CPU) ---
def _buggy_interleaved_gqa(h, Hq, Hkv):
    return h % Hkv


def _buggy_visible(P, W):
    return P + W - 1


def _buggy_mask_causal(P, W, S):
    return opbd.causal_window_mask(P, W, S)


def _mk_attention_bug(kind):
    real = opbd.window_attention

    def wrapped(q, k_cache, v_cache, seq_lens, scale, mask="pbd", return_probs=False):
        if kind == "scale":
            scale = scale * 2.0
        elif kind == "kv_swapped":
            k_cache, v_cache = v_cache, k_cache
        elif kind == "k_transposed_heads":
            k_cache = np.ascontiguousarray(opbd._f64(k_cache)[:, ::-1])
        return real(q, k_cache, v_cache, seq_lens, scale, mask=mask, return_probs=return_probs)
    return wrapped


_real_append = opbd.kv_append


def _buggy_append(k_cache, v_cache, k_new, v_new, seq_lens):
    # Window written one row too late.
    return _real_append(k_cache, v_cache, k_new, v_new, np.asarray(seq_lens) + 1)


def _buggy_mask_all(P, W, S):
    return np.ones((W, S), dtype=bool)


_real_varwin = opbd.window_attention_varwin


def _buggy_varwin_max_window(q, k_cache, v_cache, seq_lens, window_lens, scale, mask="pbd"):
    # Every sequence treated as if it had the longest window.
    wmax = np.full(len(np.asarray(window_lens)), np.asarray(q).shape[1] if hasattr(q, "shape") else 0)
    return _real_varwin(q, k_cache, v_cache, seq_lens, wmax, scale, mask=mask)


_real_append_varwin = opbd.kv_append_varwin


def _buggy_append_varwin(k_cache, v_cache, k_new, v_new, seq_lens, window_lens):
    # All W_max rows appended, padding included.
    W_max = np.asarray(opbd._f64(k_new)).shape[1]
    return _real_append_varwin(k_cache, v_cache, k_new, v_new, seq_lens,
                               np.full(len(np.asarray(seq_lens)), W_max))


MISTAKES = {
    "varwin_uses_max_window": ("window_attention_varwin", _buggy_varwin_max_window),
    "varwin_appends_padding": ("kv_append_varwin", _buggy_append_varwin),
    "gqa_interleaved": ("kv_head_of", _buggy_interleaved_gqa),
    "visible_off_by_one": ("visible_keys", _buggy_visible),
    "causal_window_mask": ("pbd_window_mask", _buggy_mask_causal),
    "mask_dropped": ("pbd_window_mask", _buggy_mask_all),
    "scale_doubled": ("window_attention", _mk_attention_bug("scale")),
    "k_v_swapped": ("window_attention", _mk_attention_bug("kv_swapped")),
    "kv_heads_reversed": ("window_attention", _mk_attention_bug("k_transposed_heads")),
    "append_shifted": ("kv_append", _buggy_append),
}


@pytest.mark.parametrize("name", sorted(MISTAKES))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, repl = MISTAKES[name]
    monkeypatch.setattr(opbd, attr, repl)
    failures = 0
    for pin in PINS:
        try:
            pin(opbd)
        except Exception:  # an assertion, or the broken oracle failing outright
            failures += 1
    assert failures > 0, f"no pin caught the planted mistake {name!r}"
