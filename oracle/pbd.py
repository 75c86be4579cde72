"""fp64 CPU oracle for Parallel Box Decoding (PBD) window attention.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU-baseline legs, never by the CUDA library.

What the method computes, and where the pages fix it
----------------------------------------------------
* LocateAnything-3B for RK3588 model card, "How it differs from the original",
  item 1: a PBD step evaluates a 6-token window (the last accepted token plus 5
  ``<text_mask>`` tokens). Attention is bidirectional inside the window; the
  model was trained that way, and a causal mask inside the window is only an
  approximation (the RKLLM port uses it). The engine sends the accepted tokens
  plus 5 mask tokens each step and reuses the KV cache of the common prefix with
  no explicit rollback; window token positions follow the original layout.
* LocateAnything-3B ONNX WebGPU INT4 model card, "KV-cache graph for in-browser
  use": 36 layers of grouped-query past K/V tensors shaped ``[1, 2, seq, 128]``;
  "Why this repo exists": hidden size 2048, hence 16 query heads of width 128.
* "LocateAnything-3B on a 12 GB RTX 4000 Ada" page, "Architecture footprint":
  bf16 throughout. SKILL.md page, "Inference API": ``slow`` mode is plain
  next-token prediction, i.e. a window of one token.

Readings where the pages are silent (each listed in the design notes):
* query head h reads KV head ``h // (Hq / Hkv)`` (contiguous grouping);
* softmax scale 1/sqrt(head_dim);
* the window's K/V land in cache rows P_b .. P_b+W-1 (P_b = committed prefix
  length of sequence b) before attention; RoPE is applied by the caller;
* "causal to the prefix" means every window row sees every prefix row: the
  window is the last block of a block-causal mask, so each of its rows sees
  keys [0, P_b + W) and nothing beyond.

Everything is computed in float64 from the bf16 inputs upcast exactly; the
result is returned in float64 (the caller rounds if it wants bf16).
"""
from __future__ import annotations

import numpy as np


def _f64(x) -> np.ndarray:
    """Exact upcast of a (bf16/fp32/fp64) torch tensor or array to float64."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


# --------------------------------------------------------------------------
# step a1: window K/V append (RK3588 card, item 1: prefix KV reused, the
# window's rows written after it, no rollback of older speculative rows)
# --------------------------------------------------------------------------
def kv_append(k_cache, v_cache, k_new, v_new, seq_lens):
    """Return copies of the caches with the window rows written.

    k_cache, v_cache: [B, Hkv, S_max, D]; k_new, v_new: [B, W, Hkv, D];
    seq_lens: [B] committed prefix lengths P_b. Row P_b + w of KV head h of
    sequence b receives k_new[b, w, h]. Rows outside [P_b, P_b + W) are kept.
    """
    k = np.array(_f64(k_cache), copy=True)
    v = np.array(_f64(v_cache), copy=True)
    kn, vn = _f64(k_new), _f64(v_new)
    P = np.asarray(_f64(seq_lens), dtype=np.int64)
    B, W = kn.shape[0], kn.shape[1]
    for b in range(B):
        for w in range(W):
            k[b, :, P[b] + w, :] = kn[b, w, :, :]
            v[b, :, P[b] + w, :] = vn[b, w, :, :]
    return k, v


# --------------------------------------------------------------------------
# step a3: the PBD block mask
# --------------------------------------------------------------------------
def visible_keys(P: int, W: int) -> int:
    """Number of keys a PBD window row sees: the whole prefix and the whole window."""
    return P + W


def pbd_window_mask(P: int, W: int, S: int) -> np.ndarray:
    """allowed[i, j] for window row i (position P+i) and cache row j < S.

    Bidirectional inside the window, causal toward the prefix (RK3588 card,
    item 1): every window row sees rows [0, P+W), nothing at or beyond P+W.
    """
    j = np.arange(S)[None, :]
    return np.broadcast_to(j < visible_keys(P, W), (W, S)).copy()


def causal_window_mask(P: int, W: int, S: int) -> np.ndarray:
    """The RKLLM approximation (RK3588 card, item 1): causal inside the window.

    Window row i (position P+i) sees rows [0, P+i].
    """
    i = np.arange(W)[:, None]
    j = np.arange(S)[None, :]
    return j <= P + i


def block_mask_bruteforce(block_ids) -> np.ndarray:
    """Full T x T block-causal mask enumerated from per-token block ids.

    Token i may attend token j when j is not after i, or when both tokens are
    in the same block (blocks are bidirectional). For a PBD step the prefix
    tokens are singleton blocks and the W window tokens share one block; for
    SDLM-style training/prefill the generated part is cut into blocks of
    ``block_size`` (SKILL.md page, "Training" / "Key Parameters").
    Written as two explicit loops so that it shares nothing with the
    vectorised masks above.
    """
    ids = list(block_ids)
    T = len(ids)
    m = np.zeros((T, T), dtype=bool)
    for i in range(T):
        for j in range(T):
            m[i, j] = (j <= i) or (ids[i] == ids[j])
    return m


def pbd_block_ids(P: int, W: int, causal_window: bool = False):
    """Block ids of one PBD step: singleton prefix blocks, one window block.

    With ``causal_window`` every window token is its own block (RKLLM mode).
    """
    if causal_window:
        return list(range(P + W))
    return list(range(P)) + [P] * W


# --------------------------------------------------------------------------
# GQA mapping (ONNX card: K/V have 2 heads, hidden 2048 -> 16 query heads)
# --------------------------------------------------------------------------
def kv_head_of(h: int, Hq: int, Hkv: int) -> int:
    """KV head read by query head h: contiguous groups of Hq/Hkv query heads."""
    return h // (Hq // Hkv)


# --------------------------------------------------------------------------
# steps a2 + a4 + a5 + a6: scores, softmax, PV (the plain definition)
# --------------------------------------------------------------------------
def window_attention(q, k_cache, v_cache, seq_lens, scale: float,
                     mask: str = "pbd", return_probs: bool = False):
    """Explicit-mask softmax attention of each window row over the cache.

    q: [B, W, Hq, D]; k_cache, v_cache: [B, Hkv, S, D] (window rows already
    appended); seq_lens: [B] prefix lengths. For every b, query head h and
    window row i:
        s_j   = scale * <q[b,i,h,:], k[b, kv(h), j, :]>        for all j < S
        p_j   = M[i,j] exp(s_j - max_M s) / sum_M exp(s - max_M s)
        out   = sum_j p_j v[b, kv(h), j, :]
    with M the PBD window mask (``mask="pbd"``) or the causal-window mask
    (``mask="causal"``). Returns float64 out [B, W, Hq, D] and, when asked,
    p as [B, Hq, W, S].
    """
    qf, kf, vf = _f64(q), _f64(k_cache), _f64(v_cache)
    P = np.asarray(_f64(seq_lens), dtype=np.int64)
    B, W, Hq, D = qf.shape
    Hkv, S = kf.shape[1], kf.shape[2]
    out = np.zeros((B, W, Hq, D), dtype=np.float64)
    probs = np.zeros((B, Hq, W, S), dtype=np.float64) if return_probs else None
    for b in range(B):
        if mask == "pbd":
            M = pbd_window_mask(int(P[b]), W, S)
        elif mask == "causal":
            M = causal_window_mask(int(P[b]), W, S)
        else:
            raise ValueError(mask)
        # The sums run over keys some window row may see, j < T; rows at or beyond T are
        # never part of the definition (their content may be anything, even non-finite).
        cols = np.nonzero(M.any(axis=0))[0]
        T = int(cols.max()) + 1 if cols.size else 0
        Mt = M[:, :T]
        for h in range(Hq):
            g = kv_head_of(h, Hq, Hkv)
            s = scale * (qf[b, :, h, :] @ kf[b, g, :T, :].T)          # [W, T]
            s = np.where(Mt, s, -np.inf)
            s = s - s.max(axis=1, keepdims=True)
            e = np.where(Mt, np.exp(s), 0.0)
            p = e / e.sum(axis=1, keepdims=True)
            out[b, :, h, :] = p @ vf[b, g, :T, :]
            if return_probs:
                probs[b, h, :, :T] = p
    if return_probs:
        return out, probs
    return out


def pbd_step(q, k_cache, v_cache, k_new, v_new, seq_lens, scale: float,
             mask: str = "pbd", return_probs: bool = False):
    """One PBD layer call: append the window K/V, then window attention."""
    k, v = kv_append(k_cache, v_cache, k_new, v_new, seq_lens)
    return window_attention(q, k, v, seq_lens, scale, mask=mask, return_probs=return_probs)


# --------------------------------------------------------------------------
# variable window per sequence (the RKLLM engine's step: the a_b accepted tokens plus
# 5 <text_mask> tokens, so W_b = a_b + 5 differs between sequences of a batch)
# --------------------------------------------------------------------------
def kv_append_varwin(k_cache, v_cache, k_new, v_new, seq_lens, window_lens):
    """Window rows w < W_b of sequence b go to cache rows P_b + w; k_new, v_new are
    [B, W_max, Hkv, D] with rows w >= W_b unused. Sequences with P_b < 0, W_b < 1,
    W_b > W_max or P_b + W_b > S are left untouched."""
    k = _f64(k_cache).copy()
    v = _f64(v_cache).copy()
    kn, vn = _f64(k_new), _f64(v_new)
    P = np.asarray(_f64(seq_lens), dtype=np.int64)
    Wb = np.asarray(_f64(window_lens), dtype=np.int64)
    W_max, S = kn.shape[1], k.shape[2]
    for b in range(k.shape[0]):
        w = int(Wb[b])
        if P[b] < 0 or w < 1 or w > W_max or P[b] + w > S:
            continue
        for i in range(w):
            k[b, :, P[b] + i, :] = kn[b, i]
            v[b, :, P[b] + i, :] = vn[b, i]
    return k, v


def window_attention_varwin(q, k_cache, v_cache, seq_lens, window_lens, scale: float,
                            mask: str = "pbd"):
    """Window attention with a window length W_b per sequence.

    q: [B, W_max, Hq, D]; row i < W_b of sequence b sits at position P_b + i and attends
    exactly as in ``window_attention`` for a window of W_b rows (every row sees keys
    [0, P_b + W_b) under the PBD mask). Rows i >= W_b are padding: their output is zero.
    """
    qf = _f64(q)
    P = np.asarray(_f64(seq_lens), dtype=np.int64)
    Wb = np.asarray(_f64(window_lens), dtype=np.int64)
    out = np.zeros_like(qf)
    for b in range(qf.shape[0]):
        w = int(Wb[b])
        out[b, :w] = window_attention(qf[b:b + 1, :w], k_cache[b:b + 1], v_cache[b:b + 1],
                                      np.array([P[b]]), scale, mask=mask)[0]
    return out


def pbd_step_varwin(q, k_cache, v_cache, k_new, v_new, seq_lens, window_lens, scale: float,
                    mask: str = "pbd"):
    """One layer call with per-sequence windows: append, then window attention."""
    k, v = kv_append_varwin(k_cache, v_cache, k_new, v_new, seq_lens, window_lens)
    return window_attention_varwin(q, k, v, seq_lens, window_lens, scale, mask=mask)


def block_prefill_attention(q, k, v, block_ids, scale: float):
    """Block-causal attention over whole sequences (SDLM block mask).

    q: [T, Hq, D], k, v: [T, Hkv, D] for one sequence; block_ids: [T].
    Token i attends j when j <= i or block(i) == block(j).
    """
    qf, kf, vf = _f64(q), _f64(k), _f64(v)
    T, Hq, D = qf.shape
    Hkv = kf.shape[1]
    ids = np.asarray(block_ids)
    same = ids[:, None] == ids[None, :]
    M = (np.arange(T)[None, :] <= np.arange(T)[:, None]) | same
    out = np.zeros_like(qf)
    for h in range(Hq):
        g = kv_head_of(h, Hq, Hkv)
        s = scale * (qf[:, h, :] @ kf[:, g, :].T)
        s = np.where(M, s, -np.inf)
        s = s - s.max(axis=1, keepdims=True)
        e = np.where(M, np.exp(s), 0.0)
        out[:, h, :] = (e / e.sum(axis=1, keepdims=True)) @ vf[:, g, :]
    return out


def block_prefill_row(q_row, k, v, i: int, block_ids, scale: float):
    """Output of query row i alone (all heads) under the block-causal mask of
    ``block_prefill_attention``: the same definition evaluated for one row, so that long
    sequences can be checked at sampled rows. q_row: [Hq, D]; k, v: [T, Hkv, D]."""
    qf, kf, vf = _f64(q_row), _f64(k), _f64(v)
    Hq, D = qf.shape
    T, Hkv = kf.shape[0], kf.shape[1]
    ids = np.asarray(block_ids)
    allowed = (np.arange(T) <= i) | (ids == ids[i])
    out = np.zeros((Hq, D), dtype=np.float64)
    for h in range(Hq):
        g = kv_head_of(h, Hq, Hkv)
        s = scale * (kf[allowed, g, :] @ qf[h])
        e = np.exp(s - s.max())
        out[h] = (e / e.sum()) @ vf[allowed, g, :]
    return out
