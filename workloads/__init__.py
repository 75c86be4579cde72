"""Seeded synthetic inputs for PBD window attention.

This module only draws random numbers and lays them out. It holds none of the
method's arithmetic (no scores, no softmax, no cache append): both the fp64
oracle and the CUDA path consume what it returns, and neither is imported here.

Workload shapes follow the pages:

* decoder = Qwen2.5-3B: 36 layers, hidden 2048, KV cache tensors of shape
  ``[1, 2, seq, 128]`` (LocateAnything-3B ONNX WebGPU INT4 model card,
  "KV-cache graph for in-browser use"; "Why this repo exists" for hidden 2048),
  so 16 query heads share 2 KV heads;
* one PBD step attends a 6-token window, the last accepted token plus 5
  ``<text_mask>`` tokens (LocateAnything-3B for RK3588 model card, "How it
  differs from the original", item 1);
* a 448x448 image gives 256 visual tokens (same card, "Files" and item 2), and
  the RKLLM build has a 4096-token maximum context (same card, "Files").

Draw order per configuration (CPU ``torch.Generator`` seeded once):
  1. ragged prefix lengths (batched ragged workload only): L_b ~ U{512..4096},
     accepted count a_b ~ U{1..5}, prefix P_b = L_b + a_b;
  2. per-sequence K mean offsets c_b ~ N(0, 0.5^2) (long-context workload only);
  3. per layer: outlier channel picks (single-image workload only), then the
     K cache, V cache, new window K, new window V and Q, all N(0, 1) in fp32,
     K transforms applied in fp32, then every tensor rounded to bf16 (RNE).

The caches are drawn for all ``max_seq`` rows: rows at and beyond ``P_b`` are
stale content of earlier speculative windows. The window append overwrites rows
[P_b, P_b + W); rows at or beyond P_b + W must never influence the result.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import torch

HEAD_DIM = 128
NUM_Q_HEADS = 16
NUM_KV_HEADS = 2
NUM_LAYERS = 36
PBD_WINDOW = 6


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    layers: int
    prefix: Optional[int]          # None = ragged (drawn from the seed)
    window: int
    seed: int
    num_q_heads: int = NUM_Q_HEADS
    num_kv_heads: int = NUM_KV_HEADS
    head_dim: int = HEAD_DIM
    k_outlier_frac: float = 0.0    # fraction of (kv head, channel) pairs of K scaled
    k_outlier_gain: float = 1.0
    k_seq_offset_std: float = 0.0  # std of a per-sequence scalar added to all of K
    description: str = ""

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    def with_window(self, window: int) -> "Workload":
        return dataclasses.replace(self, name=f"{self.name}_w{window}", window=window)


WORKLOADS = {
    "tiny": Workload(
        "tiny", batch=1, layers=1, prefix=64, window=PBD_WINDOW, seed=0,
        description="batch 1, 1 layer, prefix 64 + window 6, Q/K/V iid N(0,1)"),
    "single_image": Workload(
        "single_image", batch=1, layers=NUM_LAYERS, prefix=1024, window=PBD_WINDOW, seed=1,
        k_outlier_frac=0.01, k_outlier_gain=8.0,
        description="batch 1, 36 layers, prefix 1024 (256 visual + 768 text/box), window 6, "
                    "1% of K channels x8"),
    "max_context": Workload(
        "max_context", batch=1, layers=NUM_LAYERS, prefix=4096, window=PBD_WINDOW, seed=2,
        description="batch 1, 36 layers, prefix 4096, window 6 (window 1 = NTP variant)"),
    "ragged": Workload(
        "ragged", batch=64, layers=1, prefix=None, window=PBD_WINDOW, seed=3,
        description="64 sequences, L_b ~ U{512..4096} plus accepted a_b ~ U{1..5}, window 6"),
    "long": Workload(
        "long", batch=8, layers=1, prefix=32768, window=PBD_WINDOW, seed=4,
        k_seq_offset_std=0.5,
        description="batch 8, prefix 32768, window 6, per-sequence K offset N(0, 0.5^2)"),
}
# NTP fallback on the max-context caches (same seed, same max_seq, window 1).
WORKLOADS["max_context_w1"] = WORKLOADS["max_context"].with_window(1)
# The longest window the RKLLM engine sends (5 accepted tokens + 5 <text_mask> tokens, RK3588
# model card, item 1) on the ragged batch: a timing case for the kernel choice at 80 rows.
WORKLOADS["ragged_w10"] = WORKLOADS["ragged"].with_window(10)

ORDER = ["tiny", "single_image", "max_context", "max_context_w1", "ragged", "long"]


def _round_up(x: int, m: int) -> int:
    return (x + m - 1) // m * m


@dataclasses.dataclass
class LayerInputs:
    q: torch.Tensor        # bf16 [B, W, Hq, D]
    k_cache: torch.Tensor  # bf16 [B, Hkv, S_max, D] (rows >= P_b are stale)
    v_cache: torch.Tensor  # bf16 [B, Hkv, S_max, D]
    k_new: torch.Tensor    # bf16 [B, W, Hkv, D] window keys at positions P_b .. P_b+W-1
    v_new: torch.Tensor    # bf16 [B, W, Hkv, D]


@dataclasses.dataclass
class WorkloadInputs:
    workload: Workload
    seq_lens: torch.Tensor   # int32 [B], committed prefix length P_b
    max_seq: int             # cache capacity S_max
    layers: List[LayerInputs]


def draw_seq_lens(wl: Workload, gen: torch.Generator) -> torch.Tensor:
    if wl.prefix is not None:
        return torch.full((wl.batch,), wl.prefix, dtype=torch.int32)
    base = torch.randint(512, 4096 + 1, (wl.batch,), generator=gen, dtype=torch.int64)
    accepted = torch.randint(1, 5 + 1, (wl.batch,), generator=gen, dtype=torch.int64)
    return (base + accepted).to(torch.int32)


def max_seq_for(wl: Workload, seq_lens: torch.Tensor) -> int:
    # Capacity rounded to 64 rows so that the window-1 variant of a workload
    # shares the caches of its window-6 draw.
    return _round_up(int(seq_lens.max().item()) + max(wl.window, PBD_WINDOW), 64)


def generate(wl: Workload, layers: Optional[int] = None,
             max_seq: Optional[int] = None) -> WorkloadInputs:
    """Draw the workload's inputs on the CPU (fp32 draws rounded to bf16)."""
    gen = torch.Generator().manual_seed(wl.seed)
    seq_lens = draw_seq_lens(wl, gen)
    offsets = None
    if wl.k_seq_offset_std > 0:
        offsets = torch.randn(wl.batch, generator=gen) * wl.k_seq_offset_std
    s_max = max_seq if max_seq is not None else max_seq_for(wl, seq_lens)
    B, W, Hq, Hkv, D = wl.batch, wl.window, wl.num_q_heads, wl.num_kv_heads, wl.head_dim
    n_layers = wl.layers if layers is None else layers
    out = []
    for _ in range(n_layers):
        gain = None
        if wl.k_outlier_frac > 0:
            n_out = math.ceil(wl.k_outlier_frac * Hkv * D)
            picks = torch.randperm(Hkv * D, generator=gen)[:n_out]
            gain = torch.ones(Hkv * D)
            gain[picks] = wl.k_outlier_gain
            gain = gain.view(Hkv, D)
        k_cache = torch.randn(B, Hkv, s_max, D, generator=gen)
        v_cache = torch.randn(B, Hkv, s_max, D, generator=gen)
        k_new = torch.randn(B, W, Hkv, D, generator=gen)
        v_new = torch.randn(B, W, Hkv, D, generator=gen)
        q = torch.randn(B, W, Hq, D, generator=gen)
        if gain is not None:
            k_cache = k_cache * gain.view(1, Hkv, 1, D)
            k_new = k_new * gain.view(1, 1, Hkv, D)
        if offsets is not None:
            k_cache = k_cache + offsets.view(B, 1, 1, 1)
            k_new = k_new + offsets.view(B, 1, 1, 1)
        bf = torch.bfloat16
        out.append(LayerInputs(q.to(bf), k_cache.to(bf), v_cache.to(bf),
                               k_new.to(bf), v_new.to(bf)))
    return WorkloadInputs(wl, seq_lens, s_max, out)


def random_case(batch: int, prefix_lens, window: int, num_q_heads: int = NUM_Q_HEADS,
                num_kv_heads: int = NUM_KV_HEADS, head_dim: int = HEAD_DIM,
                seed: int = 1234, max_seq: Optional[int] = None,
                stale_fill: Optional[float] = None) -> WorkloadInputs:
    """A small seeded case with explicit prefix lengths (edge-case tests).

    ``stale_fill`` (e.g. NaN) overwrites cache rows at and beyond P_b + W so a
    read of a row outside the visible range shows up in the output.
    """
    gen = torch.Generator().manual_seed(seed)
    seq_lens = torch.tensor(list(prefix_lens), dtype=torch.int32)
    assert seq_lens.numel() == batch
    s_max = max_seq if max_seq is not None else _round_up(int(seq_lens.max()) + window, 8)
    B, W, Hq, Hkv, D = batch, window, num_q_heads, num_kv_heads, head_dim
    k_cache = torch.randn(B, Hkv, s_max, D, generator=gen)
    v_cache = torch.randn(B, Hkv, s_max, D, generator=gen)
    k_new = torch.randn(B, W, Hkv, D, generator=gen)
    v_new = torch.randn(B, W, Hkv, D, generator=gen)
    q = torch.randn(B, W, Hq, D, generator=gen)
    if stale_fill is not None:
        for b in range(B):
            lo = int(seq_lens[b]) + W
            k_cache[b, :, lo:, :] = stale_fill
            v_cache[b, :, lo:, :] = stale_fill
    wl = Workload(f"case_s{seed}", batch=B, layers=1, prefix=None, window=W, seed=seed,
                  num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D)
    bf = torch.bfloat16
    return WorkloadInputs(wl, seq_lens, s_max,
                          [LayerInputs(q.to(bf), k_cache.to(bf), v_cache.to(bf),
                                       k_new.to(bf), v_new.to(bf))])


def algorithmic_bytes(seq_lens, window: int, num_q_heads: int = NUM_Q_HEADS,
                      num_kv_heads: int = NUM_KV_HEADS, head_dim: int = HEAD_DIM) -> int:
    """Bytes one attention call must move at minimum (bf16 everywhere).

    K and V rows [0, P_b + W) of every KV head are read once; Q is read and the
    output written once. The window append adds its new rows (read + write).
    """
    tokens = sum(int(p) + window for p in seq_lens)
    kv = 2 * num_kv_heads * tokens * head_dim * 2
    qo = 2 * len(seq_lens) * window * num_q_heads * head_dim * 2
    return kv + qo


def append_bytes(batch: int, window: int, num_kv_heads: int = NUM_KV_HEADS,
                 head_dim: int = HEAD_DIM) -> int:
    """Bytes of one window append: new K and V rows read once and written once."""
    return 2 * 2 * batch * window * num_kv_heads * head_dim * 2


@dataclasses.dataclass
class PrefillInputs:
    q: torch.Tensor          # bf16 [B, T, Hq, D]
    k_cache: torch.Tensor    # bf16 [B, Hkv, S, D], rows [0, T_b) hold sequence b
    v_cache: torch.Tensor    # bf16 [B, Hkv, S, D]
    seq_lens: torch.Tensor   # int32 [B] = T_b
    scale: float


def prefill_case(lens, num_q_heads: int = NUM_Q_HEADS, num_kv_heads: int = NUM_KV_HEADS,
                 head_dim: int = HEAD_DIM, seed: int = 1234, t_max: Optional[int] = None,
                 max_seq: Optional[int] = None, stale_fill: Optional[float] = None) -> PrefillInputs:
    """Seeded inputs of a block-causal prefill: N(0,1) fp32 draws rounded to bf16, drawn in
    the order K cache, V cache, Q. ``stale_fill`` overwrites cache rows at and beyond T_b and
    q rows at and beyond T_b (padding) so that a read outside the valid range shows."""
    gen = torch.Generator().manual_seed(seed)
    lens = [int(x) for x in lens]
    B = len(lens)
    T = t_max if t_max is not None else max(1, max(lens))
    S = max_seq if max_seq is not None else _round_up(T, 8)
    k = torch.randn(B, num_kv_heads, S, head_dim, generator=gen).to(torch.bfloat16)
    v = torch.randn(B, num_kv_heads, S, head_dim, generator=gen).to(torch.bfloat16)
    q = torch.randn(B, T, num_q_heads, head_dim, generator=gen).to(torch.bfloat16)
    if stale_fill is not None:
        for b, n in enumerate(lens):
            k[b, :, n:] = stale_fill
            v[b, :, n:] = stale_fill
            q[b, n:] = stale_fill
    return PrefillInputs(q, k, v, torch.tensor(lens, dtype=torch.int32),
                         1.0 / math.sqrt(head_dim))
