"""Seeded synthetic workloads for the DeepSeek Sparse Attention hot path.

This module only draws random numbers and arranges them into the shapes the
hot path consumes.  It holds none of the method's arithmetic (no Hadamard
rotation, no FP8 quantisation, no scoring, no selection, no attention), so the
CPU oracle and the CUDA path can both read the same inputs without sharing any
of the computation.

Shapes follow the V3.2-Exp sizes shown on the pages:
  * "DeepSeek-V3.2-Exp - Split indexer heads", Indexer.forward: indexer queries
    [B, S, H=64, D=128], one shared key per token [B, S, D], per-head weights
    [B, S, H].
  * "DeepSeek Sparse Attention, one decode step in one layer (V3.2 sizes)"
    diagram: top-k = 2048, core attention with 128 heads over 576-wide latent
    rows (512 latent + 64 rotary), each latent row being key and value.

Every tensor is drawn in fp32 from ``torch.Generator('cpu')`` and then cast to
the stated dtype.  Seeds: 0 for the tiny prefill case; ``1000 * cfg + b`` for
sequence ``b`` of every other case, so one sequence can be regenerated alone.
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    cfg: int
    name: str
    mode: str            # "prefill" (S = T, start_pos = 0) or "decode" (S = 1)
    B: int
    T: int               # end_pos: tokens visible to the step
    H: int               # indexer heads
    D: int               # indexer head dim (= act_quant block)
    rope: int            # rotary part of the indexer head (layout only)
    topk: int            # index_topk
    Hq: int              # MLA heads
    dc: int              # latent (kv_lora_rank)
    dr: int              # shared rotary key width
    attn_dtype: str      # "f32" (test mode) or "bf16"
    planted_frac: float = 0.0

    @property
    def K(self) -> int:
        """Selected slots per query: min(index_topk, end_pos)."""
        return min(self.topk, self.T)

    @property
    def dqk(self) -> int:
        return self.dc + self.dr

    @property
    def softmax_scale_idx(self) -> float:
        """Indexer softmax scale: D^-1/2 (the pages leave it unstated)."""
        return self.D ** -0.5

    @property
    def sm_scale(self) -> float:
        """Latent-attention scale: (dc + dr)^-1/2 (an explicit argument)."""
        return (self.dc + self.dr) ** -0.5

    def seed(self, b: int) -> int:
        return 0 if self.cfg == 0 else 1000 * self.cfg + b


WORKLOADS = {
    0: Workload(0, "tiny_prefill_T128", "prefill", B=1, T=128, H=4, D=64, rope=16,
                topk=16, Hq=8, dc=64, dr=16, attn_dtype="f32"),
    1: Workload(1, "decode_B1_T4096", "decode", B=1, T=4096, H=64, D=128, rope=64,
                topk=2048, Hq=128, dc=512, dr=64, attn_dtype="bf16"),
    2: Workload(2, "decode_B32_T32768", "decode", B=32, T=32768, H=64, D=128, rope=64,
                topk=2048, Hq=128, dc=512, dr=64, attn_dtype="bf16"),
    3: Workload(3, "prefill_T8192", "prefill", B=1, T=8192, H=64, D=128, rope=64,
                topk=2048, Hq=128, dc=512, dr=64, attn_dtype="bf16"),
    4: Workload(4, "decode_B8_T131072_planted", "decode", B=8, T=131072, H=64, D=128,
                rope=64, topk=2048, Hq=128, dc=512, dr=64, attn_dtype="bf16",
                planted_frac=0.01),
}


def _torch_dtype(name: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def _randn(g: torch.Generator, *shape: int) -> torch.Tensor:
    return torch.randn(*shape, generator=g, dtype=torch.float32)


def decode_sequence(wl: Workload, b: int, T: int | None = None) -> dict:
    """Inputs of one decode step for sequence ``b`` (CPU tensors).

    keys      [T, D]       fp32 raw indexer keys (post-RoPE, pre-rotation);
                           position T-1 is the new token's key.
    q_idx     [H, D]       fp32 new token's indexer queries (post-RoPE).
    w         [H]          fp32 per-head weights (weights_proj output).
    q_mla     [Hq, dc+dr]  attention query in latent space (absorbed), attn dtype.
    kv        [T, dc+dr]   latent rows [c | k_pe], attn dtype; row T-1 is the new one.
    planted   [n] int64    positions whose keys were planted (empty if none).
    """
    T = wl.T if T is None else T
    g = torch.Generator().manual_seed(wl.seed(b))
    q_idx = _randn(g, wl.H, wl.D)
    w = _randn(g, wl.H)
    keys = _randn(g, T, wl.D)
    q_mla = _randn(g, wl.Hq, wl.dqk)
    kv = _randn(g, T, wl.dqk)
    n_plant = int(math.floor(wl.planted_frac * T))
    planted = torch.empty(0, dtype=torch.int64)
    if n_plant > 0:
        planted = torch.randperm(T, generator=g)[:n_plant].sort().values
        # A key aligned with the positively weighted queries: k = sqrt(D) r/|r|,
        # r = sum over heads with w_h > 0 of w_h q_h.  Such keys score high.
        pos = w > 0
        r = (w[pos, None] * q_idx[pos]).sum(0)
        k_hot = r * (math.sqrt(wl.D) / float(r.norm()))
        keys[planted] = k_hot
    dt = _torch_dtype(wl.attn_dtype)
    return dict(q_idx=q_idx, w=w, keys=keys, q_mla=q_mla.to(dt), kv=kv.to(dt),
                planted=planted)


def prefill_inputs(wl: Workload, T: int | None = None) -> dict:
    """Inputs of one prefill pass (B sequences, S = T queries, start_pos = 0).

    q_idx [B,T,H,D] fp32, keys [B,T,D] fp32, w [B,T,H] fp32,
    q_mla [B,T,Hq,dc+dr] and kv [B,T,dc+dr] in the attention dtype.
    """
    T = wl.T if T is None else T
    qs, ks, ws, qm, kvs = [], [], [], [], []
    for b in range(wl.B):
        g = torch.Generator().manual_seed(wl.seed(b))
        qs.append(_randn(g, T, wl.H, wl.D))
        ws.append(_randn(g, T, wl.H))
        ks.append(_randn(g, T, wl.D))
        qm.append(_randn(g, T, wl.Hq, wl.dqk))
        kvs.append(_randn(g, T, wl.dqk))
    dt = _torch_dtype(wl.attn_dtype)
    return dict(q_idx=torch.stack(qs), w=torch.stack(ws), keys=torch.stack(ks),
                q_mla=torch.stack(qm).to(dt), kv=torch.stack(kvs).to(dt))


def score_rows(rows: int, T: int, seed: int, tie_frac: float = 0.0) -> torch.Tensor:
    """Synthetic fp32 score rows [rows, T] ~N(0,1) for selection tests.

    With ``tie_frac`` > 0 that fraction of each row is overwritten with copies
    of a few shared values, so that exact ties occur (also at the k-th place).
    """
    g = torch.Generator().manual_seed(seed)
    s = _randn(g, rows, T)
    if tie_frac > 0:
        n = max(1, int(tie_frac * T))
        for r in range(rows):
            pos = torch.randperm(T, generator=g)[:n]
            vals = _randn(g, 4)
            s[r, pos] = vals[torch.randint(0, 4, (n,), generator=g)]
    return s


def random_indices(B: int, S: int, K: int, T: int, start_pos: int, seed: int,
                   fill: float = 1.0) -> torch.Tensor:
    """Distinct causal indices [B, S, K] int32 with -1 in unused slots.

    Row (b, s) may use positions 0..start_pos+s; it gets
    round(fill * min(K, start_pos+s+1)) of them, in random order.
    """
    g = torch.Generator().manual_seed(seed)
    out = torch.full((B, S, K), -1, dtype=torch.int32)
    for b in range(B):
        for s in range(S):
            n_valid = min(T, start_pos + s + 1)
            m = int(round(fill * min(K, n_valid)))
            pick = torch.randperm(n_valid, generator=g)[:m]
            slots = torch.randperm(K, generator=g)[:m]
            out[b, s, slots] = pick.to(torch.int32)
    return out
