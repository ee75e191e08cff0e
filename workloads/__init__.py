"""Seeded synthetic inputs for causal self-attention, shared by the oracle side and the CUDA side.

This module holds no attention arithmetic: it only names the workloads and draws their inputs. Both the
float64 oracle (``oracle/``) and the CUDA path (``causal_self_attention_bf16_b200``) receive the same bf16
tensors from here, so that a parity comparison sees identical bytes.

Shapes follow nanochat's single depth dial: the model width is 64 * depth and every head has 128 dims, so
depth d gives H = d / 2 heads (apidog "Train your own ChatGPT", section "Philosophy: one dial"; aisight.pl
nanochat review, "Model and scaling assumptions": d20 = 1280 channels, 10 heads of 128). Rows are full
2048-token packed sequences (apidog, section 4 "Data loading", best-fit packing to 2048), and the device batch
is 32, halved to 16 for d24/d26 (ja.news.hada.io summary, "Bigger models"; apidog leaderboard run 6 flags).

Layout of every tensor: [B, T, H, D] contiguous, the layout the pages' model reshapes into before calling
``flash_attn_func`` (apidog, section 1 "GPT model", the value-embedding ``view(B, T, n_kv_head, head_dim)``).
Grouped-query workloads (the same section lists grouped-query attention, fewer key/value heads than query
heads) give k and v H_kv heads: [B, T, H_kv, D].
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import torch

HEAD_DIM = 128


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic attention workload: shape, value recipe and seed."""

    name: str
    B: int
    H: int
    T: int
    D: int = HEAD_DIM
    Hkv: int = 0                 # key/value heads (grouped-query attention); 0 means H
    window: int = -1             # sliding window: a query sees itself and this many keys before it; -1: none
    seed: int = 0
    qk_prescale: float = 1.0     # multiply the fp32 draws of q and k by this before the bf16 cast
    key_bias: bool = False       # add one shared N(0,1) vector of length D to every key row
    recipe: str = ""

    @property
    def kv_heads(self) -> int:
        return self.Hkv if self.Hkv else self.H

    @property
    def scale(self) -> float:
        """Softmax scale 1/sqrt(D) (the usual choice; the pages do not print it)."""
        return 1.0 / math.sqrt(self.D)

    @property
    def fwd_flops(self) -> float:
        """Causal forward FLOPs by the convention 2*B*H*T^2*D (half of the dense 4*B*H*T^2*D); with a sliding
        window, scaled by the fraction of the causal (query, key) pairs that stay inside the window."""
        f = 2.0 * self.B * self.H * self.T * self.T * self.D
        if self.window >= 0:
            T, W = self.T, self.window
            kept = sum(min(i, W) + 1 for i in range(T)) if T <= 1 << 16 else T * (W + 1) - W * (W + 1) / 2
            f *= kept / (T * (T + 1) / 2)
        return f

    @property
    def bwd_flops(self) -> float:
        """Backward FLOPs counted as 2.5x the forward."""
        return 2.5 * self.fwd_flops

    def with_shape(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", B=1, H=2, T=128,
                     recipe="q,k,v,dO ~ N(0,1) fp32 from seed 0, cast to bf16"),
    "d12": Workload("d12", B=32, H=6, T=2048, qk_prescale=0.5,
                    recipe="q,k,v,dO ~ N(0,1); q,k multiplied by 0.5 before the bf16 cast"),
    "d20": Workload("d20", B=32, H=10, T=2048,
                    recipe="q,k,v,dO ~ N(0,1) fp32 from seed 0, cast to bf16"),
    "d24": Workload("d24", B=16, H=12, T=2048, key_bias=True,
                    recipe="q,k,v,dO ~ N(0,1); one shared bias b ~ N(0,1)^D added to every key row"),
    "d26": Workload("d26", B=16, H=13, T=2048,
                    recipe="q,k,v,dO ~ N(0,1) fp32 from seed 0, cast to bf16"),
    # Grouped-query attention (the pages give no head counts for it; groups of 2 and 3 query heads per
    # key/value head here).
    "tiny_gqa": Workload("tiny_gqa", B=1, H=4, T=128, Hkv=2,
                         recipe="q,dO [B,T,4,D], k,v [B,T,2,D] ~ N(0,1) fp32 from seed 0, cast to bf16"),
    "d12_gqa": Workload("d12_gqa", B=32, H=6, T=2048, Hkv=2, qk_prescale=0.5,
                        recipe="d12 with 2 key/value heads: q,dO [B,T,6,D], k,v [B,T,2,D]; q,k times 0.5"),
    "d20_gqa": Workload("d20_gqa", B=32, H=10, T=2048, Hkv=5,
                        recipe="d20 with 5 key/value heads: q,dO [B,T,10,D], k,v [B,T,5,D] ~ N(0,1)"),
    # Sliding-window attention (the pages' "SSSL" layers: short-window layers between full-context ones; the
    # window length is not on the pages: a quarter of the context here).
    "tiny_sw": Workload("tiny_sw", B=1, H=2, T=300, window=100,
                        recipe="q,k,v,dO ~ N(0,1) fp32 from seed 0, cast to bf16; window 100"),
    "d20_sw": Workload("d20_sw", B=32, H=10, T=2048, window=512,
                       recipe="d20 shape and recipe, sliding window of 512 keys"),
}
# d26 sequence-length sweep at a fixed B*T = 32768 tokens per device.
for _T in (512, 1024, 2048, 4096):
    WORKLOADS[f"d26_T{_T}"] = Workload(f"d26_T{_T}", B=32768 // _T, H=13, T=_T,
                                       recipe="d26 heads, B*T = 32768 tokens, q,k,v,dO ~ N(0,1)")

HEADLINE = "d20"


def make_inputs(w: Workload, device: Optional[torch.device] = None, need_grad_input: bool = True):
    """Draw (q, k, v, dO) for a workload as bf16 tensors: q, dO [B, T, H, D]; k, v [B, T, H_kv, D].

    One CPU ``torch.Generator`` seeded with ``w.seed`` draws fp32 standard normals in the order q, k, v, dO and
    then (d24 only) the key bias. Pre-scaling and the bias are applied in fp32, then each tensor is rounded to
    bf16 (round to nearest even). The same bytes go to the GPU and, upcast exactly, to the oracle.
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed)
    shape = (w.B, w.T, w.H, w.D)
    kv_shape = (w.B, w.T, w.kv_heads, w.D)
    q = torch.randn(shape, generator=g, dtype=torch.float32)
    k = torch.randn(kv_shape, generator=g, dtype=torch.float32)
    v = torch.randn(kv_shape, generator=g, dtype=torch.float32)
    do = torch.randn(shape, generator=g, dtype=torch.float32) if need_grad_input else None
    if w.qk_prescale != 1.0:
        q.mul_(w.qk_prescale)
        k.mul_(w.qk_prescale)
    if w.key_bias:
        bias = torch.randn((w.D,), generator=g, dtype=torch.float32)
        k.add_(bias)
    out = [t.to(torch.bfloat16) if t is not None else None for t in (q, k, v, do)]
    if device is not None:
        out = [t.to(device) if t is not None else None for t in out]
    return tuple(out)


def key_bias_vector(w: Workload) -> torch.Tensor:
    """The shared key bias of a ``key_bias`` workload (fp32, length D), redrawn from the same stream."""
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed)
    n, nkv = w.B * w.T * w.H * w.D, w.B * w.T * w.kv_heads * w.D
    for size in (n, nkv, nkv, n):
        torch.randn((size,), generator=g, dtype=torch.float32)
    return torch.randn((w.D,), generator=g, dtype=torch.float32)


def sample_slices(w: Workload, k: int = 4, seed: int = 1234):
    """Seeded sample of (b, h) slices, always including (0, 0) and (B-1, H-1)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    picks = [(0, 0), (w.B - 1, w.H - 1)]
    while len(picks) < min(k, w.B * w.H):
        b = int(torch.randint(0, w.B, (1,), generator=g))
        h = int(torch.randint(0, w.H, (1,), generator=g))
        if (b, h) not in picks:
            picks.append((b, h))
    return picks


@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    """New queries against a key/value cache (the inference engine's cached decode): q [B, Tq, H, D], caches
    [B, Tk, H_kv, D], cache_seqlens [B] drawn uniformly from [min_len, Tk] (a seeded mix of lengths)."""

    name: str
    B: int
    H: int
    Hkv: int
    Tq: int
    Tk: int
    D: int = HEAD_DIM
    min_len: int = 1
    seed: int = 0
    window: int = -1             # sliding window (the model's short-window layers); -1: none
    recipe: str = ""

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)


DECODE_WORKLOADS: Dict[str, DecodeWorkload] = {
    "decode_tiny": DecodeWorkload("decode_tiny", B=3, H=4, Hkv=2, Tq=2, Tk=300, seed=1,
                                  recipe="q, caches ~ N(0,1) bf16; lengths uniform in [1, 300]"),
    "decode_d20": DecodeWorkload("decode_d20", B=64, H=10, Hkv=10, Tq=1, Tk=2048, seed=2,
                                 recipe="d20 heads, one new token per sequence, 64 sequences with cached lengths "
                                        "uniform in [1, 2048]; q, caches ~ N(0,1) bf16"),
    "decode_d20_gqa": DecodeWorkload("decode_d20_gqa", B=64, H=10, Hkv=5, Tq=1, Tk=2048, seed=3,
                                     recipe="decode_d20 with 5 key/value heads"),
    "decode_d20_sw": DecodeWorkload("decode_d20_sw", B=64, H=10, Hkv=10, Tq=1, Tk=2048, seed=2, window=512,
                                    recipe="decode_d20 through a short-window layer: window 512"),
}


def make_decode_inputs(w: DecodeWorkload, device: Optional[torch.device] = None):
    """(q, k_cache, v_cache, cache_seqlens): bf16 tensors and int32 lengths from one seeded CPU generator, in
    the order lengths, q, k_cache, v_cache."""
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed)
    lens = torch.randint(w.min_len, w.Tk + 1, (w.B,), generator=g, dtype=torch.int64).to(torch.int32)
    q = torch.randn((w.B, w.Tq, w.H, w.D), generator=g, dtype=torch.float32).to(torch.bfloat16)
    kc = torch.randn((w.B, w.Tk, w.Hkv, w.D), generator=g, dtype=torch.float32).to(torch.bfloat16)
    vc = torch.randn((w.B, w.Tk, w.Hkv, w.D), generator=g, dtype=torch.float32).to(torch.bfloat16)
    out = (q, kc, vc, lens)
    if device is not None:
        out = tuple(t.to(device) for t in out)
    return out



@dataclasses.dataclass(frozen=True)
class PrologueWorkload:
    """Raw q [B, T, H, D] and k [B, T, H_kv, D] before QK normalisation and the rotary embedding, plus the
    gradients of the prologue's outputs for its backward. Entries are N(0,1) times a per-row factor
    exp(N(0, 0.5^2)), so row norms differ as projections of a residual stream do; with `offsets`, each
    sequence starts at a position drawn uniformly from [0, max_offset] (decode's new tokens after a cache)."""

    name: str
    B: int
    T: int
    H: int
    Hkv: int
    D: int = HEAD_DIM
    rope_base: float = 10000.0
    eps: float = 1e-6
    pairing: str = "interleaved"
    max_offset: int = 0
    seed: int = 0
    recipe: str = ""


PROLOGUE_WORKLOADS: Dict[str, PrologueWorkload] = {
    "rope_tiny": PrologueWorkload("rope_tiny", B=2, T=37, H=5, Hkv=2, max_offset=100000, seed=11,
                                  recipe="ragged positions (74 < 5 blocks of 16), 7 rows per position, offsets up "
                                         "to 1e5"),
    "rope_d20": PrologueWorkload("rope_d20", B=32, T=2048, H=10, Hkv=10, seed=12,
                                 recipe="d20 training batch: 32 x 2048 tokens, 10 query and 10 key heads"),
    "rope_d20_gqa": PrologueWorkload("rope_d20_gqa", B=32, T=2048, H=10, Hkv=5, pairing="half", seed=13,
                                     recipe="rope_d20 with 5 key heads and the half pairing"),
}


def make_prologue_inputs(w: PrologueWorkload, device: Optional[torch.device] = None):
    """(q, k, dq_out, dk_out, offsets): bf16 tensors and int32 [B] offsets (None when max_offset is 0) from
    one seeded CPU generator, in the order q, q row factors, k, k row factors, dq_out, dk_out, offsets."""
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed)

    def rows(heads):
        x = torch.randn((w.B, w.T, heads, w.D), generator=g, dtype=torch.float32)
        f = torch.exp(0.5 * torch.randn((w.B, w.T, heads, 1), generator=g, dtype=torch.float32))
        return (x * f).to(torch.bfloat16)

    q, k = rows(w.H), rows(w.Hkv)
    dq = torch.randn((w.B, w.T, w.H, w.D), generator=g, dtype=torch.float32).to(torch.bfloat16)
    dk = torch.randn((w.B, w.T, w.Hkv, w.D), generator=g, dtype=torch.float32).to(torch.bfloat16)
    offs = None
    if w.max_offset > 0:
        offs = torch.randint(0, w.max_offset + 1, (w.B,), generator=g, dtype=torch.int64).to(torch.int32)
    out = (q, k, dq, dk, offs)
    if device is not None:
        out = tuple(None if t is None else t.to(device) for t in out)
    return out
