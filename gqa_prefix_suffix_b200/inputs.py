"""Seeded synthetic inputs for the suffix attention, shared by the CUDA path's
tests/benchmark and by the oracle's tests.

This module draws random numbers and lays them out; it holds none of the
attention arithmetic.  Recipe (one generator per call, fixed draw order):

1. ``torch.Generator().manual_seed(seed)`` on the CPU.
2. If the valid length is random, draw it first (integer, inclusive range).
3. Draw fp32 N(0,1) for Q [B,Hq,S,D], K_prefix, V_prefix [B,Hkv,P,D],
   K_suffix, V_suffix [B,Hkv,S,D], in that order.
4. Peaked keys: per sample, ``round(peak_frac * P)`` prefix rows chosen
   uniformly without replacement over [0, P); those K rows (all KV heads) are
   multiplied by ``peak_mult``.  This makes some logits large, so the softmax
   is peaked.
5. Extra mask: per sample, ``round(mask_frac * valid_len)`` positions in
   [0, valid_len) chosen without replacement are hidden (mask byte 0).
6. Every value is rounded once to bf16 (round to nearest even).

Padding rows [valid_len, P) keep ordinary N(0,1) data (not zeros), so that a
kernel that wrongly reads them changes its result.

Shapes follow the pages: head_dim 256 and 8 query heads over 4 KV heads
(page "TensorRT+Triton+FlexAttention: OpenDM VLA 快速推理加速栈深度剖析", section
2.2 shape table), action chunks of 50 (base model, RoboTwin) and 10 (LIBERO)
(page "DM05 推理指南", section 2 table), prefix buckets 576/704/768/896/1024
(same page, section "Fast Backend 约束") and a single 2048 bucket for the
history demos (first page, section 3).  The pages name LIBERO and RoboTwin
only as checkpoints; no dataset item is used or needed: these synthetic
tensors stand in for the prefix/suffix activations.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional

import torch

HQ, HKV, HEAD_DIM = 8, 4, 256
PREFIX_BUCKETS = (576, 704, 768, 896, 1024)


@dataclass
class SuffixAttnInputs:
    name: str
    B: int
    Hq: int
    Hkv: int
    P: int
    S: int
    D: int
    q: torch.Tensor                      # bf16 [B,Hq,S,D]
    k_prefix: torch.Tensor               # bf16 [B,Hkv,P,D]
    v_prefix: torch.Tensor               # bf16 [B,Hkv,P,D]
    k_suffix: torch.Tensor               # bf16 [B,Hkv,S,D]
    v_suffix: torch.Tensor               # bf16 [B,Hkv,S,D]
    prefix_valid_len: Optional[torch.Tensor] = None   # int32 [B]
    prefix_mask: Optional[torch.Tensor] = None        # uint8 [B,P], 1 = visible
    meta: dict = field(default_factory=dict)

    def tensors(self):
        return dict(q=self.q, k_prefix=self.k_prefix, v_prefix=self.v_prefix,
                    prefix_valid_len=self.prefix_valid_len, prefix_mask=self.prefix_mask,
                    k_suffix=self.k_suffix, v_suffix=self.v_suffix)

    def dims(self):
        return dict(B=self.B, Hq=self.Hq, Hkv=self.Hkv, P=self.P, S=self.S, D=self.D)

    def to(self, device, non_blocking=False):
        def mv(t):
            return None if t is None else t.to(device, non_blocking=non_blocking)
        return SuffixAttnInputs(self.name, self.B, self.Hq, self.Hkv, self.P, self.S, self.D,
                                mv(self.q), mv(self.k_prefix), mv(self.v_prefix),
                                mv(self.k_suffix), mv(self.v_suffix),
                                mv(self.prefix_valid_len), mv(self.prefix_mask), dict(self.meta))


def _randn(gen, shape):
    return torch.randn(shape, generator=gen, dtype=torch.float32)


def make_inputs(B: int, Hq: int, Hkv: int, P: int, S: int, D: int, seed: int, *,
                valid_len=None, valid_range=None, peak_frac: float = 0.0,
                peak_mult: float = 1.0, mask_frac: float = 0.0,
                name: str = "custom", prefix=None) -> SuffixAttnInputs:
    """Draw one seeded input set following the module recipe.

    valid_len: None (no valid-length tensor: every prefix row visible), an int
    (same for all samples) or a list of B ints.  valid_range=(lo, hi) draws
    each sample's valid length uniformly from the inclusive range instead.
    prefix=(k_prefix, v_prefix) reuses an existing prefix cache (fp32 draws
    for it are then skipped)."""
    gen = torch.Generator().manual_seed(int(seed))
    if valid_range is not None:
        lo, hi = valid_range
        vl = torch.randint(int(lo), int(hi) + 1, (B,), generator=gen, dtype=torch.int64).to(torch.int32)
    elif valid_len is None:
        vl = None
    elif isinstance(valid_len, int):
        vl = torch.full((B,), valid_len, dtype=torch.int32)
    else:
        vl = torch.tensor(list(valid_len), dtype=torch.int32)
        assert vl.numel() == B
    q = _randn(gen, (B, Hq, S, D))
    if prefix is None:
        kp = _randn(gen, (B, Hkv, P, D))
        vp = _randn(gen, (B, Hkv, P, D))
    ks = _randn(gen, (B, Hkv, S, D))
    vs = _randn(gen, (B, Hkv, S, D))
    peaks: List[List[int]] = []
    if prefix is None and peak_frac > 0.0 and P > 0:
        n_peak = int(round(peak_frac * P))
        for b in range(B):
            rows = torch.randperm(P, generator=gen)[:n_peak]
            kp[b, :, rows, :] *= peak_mult
            peaks.append(sorted(rows.tolist()))
    mask = None
    if mask_frac > 0.0:
        mask = torch.ones((B, P), dtype=torch.uint8)
        for b in range(B):
            v = P if vl is None else max(0, min(P, int(vl[b])))
            n_hide = int(round(mask_frac * v))
            if n_hide > 0:
                hide = torch.randperm(v, generator=gen)[:n_hide]
                mask[b, hide] = 0
    bf = torch.bfloat16
    if prefix is None:
        kp_b, vp_b = kp.to(bf), vp.to(bf)
    else:
        kp_b, vp_b = prefix
    return SuffixAttnInputs(name, B, Hq, Hkv, P, S, D, q.to(bf), kp_b, vp_b, ks.to(bf), vs.to(bf),
                            vl, mask, dict(seed=int(seed), peak_rows=peaks,
                                           peak_frac=peak_frac, peak_mult=peak_mult,
                                           mask_frac=mask_frac))


# --- the five workloads -------------------------------------------------------

def libero_tiny() -> SuffixAttnInputs:
    """LIBERO-shape chunk: B=1, P=576 bucket, 512 valid prefix rows, S=10."""
    return make_inputs(1, HQ, HKV, 576, 10, HEAD_DIM, 1000, valid_len=512,
                       name="libero_tiny_b1_p576_v512_s10")


def base_chunk() -> SuffixAttnInputs:
    """Base-model chunk: B=1, P=1024 bucket, 900 valid rows, S=50; 5 % of the
    prefix K rows scaled by 3.0 (peaked softmax)."""
    return make_inputs(1, HQ, HKV, 1024, 50, HEAD_DIM, 1001, valid_len=900,
                       peak_frac=0.05, peak_mult=3.0, name="base_chunk_b1_p1024_v900_s50")


def bucket_sweep() -> List[SuffixAttnInputs]:
    """S=50 over every default prefix bucket, valid length ~ U[P-128, P],
    five calls per bucket with seed 2000 + 10*bucket_index + call."""
    out = []
    for bi, P in enumerate(PREFIX_BUCKETS):
        for call in range(5):
            out.append(make_inputs(1, HQ, HKV, P, 50, HEAD_DIM, 2000 + 10 * bi + call,
                                   valid_range=(P - 128, P),
                                   name=f"bucket_sweep_b1_p{P}_s50_call{call}"))
    return out


def history_loop(n_steps: int = 10) -> List[SuffixAttnInputs]:
    """Long-prefix denoising loop: one P=2048 prefix cache (seed 3000, 1900
    valid rows) reused by n_steps calls with fresh suffix Q/K/V (seeds
    3001...)."""
    base = make_inputs(1, HQ, HKV, 2048, 50, HEAD_DIM, 3000, valid_len=1900,
                       name="history_prefix")
    calls = []
    for step in range(n_steps):
        calls.append(make_inputs(1, HQ, HKV, 2048, 50, HEAD_DIM, 3001 + step, valid_len=1900,
                                 prefix=(base.k_prefix, base.v_prefix),
                                 name=f"history_b1_p2048_v1900_s50_step{step}"))
    return calls


def batched_mask() -> SuffixAttnInputs:
    """Batched throughput: B=32, P=1024, S=50, valid length ~ U[576, 1024],
    a further 10 % of in-range positions hidden, 1 % of K rows scaled by 4."""
    return make_inputs(32, HQ, HKV, 1024, 50, HEAD_DIM, 4000, valid_range=(576, 1024),
                       peak_frac=0.01, peak_mult=4.0, mask_frac=0.10,
                       name="batched_b32_p1024_s50_mask")


# --- prefix prefill (the step that fills the prefix KV cache) ---------------

@dataclass
class PrefillInputs:
    """One prefix-prefill attention call: the P prefix positions attend to
    the prefix K/V of the same call under the prefix-causal mask."""
    name: str
    B: int
    Hq: int
    Hkv: int
    P: int
    D: int
    q: torch.Tensor                      # bf16 [B,Hq,P,D]
    k: torch.Tensor                      # bf16 [B,Hkv,P,D]
    v: torch.Tensor                      # bf16 [B,Hkv,P,D]
    valid_len: Optional[torch.Tensor] = None   # int32 [B]

    def to(self, device):
        mv = lambda t: None if t is None else t.to(device)
        return PrefillInputs(self.name, self.B, self.Hq, self.Hkv, self.P, self.D, mv(self.q), mv(self.k),
                             mv(self.v), mv(self.valid_len))

    def tensors(self):
        return dict(q=self.q, k=self.k, v=self.v, valid_len=self.valid_len)


def make_prefill_inputs(B: int, Hq: int, Hkv: int, P: int, D: int, seed: int, *, valid_len=None,
                        valid_range=None, name: str = "prefill") -> PrefillInputs:
    """Seeded prefill inputs: valid length (fixed, per-sample list, or drawn
    from an inclusive range first), then fp32 N(0,1) Q [B,Hq,P,D], K, V
    [B,Hkv,P,D] in that order, each rounded once to bf16.  Padding rows keep
    ordinary data."""
    gen = torch.Generator().manual_seed(int(seed))
    if valid_range is not None:
        lo, hi = valid_range
        vl = torch.randint(int(lo), int(hi) + 1, (B,), generator=gen, dtype=torch.int64).to(torch.int32)
    elif valid_len is None:
        vl = None
    elif isinstance(valid_len, int):
        vl = torch.full((B,), valid_len, dtype=torch.int32)
    else:
        vl = torch.tensor(list(valid_len), dtype=torch.int32)
    bf = torch.bfloat16
    q = _randn(gen, (B, Hq, P, D)).to(bf)
    k = _randn(gen, (B, Hkv, P, D)).to(bf)
    v = _randn(gen, (B, Hkv, P, D)).to(bf)
    return PrefillInputs(name, B, Hq, Hkv, P, D, q, k, v, vl)


def prefill_base() -> PrefillInputs:
    """Prefix prefill of the base-model chunk's prefix: B=1, P=1024 bucket
    with 900 valid positions, 8/4 heads (the prefix decoder's shape), D=256."""
    return make_prefill_inputs(1, HQ, HKV, 1024, HEAD_DIM, 5001, valid_len=900, name="prefill_b1_p1024_v900")


def prefill_history() -> PrefillInputs:
    """Prefix prefill of the history demo's prefix: B=1, P=2048, 1900 valid."""
    return make_prefill_inputs(1, HQ, HKV, 2048, HEAD_DIM, 5002, valid_len=1900, name="prefill_b1_p2048_v1900")


# --- suffix prologue (QKV projection + QK-Norm + RoPE) -----------------------

@dataclass
class PrologueInputs:
    """One suffix-prologue call: the action tokens' hidden states, the QKV
    weight and the QK-Norm weights, and each token's position."""
    name: str
    B: int
    S: int
    H: int
    Hq: int
    Hkv: int
    D: int
    x: torch.Tensor        # bf16 [B*S, H]
    w: torch.Tensor        # bf16 [(Hq + 2*Hkv)*D, H]: query heads, key heads, value heads
    qw: torch.Tensor       # bf16 [D]
    kw: torch.Tensor       # bf16 [D]
    pos: torch.Tensor      # int32 [B*S]

    def to(self, device):
        return PrologueInputs(self.name, self.B, self.S, self.H, self.Hq, self.Hkv, self.D, self.x.to(device),
                              self.w.to(device), self.qw.to(device), self.kw.to(device), self.pos.to(device))

    def tensors(self):
        return dict(x=self.x, w=self.w, qw=self.qw, kw=self.kw, pos=self.pos)


def make_prologue_inputs(B: int, S: int, seed: int, *, H: int = 1024, Hq: int = HQ, Hkv: int = HKV,
                         D: int = HEAD_DIM, pos0=0, name: str = "prologue") -> PrologueInputs:
    """Seeded prologue inputs: fp32 N(0,1) hidden states x [B*S, H]; the QKV
    weight N(0,1) / sqrt(H) (so projections are O(1)); QK-Norm weights
    1 + 0.1 N(0,1); all rounded once to bf16.  Token i of sample b sits at
    position pos0[b] + i (pos0 an int or a list of B ints: the suffix follows
    the prefix)."""
    gen = torch.Generator().manual_seed(int(seed))
    bf = torch.bfloat16
    x = _randn(gen, (B * S, H)).to(bf)
    w = (_randn(gen, ((Hq + 2 * Hkv) * D, H)) / (H ** 0.5)).to(bf)
    qw = (1.0 + 0.1 * _randn(gen, (D,))).to(bf)
    kw = (1.0 + 0.1 * _randn(gen, (D,))).to(bf)
    p0 = [pos0] * B if isinstance(pos0, int) else list(pos0)
    pos = torch.tensor([p0[b] + i for b in range(B) for i in range(S)], dtype=torch.int32)
    return PrologueInputs(name, B, S, H, Hq, Hkv, D, x, w, qw, kw, pos)


def prologue_base() -> PrologueInputs:
    """The base-model chunk's prologue: B=1, S=50 action tokens after a
    900-token prefix, hidden 1024, 8/4 heads, D=256 (the action expert's
    shape)."""
    return make_prologue_inputs(1, 50, 6001, pos0=900, name="prologue_b1_s50_h1024")


def prologue_batched() -> PrologueInputs:
    """The batched workload's prologue: B=32 chunks of S=50 tokens."""
    gen = torch.Generator().manual_seed(6002)
    starts = torch.randint(576, 1025, (32,), generator=gen).tolist()
    return make_prologue_inputs(32, 50, 6003, pos0=starts, name="prologue_b32_s50_h1024")


# --- post-attention block (output projection, Adarms, GEGLU, MLP down) -------

@dataclass
class PostAttnInputs:
    """One post-attention block call of an action-expert layer."""
    name: str
    B: int
    S: int
    Hq: int
    D: int
    Hd: int
    F: int
    attn: torch.Tensor    # bf16 [B, Hq, S, D]: the suffix attention's output
    h: torch.Tensor       # bf16 [B*S, Hd]: residual stream entering the layer
    scale: torch.Tensor   # bf16 [B, Hd]: time modulation (per sample)
    shift: torch.Tensor   # bf16 [B, Hd]
    gate: torch.Tensor    # bf16 [B, Hd]
    wo: torch.Tensor      # bf16 [Hd, Hq*D]
    wgu: torch.Tensor     # bf16 [2F, Hd]: gate rows, then up rows
    wd: torch.Tensor      # bf16 [Hd, F]

    def to(self, device):
        f = {k: getattr(self, k).to(device) for k in self.tensors()}
        return PostAttnInputs(self.name, self.B, self.S, self.Hq, self.D, self.Hd, self.F, **f)

    def tensors(self):
        return dict(attn=self.attn, h=self.h, scale=self.scale, shift=self.shift, gate=self.gate, wo=self.wo,
                    wgu=self.wgu, wd=self.wd)


def make_post_inputs(B: int, S: int, seed: int, *, Hq: int = HQ, D: int = HEAD_DIM, Hd: int = 1024,
                     F: int = 4096, name: str = "post") -> PostAttnInputs:
    """Seeded post-attention inputs, drawn in this order as fp32 N(0,1) and
    rounded once to bf16: attention output, residual, then the time
    modulation scale and shift (x 0.1) and gate (x 0.5), then the weights
    scaled by 1/sqrt(fan-in) so every projection is O(1)."""
    gen = torch.Generator().manual_seed(int(seed))
    bf = torch.bfloat16
    attn = _randn(gen, (B, Hq, S, D)).to(bf)
    h = _randn(gen, (B * S, Hd)).to(bf)
    scale = (0.1 * _randn(gen, (B, Hd))).to(bf)
    shift = (0.1 * _randn(gen, (B, Hd))).to(bf)
    gate = (0.5 * _randn(gen, (B, Hd))).to(bf)
    wo = (_randn(gen, (Hd, Hq * D)) / (Hq * D) ** 0.5).to(bf)
    wgu = (_randn(gen, (2 * F, Hd)) / Hd ** 0.5).to(bf)
    wd = (_randn(gen, (Hd, F)) / F ** 0.5).to(bf)
    return PostAttnInputs(name, B, S, Hq, D, Hd, F, attn, h, scale, shift, gate, wo, wgu, wd)


def post_base() -> PostAttnInputs:
    """The base-model chunk's post-attention block: B=1, S=50, hidden 1024,
    intermediate 4096, 8 heads of 256."""
    return make_post_inputs(1, 50, 8001, name="post_b1_s50_h1024_f4096")


def post_batched() -> PostAttnInputs:
    """The batched workload's post-attention block: B=32, S=50."""
    return make_post_inputs(32, 50, 8002, name="post_b32_s50_h1024_f4096")


WORKLOADS = {
    "libero_tiny": libero_tiny,
    "base_chunk": base_chunk,
    "bucket_sweep": bucket_sweep,
    "history_loop": history_loop,
    "batched_mask": batched_mask,
}
