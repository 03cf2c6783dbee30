"""Checks that tie the fp64 oracle to facts outside itself.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises AssertionError
when the oracle disagrees with a fact that the pages or the mathematics fix:
a library routine that computes a special case (float64 scaled-dot-product
attention), a closed form, an invariant, or a brute force in independent
arithmetic.  ``test_oracle.py`` runs them on the real oracle;
``test_oracle_mutations.py`` shows that each planted mistake in a copy of the
oracle fails at least one of them.

The attention these pins describe is the action-expert suffix attention of
the page "TensorRT+Triton+FlexAttention: OpenDM VLA 快速推理加速栈深度剖析",
section 2.2: logits over the prefix KV cache and the suffix K/V under the
prefix-visibility mask, softmax, value-weighted sum; GQA with head_dim 256
and 8/4 heads (same section's shape table).
"""
from __future__ import annotations

import decimal
import math

import numpy as np
import torch

BF = torch.bfloat16


def bf16_rand(gen, shape, mult=1.0):
    return (torch.randn(shape, generator=gen, dtype=torch.float32) * mult).to(BF)


def rand_case(seed, B, Hq, Hkv, P, S, D, vl=None, mask_p=0.0, mult=1.0):
    gen = torch.Generator().manual_seed(seed)
    q = bf16_rand(gen, (B, Hq, S, D), mult)
    kp = bf16_rand(gen, (B, Hkv, P, D), mult)
    vp = bf16_rand(gen, (B, Hkv, P, D))
    ks = bf16_rand(gen, (B, Hkv, S, D), mult)
    vs = bf16_rand(gen, (B, Hkv, S, D))
    if vl is None:
        vlt = torch.randint(0, P + 1, (B,), generator=gen, dtype=torch.int64).to(torch.int32)
    else:
        vlt = torch.tensor(vl, dtype=torch.int32)
    mask = None
    if mask_p > 0.0:
        mask = (torch.rand((B, P), generator=gen) >= mask_p).to(torch.uint8)
    return dict(q=q, k_prefix=kp, v_prefix=vp, prefix_valid_len=vlt, prefix_mask=mask,
                k_suffix=ks, v_suffix=vs, B=B, Hq=Hq, Hkv=Hkv, P=P, S=S, D=D)


def run(orc, c, **kw):
    return orc.suffix_attn(c["q"], c["k_prefix"], c["v_prefix"], c["prefix_valid_len"],
                           c["prefix_mask"], c["k_suffix"], c["v_suffix"],
                           c["B"], c["Hq"], c["Hkv"], c["P"], c["S"], c["D"], **kw)


def visible_keys(c, b):
    """Boolean visibility of the P+S keys of sample b (prefix, then suffix)."""
    P, S = c["P"], c["S"]
    vl = P if c["prefix_valid_len"] is None else int(c["prefix_valid_len"][b])
    vl = max(0, min(P, vl))
    vis = np.zeros(P + S, dtype=bool)
    vis[:vl] = True
    if c["prefix_mask"] is not None:
        vis[:P] &= c["prefix_mask"][b].numpy() != 0
    vis[P:] = True
    return vis


def sdpa_reference(c):
    """float64 torch scaled_dot_product_attention on the concatenated keys.

    The KV heads are expanded to the query heads with repeat_interleave (head
    h reads KV head h // G).  The LSE comes from the same library call: one
    extra key with an all-zero K row (logit exactly 0) and a value that is 1
    in an extra output column receives weight 1 / (1 + Z), where Z is the sum
    of exp(logit) over the real visible keys; so LSE = ln(1/w - 1)."""
    B, Hq, Hkv, P, S, D = (c[k] for k in ("B", "Hq", "Hkv", "P", "S", "D"))
    G = Hq // Hkv
    f = lambda t: t.to(torch.float64)
    k = torch.cat([f(c["k_prefix"]), f(c["k_suffix"])], dim=2)      # [B,Hkv,P+S,D]
    v = torch.cat([f(c["v_prefix"]), f(c["v_suffix"])], dim=2)
    k = k.repeat_interleave(G, dim=1)
    v = v.repeat_interleave(G, dim=1)
    vis = torch.stack([torch.from_numpy(visible_keys(c, b)) for b in range(B)])  # [B,P+S]
    attn_mask = vis[:, None, None, :].expand(B, Hq, S, P + S)
    q = f(c["q"])
    out = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=attn_mask)
    # LSE through the extra-key construction
    k_x = torch.cat([k, torch.zeros(B, Hq, 1, D, dtype=torch.float64)], dim=2)
    v_x = torch.cat([torch.cat([v, torch.zeros(B, Hq, P + S, 1, dtype=torch.float64)], dim=3),
                     torch.cat([torch.zeros(B, Hq, 1, D, dtype=torch.float64),
                                torch.ones(B, Hq, 1, 1, dtype=torch.float64)], dim=3)], dim=2)
    mask_x = torch.cat([attn_mask, torch.ones(B, Hq, S, 1, dtype=torch.bool)], dim=3)
    out_x = torch.nn.functional.scaled_dot_product_attention(q, k_x, v_x, attn_mask=mask_x)
    w = out_x[..., D]
    lse = torch.log(1.0 / w - 1.0)
    return out.numpy(), lse.numpy()


# --------------------------------------------------------------------------

SDPA_SHAPES = [
    # seed, B, Hq, Hkv, P, S, D, mask_p
    (11, 1, 2, 1, 5, 1, 4, 0.0),
    (12, 2, 4, 2, 7, 3, 8, 0.3),
    (13, 2, 8, 4, 8, 4, 16, 0.2),
    (14, 1, 4, 1, 6, 2, 256, 0.4),
    (15, 2, 2, 2, 3, 4, 8, 0.0),
    (16, 1, 8, 4, 0, 3, 8, 0.0),
]


def pin_sdpa_float64(orc):
    """O and LSE equal float64 library attention on tiny random shapes."""
    for seed, B, Hq, Hkv, P, S, D, mp in SDPA_SHAPES:
        c = rand_case(seed, B, Hq, Hkv, P, S, D, mask_p=mp)
        o, lse = run(orc, c)
        o_ref, lse_ref = sdpa_reference(c)
        np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12,
                                   err_msg=f"O vs float64 SDPA, case seed {seed}")
        np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-9,
                                   err_msg=f"LSE vs float64 SDPA, case seed {seed}")


def pin_uniform_logits(orc):
    """Q = 0 makes every logit 0: O is the mean of the visible V rows and LSE is
    ln(number of visible keys)."""
    c = rand_case(21, 2, 4, 2, 9, 3, 8, mask_p=0.3)
    c["q"] = torch.zeros_like(c["q"])
    o, lse = run(orc, c)
    G = c["Hq"] // c["Hkv"]
    for b in range(c["B"]):
        vis = visible_keys(c, b)
        for h in range(c["Hq"]):
            kv = h // G
            rows = torch.cat([c["v_prefix"][b, kv], c["v_suffix"][b, kv]], 0).to(torch.float64).numpy()
            mean = rows[vis].mean(axis=0)
            for i in range(c["S"]):
                np.testing.assert_allclose(o[b, h, i], mean, rtol=0, atol=1e-13)
                assert abs(lse[b, h, i] - math.log(int(vis.sum()))) < 1e-13


def pin_constant_v_gqa(orc):
    """Every V row of KV head g holds the constant c_g: head h must output
    c_{h // G} (pins the GQA head mapping and the normalisation)."""
    consts = [0.5, -1.25, 2.0, 3.5]
    c = rand_case(22, 2, 8, 4, 6, 3, 8, mask_p=0.2)
    for g, val in enumerate(consts):
        c["v_prefix"][:, g] = val
        c["v_suffix"][:, g] = val
    o, _ = run(orc, c)
    for h in range(8):
        np.testing.assert_allclose(o[:, h], consts[h // 2], rtol=0, atol=1e-13,
                                   err_msg=f"head {h}")


def pin_masked_rows_ignored(orc):
    """Large finite values in masked prefix rows, and NaN in rows at or past
    the valid length, change nothing."""
    c = rand_case(23, 2, 4, 2, 10, 2, 8, vl=[7, 4], mask_p=0.3)
    o0, l0 = run(orc, c)
    for b in range(c["B"]):
        vl = int(c["prefix_valid_len"][b])
        hidden = np.where(c["prefix_mask"][b].numpy()[:vl] == 0)[0]
        for t in ("k_prefix", "v_prefix"):
            c[t][b, :, hidden.tolist(), :] = 1.0e4
            c[t][b, :, vl:, :] = float("nan")
    o1, l1 = run(orc, c)
    assert np.array_equal(o0, o1) and np.array_equal(l0, l1)


def pin_single_suffix_key(orc):
    """S = 1 with no visible prefix key: O is the one suffix V row and LSE is
    its logit <q, k_s> / sqrt(D)."""
    for P in (0, 4):
        c = rand_case(24 + P, 1, 2, 1, P, 1, 16, vl=[0])
        o, lse = run(orc, c)
        ks = c["k_suffix"][0, 0, 0].to(torch.float64).numpy()
        vs = c["v_suffix"][0, 0, 0].to(torch.float64).numpy()
        for h in range(2):
            q = c["q"][0, h, 0].to(torch.float64).numpy()
            np.testing.assert_array_equal(o[0, h, 0], vs)
            assert abs(lse[0, h, 0] - float(np.dot(q, ks)) / 4.0) < 1e-12


def pin_dominant_key(orc):
    """One prefix key aligned with every query and scaled far above the
    others takes essentially all the weight."""
    B, Hq, Hkv, P, S, D = 1, 2, 1, 6, 2, 4
    c = rand_case(25, B, Hq, Hkv, P, S, D, vl=[6])
    for t in ("q", "k_prefix", "k_suffix"):
        c[t] = (c[t].to(torch.float32) * 0.01).to(BF)
    c["q"][..., 0] = 8.0
    c["k_prefix"][0, 0, 3, :] = 0.0
    c["k_prefix"][0, 0, 3, 0] = 8.0      # logit exactly 8*8/sqrt(4) = 32 (others ~ 0.04)
    o, lse = run(orc, c)
    v3 = c["v_prefix"][0, 0, 3].to(torch.float64).numpy()
    for h in range(Hq):
        for i in range(S):
            np.testing.assert_allclose(o[0, h, i], v3, rtol=0, atol=1e-11)
            assert abs(lse[0, h, i] - 32.0) < 1e-11


def pin_prefix_permutation(orc):
    """Permuting the prefix rows inside the valid range (with their mask
    bytes) permutes nothing in the result."""
    c = rand_case(26, 1, 4, 2, 12, 3, 8, vl=[10], mask_p=0.25)
    o0, l0 = run(orc, c)
    perm = torch.randperm(10, generator=torch.Generator().manual_seed(5))
    full = torch.cat([perm, torch.arange(10, 12)])
    c["k_prefix"] = c["k_prefix"][:, :, full].contiguous()
    c["v_prefix"] = c["v_prefix"][:, :, full].contiguous()
    c["prefix_mask"] = c["prefix_mask"][:, full].contiguous()
    o1, l1 = run(orc, c)
    np.testing.assert_allclose(o1, o0, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l1, l0, rtol=0, atol=1e-13)


def pin_split_merge(orc):
    """Attention over disjoint key ranges merged by the log-sum-exp identity
    equals attention over the union (the split-KV combine)."""
    c = rand_case(27, 2, 4, 2, 11, 3, 8, vl=[9, 11], mask_p=0.2)
    o_full, l_full = run(orc, c)
    P, S = c["P"], c["S"]
    cuts = [0, 4, 9, P + 1, P + S]
    parts_o, parts_l = [], []
    for lo, hi in zip(cuts[:-1], cuts[1:]):
        o, l = run(orc, c, key_range=(lo, hi))
        parts_o.append(o.reshape(-1, c["D"]))
        parts_l.append(l.reshape(-1))
    o_m, l_m = orc.merge_parts(np.stack(parts_o), np.stack(parts_l))
    np.testing.assert_allclose(o_m, o_full.reshape(-1, c["D"]), rtol=0, atol=1e-13)
    np.testing.assert_allclose(l_m, l_full.reshape(-1), rtol=0, atol=1e-13)


def _dec_bf16(t):
    return [decimal.Decimal(float(x)) for x in t.to(torch.float32).reshape(-1).tolist()]


def pin_decimal_bruteforce(orc):
    """A 60-digit decimal brute force of softmax(q K^T / sqrt(D)) V on a tiny
    case (every bf16 value is exact in decimal)."""
    decimal.getcontext().prec = 60
    c = rand_case(28, 1, 2, 1, 4, 2, 4, vl=[3])
    c["prefix_mask"] = torch.tensor([[1, 0, 1, 1]], dtype=torch.uint8)
    o, lse = run(orc, c)
    P, S, D = 4, 2, 4
    vis = visible_keys(c, 0)
    K = _dec_bf16(torch.cat([c["k_prefix"][0, 0], c["k_suffix"][0, 0]], 0))
    V = _dec_bf16(torch.cat([c["v_prefix"][0, 0], c["v_suffix"][0, 0]], 0))
    half = decimal.Decimal(1) / decimal.Decimal(D).sqrt()
    for h in range(2):
        for i in range(S):
            qrow = _dec_bf16(c["q"][0, h, i])
            logits = {}
            for x in range(P + S):
                if vis[x]:
                    logits[x] = half * sum(qrow[d] * K[x * D + d] for d in range(D))
            z = sum(l.exp() for l in logits.values())
            want_lse = z.ln()
            for d in range(D):
                want = sum((l.exp() / z) * V[x * D + d] for x, l in logits.items())
                assert abs(float(want) - o[0, h, i, d]) < 1e-14
            assert abs(float(want_lse) - lse[0, h, i]) < 1e-14


def pin_valid_len_clamp_and_boundary(orc):
    """Valid lengths outside [0, P] clamp to the range; the key at index
    valid_len - 1 is seen and the key at valid_len is not."""
    c = rand_case(29, 1, 2, 1, 6, 2, 8, vl=[3])
    base_o, _ = run(orc, c)
    for vl, same_as in ((-5, 0), (13, 6)):
        c1 = dict(c, prefix_valid_len=torch.tensor([vl], dtype=torch.int32))
        c2 = dict(c, prefix_valid_len=torch.tensor([same_as], dtype=torch.int32))
        assert np.array_equal(run(orc, c1)[0], run(orc, c2)[0])
    c3 = dict(c, prefix_valid_len=None)
    c4 = dict(c, prefix_valid_len=torch.tensor([6], dtype=torch.int32))
    assert np.array_equal(run(orc, c3)[0], run(orc, c4)[0])
    # boundary: change row vl-1 -> output moves; change row vl -> it does not
    c5 = dict(c, v_prefix=c["v_prefix"].clone())
    c5["v_prefix"][0, 0, 3] = 100.0
    assert np.array_equal(run(orc, c5)[0], base_o)
    c6 = dict(c, v_prefix=c["v_prefix"].clone())
    c6["v_prefix"][0, 0, 2] = 100.0
    assert not np.allclose(run(orc, c6)[0], base_o)


# --------------------------------------------------------------------------
# Prefix-prefill attention under the prefix-causal mask (page
# "TensorRT+Triton+FlexAttention: OpenDM VLA 快速推理加速栈深度剖析", section
# 2.3): prefix query i sees prefix key j iff j <= i and j < valid length;
# query rows at or past the valid length are not computed.

def prefill_case(seed, B, Hq, Hkv, P, D, vl=None):
    gen = torch.Generator().manual_seed(seed)
    q = bf16_rand(gen, (B, Hq, P, D))
    k = bf16_rand(gen, (B, Hkv, P, D))
    v = bf16_rand(gen, (B, Hkv, P, D))
    vlt = None if vl is None else torch.tensor(vl, dtype=torch.int32)
    return dict(q=q, k=k, v=v, valid_len=vlt, B=B, Hq=Hq, Hkv=Hkv, P=P, D=D)


def run_prefill(orc, c, fill=float("nan"), **kw):
    return orc.prefix_causal_attn(c["q"], c["k"], c["v"], c["valid_len"], c["B"], c["Hq"], c["Hkv"], c["P"],
                                  c["D"], fill=fill, **kw)


def prefill_sdpa_reference(c):
    """float64 library attention with a boolean mask built from the rule
    (key j visible to query i iff j <= i and j < valid length), LSE through
    the extra all-zero key as in sdpa_reference."""
    B, Hq, Hkv, P, D = (c[k] for k in ("B", "Hq", "Hkv", "P", "D"))
    G = Hq // Hkv
    f = lambda t: t.to(torch.float64)
    q, k, v = f(c["q"]), f(c["k"]).repeat_interleave(G, 1), f(c["v"]).repeat_interleave(G, 1)
    vl = [P] * B if c["valid_len"] is None else [max(0, min(P, int(x))) for x in c["valid_len"]]
    i = torch.arange(P)[:, None]
    j = torch.arange(P)[None, :]
    mask = torch.stack([(j <= i) & (j < vl[b]) for b in range(B)])[:, None].expand(B, Hq, P, P)
    out = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask)
    k_x = torch.cat([k, torch.zeros(B, Hq, 1, D, dtype=torch.float64)], dim=2)
    v_x = torch.cat([torch.cat([v, torch.zeros(B, Hq, P, 1, dtype=torch.float64)], dim=3),
                     torch.cat([torch.zeros(B, Hq, 1, D, dtype=torch.float64),
                                torch.ones(B, Hq, 1, 1, dtype=torch.float64)], dim=3)], dim=2)
    mask_x = torch.cat([mask, torch.ones(B, Hq, P, 1, dtype=torch.bool)], dim=3)
    w = torch.nn.functional.scaled_dot_product_attention(q, k_x, v_x, attn_mask=mask_x)[..., D]
    return out.numpy(), torch.log(1.0 / w - 1.0).numpy(), vl


PREFILL_SHAPES = [
    # seed, B, Hq, Hkv, P, D, valid lengths
    (41, 1, 2, 1, 5, 4, None),
    (42, 2, 4, 2, 7, 8, [7, 3]),
    (43, 2, 8, 4, 9, 16, [9, 1]),
    (44, 1, 4, 1, 6, 256, [4]),
]


def pin_prefill_sdpa_float64(orc):
    """Computed rows equal float64 library attention under the causal and
    padding mask; rows at or past the valid length are left untouched."""
    for seed, B, Hq, Hkv, P, D, vl in PREFILL_SHAPES:
        c = prefill_case(seed, B, Hq, Hkv, P, D, vl)
        o, lse = run_prefill(orc, c, fill=-7.0)
        o_ref, l_ref, vls = prefill_sdpa_reference(c)
        for b in range(B):
            n = vls[b]
            np.testing.assert_allclose(o[b, :, :n], o_ref[b, :, :n], rtol=0, atol=1e-12,
                                       err_msg=f"prefill O vs float64 SDPA, seed {seed}")
            np.testing.assert_allclose(lse[b, :, :n], l_ref[b, :, :n], rtol=0, atol=1e-9,
                                       err_msg=f"prefill LSE vs float64 SDPA, seed {seed}")
            assert (o[b, :, n:] == -7.0).all() and (lse[b, :, n:] == -7.0).all(), "padding rows written"


def pin_prefill_first_row_and_uniform(orc):
    """Row 0 sees only key 0: O = V row 0 and LSE = <q_0, k_0> / sqrt(D).
    With Q = 0 every visible logit is 0: row i is the mean of V rows 0..i and
    its LSE is ln(i + 1)."""
    c = prefill_case(45, 1, 4, 2, 8, 16)
    o, lse = run_prefill(orc, c)
    for h in range(4):
        kv = h // 2
        q0 = c["q"][0, h, 0].to(torch.float64).numpy()
        k0 = c["k"][0, kv, 0].to(torch.float64).numpy()
        np.testing.assert_array_equal(o[0, h, 0], c["v"][0, kv, 0].to(torch.float64).numpy())
        assert abs(lse[0, h, 0] - float(np.dot(q0, k0)) / 4.0) < 1e-12
    c["q"] = torch.zeros_like(c["q"])
    o, lse = run_prefill(orc, c)
    v = c["v"].to(torch.float64).numpy()
    for h in range(4):
        for i in range(8):
            np.testing.assert_allclose(o[0, h, i], v[0, h // 2, :i + 1].mean(axis=0), rtol=0, atol=1e-13)
            assert abs(lse[0, h, i] - math.log(i + 1)) < 1e-13


def pin_prefill_future_keys_ignored(orc):
    """NaN in the K/V rows from position t on changes no row before t
    (causality); NaN at or past the valid length changes no computed row."""
    c = prefill_case(46, 2, 4, 2, 10, 8, [10, 6])
    o0, l0 = run_prefill(orc, c, fill=0.0)
    t = 5
    c1 = dict(c, k=c["k"].clone(), v=c["v"].clone())
    c1["k"][:, :, t:] = float("nan")
    c1["v"][:, :, t:] = float("nan")
    o1, l1 = run_prefill(orc, c1, fill=0.0)
    assert np.array_equal(o1[:, :, :t], o0[:, :, :t]) and np.array_equal(l1[:, :, :t], l0[:, :, :t])
    c2 = dict(c, k=c["k"].clone(), v=c["v"].clone())
    c2["k"][1, :, 6:] = float("nan")
    c2["v"][1, :, 6:] = float("nan")
    o2, l2 = run_prefill(orc, c2, fill=0.0)
    assert np.array_equal(o2, o0) and np.array_equal(l2, l0)


def pin_prefill_decimal_bruteforce(orc):
    """60-digit decimal brute force of the causal softmax on a tiny case."""
    decimal.getcontext().prec = 60
    c = prefill_case(47, 1, 2, 1, 5, 4, [4])
    o, lse = run_prefill(orc, c)
    D = 4
    K = _dec_bf16(c["k"][0, 0])
    V = _dec_bf16(c["v"][0, 0])
    half = decimal.Decimal(1) / decimal.Decimal(D).sqrt()
    for h in range(2):
        for i in range(4):
            qrow = _dec_bf16(c["q"][0, h, i])
            logits = [half * sum(qrow[d] * K[j * D + d] for d in range(D)) for j in range(i + 1)]
            z = sum(l.exp() for l in logits)
            for d in range(D):
                want = sum((l.exp() / z) * V[j * D + d] for j, l in enumerate(logits))
                assert abs(float(want) - o[0, h, i, d]) < 1e-14
            assert abs(float(z.ln()) - lse[0, h, i]) < 1e-14


# --------------------------------------------------------------------------
# Suffix prologue: QKV projection + QK-Norm + RoPE (page "TensorRT+Triton+
# FlexAttention: OpenDM VLA 快速推理加速栈深度剖析", section 2.2).  Readings:
# one weight matrix (query heads, then key heads, then value heads), RMS
# norm over each head's features with a learned weight (eps 1e-6), rotate-half
# RoPE with theta 10000 on the normalised queries and keys.

def prologue_case(seed, B=1, S=3, H=32, Hq=4, Hkv=2, D=16, pos0=0):
    gen = torch.Generator().manual_seed(seed)
    x = bf16_rand(gen, (B * S, H))
    w = bf16_rand(gen, ((Hq + 2 * Hkv) * D, H), mult=0.2)
    qw = (1.0 + 0.1 * torch.randn(D, generator=gen)).to(BF)
    kw = (1.0 + 0.1 * torch.randn(D, generator=gen)).to(BF)
    pos = torch.arange(B * S, dtype=torch.int32) % S + pos0
    return dict(x=x, w=w, qw=qw, kw=kw, pos=pos, B=B, S=S, H=H, Hq=Hq, Hkv=Hkv, D=D)


def run_prologue(orc, c, **kw):
    return orc.qkv_prologue(c["x"], c["w"], c["qw"], c["kw"], c["pos"], c["B"], c["S"], c["H"], c["Hq"], c["Hkv"],
                            c["D"], **kw)


def prologue_library_reference(c, eps=1e-6, theta=10000.0):
    """float64 library routines: linear, rms_norm, and the rotation done as a
    complex multiplication of the pairs (d, d + D/2) by exp(i * angle)."""
    B, S, H, Hq, Hkv, D = (c[k] for k in ("B", "S", "H", "Hq", "Hkv", "D"))
    f = lambda t: t.to(torch.float64)
    proj = torch.nn.functional.linear(f(c["x"]), f(c["w"]))                  # [B*S, (Hq+2Hkv)*D]
    heads = proj.view(B * S, Hq + 2 * Hkv, D)
    q = torch.nn.functional.rms_norm(heads[:, :Hq], (D,), weight=f(c["qw"]), eps=eps)
    k = torch.nn.functional.rms_norm(heads[:, Hq:Hq + Hkv], (D,), weight=f(c["kw"]), eps=eps)
    v = heads[:, Hq + Hkv:]
    half = D // 2
    inv = theta ** (-2.0 * torch.arange(half, dtype=torch.float64) / D)
    ang = c["pos"].to(torch.float64)[:, None] * inv[None, :]                 # [B*S, half]
    rot = torch.polar(torch.ones_like(ang), ang)[:, None, :]

    def rope(t):
        z = torch.complex(t[..., :half], t[..., half:]) * rot
        return torch.cat([z.real, z.imag], dim=-1)

    def lay(t, n):
        return t.view(B, S, n, D).permute(0, 2, 1, 3).numpy()
    return lay(rope(q), Hq), lay(rope(k), Hkv), lay(v, Hkv)


def pin_prologue_library_float64(orc):
    """Equal to float64 library projection, RMS norm and complex rotation."""
    for seed, B, S, pos0 in ((51, 1, 3, 0), (52, 2, 5, 900), (53, 1, 4, 1900)):
        c = prologue_case(seed, B=B, S=S, pos0=pos0)
        got = run_prologue(orc, c)
        want = prologue_library_reference(c)
        for g, w_, name in zip(got, want, "qkv"):
            np.testing.assert_allclose(g, w_, rtol=0, atol=1e-11, err_msg=f"prologue {name}, seed {seed}")


def pin_prologue_position_zero_and_norm(orc):
    """At position 0 the rotation is the identity; with unit norm weights
    every normalised query and key row has squared length D * ms / (ms + eps)
    (a rotation keeps lengths); values are the plain projection."""
    c = prologue_case(54, B=1, S=4, pos0=0)
    c["pos"] = torch.zeros_like(c["pos"])
    c["qw"] = torch.ones_like(c["qw"])
    c["kw"] = torch.ones_like(c["kw"])
    q, k, v = run_prologue(orc, c)
    proj = c["x"].to(torch.float64) @ c["w"].to(torch.float64).T
    D, Hq, Hkv = c["D"], c["Hq"], c["Hkv"]
    for t in range(4):
        for h in range(Hq + 2 * Hkv):
            y = proj[t, h * D:(h + 1) * D].numpy()
            ms = float((y * y).mean())
            if h < Hq:
                got = q[0, h, t]
            elif h < Hq + Hkv:
                got = k[0, h - Hq, t]
            else:
                np.testing.assert_allclose(v[0, h - Hq - Hkv, t], y, rtol=0, atol=1e-12)
                continue
            np.testing.assert_allclose(got, y / math.sqrt(ms + 1e-6), rtol=0, atol=1e-12)
    c["pos"] = torch.arange(4, dtype=torch.int32) * 37
    q2, k2, _ = run_prologue(orc, c)
    for t in range(4):
        for h in range(Hq):
            assert abs(float((q2[0, h, t] ** 2).sum()) - float((q[0, h, t] ** 2).sum())) < 1e-10


def pin_prologue_relative_position(orc):
    """<q at position m, k at position n> depends only on m - n: shifting
    every position by the same amount leaves all query-key dot products
    unchanged (pins the rotation's pairing, sign and shared angles)."""
    c = prologue_case(55, B=1, S=5, pos0=3)
    q0, k0, _ = run_prologue(orc, c)
    c2 = dict(c, pos=c["pos"] + 250)
    q1, k1, _ = run_prologue(orc, c2)
    d0 = np.einsum("bhid,bgjd->bhgij", q0, k0)
    d1 = np.einsum("bhid,bgjd->bhgij", q1, k1)
    np.testing.assert_allclose(d1, d0, rtol=0, atol=1e-9)
    assert not np.allclose(q1, q0)


def pin_prologue_decimal_bruteforce(orc):
    """60-digit decimal projection and RMS norm at position 0 (no trigonometry
    needed there) on a tiny case."""
    decimal.getcontext().prec = 60
    c = prologue_case(56, B=1, S=2, H=8, Hq=2, Hkv=1, D=4)
    c["pos"] = torch.zeros_like(c["pos"])
    q, k, v = run_prologue(orc, c)
    X = _dec_bf16(c["x"])
    W = _dec_bf16(c["w"])
    QW, KW = _dec_bf16(c["qw"]), _dec_bf16(c["kw"])
    H, D = 8, 4
    eps = decimal.Decimal("1e-6")
    for t in range(2):
        for h in range(4):
            y = [sum(W[(h * D + d) * H + cc] * X[t * H + cc] for cc in range(H)) for d in range(D)]
            if h == 3:
                for d in range(D):
                    assert abs(float(y[d]) - v[0, 0, t, d]) < 1e-14
                continue
            ms = sum(e * e for e in y) / D
            r = (ms + eps).sqrt()
            nw = QW if h < 2 else KW
            for d in range(D):
                want = float(y[d] / r * nw[d])
                got = q[0, h, t, d] if h < 2 else k[0, 0, t, d]
                assert abs(want - got) < 1e-13


# --------------------------------------------------------------------------
# Post-attention block (page "TensorRT+Triton+FlexAttention: OpenDM VLA
# 快速推理加速栈深度剖析", section 2.2: Adarms time modulation, GEGLU gate-up,
# MLP down).  Readings: output projection + residual, an RMS norm whose
# weight (1 + scale) and bias (shift) come from the time embedding, GEGLU with
# the tanh GELU, MLP down, and a residual gated by the time embedding's gate.

def post_case(seed, B=2, S=3, Hq=2, D=8, Hd=16, F=24, wscale=0.3):
    gen = torch.Generator().manual_seed(seed)
    return dict(attn=bf16_rand(gen, (B, Hq, S, D)), h=bf16_rand(gen, (B * S, Hd)),
                scale=bf16_rand(gen, (B, Hd), 0.2), shift=bf16_rand(gen, (B, Hd), 0.2),
                gate=bf16_rand(gen, (B, Hd), 0.5), wo=bf16_rand(gen, (Hd, Hq * D), wscale),
                wgu=bf16_rand(gen, (2 * F, Hd), wscale), wd=bf16_rand(gen, (Hd, F), wscale),
                B=B, S=S, Hq=Hq, D=D, Hd=Hd, F=F)


def run_post(orc, c, **kw):
    return orc.post_attention(c["attn"], c["h"], c["scale"], c["shift"], c["gate"], c["wo"], c["wgu"], c["wd"],
                              c["B"], c["S"], c["Hq"], c["D"], c["Hd"], c["F"], **kw)


def post_library_reference(c, eps=1e-6):
    """float64 library routines: linear, rms_norm, gelu (tanh approximation)."""
    B, S, Hq, D, Hd, F = (c[k] for k in ("B", "S", "Hq", "D", "Hd", "F"))
    f = lambda t: t.to(torch.float64)
    a = f(c["attn"]).permute(0, 2, 1, 3).reshape(B * S, Hq * D)
    h1 = f(c["h"]) + torch.nn.functional.linear(a, f(c["wo"]))
    per_tok = lambda t: f(t).repeat_interleave(S, dim=0)               # [B*S, Hd]
    u = torch.nn.functional.rms_norm(h1, (Hd,), eps=eps) * (1.0 + per_tok(c["scale"])) + per_tok(c["shift"])
    gu = torch.nn.functional.linear(u, f(c["wgu"]))
    m = torch.nn.functional.gelu(gu[:, :F], approximate="tanh") * gu[:, F:]
    return (h1 + per_tok(c["gate"]) * torch.nn.functional.linear(m, f(c["wd"]))).numpy()


def pin_post_library_float64(orc):
    """Equal to float64 library linear, rms_norm and tanh-GELU on tiny shapes."""
    for seed in (61, 62, 63):
        c = post_case(seed)
        np.testing.assert_allclose(run_post(orc, c), post_library_reference(c), rtol=0, atol=1e-11,
                                   err_msg=f"post-attention block vs float64 library, seed {seed}")


def pin_post_closed_forms(orc):
    """A zero gate leaves out = h + Wo a (the residual after the projection);
    scale = -1 and shift = 0 make the MLP input zero, so out = h + Wo a too;
    zero projections leave out = h."""
    c = post_case(64)
    B, S, Hq, D = c["B"], c["S"], c["Hq"], c["D"]
    a = c["attn"].to(torch.float64).permute(0, 2, 1, 3).reshape(B * S, Hq * D)
    h1 = (c["h"].to(torch.float64) + a @ c["wo"].to(torch.float64).T).numpy()
    np.testing.assert_allclose(run_post(orc, dict(c, gate=torch.zeros_like(c["gate"]))), h1, rtol=0, atol=1e-12)
    c2 = dict(c, scale=torch.full_like(c["scale"], -1.0), shift=torch.zeros_like(c["shift"]))
    np.testing.assert_allclose(run_post(orc, c2), h1, rtol=0, atol=1e-12)
    c3 = dict(c, wo=torch.zeros_like(c["wo"]), wd=torch.zeros_like(c["wd"]))
    np.testing.assert_allclose(run_post(orc, c3), c["h"].to(torch.float64).numpy(), rtol=0, atol=0)


def pin_post_gelu_value(orc):
    """One token, one intermediate feature: u_0 = 1 exactly (shift 1, scale
    -1 so the norm term vanishes), gate row picks u_0, up row picks u_0, down
    weight 1 and gate 1: out - h1 = gelu_tanh(1) * 1, the textbook value
    0.5 * (1 + tanh(sqrt(2/pi) * 1.044715))."""
    c = post_case(65, B=1, S=1, Hq=1, D=4, Hd=4, F=1)
    c["scale"] = torch.full_like(c["scale"], -1.0)
    c["shift"] = torch.tensor([[1.0, 0.0, 0.0, 0.0]], dtype=BF)
    c["gate"] = torch.ones_like(c["gate"])
    c["wgu"] = torch.tensor([[1.0, 0.0, 0.0, 0.0], [1.0, 0.0, 0.0, 0.0]], dtype=BF)
    c["wd"] = torch.tensor([[1.0], [0.0], [0.0], [0.0]], dtype=BF)
    out = run_post(orc, c)
    h1 = (c["h"].to(torch.float64) + c["attn"].to(torch.float64).reshape(1, 4) @ c["wo"].to(torch.float64).T).numpy()
    want = 0.5 * (1.0 + math.tanh(math.sqrt(2.0 / math.pi) * 1.044715))
    assert abs((out - h1)[0, 0] - want) < 1e-15 and abs(want - 0.8411919906082768) < 1e-15
    np.testing.assert_allclose((out - h1)[0, 1:], 0.0, atol=0)


def pin_post_decimal_bruteforce(orc):
    """60-digit decimal evaluation of the whole block on a tiny case (tanh from
    the decimal exponential)."""
    decimal.getcontext().prec = 60
    c = post_case(66, B=1, S=2, Hq=1, D=4, Hd=4, F=3)
    out = run_post(orc, c)
    Dc = decimal.Decimal
    A = _dec_bf16(c["attn"])
    Hh = _dec_bf16(c["h"])
    SC, SH, GT = _dec_bf16(c["scale"]), _dec_bf16(c["shift"]), _dec_bf16(c["gate"])
    WO, WGU, WD = _dec_bf16(c["wo"]), _dec_bf16(c["wgu"]), _dec_bf16(c["wd"])
    Hd, F = 4, 3
    k = (Dc(2) / Dc("3.14159265358979323846264338327950288419716939937510")).sqrt()

    def tanh(x):
        e = (2 * x).exp()
        return (e - 1) / (e + 1)

    for t in range(2):
        a = [A[t * 4 + d] for d in range(4)]          # attn [1, 1, S=2, D=4]: query t, feature d
        h1 = [Hh[t * Hd + o] + sum(WO[o * 4 + cc] * a[cc] for cc in range(4)) for o in range(Hd)]
        r = (sum(x * x for x in h1) / Hd + Dc("1e-6")).sqrt()
        u = [h1[o] / r * (1 + SC[o]) + SH[o] for o in range(Hd)]
        m = []
        for f in range(F):
            g = sum(WGU[f * Hd + cc] * u[cc] for cc in range(Hd))
            up = sum(WGU[(F + f) * Hd + cc] * u[cc] for cc in range(Hd))
            m.append(g / 2 * (1 + tanh(k * (g + Dc("0.044715") * g * g * g))) * up)
        for o in range(Hd):
            want = h1[o] + GT[o] * sum(WD[o * F + f] * m[f] for f in range(F))
            assert abs(float(want) - out[t, o]) < 1e-13


ALL_PINS = [pin_sdpa_float64, pin_uniform_logits, pin_constant_v_gqa, pin_masked_rows_ignored,
            pin_single_suffix_key, pin_dominant_key, pin_prefix_permutation, pin_split_merge,
            pin_decimal_bruteforce, pin_valid_len_clamp_and_boundary,
            pin_prefill_sdpa_float64, pin_prefill_first_row_and_uniform, pin_prefill_future_keys_ignored,
            pin_prefill_decimal_bruteforce,
            pin_prologue_library_float64, pin_prologue_position_zero_and_norm, pin_prologue_relative_position,
            pin_prologue_decimal_bruteforce,
            pin_post_library_float64, pin_post_closed_forms, pin_post_gelu_value, pin_post_decimal_bruteforce]
