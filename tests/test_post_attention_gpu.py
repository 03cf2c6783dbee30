"""The post-attention block (dm05_post_attention: output projection + residual,
Adarms, GEGLU, MLP down + gated residual) against the fp64 oracle, element by
element.

Tolerance, from the kernels' arithmetic: they accumulate in fp32, but the two
GEMM inputs built on the way -- u (the Adarms output) and m (the GEGLU
output) -- are rounded to bf16, the tensor cores' input type, and out is
rounded once to bf16.  Each rounding is an independent error, uniform within
half a bf16 ulp (variance ulp^2 / 12).  Linearised through the block:
  Var(dg_f), Var(dup_f) = sum_k W_fk^2 Var(du_k)           (gate and up rows)
  Var(dm_f) <= 2 (gelu'(g_f) up_f)^2 Var(dg_f) + 2 gelu(g_f)^2 Var(dup_f)
               + ulp(m_f)^2 / 12                            (2x: their covariance)
  sigma_ti^2 = gate_i^2 sum_f Wd_if^2 Var(dm_f)
with g, up, m the exact (fp64) intermediates.  Every element must satisfy
|out - ref| <= ulp(ref) + 6 sigma_ti + 1e-4 (one output ulp for the final
rounding, 1e-4 for the fp32 sums), and the mean error must stay within twice
the mean error of the correctly rounded result plus 1e-3.  Measured on 1.2M
elements, the largest error minus half an output ulp is 3.6 sigma."""
import numpy as np
import pytest
import torch

import oracle
from gqa_prefix_suffix_b200 import binding as bd
from gqa_prefix_suffix_b200 import inputs as gen

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gqa_prefix_suffix_b200 import build
    build.build()
    bd.lib()


def bf16_ulp(x):
    """The bf16 ulp at |x| (8 significant bits)."""
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** -126)))
    return 2.0 ** (e - 7)


def _gelu(z):
    return 0.5 * z * (1.0 + np.tanh(0.7978845608028654 * (z + 0.044715 * z ** 3)))


def _gelu_prime(z):
    k0, k1 = 0.7978845608028654, 0.044715
    t = np.tanh(k0 * (z + k1 * z ** 3))
    return 0.5 * (1.0 + t) + 0.5 * z * (1.0 - t * t) * k0 * (1.0 + 3.0 * k1 * z * z)


def rounding_sigma(inp, eps=1e-6):
    """Per-element standard deviation of the error that the bf16 roundings of
    u and m put into out (the model of the module docstring), from fp64
    intermediates of the inputs alone."""
    B, S, Hq, D, Hd, F = inp.B, inp.S, inp.Hq, inp.D, inp.Hd, inp.F
    T = B * S
    f = lambda x: x.float().double().numpy()
    a = f(inp.attn).reshape(B, Hq, S, D).transpose(0, 2, 1, 3).reshape(T, Hq * D)
    bi = np.repeat(np.arange(B), S)
    h1 = f(inp.h) + a @ f(inp.wo).T
    u = h1 / np.sqrt((h1 ** 2).mean(1, keepdims=True) + eps) * (1.0 + f(inp.scale)[bi]) + f(inp.shift)[bi]
    wgu, wd = f(inp.wgu), f(inp.wd)
    gu = u @ wgu.T
    g, up = gu[:, :F], gu[:, F:]
    var_gu = (bf16_ulp(u) ** 2 / 12.0) @ (wgu ** 2).T
    var_m = (2.0 * (_gelu_prime(g) * up) ** 2 * var_gu[:, :F] + 2.0 * _gelu(g) ** 2 * var_gu[:, F:]
             + bf16_ulp(_gelu(g) * up) ** 2 / 12.0)
    return np.abs(f(inp.gate)[bi]) * np.sqrt(var_m @ (wd ** 2).T)


def run_and_check(inp, what):
    d = inp.to("cuda")
    out = bd.post_attention(d.attn, d.h, d.scale, d.shift, d.gate, d.wo, d.wgu, d.wd)
    torch.cuda.synchronize()
    rc, word = bd.dm05_get_error_word(None)
    assert rc == 0 and word == 0, hex(word)
    ref = oracle.post_attention(inp.attn, inp.h, inp.scale, inp.shift, inp.gate, inp.wo, inp.wgu, inp.wd, inp.B,
                                inp.S, inp.Hq, inp.D, inp.Hd, inp.F, nthreads=min(16, oracle.max_threads()))
    g = out.float().cpu().double().numpy()
    err = np.abs(g - ref)
    floor = np.abs(torch.from_numpy(ref).to(torch.bfloat16).double().numpy() - ref).mean()
    sig = rounding_sigma(inp)
    bound = bf16_ulp(ref) + 6.0 * sig + 1e-4
    z = np.maximum(err - bf16_ulp(ref) / 2, 0.0) / sig
    print(f"[{what}] max err {err.max():.4g}, mean {err.mean():.4g} (rounding floor {floor:.4g}), "
          f"max |ref| {np.abs(ref).max():.3g}, largest (err - ulp/2) / sigma {z.max():.3g}")
    assert (err <= bound).all(), f"{what}: {int((err > bound).sum())} elements over the bound, max {err.max():.4g}"
    assert err.mean() <= 2.0 * floor + 1e-3, f"{what}: mean err {err.mean():.4g}"


CASES = [
    # B, S, Hq, D, Hd, F
    (1, 1, 2, 64, 128, 64),
    (2, 7, 2, 128, 256, 320),
    (1, 50, 8, 256, 1024, 4096),
    (3, 70, 4, 64, 256, 512),       # S > 64: two token tiles per sample
    # one-wave grids: 100 tokens in one 128-token tile (GEGLU on M = 64 in
    # four-chunk stages, the ring wrapping over four 256-column groups), and
    # F = 8192 (GEGLU on M = 128, MLP down split 16 ways of 8 chunks)
    (1, 100, 8, 256, 1024, 2048),
    (1, 64, 8, 256, 1024, 8192),
    # grids of several waves: 1200 tokens (the last 128-token tile holding
    # 48), and 4800 tokens of a narrow MLP (last tile 64 tokens)
    (24, 50, 8, 256, 1024, 4096),
    (80, 60, 2, 64, 256, 1024),
]


@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}_S{c[1]}_Hq{c[2]}_D{c[3]}_Hd{c[4]}_F{c[5]}" for c in CASES])
def test_post_attention_shapes(case):
    B, S, Hq, D, Hd, F = case
    inp = gen.make_post_inputs(B, S, 8100 + B * 7 + S, Hq=Hq, D=D, Hd=Hd, F=F)
    run_and_check(inp, f"B={B} S={S} Hd={Hd} F={F}")


def test_post_attention_batched():
    run_and_check(gen.post_batched(), "batched B=32")


def test_post_attention_is_deterministic():
    d = gen.post_base().to("cuda")
    a = bd.post_attention(d.attn, d.h, d.scale, d.shift, d.gate, d.wo, d.wgu, d.wd)
    b = bd.post_attention(d.attn, d.h, d.scale, d.shift, d.gate, d.wo, d.wgu, d.wd)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_post_attention_rejects_bad_arguments():
    fake = 0x7f0000001000
    a = [fake] * 9
    assert bd.dm05_post_attention(*a, 1, 50, 8, 256, 1000, 4096, 1e-6, None) == bd.DM05_ERR_UNSUPPORTED
    assert bd.dm05_post_attention(*a, 1, 50, 8, 100, 1024, 4096, 1e-6, None) == bd.DM05_ERR_UNSUPPORTED
    assert bd.dm05_post_attention(*a, 0, 50, 8, 256, 1024, 4096, 1e-6, None) == bd.DM05_ERR_SHAPE
    b = list(a)
    b[0] = fake + 8
    assert bd.dm05_post_attention(*b, 1, 50, 8, 256, 1024, 4096, 1e-6, None) == bd.DM05_ERR_ALIGN
    b = list(a)
    b[5] = None
    assert bd.dm05_post_attention(*b, 1, 50, 8, 256, 1024, 4096, 1e-6, None) == bd.DM05_ERR_NULL
