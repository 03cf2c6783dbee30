"""Multi-step calls (dm05_suffix_attn_steps_*): the 10 denoising-step calls of
the history loop over one prefix cache, captured once and replayed with one
launch, against the fp64 oracle for every step.

The chained case feeds each step's output back as the next step's queries
(out has the query layout), so the launch must order the steps; the oracle
chains its own results (each rounded once to bf16, as the kernel rounds its
output) and never sees a GPU value."""
import pytest
import torch

import oracle
from gqa_prefix_suffix_b200 import binding as bd
from gqa_prefix_suffix_b200 import inputs as gen
from parity import check_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gqa_prefix_suffix_b200 import build
    build.build()
    bd.lib()


def _ptr(t):
    return None if t is None else t.data_ptr()


@pytest.mark.parametrize("flags", [0, bd.DM05_FLAG_PREFIX_STATIC])
def test_history_loop_steps_match_the_oracle(flags):
    calls = gen.history_loop()
    ds = [c.to("cuda") for c in calls]
    d0 = ds[0]
    outs = [torch.full_like(d.q, float("nan")) for d in ds]
    lses = [torch.full(d.q.shape[:3], float("nan"), dtype=torch.float32, device="cuda") for d in ds]
    steps = [(_ptr(d.q), _ptr(d.k_suffix), _ptr(d.v_suffix), _ptr(o), _ptr(l)) for d, o, l in zip(ds, outs, lses)]
    rc, h = bd.dm05_suffix_attn_steps_create(steps, _ptr(d0.k_prefix), _ptr(d0.v_prefix), _ptr(d0.prefix_valid_len),
                                             None, 1, 8, 4, 2048, 50, 256, flags)
    assert rc == 0, bd.dm05_status_string(rc)
    try:
        for rep in range(2):  # the same graph twice: the second launch reuses it
            for o in outs:
                o.fill_(float("nan"))
            assert bd.dm05_suffix_attn_steps_launch(h, None) == 0
            torch.cuda.synchronize()
            for c, o, l in zip(calls, outs, lses):
                o_ref, l_ref = oracle.inputs_call(c, nthreads=8)
                check_close(o.cpu(), l.cpu(), o_ref, l_ref, f"{c.name} launch {rep}")
        rc, word = bd.dm05_get_error_word(None)
        assert rc == 0 and word == 0
    finally:
        assert bd.dm05_suffix_attn_steps_destroy(h) == 0


def test_chained_steps_are_ordered():
    # step t + 1 reads step t's output as its queries: 4 chained steps
    n = 4
    base = gen.make_inputs(1, 8, 4, 1024, 50, 256, 7001, valid_len=900)
    d = base.to("cuda")
    outs = [torch.empty_like(d.q) for _ in range(n)]
    qs = [d.q] + outs[:-1]
    steps = [(_ptr(q), _ptr(d.k_suffix), _ptr(d.v_suffix), _ptr(o), None) for q, o in zip(qs, outs)]
    rc, h = bd.dm05_suffix_attn_steps_create(steps, _ptr(d.k_prefix), _ptr(d.v_prefix), _ptr(d.prefix_valid_len),
                                             None, 1, 8, 4, 1024, 50, 256, bd.DM05_FLAG_PREFIX_STATIC)
    assert rc == 0
    try:
        assert bd.dm05_suffix_attn_steps_launch(h, None) == 0
        torch.cuda.synchronize()
    finally:
        bd.dm05_suffix_attn_steps_destroy(h)
    cur = base
    for t in range(n):
        o_ref, l_ref = oracle.inputs_call(cur, nthreads=8)
        check_close(outs[t].cpu(), None, o_ref, l_ref, f"chained step {t}")
        nxt = gen.make_inputs(1, 8, 4, 1024, 50, 256, 7001, valid_len=900)
        nxt.q = torch.from_numpy(o_ref).to(torch.bfloat16)   # the oracle's own rounded result
        cur = nxt


def test_steps_reject_bad_arguments():
    fake = 0x7f0000001000
    st = [(fake, fake, fake, fake, None)]
    assert bd.dm05_suffix_attn_steps_create([], fake, fake, None, None, 1, 8, 4, 64, 10, 256)[0] == bd.DM05_ERR_SHAPE
    assert bd.dm05_suffix_attn_steps_create(st, fake, fake, None, None, 1, 8, 4, 64, 10, 128)[0] == \
        bd.DM05_ERR_UNSUPPORTED
    bad = [(fake + 8, fake, fake, fake, None)]
    assert bd.dm05_suffix_attn_steps_create(bad, fake, fake, None, None, 1, 8, 4, 64, 10, 256)[0] == bd.DM05_ERR_ALIGN
    assert bd.dm05_suffix_attn_steps_create(st, fake, fake, None, None, 1, 8, 4, 64, 10, 256, 0x10)[0] == \
        bd.DM05_ERR_SHAPE
    assert bd.dm05_suffix_attn_steps_launch(None, None) == bd.DM05_ERR_NULL
