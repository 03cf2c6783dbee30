"""CUDA path against the fp64 oracle, element by element, on seeded inputs,
with the tolerance stated in parity.py."""
import math
import zlib

import numpy as np
import pytest
import torch

import oracle
from gqa_prefix_suffix_b200 import binding as bd
from gqa_prefix_suffix_b200 import inputs as gen
from parity import LSE_ABS, MEAN_ABS, bf16_ulp, check_close, visible_keys

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gqa_prefix_suffix_b200 import build
    build.build()
    bd.lib()
    yield
    bd.dm05_set_split_override(0)
    bd.dm05_set_row_block_override(0)


def run_gpu(inp, splits=0, with_lse=True, stream=None, row_blocks=0):
    d = inp.to("cuda")
    assert bd.dm05_set_split_override(splits) == 0
    assert bd.dm05_set_row_block_override(row_blocks) == 0
    try:
        out, lse = bd.suffix_attn(d.q, d.k_prefix, d.v_prefix, d.k_suffix, d.v_suffix,
                                  prefix_valid_len=d.prefix_valid_len, prefix_mask=d.prefix_mask,
                                  want_lse=with_lse, stream=stream)
        torch.cuda.synchronize()
    finally:
        bd.dm05_set_split_override(0)
        bd.dm05_set_row_block_override(0)
    rc, word = bd.dm05_get_error_word(None)
    assert rc == 0
    return out.cpu(), (lse.cpu() if lse is not None else None), word


def ref(inp):
    return oracle.inputs_call(inp, nthreads=min(8, oracle.max_threads()))


# ---------------------------------------------------------------- small / ragged shapes

SMALL = [
    # name, B, Hq, Hkv, P, S, valid (None|int|list|'rand'), mask_frac, peak(frac, mult)
    ("no_prefix", 1, 8, 4, 0, 1, None, 0.0, None),
    ("one_prefix_row", 1, 8, 4, 1, 1, 1, 0.0, None),
    ("p63_s10", 2, 8, 4, 63, 10, "rand", 0.0, None),
    ("p64_s50", 1, 8, 4, 64, 50, 64, 0.0, None),
    ("p65_s50", 2, 8, 4, 65, 50, [65, 1], 0.0, None),
    ("p127_s7", 1, 8, 4, 127, 7, 127, 0.2, None),
    ("p128_s64", 1, 8, 4, 128, 64, [100], 0.0, None),
    ("p129_s33", 3, 8, 4, 129, 33, "rand", 0.1, (0.05, 3.0)),
    ("g1_s128", 1, 4, 4, 200, 128, 150, 0.0, None),
    ("g4_s32", 2, 8, 2, 300, 32, "rand", 0.1, None),
    ("g8_s16", 1, 8, 1, 333, 16, 321, 0.0, None),
    ("valid_zero", 2, 8, 4, 256, 20, [0, 0], 0.0, None),
    ("p576_s10_mask", 2, 8, 4, 576, 10, [512, 300], 0.3, (0.02, 4.0)),
    ("p1000_s50_peaks", 1, 8, 4, 1000, 50, 999, 0.0, (0.05, 5.0)),
]


def make_small(name, B, Hq, Hkv, P, S, valid, mask_frac, peak, seed=7):
    kw = {}
    if valid == "rand":
        kw["valid_range"] = (0, P)
    elif valid is not None:
        kw["valid_len"] = valid
    if peak is not None:
        kw["peak_frac"], kw["peak_mult"] = peak
    return gen.make_inputs(B, Hq, Hkv, P, S, 256, seed + zlib.crc32(name.encode()) % 1000, mask_frac=mask_frac,
                           name=name, **kw)


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_small_shapes(case):
    inp = make_small(*case)
    out, lse, word = run_gpu(inp)
    o_ref, l_ref = ref(inp)
    check_close(out, lse, o_ref, l_ref, case[0], keys=visible_keys(inp))
    assert word == 0


@pytest.mark.parametrize("splits", [1, 2, 4, 8, 16])
def test_every_split_count(splits):
    inp = gen.make_inputs(1, 8, 4, 1024, 50, 256, 99, valid_len=900, peak_frac=0.05, peak_mult=3.0,
                          mask_frac=0.05)
    out, lse, _ = run_gpu(inp, splits=splits)
    o_ref, l_ref = ref(inp)
    check_close(out, lse, o_ref, l_ref, f"splits={splits}")


# Query row blocks forced (the automatic plan picks them from occupancy, so a
# different SM count would reach other block counts): each (sample, KV head)'s
# S queries cut into `rb` blocks of ceil(S / rb) queries per head, the last
# one short, for 1, 2, 4 and 8 query heads per KV head, with a prefix mask.
ROW_BLOCK_CASES = [
    # Hq, Hkv, S, row_blocks, splits: queries per head per block, last block
    (8, 4, 50, 2, 2),    # 25 / 25
    (8, 4, 50, 4, 8),    # 13 / 13 / 13 / 11
    (8, 4, 50, 4, 2),
    (8, 4, 60, 8, 8),    # 8 x 7 / 4
    (8, 4, 64, 8, 2),    # 8 x 8
    (4, 4, 50, 4, 8),    # G = 1
    (4, 4, 100, 8, 2),   # G = 1: 13 x 7 / 9
    (4, 4, 128, 16, 8),  # G = 1: 16 blocks of 8
    (8, 2, 30, 2, 8),    # G = 4: 15 / 15
    (8, 2, 30, 4, 2),    # G = 4: 8 / 8 / 8 / 6
    (8, 1, 16, 2, 4),    # G = 8: 8 / 8
]


@pytest.mark.parametrize("case", ROW_BLOCK_CASES, ids=[f"G{c[0] // c[1]}_S{c[2]}_rb{c[3]}_c{c[4]}" for c in ROW_BLOCK_CASES])
def test_forced_row_blocks(case):
    Hq, Hkv, S, rb, splits = case
    P = 700
    inp = gen.make_inputs(2, Hq, Hkv, P, S, 256, 500 + rb * 10 + splits, valid_range=(300, P),
                          mask_frac=0.1, peak_frac=0.02, peak_mult=4.0)
    assert bd.dm05_set_split_override(splits) == 0 and bd.dm05_set_row_block_override(rb) == 0
    try:
        rc, got_splits, _, got_rb = bd.dm05_suffix_attn_plan(2, Hq, Hkv, P, S, 256)
    finally:
        bd.dm05_set_split_override(0)
        bd.dm05_set_row_block_override(0)
    assert rc == 0 and (got_splits, got_rb) == (splits, rb), (got_splits, got_rb)
    out, lse, word = run_gpu(inp, splits=splits, row_blocks=rb)
    assert word == 0
    check_close(out, lse, *ref(inp), what=f"G={Hq // Hkv} S={S} row_blocks={rb} splits={splits}")


def test_row_block_override_falls_back_when_blocks_would_be_too_small():
    # 8 blocks of S=50 would hold 7 queries per head (< 8): one block is used
    assert bd.dm05_set_split_override(4) == 0 and bd.dm05_set_row_block_override(8) == 0
    try:
        rc, splits, _, rb = bd.dm05_suffix_attn_plan(1, 8, 4, 1024, 50, 256)
    finally:
        bd.dm05_set_split_override(0)
        bd.dm05_set_row_block_override(0)
    assert rc == 0 and splits == 4 and rb == 1


def test_splits_beyond_tiles():
    # 16 CTAs for a unit with only 2 tiles: most CTAs get no work
    inp = gen.make_inputs(2, 8, 4, 64, 10, 256, 5, valid_len=[40, 0])
    out, lse, _ = run_gpu(inp, splits=16)
    o_ref, l_ref = ref(inp)
    check_close(out, lse, o_ref, l_ref, "splits beyond tiles", keys=visible_keys(inp))


def ramp_case(top):
    # K rows scaled by a factor that grows along the prefix, so the running
    # max of every row moves by more than 2^8 (log2 units) between tiles.
    inp = gen.make_inputs(1, 8, 4, 512, 20, 256, 11, valid_len=512)
    ramp = torch.linspace(0.2, top, 512).view(1, 1, 512, 1)
    inp.k_prefix = (inp.k_prefix.float() * ramp).to(torch.bfloat16)
    return inp


def test_growing_logits():
    # x4, the largest K multiplier of the workloads: every row rescales O at
    # least once
    inp = ramp_case(4.0)
    o_ref, l_ref = ref(inp)
    for splits in (1, 2):
        out, lse, _ = run_gpu(inp, splits=splits)
        check_close(out, lse, o_ref, l_ref, f"ramp x4 splits={splits}")


def test_lazy_rescale_path():
    # K up to x40: the row maxima grow by far more than 2^8 over the prefix,
    # so O and the sums are rescaled, most rows several times
    inp = ramp_case(40.0)
    o_ref, l_ref = ref(inp)
    for splits in (1, 2):
        out, lse, _ = run_gpu(inp, splits=splits)
        check_close(out, lse, o_ref, l_ref, f"ramp x40 splits={splits}")


def test_peaked_precision_model():
    """On a sharper input (K up to x6) the error is still the one the bf16
    probabilities allow.  With p_j rounded to bf16 (relative error
    u = 2^-8) and O normalised by the sum of the rounded p_j, to first order
    |O_gpu - O| <= 2u max_j |v_j - O|; the output adds half a bf16 ulp."""
    inp = ramp_case(6.0)
    o_ref, l_ref = ref(inp)
    G = inp.Hq // inp.Hkv
    v_all = torch.cat([inp.v_prefix, inp.v_suffix], dim=2).double().numpy()   # [B,Hkv,P+S,D]
    vmax = np.abs(v_all).max(axis=2)                                           # [B,Hkv,D]
    vmax_q = np.repeat(vmax, G, axis=1)[:, :, None, :]                         # [B,Hq,1,D]
    bound = 0.5 * bf16_ulp(o_ref) + 2.0 ** -7 * (vmax_q + np.abs(o_ref)) + 1e-5
    for splits in (1, 2):
        out, lse, _ = run_gpu(inp, splits=splits)
        err = np.abs(out.float().double().numpy() - o_ref)
        assert (err <= bound).all(), f"splits={splits}: max err {err.max():.5f}"
        assert err.mean() <= MEAN_ABS
        assert np.abs(lse.double().numpy() - l_ref).max() <= LSE_ABS


def test_rows_past_valid_len_are_never_used():
    inp = gen.make_inputs(2, 8, 4, 200, 30, 256, 12, valid_len=[130, 65], mask_frac=0.1)
    o_ref, l_ref = ref(inp)
    for b, vl in enumerate((130, 65)):
        inp.k_prefix[b, :, vl:] = float("nan")
        inp.v_prefix[b, :, vl:] = float("nan")
        hidden = (inp.prefix_mask[b, :vl] == 0).nonzero().flatten()
        inp.k_prefix[b, :, hidden] = 1.0e4
        inp.v_prefix[b, :, hidden] = 1.0e4
    for splits in (0, 1, 4):
        out, lse, _ = run_gpu(inp, splits=splits)
        assert torch.isfinite(out.float()).all()
        check_close(out, lse, o_ref, l_ref, f"nan padding splits={splits}")


def test_valid_len_out_of_range_is_clamped_and_flagged():
    inp = gen.make_inputs(2, 8, 4, 128, 10, 256, 13, valid_len=[-5, 500])
    out, lse, word = run_gpu(inp)
    assert word & bd.DM05_EW_VALID_LEN_CLAMPED
    o_ref, l_ref = ref(inp)  # the oracle clamps to [0, P] too
    check_close(out, lse, o_ref, l_ref, "clamped")


def test_no_valid_len_and_no_lse():
    inp = gen.make_inputs(1, 8, 4, 96, 12, 256, 14, valid_len=None)
    out, lse, _ = run_gpu(inp, with_lse=False)
    assert lse is None
    o_ref, l_ref = ref(inp)
    check_close(out, None, o_ref, l_ref, "no valid_len")


def test_deterministic():
    inp = gen.base_chunk()
    a, la, _ = run_gpu(inp)
    b, lb, _ = run_gpu(inp)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert torch.equal(la, lb)


def test_no_writes_outside_outputs():
    inp = gen.make_inputs(2, 8, 4, 300, 50, 256, 15, valid_range=(0, 300))
    d = inp.to("cuda")
    n_out = 2 * 8 * 50 * 256
    pad = 4096
    canary = torch.full((n_out + 2 * pad,), 7.0, dtype=torch.bfloat16, device="cuda")
    lcan = torch.full((2 * 8 * 50 + 2 * pad,), 7.0, dtype=torch.float32, device="cuda")
    out = canary[pad:pad + n_out].view(2, 8, 50, 256)
    lse = lcan[pad:pad + 2 * 8 * 50].view(2, 8, 50)
    for splits in (1, 16):
        bd.dm05_set_split_override(splits)
        bd.suffix_attn(d.q, d.k_prefix, d.v_prefix, d.k_suffix, d.v_suffix,
                       prefix_valid_len=d.prefix_valid_len, out=out, lse=lse)
        torch.cuda.synchronize()
        bd.dm05_set_split_override(0)
        assert bool((canary[:pad] == 7.0).all()) and bool((canary[pad + n_out:] == 7.0).all())
        assert bool((lcan[:pad] == 7.0).all()) and bool((lcan[pad + 2 * 8 * 50:] == 7.0).all())
    o_ref, l_ref = ref(inp)
    check_close(out.cpu(), lse.cpu(), o_ref, l_ref, "canary")


def test_waits_for_the_producer_of_its_inputs():
    # q is written by a torch kernel right before the call on the same stream;
    # the call (launched with programmatic dependent launch) must see it.
    inp = gen.base_chunk()
    d = inp.to("cuda")
    q2 = torch.empty_like(d.q)
    out = torch.empty_like(d.q)
    for _ in range(3):
        torch.mul(d.q, -1.0, out=q2)
        bd.suffix_attn(q2, d.k_prefix, d.v_prefix, d.k_suffix, d.v_suffix,
                       prefix_valid_len=d.prefix_valid_len, out=out, want_lse=False)
    torch.cuda.synchronize()
    inp2 = gen.base_chunk()
    inp2.q = -inp2.q
    o_ref, l_ref = ref(inp2)
    check_close(out.cpu(), None, o_ref, l_ref, "pdl producer")


def test_cuda_graph_capture_and_replay():
    calls = gen.history_loop(3)
    ds = [c.to("cuda") for c in calls]
    s = torch.cuda.Stream()
    bd.reserve_for(ds[0].q, ds[0].k_prefix, stream=s)
    outs = [torch.empty_like(d.q) for d in ds]
    lses = [torch.empty(d.q.shape[:3], dtype=torch.float32, device="cuda") for d in ds]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for d, o, l in zip(ds, outs, lses):
            bd.suffix_attn(d.q, d.k_prefix, d.v_prefix, d.k_suffix, d.v_suffix,
                           prefix_valid_len=d.prefix_valid_len, out=o, lse=l, stream=s)
    for o in outs:
        o.zero_()
    g.replay()
    torch.cuda.synchronize()
    for c, o, l in zip(calls, outs, lses):
        o_ref, l_ref = ref(c)
        check_close(o.cpu(), l.cpu(), o_ref, l_ref, c.name)


# ---------------------------------------------------------------- the five workloads, full size

def test_libero_tiny():
    inp = gen.libero_tiny()
    out, lse, _ = run_gpu(inp)
    check_close(out, lse, *ref(inp), what=inp.name)


def test_base_chunk():
    inp = gen.base_chunk()
    out, lse, _ = run_gpu(inp)
    check_close(out, lse, *ref(inp), what=inp.name)


def test_bucket_sweep():
    for inp in gen.bucket_sweep():
        out, lse, _ = run_gpu(inp)
        check_close(out, lse, *ref(inp), what=inp.name)


def test_history_loop():
    for inp in gen.history_loop():
        out, lse, _ = run_gpu(inp)
        check_close(out, lse, *ref(inp), what=inp.name)


def test_batched_mask():
    inp = gen.batched_mask()
    out, lse, _ = run_gpu(inp)
    mx, mean = check_close(out, lse, *ref(inp), what=inp.name)
    assert math.isfinite(mx)


# ---------------------------------------------------------------- size limits

def test_longest_prefix():
    # P = 65535, the longest prefix the supported range is read to cover:
    # 1024 key tiles per (sample, KV head), the last one ragged (63 rows)
    inp = gen.make_inputs(1, 8, 4, 65535, 4, 256, 61, valid_len=65535, mask_frac=0.02)
    plan = bd.dm05_suffix_attn_plan(1, 8, 4, 65535, 4, 256)
    assert plan[0] == 0
    out, lse, word = run_gpu(inp)
    assert word == 0
    check_close(out, lse, *ref(inp), what=f"P=65535 plan {plan[1:]}")


def test_many_units_several_waves():
    # 1024 (sample, KV head) units: one CTA each, about seven waves on 148 SMs
    inp = gen.make_inputs(256, 8, 4, 256, 10, 256, 62, valid_range=(0, 256), mask_frac=0.1)
    out, lse, word = run_gpu(inp)
    assert word == 0
    check_close(out, lse, *ref(inp), what="B=256")


def test_long_prefix_every_split():
    # a long valid range cut 1..16 ways: up to 469 tiles per CTA
    inp = gen.make_inputs(1, 8, 4, 30016, 16, 256, 63, valid_len=30001, peak_frac=0.01, peak_mult=4.0)
    o_ref, l_ref = ref(inp)
    for splits in (1, 4, 16):
        out, lse, _ = run_gpu(inp, splits=splits)
        check_close(out, lse, o_ref, l_ref, f"P=30016 splits={splits}")


def test_per_thread_streams_from_two_threads():
    # cudaStreamPerThread is a different stream on each thread: two threads
    # issuing split calls through it at the same time must not share a
    # workspace.  Every result must equal the single-threaded one bit for bit.
    import threading
    cases = [gen.make_inputs(1, 8, 4, 1024, 50, 256, 71, valid_len=900),
             gen.make_inputs(2, 8, 4, 640, 30, 256, 72, valid_range=(0, 640), mask_frac=0.1)]
    refs = [run_gpu(c)[:2] for c in cases]
    per_thread = 2  # cudaStreamPerThread
    n_calls = 30
    devs = [c.to("cuda") for c in cases]
    outs = [[(torch.empty_like(d.q), torch.empty(d.q.shape[:3], dtype=torch.float32, device="cuda"))
             for _ in range(n_calls)] for d in devs]
    torch.cuda.synchronize()
    ptr = lambda x: None if x is None else x.data_ptr()
    errors = []

    def worker(i):
        try:
            d = devs[i]
            B, Hq, S, D = d.q.shape
            for o, l in outs[i]:
                rc = bd.dm05_suffix_attn(ptr(d.q), ptr(d.k_prefix), ptr(d.v_prefix), ptr(d.prefix_valid_len),
                                         ptr(d.prefix_mask), ptr(d.k_suffix), ptr(d.v_suffix), ptr(o), ptr(l),
                                         B, Hq, d.k_prefix.shape[1], d.k_prefix.shape[2], S, D, per_thread)
                assert rc == 0, rc
            rc, word = bd.dm05_get_error_word(per_thread)  # synchronises this thread's stream
            assert rc == 0 and word == 0, (rc, word)
        except Exception as e:  # reported below
            errors.append(e)

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=120)
    torch.cuda.synchronize()
    assert not errors, errors
    for i in range(2):
        for o, l in outs[i]:
            assert torch.equal(o.cpu().view(torch.int16), refs[i][0].view(torch.int16))
            assert torch.equal(l.cpu(), refs[i][1])


def test_wait_timeout_is_reported_and_the_context_stays_usable():
    # A wait that runs out (a barrier nothing completes, 50 ms limit) sets
    # DM05_EW_WAIT_TIMEOUT and returns; the next attention call on the same
    # context then runs normally with a clean error word.
    s = torch.cuda.Stream()
    sh = s.cuda_stream
    assert bd.dm05_get_error_word(sh)[0] == 0  # clears earlier bits
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s)
    assert bd.dm05_selftest_wait_timeout(50, sh) == 0
    e1.record(s)
    rc, word = bd.dm05_get_error_word(sh)
    assert rc == 0 and word & bd.DM05_EW_WAIT_TIMEOUT, word
    assert e0.elapsed_time(e1) >= 45.0
    inp = gen.make_inputs(1, 8, 4, 200, 10, 256, 81, valid_len=150)
    out, lse, word = run_gpu(inp)
    assert word == 0
    check_close(out, lse, *ref(inp), what="after a wait time-out")


# ---------------------------------------------------------------- static prefix (DM05_FLAG_PREFIX_STATIC)

@pytest.mark.parametrize("case", ["base_chunk", "libero_tiny", "batched_mask"])
def test_prefix_static_flag_gives_the_same_bits(case):
    # the flag only lets the prefix tiles be requested earlier: the result is
    # bit-identical to the default call, for every split count that the
    # automatic plan or the override gives
    inp = gen.WORKLOADS[case]()
    d = inp.to("cuda")
    for splits in (0, 1, 3):
        assert bd.dm05_set_split_override(splits) == 0
        try:
            a = bd.suffix_attn(d.q, d.k_prefix, d.v_prefix, d.k_suffix, d.v_suffix,
                               prefix_valid_len=d.prefix_valid_len, prefix_mask=d.prefix_mask)
            b = bd.suffix_attn(d.q, d.k_prefix, d.v_prefix, d.k_suffix, d.v_suffix,
                               prefix_valid_len=d.prefix_valid_len, prefix_mask=d.prefix_mask, prefix_static=True)
            torch.cuda.synchronize()
        finally:
            bd.dm05_set_split_override(0)
        assert torch.equal(a[0].view(torch.int16), b[0].view(torch.int16)), f"splits={splits}"
        assert torch.equal(a[1], b[1])
    o_ref, l_ref = ref(inp)
    check_close(b[0].cpu(), b[1].cpu(), o_ref, l_ref, f"{case} prefix_static")


def test_prefix_static_still_waits_for_q_and_the_suffix():
    # q, k_suffix and v_suffix are rewritten by torch kernels right before
    # each call; with the static-prefix flag the call must still see them
    inp = gen.base_chunk()
    d = inp.to("cuda")
    q2, ks2, vs2 = torch.empty_like(d.q), torch.empty_like(d.k_suffix), torch.empty_like(d.v_suffix)
    out = torch.empty_like(d.q)
    lse = torch.empty(d.q.shape[:3], dtype=torch.float32, device="cuda")
    for _ in range(3):
        torch.mul(d.q, -1.0, out=q2)
        torch.mul(d.k_suffix, 2.0, out=ks2)
        torch.mul(d.v_suffix, -0.5, out=vs2)
        bd.suffix_attn(q2, d.k_prefix, d.v_prefix, ks2, vs2, prefix_valid_len=d.prefix_valid_len, out=out,
                       lse=lse, prefix_static=True)
    torch.cuda.synchronize()
    inp2 = gen.base_chunk()
    inp2.q = -inp2.q
    inp2.k_suffix = (inp2.k_suffix.float() * 2.0).to(torch.bfloat16)
    inp2.v_suffix = (inp2.v_suffix.float() * -0.5).to(torch.bfloat16)
    o_ref, l_ref = ref(inp2)
    check_close(out.cpu(), lse.cpu(), o_ref, l_ref, "static prefix after producers")


def test_prefix_static_rejects_unknown_flags():
    fake = 0x7f0000001000
    rc = bd.dm05_suffix_attn_ex(fake, fake, fake, None, None, fake, fake, fake, None, 1, 8, 4, 64, 10, 256,
                                0x80, None)
    assert rc == bd.DM05_ERR_SHAPE
