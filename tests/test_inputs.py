"""The seeded input generators: shapes taken from the pages, recipe
properties, determinism.  CPU only."""
import json
import os

import torch

from gqa_prefix_suffix_b200 import inputs

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_shapes.json")))


def test_head_geometry_matches_pages():
    g = GOLDEN["suffix_attention_heads"]
    assert (inputs.HQ, inputs.HKV, inputs.HEAD_DIM) == (g["q_heads"], g["kv_heads"], g["head_dim"])
    # the suffix attention reads the prefix decoder's KV cache: same KV geometry
    p = GOLDEN["prefix_decoder_heads"]
    assert (p["kv_heads"], p["head_dim"]) == (g["kv_heads"], g["head_dim"])


def test_buckets_and_chunks_match_pages():
    assert list(inputs.PREFIX_BUCKETS) == GOLDEN["prefix_buckets_default"]["values"]
    chunks = GOLDEN["action_chunk_sizes"]
    assert inputs.libero_tiny().S == chunks["libero"]
    assert inputs.base_chunk().S == chunks["base_model"]
    h = inputs.history_loop(2)
    assert h[0].P == GOLDEN["prefix_bucket_history"]["value"]
    assert len(inputs.history_loop()) == GOLDEN["diffusion_steps_default"]["value"]


def test_shapes_dtypes():
    for x in (inputs.libero_tiny(), inputs.base_chunk(), inputs.batched_mask()):
        B, Hq, Hkv, P, S, D = x.B, x.Hq, x.Hkv, x.P, x.S, x.D
        assert x.q.shape == (B, Hq, S, D) and x.q.dtype == torch.bfloat16
        assert x.k_prefix.shape == (B, Hkv, P, D) and x.v_prefix.shape == (B, Hkv, P, D)
        assert x.k_suffix.shape == (B, Hkv, S, D) and x.v_suffix.shape == (B, Hkv, S, D)
        assert x.prefix_valid_len.dtype == torch.int32 and x.prefix_valid_len.shape == (B,)


def test_determinism():
    a, b = inputs.base_chunk(), inputs.base_chunk()
    for k, t in a.tensors().items():
        if t is not None:
            assert torch.equal(t, b.tensors()[k])


def test_peaked_rows_recipe():
    x = inputs.base_chunk()
    rows = x.meta["peak_rows"][0]
    assert len(rows) == round(0.05 * 1024) == 51
    # regenerate without the peak step: only the chosen rows differ, by x3.0
    gen = torch.Generator().manual_seed(1001)
    torch.randn((1, 8, 50, 256), generator=gen)
    kp = torch.randn((1, 4, 1024, 256), generator=gen)
    other = sorted(set(range(1024)) - set(rows))
    assert torch.equal(x.k_prefix[0, :, other], kp[0, :, other].to(torch.bfloat16))
    assert torch.equal(x.k_prefix[0, :, rows], (kp[0, :, rows] * 3.0).to(torch.bfloat16))


def test_batched_mask_recipe():
    x = inputs.batched_mask()
    vl = x.prefix_valid_len
    assert int(vl.min()) >= 576 and int(vl.max()) <= 1024
    for b in range(x.B):
        v = int(vl[b])
        hidden = int((x.prefix_mask[b, :v] == 0).sum())
        assert hidden == round(0.10 * v)
        assert bool((x.prefix_mask[b, v:] == 1).all())
        assert len(x.meta["peak_rows"][b]) == round(0.01 * 1024)


def test_bucket_sweep_ranges():
    calls = inputs.bucket_sweep()
    assert len(calls) == 25
    for c in calls:
        v = int(c.prefix_valid_len[0])
        assert c.P - 128 <= v <= c.P


def test_history_shares_prefix():
    h = inputs.history_loop(3)
    assert h[0].k_prefix.data_ptr() == h[1].k_prefix.data_ptr()
    assert not torch.equal(h[0].q, h[1].q)
