"""The seeded synthetic inputs follow their stated recipes (shapes, length
ranges, value distributions), and the same seed gives the same bits.  The
generators hold no replay arithmetic; both the oracle and the GPU path read
them, so a drift here would move both sides at once."""
import math

import pytest
import torch

import workloads as W


def test_same_seed_same_bits_and_names_are_independent():
    a = W.normal(5, "q", (64, 8))
    assert torch.equal(a, W.normal(5, "q", (64, 8)))
    assert not torch.equal(a, W.normal(5, "k", (64, 8)))
    assert not torch.equal(a, W.normal(6, "q", (64, 8)))


def test_raw_small_recipe():
    x = W.raw_small()
    assert x.lengths == [256]
    assert tuple(x.q.shape) == (256, 2, 64) and tuple(x.k.shape) == (256, 2, 64)
    assert tuple(x.v.shape) == (256, 4, 64) and tuple(x.g.shape) == (256, 4)
    assert x.q.dtype == torch.bfloat16 and x.g.dtype == torch.float32
    # q and k unit-normalised per head (up to their bf16 rounding)
    for t in (x.q, x.k):
        n = t.double().norm(dim=-1)
        assert torch.all((n - 1).abs() < 1e-2)
    assert x.g.min() >= -0.1 and x.g.max() <= -0.001
    assert x.beta.min() >= 0 and x.beta.max() <= 1
    assert x.h0 is None and x.scale == pytest.approx(1 / 8)


def test_raw_qwen_recipe():
    x = W.raw_qwen()
    assert x.n_seqs == 8 and all(512 <= n <= 2048 for n in x.lengths)
    T = sum(x.lengths)
    assert tuple(x.q.shape) == (T, 16, 128) and tuple(x.v.shape) == (T, 32, 128)
    # k normalised, q raw N(0, 1): its per-head norms sit near sqrt(128)
    assert torch.all((x.k.double().norm(dim=-1) - 1).abs() < 1e-2)
    assert abs(x.q.double().norm(dim=-1).mean().item() - math.sqrt(128)) < 0.5
    assert abs(x.v.double().std().item() - 1) < 0.02


def test_suffix_lengths_and_sparse_constants():
    # k = ceil(r m) for the matched prefixes of the whole-model cases
    want = {(8192, 0.05): 410, (16384, 0.05): 820, (32768, 0.05): 1639,
            (8192, 0.10): 820, (16384, 0.10): 1639, (32768, 0.10): 3277}
    assert {c: W.model_suffix(*c) for c in W.MODEL_CASES} == want
    assert W.GROUP_SUFFIX == math.floor(0.05 * 32768)
    pages = W.SPARSE_PREFIX // W.SPARSE_PAGE
    assert pages * W.SPARSE_PER_PAGE == 2048 and W.SPARSE_PER_PAGE / W.SPARSE_PAGE == 1 / 16
    assert min(math.ceil(0.05 * W.SPARSE_PREFIX), W.SPARSE_K_MAX) == 512
    bt = W.block_table(pages, 7)
    assert sorted(bt) == list(range(pages)) and bt == W.block_table(pages, 7)


def test_layer_weight_recipe_on_a_small_shape():
    s = W.LayerShape(hidden=256, inter=512, h_k=2, h_v=4, d_k=128, d_v=128)
    gi = W.group_inputs(3, [100, 30], n_layers=2, shape=s)
    assert gi.lengths == [100, 30] and tuple(gi.anchors.shape) == (130, 256)
    lw = gi.layers[0]
    # projection rows [q | k | v | z | b | a]
    assert tuple(lw.w_in.shape) == (2 * 2 * 128 + 2 * 4 * 128 + 2 * 4, 256)
    assert tuple(lw.conv_w.shape) == (2 * 2 * 128 + 4 * 128, 4)
    assert abs(lw.w_in.double().std().item() - 0.02) < 1e-3
    assert torch.all(lw.w_in_norm == 1) and torch.all(lw.w_gnorm == 1) and torch.all(lw.w_post_norm == 1)
    assert torch.all(lw.dt_bias == 0)
    assert lw.a_log.min() >= 0 and lw.a_log.max() <= math.log(16)
    assert not torch.equal(gi.layers[0].w_in, gi.layers[1].w_in)


def test_full_group_shape_constants():
    s = W.LayerShape()
    assert (s.hidden, s.inter, s.h_k, s.h_v, s.d_k, s.d_v) == (2560, 9216, 16, 32, 128, 128)
    assert s.proj_dim == 12352 and s.conv_w == 4


def test_mamba2_recipe():
    lengths = W.mamba2_lengths()
    assert len(lengths) == 64 and all(256 <= n <= 4096 for n in lengths)
    m = W.mamba2_inputs(4, [300, 0, 65])  # the full workload's distributions on a small case
    assert tuple(m.x.shape) == (365, 64, 64) and tuple(m.B.shape) == (365, 1, 128)
    assert torch.all(m.dt > 0)
    sp = torch.nn.functional.softplus
    assert torch.allclose(m.dt, sp(torch.randn(365, 64, generator=W.substream(4, "dt"))))
    assert torch.all(m.A <= -1) and torch.all(m.A >= -math.exp(2))
    assert m.lengths == [300, 0, 65]
