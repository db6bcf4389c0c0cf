"""Seeded synthetic inputs for suffix-replay state reconstruction.

This module only *draws* inputs.  It holds none of the replay arithmetic:
no recurrence, no layer math, no chunking.  Both the fp64 oracle (via the
tests) and the CUDA path (via the tests, ``bench.py`` and the smoke check)
take their inputs from here, so that the two sides see bit-identical data.

Every tensor is drawn from its own counter-free substream: the torch CPU
generator seeded with a 64-bit hash of ``(base_seed, tensor_name)``.  Data
that the workloads specify as bf16 is drawn in fp32 and rounded to bf16
(round-to-nearest-even, ``Tensor.to(torch.bfloat16)``); the fp64 value of a
bf16 element is exact, so the oracle consumes exactly what the GPU reads.

Workloads (sizes follow the method's own evaluation settings: 8K/16K/32K
matched prefixes replayed at 5 % and 10 %, "Tail-Replay", Sec. 3 and 4):

* ``raw_small``   one GDN layer, N=1, T=256, 2 QK / 4 V heads, d=64.
* ``raw_qwen``    one GDN layer, 8 sequences of U{512..2048} tokens,
                  16 QK / 32 V heads, d=128 (Qwen3.5-4B-like head shapes).
* ``group``       one replay group of 3 GDN layers + SwiGLU MLPs over a
                  1638-token anchor suffix, hidden 2560, intermediate 9216.
* ``model``       8 independent groups, suffix k = ceil(r*m) for
                  m in {8K,16K,32K}, r in {5 %, 10 %}.
* ``mamba2``      64 sequences of U{256..4096} tokens, 64 heads, P=64, N=128.
"""
from __future__ import annotations

import hashlib
import math
from dataclasses import dataclass, field

import torch

# ---------------------------------------------------------------- helpers


def substream(base_seed: int, name: str) -> torch.Generator:
    """Independent torch CPU generator for one named tensor."""
    h = hashlib.sha256(f"{base_seed}:{name}".encode()).digest()
    return torch.Generator().manual_seed(int.from_bytes(h[:8], "little") & ((1 << 63) - 1))


def normal(base_seed, name, shape, std=1.0, dtype=torch.bfloat16):
    t = torch.randn(*shape, generator=substream(base_seed, name), dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def uniform(base_seed, name, shape, lo, hi, dtype=torch.float32):
    t = torch.rand(*shape, generator=substream(base_seed, name), dtype=torch.float32)
    return (t * (hi - lo) + lo).to(dtype)


def randint_lengths(base_seed, name, n, lo, hi):
    """n sequence lengths drawn uniformly from the inclusive range [lo, hi]."""
    return torch.randint(lo, hi + 1, (n,), generator=substream(base_seed, name)).tolist()


def cu_from_lengths(lengths) -> torch.Tensor:
    cu = [0]
    for n in lengths:
        cu.append(cu[-1] + int(n))
    return torch.tensor(cu, dtype=torch.int32)


def l2_normalised_bf16(base_seed, name, shape):
    """N(0,1) rows, scaled to unit L2 norm over the last axis, then rounded to
    bf16 (the workload recipe asks for normalised q / k as *inputs*)."""
    t = torch.randn(*shape, generator=substream(base_seed, name), dtype=torch.float64)
    t = t / t.norm(dim=-1, keepdim=True)
    return t.to(torch.float32).to(torch.bfloat16)


# ---------------------------------------------------------------- raw GDN


@dataclass
class GdnInputs:
    q: torch.Tensor          # [T, Hk, dk]  bf16 (or fp32)
    k: torch.Tensor          # [T, Hk, dk]
    v: torch.Tensor          # [T, Hv, dv]
    g: torch.Tensor          # [T, Hv] fp32, natural-log decay (alpha = exp(g))
    beta: torch.Tensor       # [T, Hv] fp32
    cu_seqlens: torch.Tensor  # [N+1] int32
    h0: torch.Tensor | None = None  # [N, Hv, dv, dk] fp32
    scale: float = 0.0

    @property
    def n_seqs(self):
        return self.cu_seqlens.numel() - 1

    @property
    def lengths(self):
        c = self.cu_seqlens.tolist()
        return [c[i + 1] - c[i] for i in range(len(c) - 1)]

    @property
    def max_seqlen(self):
        return max(self.lengths) if self.n_seqs else 0


def gdn_inputs(seed, lengths, h_k, h_v, d_k, d_v, *, norm_q=True, norm_k=True,
               g_range=(-0.1, -0.001), beta_range=(0.0, 1.0), h0_std=None,
               dtype=torch.bfloat16) -> GdnInputs:
    """Raw gated-delta replay inputs: q/k/v ~ N(0,1) (optionally L2-normalised
    per head), g ~ U(g_range), beta ~ U(beta_range), S_0 = 0 unless h0_std."""
    T = int(sum(lengths))
    if norm_q:
        q = l2_normalised_bf16(seed, "q", (T, h_k, d_k))
    else:
        q = normal(seed, "q", (T, h_k, d_k))
    if norm_k:
        k = l2_normalised_bf16(seed, "k", (T, h_k, d_k))
    else:
        k = normal(seed, "k", (T, h_k, d_k))
    v = normal(seed, "v", (T, h_v, d_v))
    if dtype == torch.float32:
        # fp32-input mode: full-precision draws of the same distributions
        q = torch.randn(T, h_k, d_k, generator=substream(seed, "q32"))
        k = torch.randn(T, h_k, d_k, generator=substream(seed, "k32"))
        v = torch.randn(T, h_v, d_v, generator=substream(seed, "v32"))
        if norm_q:
            q = q / q.norm(dim=-1, keepdim=True)
        if norm_k:
            k = k / k.norm(dim=-1, keepdim=True)
    g = uniform(seed, "g", (T, h_v), *g_range)
    beta = uniform(seed, "beta", (T, h_v), *beta_range)
    h0 = None
    if h0_std is not None:
        h0 = normal(seed, "h0", (len(lengths), h_v, d_v, d_k), std=h0_std, dtype=torch.float32)
    return GdnInputs(q, k, v, g, beta, cu_from_lengths(lengths), h0, 1.0 / math.sqrt(d_k))


def raw_small(seed=0x5EED0000) -> GdnInputs:
    """One GDN layer: N=1, T=256, H_k=2, H_v=4, d=64, q and k normalised."""
    return gdn_inputs(seed, [256], 2, 4, 64, 64, norm_q=True, norm_k=True)


def raw_qwen_lengths(seed=0x5EED0001, n=8, lo=512, hi=2048):
    return randint_lengths(seed, "lengths", n, lo, hi)


def raw_qwen(seed=0x5EED0001, lengths=None) -> GdnInputs:
    """One GDN layer at Qwen3.5-4B-like head shapes: 8 varlen suffixes drawn
    from U{512..2048}, H_k=16, H_v=32, d=128, k normalised, q raw."""
    if lengths is None:
        lengths = raw_qwen_lengths(seed)
    return gdn_inputs(seed, lengths, 16, 32, 128, 128, norm_q=False, norm_k=True)


# ---------------------------------------------------------------- group replay

HIDDEN = 2560
INTER = 9216
H_K, H_V, D_HEAD = 16, 32, 128
CONV_W = 4
EPS = 1e-6


@dataclass
class LayerShape:
    hidden: int = HIDDEN
    inter: int = INTER
    h_k: int = H_K
    h_v: int = H_V
    d_k: int = D_HEAD
    d_v: int = D_HEAD
    conv_w: int = CONV_W
    eps: float = EPS

    @property
    def qk_dim(self):
        return self.h_k * self.d_k

    @property
    def v_dim(self):
        return self.h_v * self.d_v

    @property
    def conv_dim(self):
        return 2 * self.qk_dim + self.v_dim

    @property
    def proj_dim(self):
        # [q | k | v | z | b | a]
        return self.conv_dim + self.v_dim + 2 * self.h_v


@dataclass
class LayerWeights:
    w_in_norm: torch.Tensor   # [hidden] bf16
    w_in: torch.Tensor        # [proj_dim, hidden] bf16
    conv_w: torch.Tensor      # [conv_dim, conv_w] bf16
    a_log: torch.Tensor       # [h_v] fp32
    dt_bias: torch.Tensor     # [h_v] fp32
    w_gnorm: torch.Tensor     # [d_v] bf16
    w_out: torch.Tensor       # [hidden, v_dim] bf16
    w_post_norm: torch.Tensor  # [hidden] bf16
    w_gate: torch.Tensor      # [inter, hidden] bf16
    w_up: torch.Tensor        # [inter, hidden] bf16
    w_down: torch.Tensor      # [hidden, inter] bf16


def layer_weights(seed, layer: int, s: LayerShape, std=0.02) -> LayerWeights:
    """Random-init layer weights: projections and conv ~ N(0, std) bf16,
    A_log ~ U(ln 1, ln 16), dt_bias = 0, every norm weight = 1."""
    p = f"L{layer}."
    ones_h = torch.ones(s.hidden, dtype=torch.bfloat16)
    return LayerWeights(
        w_in_norm=ones_h.clone(),
        w_in=normal(seed, p + "w_in", (s.proj_dim, s.hidden), std),
        conv_w=normal(seed, p + "conv_w", (s.conv_dim, s.conv_w), std),
        a_log=uniform(seed, p + "a_log", (s.h_v,), 0.0, math.log(16.0)),
        dt_bias=torch.zeros(s.h_v, dtype=torch.float32),
        w_gnorm=torch.ones(s.d_v, dtype=torch.bfloat16),
        w_out=normal(seed, p + "w_out", (s.hidden, s.v_dim), std),
        w_post_norm=ones_h.clone(),
        w_gate=normal(seed, p + "w_gate", (s.inter, s.hidden), std),
        w_up=normal(seed, p + "w_up", (s.inter, s.hidden), std),
        w_down=normal(seed, p + "w_down", (s.hidden, s.inter), std),
    )


@dataclass
class GroupInputs:
    anchors: torch.Tensor          # [T, hidden] bf16
    cu_seqlens: torch.Tensor       # [N+1] int32
    layers: list                   # [n_layers] LayerWeights
    shape: LayerShape = field(default_factory=LayerShape)

    @property
    def lengths(self):
        c = self.cu_seqlens.tolist()
        return [c[i + 1] - c[i] for i in range(len(c) - 1)]


def group_inputs(seed, lengths, n_layers=3, shape: LayerShape | None = None,
                 anchor_std=1.0) -> GroupInputs:
    s = shape or LayerShape()
    T = int(sum(lengths))
    anchors = normal(seed, "anchors", (T, s.hidden), anchor_std)
    layers = [layer_weights(seed, l, s) for l in range(n_layers)]
    return GroupInputs(anchors, cu_from_lengths(lengths), layers, s)


GROUP_SUFFIX = 1638  # 5 % of a 32K matched prefix (floor of 0.05 * 32768)


def group(seed=0x5EED0002) -> GroupInputs:
    """One replay group: 3 GDN layers + SwiGLU MLPs over a 1638-token suffix."""
    return group_inputs(seed, [GROUP_SUFFIX])


def model_suffix(prefix: int, ratio: float) -> int:
    """Replay length k = ceil(r * m) for a matched prefix of m tokens."""
    return int(math.ceil(ratio * prefix - 1e-9))


MODEL_CASES = [(m, r) for m in (8192, 16384, 32768) for r in (0.05, 0.10)]


def model_group(prefix, ratio, g, seed=0x5EED0003, shape=None) -> GroupInputs:
    """Group g of the 8-group whole-model replay (independent seed per group)."""
    return group_inputs(seed + g, [model_suffix(prefix, ratio)], shape=shape)


SPARSE_PREFIX = 32768     # matched prefix of the token-sparse replay workload
SPARSE_PAGE = 64          # tokens per page
SPARSE_PER_PAGE = 4       # anchors per page (density 1/16)
SPARSE_K_MAX = 512        # replay budget cap in anchors


def anchor_pool_group(pool_rows, k, seed, shape=None, n_layers=3) -> GroupInputs:
    """A group whose `anchors` is an anchor pool of pool_rows random bf16
    hiddens (N(0,1)) from which a replay of k tokens gathers its rows; the
    weights follow layer_weights."""
    s = shape or LayerShape()
    pool = normal(seed, "pool", (pool_rows, s.hidden), 1.0)
    layers = [layer_weights(seed, l, s) for l in range(n_layers)]
    return GroupInputs(pool, cu_from_lengths([k]), layers, s)


def block_table(n_pages, seed) -> list:
    """A seeded page -> pool-block permutation (the sidecar's page table)."""
    return torch.randperm(n_pages, generator=substream(seed, "block_table")).tolist()


# ---------------------------------------------------------------- Mamba2


@dataclass
class Mamba2Inputs:
    x: torch.Tensor          # [T, H, P] bf16
    B: torch.Tensor          # [T, G, Ns] bf16
    C: torch.Tensor          # [T, G, Ns] bf16
    dt: torch.Tensor         # [T, H] fp32
    A: torch.Tensor          # [H] fp32
    cu_seqlens: torch.Tensor
    h0: torch.Tensor | None = None  # [N, H, P, Ns] fp32

    @property
    def lengths(self):
        c = self.cu_seqlens.tolist()
        return [c[i + 1] - c[i] for i in range(len(c) - 1)]

    @property
    def max_seqlen(self):
        return max(self.lengths) if self.lengths else 0


def mamba2_inputs(seed, lengths, H=64, P=64, Ns=128, G=1, h0_std=None) -> Mamba2Inputs:
    """x, B, C ~ N(0,1) bf16; dt = softplus(N(0,1)) fp32; A = -exp(U(0,2))."""
    T = int(sum(lengths))
    x = normal(seed, "x", (T, H, P))
    B = normal(seed, "B", (T, G, Ns))
    C = normal(seed, "C", (T, G, Ns))
    dt = torch.nn.functional.softplus(
        torch.randn(T, H, generator=substream(seed, "dt"), dtype=torch.float32))
    A = -torch.exp(uniform(seed, "A", (H,), 0.0, 2.0))
    h0 = None
    if h0_std is not None:
        h0 = normal(seed, "h0", (len(lengths), H, P, Ns), std=h0_std, dtype=torch.float32)
    return Mamba2Inputs(x, B, C, dt, A, cu_from_lengths(lengths), h0)


def mamba2_lengths(seed=0x5EED0004, n=64, lo=256, hi=4096):
    return randint_lengths(seed, "lengths", n, lo, hi)


def mamba2(seed=0x5EED0004, lengths=None) -> Mamba2Inputs:
    if lengths is None:
        lengths = mamba2_lengths(seed)
    return mamba2_inputs(seed, lengths)
