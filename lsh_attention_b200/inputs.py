"""Seeded synthetic inputs and the named workloads.

This module only draws random numbers and names shapes; it holds none of the
attention method's arithmetic. Both the CUDA path (through the tests and the
bench) and the CPU oracle consume the tensors it returns, so the two sides see
bit-identical inputs.

Recipe (fixed, so every run reproduces the same values):

* shared-QK vectors ``x`` and values ``v``: a CPU ``torch.Generator`` seeded
  with ``data_seed`` (0) draws ``x = randn(B, H, n, d)`` and then
  ``v = randn(B, H, n, d)`` in fp32.
* clustered ``x`` (skewed bucket histograms): the same generator first draws
  ``centres = randn(32, d)``, then ``assign = randint(0, 32, (B, H, n))``, then
  ``x = centres[assign] + 0.3 * randn(B, H, n, d)``, then ``v``.
* random rotations ``R``: a second generator seeded with ``r_seed`` (1) draws
  ``randn(rounds, d, n_buckets // 2)`` in fp32.
* bf16 workloads cast the fp32 draws to bf16 (round to nearest even).

The workloads mirror the shapes the Reformer pages train on (enwik8-64K text,
imagenet64 images flattened to 12288 positions); the data itself is synthetic.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import torch

N_CLUSTERS = 32
CLUSTER_SIGMA = 0.3


@dataclass(frozen=True)
class Workload:
    """One attention problem: shapes, hashing parameters and input recipe."""

    name: str
    batch: int
    heads: int
    n: int
    d: int
    n_buckets: int
    chunk: int
    rounds: int
    causal: bool
    dtype: str  # "f32" or "bf16"
    clustered: bool = False
    data_seed: int = 0
    r_seed: int = 1

    @property
    def tokens(self) -> int:
        """Tokens per forward pass as the metric counts them (batch x length)."""
        return self.batch * self.n

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


TINY_F32 = Workload("tiny-f32", 1, 1, 1024, 64, 16, 64, 1, False, "f32")
BF16_SHORT = Workload("bf16-short", 2, 8, 4096, 64, 64, 64, 2, True, "bf16")
LONG_64K = Workload("long-64k", 1, 8, 65536, 128, 1024, 64, 4, True, "bf16")
IMAGE_12K = Workload("image-12k", 8, 8, 12288, 64, 192, 64, 8, True, "bf16", clustered=True)


def sweep_workloads() -> list[Workload]:
    """Length x rounds sweep: n in {2K, 8K, 32K, 128K}, rounds in {1, 2, 4, 8},
    one batch, eight heads, d=64, n/64 buckets, chunk 64, causal, bf16, each on
    isotropic and on 32-cluster inputs."""
    out = []
    for n in (2048, 8192, 32768, 131072):
        for rounds in (1, 2, 4, 8):
            for clustered in (False, True):
                tag = "clu" if clustered else "iso"
                out.append(Workload(f"sweep-n{n}-r{rounds}-{tag}", 1, 8, n, 64, n // 64, 64,
                                    rounds, True, "bf16", clustered=clustered))
    return out


WORKLOADS = {w.name: w for w in (TINY_F32, BF16_SHORT, LONG_64K, IMAGE_12K)}


def torch_dtype(name: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def make_qkv(w: Workload) -> tuple[torch.Tensor, torch.Tensor]:
    """Shared-QK vectors x and values v, shape [B, H, n, d], CPU, in w.dtype."""
    g = torch.Generator(device="cpu").manual_seed(w.data_seed)
    shape = (w.batch, w.heads, w.n, w.d)
    if w.clustered:
        centres = torch.randn(N_CLUSTERS, w.d, generator=g)
        assign = torch.randint(0, N_CLUSTERS, shape[:3], generator=g)
        x = centres[assign] + CLUSTER_SIGMA * torch.randn(shape, generator=g)
    else:
        x = torch.randn(shape, generator=g)
    v = torch.randn(shape, generator=g)
    dt = torch_dtype(w.dtype)
    return x.to(dt).contiguous(), v.to(dt).contiguous()


def make_rotations(w: Workload) -> torch.Tensor:
    """Random rotations R, shape [rounds, d, n_buckets/2], CPU, in w.dtype."""
    g = torch.Generator(device="cpu").manual_seed(w.r_seed)
    r = torch.randn(w.rounds, w.d, w.n_buckets // 2, generator=g)
    return r.to(torch_dtype(w.dtype)).contiguous()


def make_buckets(w: Workload, seed: int = 7) -> torch.Tensor:
    """Uniform random bucket ids, shape [B, H, rounds, n], int32 (for feeding the
    sort and the attention with caller-supplied buckets)."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    return torch.randint(0, w.n_buckets, (w.batch, w.heads, w.rounds, w.n), generator=g,
                         dtype=torch.int64).to(torch.int32)


def make_rev_weights(d_model: int, d_ff: int, seed: int = 2) -> dict:
    """Weights of a reversible block (bf16, out x in; biases fp32): N(0, 1)
    scaled by 1/sqrt(fan-in) so activations stay of unit size."""
    g = torch.Generator(device="cpu").manual_seed(seed)

    def w(out_f, in_f):
        return (torch.randn(out_f, in_f, generator=g) / in_f ** 0.5).to(torch.bfloat16)

    return {"w_qk": w(d_model, d_model), "w_v": w(d_model, d_model), "w_o": w(d_model, d_model),
            "w1": w(d_ff, d_model), "b1": 0.1 * torch.randn(d_ff, generator=g),
            "w2": w(d_model, d_ff), "b2": 0.1 * torch.randn(d_model, generator=g)}


def make_rev_inputs(batch: int, n: int, d_model: int, seed: int = 3):
    """The two halves x1, x2 [batch, n, d_model] of a reversible block's input,
    N(0, 1) in bf16."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    x1 = torch.randn(batch, n, d_model, generator=g).to(torch.bfloat16)
    x2 = torch.randn(batch, n, d_model, generator=g).to(torch.bfloat16)
    return x1, x2


def make_topk_projections(rounds: int, d: int, n_bits: int, seed: int = 1) -> torch.Tensor:
    """SimHash projections of the top-k variant, [rounds, d, n_bits], N(0, 1)
    rounded to bf16."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    return torch.randn(rounds, d, n_bits, generator=g).to(torch.bfloat16)
