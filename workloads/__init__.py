"""Seeded synthetic workloads for the causal long convolution.

This module holds no convolution arithmetic: it only draws the inputs (u, k and
the optional gates w, v and frequency mask) from seeded numpy generators and
rounds them to the I/O dtype.  Both the CUDA path's tests/benchmark and the
fp64 oracle read the same rounded values, so input rounding is not part of any
measured error.

Recipe: seed = 1000 + workload index; tensor ``t`` of a workload draws from
``np.random.default_rng([seed, TENSOR_IDS[t]])``.  Values are drawn in float32
and rounded to the dtype with round-to-nearest-even (torch ``.to``).

The workloads mirror the sequence lengths the FlashFFTConv page measures
(1K forward latency, 8K Hyena filters with 2K partial filters, the 1M-token
HyenaDNA setting and its extension to 4M tokens with partial filters, 75%
frequency sparsity); there is no dataset here, and the DNA-like workloads are
a synthetic stand-in for genome data.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

TENSOR_IDS = {"u": 1, "w": 2, "v": 3, "k": 4, "mask": 5, "proj": 6, "sym": 7, "dy": 8}
MASK_BLOCK = 32


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int          # 1-based workload number (seed = 1000 + index)
    B: int
    H: int
    N: int
    L: int              # filter length (L == N unless partial)
    dtype: str          # "f32" | "f16" | "bf16"
    gated: bool
    k_kind: str         # "scaled" (N(0,1)/sqrt(N)), "decay:<a>", "plain"
    u_kind: str = "normal"   # "normal" | "dna"
    sparsity: float = 0.0    # fraction of mask blocks zeroed (0 = no mask)
    description: str = ""
    monarch_keep: int = 0    # Monarch-aligned mask: bit c2 keeps the middle digit c2 (0 = none)
    shard: int = 0           # channel shard (one per rank); 0 = the workload itself

    @property
    def seed(self) -> int:
        return 1000 + self.index

    @property
    def elems(self) -> int:
        return self.B * self.H * self.N

    def with_shape(self, B: Optional[int] = None, H: Optional[int] = None,
                   N: Optional[int] = None, L: Optional[int] = None) -> "Workload":
        """Same recipe at another shape (the parity tests' reduced sizes)."""
        N2 = N if N is not None else self.N
        if L is not None:
            L2 = L
        elif self.L == self.N:
            L2 = N2
        else:
            L2 = max(1, self.L * N2 // self.N)
        return dataclasses.replace(self, B=B if B is not None else self.B,
                                   H=H if H is not None else self.H, N=N2, L=L2)


WORKLOADS = {
    "fp32_n1k": Workload("fp32_n1k", 1, 1, 8, 1024, 1024, "f32", False, "scaled",
                         description="fp32 causal conv B=1 H=8 N=1024, FFT size 2048"),
    "gated_bf16_n4k": Workload("gated_bf16_n4k", 2, 64, 768, 4096, 4096, "bf16", True,
                               "decay:0.001",
                               description="gated bf16 conv B=64 H=768 N=4096"),
    "fp16_n32k": Workload("fp16_n32k", 3, 8, 256, 32768, 32768, "f16", False, "scaled",
                          description="fp16 conv B=8 H=256 N=32768"),
    "dna_bf16_n1m": Workload("dna_bf16_n1m", 4, 1, 128, 1 << 20, 1 << 20, "bf16", False,
                             "decay:1e-5", u_kind="dna",
                             description="bf16 conv B=1 H=128 N=1M, DNA-like input"),
    "partial_bf16_n8k": Workload("partial_bf16_n8k", 5, 16, 768, 8192, 2048, "bf16", True,
                                 "plain",
                                 description="gated bf16 B=16 H=768 N=8192, filter length 2048"),
    "sparse_bf16_n8k": Workload("sparse_bf16_n8k", 6, 16, 768, 8192, 8192, "bf16", True,
                                "plain", sparsity=0.75,
                                description="gated bf16 B=16 H=768 N=8192, 75% block-sparse rfft(k)"),
    # the sequence extension with partial filters (1M-token filters on 4M
    # sequences), the same element count as the 1M DNA workload
    "dna_bf16_n4m_l1m": Workload("dna_bf16_n4m_l1m", 7, 1, 32, 1 << 22, 1 << 20, "bf16", False,
                                 "decay:1e-5", u_kind="dna",
                                 description="bf16 conv B=1 H=32 N=4M, filter length 1M, DNA-like input"),
    # sequence length 1K at the flagship's batch x channels (64 x 768): the
    # length of the page's kernel-level latency rows, gated and ungated
    "gated_bf16_n1k": Workload("gated_bf16_n1k", 8, 64, 768, 1024, 1024, "bf16", True, "decay:0.001",
                               description="gated bf16 conv B=64 H=768 N=1024"),
    "bf16_n1k": Workload("bf16_n1k", 9, 64, 768, 1024, 1024, "bf16", False, "scaled",
                         description="bf16 conv B=64 H=768 N=1024"),
    # sequence length 16K at cfg3's element count: the four-block fused
    # tensor-core mode (the 32K configuration runs staged)
    "fp16_n16k": Workload("fp16_n16k", 11, 16, 256, 16384, 16384, "f16", False, "scaled",
                          description="fp16 conv B=16 H=256 N=16384"),
    # the flagship shape with a Monarch-aligned 75% frequency mask: the middle
    # digits c2 in {0..3, 28..31} of the 8192-point spectrum are kept
    "monarch_bf16_n4k": Workload("monarch_bf16_n4k", 10, 64, 768, 4096, 4096, "bf16", True, "decay:0.001",
                                 monarch_keep=0xF000000F,
                                 description="gated bf16 conv B=64 H=768 N=4096, Monarch-aligned 75% sparse"),
}

# The workload the benchmark times at one GPU.
BENCH_WORKLOAD = "gated_bf16_n4k"


# Tensors every channel shard shares: the DNA symbol stream (one per batch
# row, embedded into every channel) and the frequency mask row.
SHARED_TENSORS = ("sym", "mask")


def _rng(w: Workload, tensor: str) -> np.random.Generator:
    if w.shard == 0 or tensor in SHARED_TENSORS:
        return np.random.default_rng([w.seed, TENSOR_IDS[tensor]])
    return np.random.default_rng([w.seed, TENSOR_IDS[tensor], w.shard])


def shard_of(w: Workload, rank: int) -> Workload:
    """Rank `rank`'s channel shard of the multi-GPU problem built on `w`.

    With R ranks the whole problem has H*R channels: shard r holds channels
    [r*H, (r+1)*H), drawn from its own seeded streams (u, w, v, k and the DNA
    projection take the shard id as a third seed word), while the DNA symbol
    stream and the mask row are the same on every shard.  Shard 0 is the
    workload itself, so a one-rank run is unchanged."""
    if rank < 0:
        raise ValueError(rank)
    return dataclasses.replace(w, shard=rank)


def round_to(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float32 values to `dtype` (RNE) and return them as float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "f32":
        return x
    import torch
    tdt = {"f16": torch.float16, "bf16": torch.bfloat16}[dtype]
    return torch.from_numpy(x).to(tdt).to(torch.float32).numpy()


def torch_dtype(dtype: str):
    import torch
    return {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[dtype]


def _normal(rng, shape):
    return rng.standard_normal(size=shape, dtype=np.float32)


def make_filter(w: Workload) -> np.ndarray:
    rng = _rng(w, "k")
    k = _normal(rng, (w.H, w.L))
    if w.k_kind == "scaled":
        k = k / np.float32(math.sqrt(w.N))
    elif w.k_kind.startswith("decay:"):
        a = float(w.k_kind.split(":", 1)[1])
        t = np.arange(w.L, dtype=np.float64)
        k = (k * np.exp(-a * t)[None, :]).astype(np.float32)
    elif w.k_kind != "plain":
        raise ValueError(w.k_kind)
    return round_to(k, w.dtype)


def make_input(w: Workload) -> np.ndarray:
    if w.u_kind == "normal":
        return round_to(_normal(_rng(w, "u"), (w.B, w.H, w.N)), w.dtype)
    if w.u_kind == "dna":
        # one-hot embedded 4-symbol sequence projected by a seeded 4 x H matrix:
        # u[b, h, t] = P[s[b, t], h]
        sym = _rng(w, "sym").integers(0, 4, size=(w.B, w.N))
        P = _normal(_rng(w, "proj"), (4, w.H))
        u = np.transpose(P[sym], (0, 2, 1))  # [B, H, N]
        return round_to(np.ascontiguousarray(u), w.dtype)
    raise ValueError(w.u_kind)


def make_gates(w: Workload):
    if not w.gated:
        return None, None
    g = round_to(_normal(_rng(w, "w"), (w.B, w.H, w.N)), w.dtype)
    v = round_to(_normal(_rng(w, "v"), (w.B, w.H, w.N)), w.dtype)
    return g, v


def monarch_binmask(keep: int, N: int) -> np.ndarray:
    """[2N] uint8 per-bin mask of the 2N-point spectrum that a Monarch-aligned
    keep set selects: with f = c1 + 32 c2 + 1024 c3 (the middle digit
    c2 = (f >> 5) & 31), bin f is kept iff the c2 of f and the c2 of its mirror
    (2N - f) mod 2N are both in `keep` (bit c2)."""
    M = 2 * N
    f = np.arange(M)
    c2 = (f >> 5) & 31
    c2m = (((M - f) % M) >> 5) & 31
    bit = lambda c: (np.uint64(keep) >> c.astype(np.uint64)) & np.uint64(1)
    return (bit(c2) & bit(c2m)).astype(np.uint8)


def monarch_kept_fraction(w: Workload) -> float:
    """Fraction of the rfft bins [0, N] a Monarch-aligned workload keeps."""
    m = monarch_binmask(w.monarch_keep, w.N)
    return float(m[:w.N + 1].sum()) / (w.N + 1)


def make_mask(w: Workload) -> Optional[np.ndarray]:
    """[1, N/32] uint8 block mask (1 = keep): exactly round(sparsity * N/32) blocks
    are zeroed, the first ones of a seeded permutation of block ids."""
    if w.sparsity <= 0.0:
        return None
    nblk = w.N // MASK_BLOCK
    nzero = int(round(w.sparsity * nblk))
    perm = _rng(w, "mask").permutation(nblk)
    m = np.ones((1, nblk), dtype=np.uint8)
    m[0, perm[:nzero]] = 0
    return m


def make_grad_output(w: Workload) -> np.ndarray:
    """The incoming gradient dy [B, H, N] of a backward call: standard
    normal, rounded to the workload's dtype, from its own seeded stream."""
    return round_to(_normal(_rng(w, "dy"), (w.B, w.H, w.N)), w.dtype)


def make_all(w: Workload):
    """dict(u, k, w, v, mask) of float32 numpy arrays (dtype-rounded values)."""
    g, v = make_gates(w)
    return {"u": make_input(w), "k": make_filter(w), "w": g, "v": v, "mask": make_mask(w)}


def sample_points(w: Workload, nseq: int = 16, nrand: int = 61, seed_offset: int = 0):
    """Seeded (sequence, t) sample list: t in {0, 1, N-1} plus `nrand` random t,
    on `nseq` random sequences (flattened b*H + h)."""
    rng = np.random.default_rng([w.seed, 100 + seed_offset])
    S = w.B * w.H
    seqs = rng.choice(S, size=min(nseq, S), replace=False)
    out_s, out_t = [], []
    for s in seqs:
        ts = [0, min(1, w.N - 1), w.N - 1] + list(rng.integers(0, w.N, size=nrand))
        out_s += [int(s)] * len(ts)
        out_t += [int(t) for t in ts]
    return np.asarray(out_s, dtype=np.int64), np.asarray(out_t, dtype=np.int64)
