"""Seeded synthetic inputs for the KDA forward pass.

This module is shared by the tests, the oracle checks, ``bench.py`` and
``__graft_entry__.smoke()``.  It holds none of the method's arithmetic: it only
draws random numbers, rounds them to bf16 and lays them out in the operator's
shapes, so that the CPU oracle and the CUDA path consume the same bytes.

Recipe (the operator statement on the FlashKDA pages fixes the shapes, dtypes and
the K=V=128 restriction; the value distributions are the workload recipe):

* A NumPy ``PCG64(seed)`` stream is drawn in the fixed order
  lengths -> q -> k -> v -> g -> beta -> A_log -> dt_bias -> initial_state.
* Normal values are drawn in fp32 as (mean, standard deviation) and rounded to
  bf16 with round-to-nearest-even (``torch.Tensor.to(torch.bfloat16)``).
* ``A_log[h] = log(U(1, 16))`` (fp32), ``dt_bias ~ N(0, 0.1)`` per (h, channel)
  (fp32), ``scale = 1/sqrt(K)``, ``lower_bound = -5``.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

K_HEAD = 128
V_HEAD = 128


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and distribution recipe of one synthetic KDA workload."""

    name: str
    B: int
    T: int  # tokens per sequence (fixed length) or total tokens (varlen)
    H: int
    K: int = K_HEAD
    V: int = V_HEAD
    g_std: float = 1.0
    init_state: Optional[str] = None  # None | "f32" | "bf16"
    init_std: float = 0.05
    varlen: Optional[dict] = None  # {"n": seqs, "lo": min len, "hi": max len, "total": T or None}
    lower_bound: float = -5.0


WORKLOADS = {
    # Tiny case the oracle finishes in seconds.
    0: Workload("tiny_B1_T512_H4", B=1, T=512, H=4),
    # Single long prefill with an fp32 initial state.
    1: Workload("long_B1_T8192_H32_s0f32", B=1, T=8192, H=32, init_state="f32"),
    # 16 packed sequences of 256..4096 tokens summing to 32768.
    2: Workload("varlen16_T32768_H32_s0f32", B=1, T=32768, H=32, init_state="f32",
                varlen={"n": 16, "lo": 256, "hi": 4096, "total": 32768}),
    # Long-context prefill, strong decay (g ~ N(0, 2)).
    3: Workload("long_B4_T32768_H32_g2", B=4, T=32768, H=32, g_std=2.0),
    # 1024 short sequences of 64..512 tokens, bf16 initial state.
    4: Workload("short1024_H16_s0bf16", B=1, T=0, H=16, init_state="bf16",
                varlen={"n": 1024, "lo": 64, "hi": 512, "total": None}),
}


@dataclasses.dataclass
class KDAInputs:
    """Host (CPU) tensors of one KDA forward call.

    q, k, g: bf16 [B,T,H,K]; v: bf16 [B,T,H,V]; beta: bf16 [B,T,H];
    A_log: fp32 [H]; dt_bias: fp32 [H,K]; initial_state: fp32 or bf16 [N,H,K,V]
    or None; cu_seqlens: int64 [N+1] or None (then B sequences of length T).
    """

    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    g: torch.Tensor
    beta: torch.Tensor
    A_log: torch.Tensor
    dt_bias: torch.Tensor
    scale: float
    lower_bound: float
    initial_state: Optional[torch.Tensor]
    cu_seqlens: Optional[torch.Tensor]

    @property
    def B(self) -> int:
        return self.q.shape[0]

    @property
    def T(self) -> int:
        return self.q.shape[1]

    @property
    def H(self) -> int:
        return self.q.shape[2]

    @property
    def K(self) -> int:
        return self.q.shape[3]

    @property
    def V(self) -> int:
        return self.v.shape[3]

    @property
    def num_seqs(self) -> int:
        return self.B if self.cu_seqlens is None else self.cu_seqlens.numel() - 1

    @property
    def tokens(self) -> int:
        return self.B * self.T

    def seq_bounds(self):
        """List of (batch index, start token, length) for every sequence."""
        if self.cu_seqlens is None:
            return [(b, 0, self.T) for b in range(self.B)]
        cu = self.cu_seqlens.tolist()
        return [(0, cu[s], cu[s + 1] - cu[s]) for s in range(len(cu) - 1)]


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def _normal_bf16(rng: np.random.Generator, shape, std: float, mean: float = 0.0,
                 block: int = 1 << 24) -> torch.Tensor:
    """N(mean, std) drawn in fp32 in memory order, rounded to bf16 block by block."""
    n = int(np.prod(shape)) if len(shape) else 1
    out = torch.empty(n, dtype=torch.bfloat16)
    for s in range(0, n, block):
        e = min(n, s + block)
        x = rng.standard_normal(e - s, dtype=np.float32)
        if std != 1.0:
            x *= np.float32(std)
        if mean != 0.0:
            x += np.float32(mean)
        out[s:e] = torch.from_numpy(x).to(torch.bfloat16)
    return out.view(*shape)


def draw_lengths(rng: np.random.Generator, n: int, lo: int, hi: int, total: Optional[int]):
    """Sequence lengths U{lo..hi}.  With a fixed total, all n are redrawn until the
    last one (total - sum of the first n-1) falls inside [lo, hi]."""
    if total is None:
        return rng.integers(lo, hi + 1, size=n, dtype=np.int64)
    for _ in range(100000):
        lens = rng.integers(lo, hi + 1, size=n, dtype=np.int64)
        last = total - int(lens[:-1].sum())
        if lo <= last <= hi:
            lens[-1] = last
            return lens
    raise RuntimeError("could not draw lengths with the requested total")


def make_inputs(w: Workload | int, seed: Optional[int] = None, *, T: Optional[int] = None,
                B: Optional[int] = None, H: Optional[int] = None,
                lengths: Optional[list] = None) -> KDAInputs:
    """Build the seeded inputs of workload ``w`` (an index of WORKLOADS or a Workload).

    ``seed`` defaults to the workload index.  ``T``, ``B``, ``H`` and ``lengths``
    override the recipe's sizes (for small parity cases); ``lengths`` forces a
    varlen batch with exactly those sequence lengths.
    """
    if isinstance(w, int):
        if seed is None:
            seed = w
        w = WORKLOADS[w]
    if seed is None:
        seed = 0
    rng = np.random.Generator(np.random.PCG64(seed))
    Bv = w.B if B is None else B
    Hv = w.H if H is None else H
    K, V = w.K, w.V

    cu = None
    if lengths is not None:
        lens = np.asarray(lengths, dtype=np.int64)
    elif w.varlen is not None and T is None:
        vl = w.varlen
        lens = draw_lengths(rng, vl["n"], vl["lo"], vl["hi"], vl["total"])
    else:
        lens = None
    if lens is not None:
        Bv = 1
        cu_np = np.zeros(len(lens) + 1, dtype=np.int64)
        cu_np[1:] = np.cumsum(lens)
        cu = torch.from_numpy(cu_np)
        Tv = int(cu_np[-1])
    else:
        Tv = w.T if T is None else T
    N = Bv if cu is None else cu.numel() - 1

    q = _normal_bf16(rng, (Bv, Tv, Hv, K), 1.0)
    k = _normal_bf16(rng, (Bv, Tv, Hv, K), 1.0)
    v = _normal_bf16(rng, (Bv, Tv, Hv, V), 1.0)
    g = _normal_bf16(rng, (Bv, Tv, Hv, K), w.g_std)
    beta = _normal_bf16(rng, (Bv, Tv, Hv), 1.0)
    A_log = torch.from_numpy(np.log(rng.uniform(1.0, 16.0, size=Hv)).astype(np.float32))
    dt_bias = torch.from_numpy((rng.standard_normal((Hv, K), dtype=np.float32)
                                * np.float32(0.1)).astype(np.float32))
    init = None
    if w.init_state is not None:
        s = _normal_bf16(rng, (N, Hv, K, V), w.init_std) if w.init_state == "bf16" else None
        if w.init_state == "f32":
            s = torch.from_numpy((rng.standard_normal((N, Hv, K, V), dtype=np.float32)
                                  * np.float32(w.init_std)).astype(np.float32))
        init = s
    return KDAInputs(q=q, k=k, v=v, g=g, beta=beta, A_log=A_log, dt_bias=dt_bias,
                     scale=1.0 / math.sqrt(K), lower_bound=w.lower_bound,
                     initial_state=init, cu_seqlens=cu)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Raw uint16 bit patterns of a bf16 tensor (for the CPU oracle)."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)
