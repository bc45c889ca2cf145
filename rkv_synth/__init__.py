"""Seeded synthetic inputs for the R-KV decode-time compression step.

This module only draws numbers.  It holds none of the method's arithmetic
(no attention, no norms, no similarity, no selection), so that the CPU oracle
and the CUDA path can both consume its output without sharing any of the
computation they are compared on.

The workloads follow the shapes the R-KV pages quote: a KV budget of 1024 with
a recent window of 8 and a compression every 128 decoded tokens (hysenlabs
write-up, "What the redundancy scoring actually does at decode time", and the
run_math.py flags in "Three install paths"), Llama3-8B and Qwen-14B head
counts (atlas.scime.ai summary, "Measured effects" table) and 16K generation
at a 10% budget ("Key results").  Reasoning traces are repetitive by
construction (hysenlabs write-up, "How this differs from attention-sink and
heavy-hitter eviction"), which the generator models as near-duplicate runs:

* a run of length L ~ U{4..16} placed at destination p copies the segment
  s..s+L-1 (with s+L <= p) into p..p+L-1 for both K and V, plus N(0, 0.01^2)
  noise per element, before rounding to bf16;
* run positions are drawn once per sequence and shared by every layer and KV
  head (a repeated token repeats everywhere); the noise is drawn per element;
* runs do not overlap and cover about ``dup_frac`` of the cached positions.

Tensors are laid out as the compression step consumes them:

* ``K``, ``V``: ``[n_layers, batch, n_kv_heads, cap, head_dim]`` bf16, rows at
  and beyond a sequence's current length are zero;
* ``Q``: ``[n_layers, batch, n_q_heads, window, head_dim]`` bf16, the last
  ``window`` query vectors of every query head;
* ``cur_len``: ``[batch]`` int32.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Sequence

import numpy as np
import torch

__all__ = [
    "Workload",
    "WORKLOADS",
    "dup_runs",
    "make_inputs",
    "bf16_bits",
    "pack_ragged",
    "unpack_ragged",
]


@dataclass(frozen=True)
class Workload:
    """One synthetic configuration of the compression step."""

    name: str
    n_layers: int
    batch: int
    n_kv_heads: int
    n_q_heads: int
    head_dim: int
    budgets: Sequence[int]          # one per sequence (len == batch) or a single value
    buffer: int = 128
    window: int = 8
    mix_lambda: float = 0.1
    dup_frac: Sequence[float] = (0.3,)  # one per sequence or a single value
    ar_rho: float = 0.0             # 0: i.i.d. N(0,1) keys; >0: AR(1) keys along the sequence
    seed: int = 0

    def budget_of(self, b: int) -> int:
        return int(self.budgets[b] if len(self.budgets) > 1 else self.budgets[0])

    def dup_of(self, b: int) -> float:
        return float(self.dup_frac[b] if len(self.dup_frac) > 1 else self.dup_frac[0])

    @property
    def cap(self) -> int:
        return max(self.budget_of(b) for b in range(self.batch)) + self.buffer

    def n_tokens(self) -> List[int]:
        """Cached length of every sequence at the moment its buffer fills."""
        return [self.budget_of(b) + self.buffer for b in range(self.batch)]

    def token_heads(self) -> int:
        """Cached token-heads one step compresses (all layers x heads x sequences)."""
        return self.n_layers * self.n_kv_heads * sum(self.n_tokens())


def _uniform(seed: int, lo: float, hi: float, n: int) -> List[float]:
    rng = np.random.default_rng(seed)
    return [float(x) for x in rng.uniform(lo, hi, size=n)]


def _ragged_budgets(seed: int, n: int) -> List[int]:
    rng = np.random.default_rng(seed)
    return [int(x) for x in rng.choice([512, 1024, 1536, 2048], size=n)]


# The five workloads of the R-KV step, by shape.  Sizes follow the pages'
# settings (budget 1024 / window 8 / lambda 0.1 / step 128; Llama3-8B with
# 8 KV and 32 query heads; Qwen-14B with 8 KV and 40 query heads; 16K tokens
# at a 10% budget).
WORKLOADS = {
    "single_layer": Workload("single_layer", 1, 1, 8, 32, 128, (1024,), seed=1),
    "llama3_8b_step": Workload("llama3_8b_step", 32, 1, 8, 32, 128, (1024,), seed=2),
    "qwen_14b_batched": Workload(
        "qwen_14b_batched", 48, 16, 8, 40, 128, (2048,),
        dup_frac=tuple(_uniform(303, 0.10, 0.50, 16)), seed=3),
    "ragged_batch": Workload(
        "ragged_batch", 32, 64, 8, 32, 128, tuple(_ragged_budgets(404, 64)), seed=4),
    "decode_loop_16k": Workload(
        "decode_loop_16k", 32, 32, 8, 32, 128, (1638,), ar_rho=0.9, seed=5),
}


def dup_runs(n_tokens: int, dup_frac: float, seed: int) -> List[tuple]:
    """Near-duplicate runs ``(dst, src, length)`` for one sequence, ascending in dst.

    Runs never overlap one another as destinations, and every source segment
    lies strictly before its destination (src + length <= dst), so applying
    the runs in ascending dst order copies already-final rows.
    """
    rng = np.random.default_rng(seed)
    target = int(round(dup_frac * n_tokens))
    occupied = np.zeros(n_tokens, dtype=bool)
    runs = []
    covered = 0
    attempts = 0
    while covered < target and attempts < 100 * max(1, n_tokens):
        attempts += 1
        L = int(rng.integers(4, 17))
        if 2 * L > n_tokens:
            break
        p = int(rng.integers(L, n_tokens - L + 1))
        if occupied[p:p + L].any():
            continue
        s = int(rng.integers(0, p - L + 1))
        occupied[p:p + L] = True
        runs.append((p, s, L))
        covered += L
    runs.sort()
    return runs


def _ar1(eps: torch.Tensor, rho: float, chunk: int = 64) -> torch.Tensor:
    """Stationary AR(1) along dim -2: k_0 = eps_0, k_t = rho k_{t-1} + sqrt(1-rho^2) eps_t.

    Evaluated chunk by chunk with a lower-triangular matrix of powers of rho,
    so that a long trace costs a few small matmuls instead of a Python loop.
    """
    n = eps.shape[-2]
    c = float(np.sqrt(1.0 - rho * rho))
    t = torch.arange(chunk, device=eps.device, dtype=torch.float64)
    diff = t[:, None] - t[None, :]
    toep = torch.where(diff >= 0, torch.pow(torch.tensor(rho, dtype=torch.float64,
                                                         device=eps.device), diff.clamp(min=0)),
                       torch.zeros((), dtype=torch.float64, device=eps.device)).to(torch.float32)
    carry_w = torch.pow(torch.tensor(rho, dtype=torch.float64, device=eps.device),
                        t + 1).to(torch.float32)
    drive = eps * c
    drive[..., 0, :] = eps[..., 0, :]
    out = torch.empty_like(eps)
    prev = None
    for c0 in range(0, n, chunk):
        c1 = min(n, c0 + chunk)
        m = c1 - c0
        blk = torch.matmul(toep[:m, :m], drive[..., c0:c1, :])
        if prev is not None:
            blk = blk + carry_w[:m, None] * prev[..., None, :]
        out[..., c0:c1, :] = blk
        prev = blk[..., m - 1, :]
    return out


def _ar1_from_zero(drive: torch.Tensor, rho: float, chunk: int = 64) -> torch.Tensor:
    """x_t = rho x_{t-1} + drive_t with x_{-1} = 0, along dim -2 (chunked matmuls)."""
    n = drive.shape[-2]
    t = torch.arange(chunk, device=drive.device, dtype=torch.float64)
    diff = t[:, None] - t[None, :]
    r = torch.tensor(rho, dtype=torch.float64, device=drive.device)
    toep = torch.where(diff >= 0, torch.pow(r, diff.clamp(min=0)),
                       torch.zeros((), dtype=torch.float64, device=drive.device)).to(torch.float32)
    carry_w = torch.pow(r, t + 1).to(torch.float32)
    out = torch.empty_like(drive)
    prev = None
    for c0 in range(0, n, chunk):
        c1 = min(n, c0 + chunk)
        m = c1 - c0
        blk = torch.matmul(toep[:m, :m], drive[..., c0:c1, :])
        if prev is not None:
            blk = blk + carry_w[:m, None] * prev[..., None, :]
        out[..., c0:c1, :] = blk
        prev = blk[..., m - 1, :]
    return out


def _apply_runs(x: torch.Tensor, runs, noise_gen: torch.Generator, sigma: float) -> None:
    """In place on fp32 rows ``x[..., n, D]``: copy each run's source rows plus noise."""
    for (p, s, L) in runs:
        src = x[..., s:s + L, :]
        noise = torch.randn(src.shape, generator=noise_gen, device=x.device,
                            dtype=torch.float32) * sigma
        x[..., p:p + L, :] = src + noise


def make_inputs(w: Workload, device: str = "cpu", layers: Optional[Sequence[int]] = None,
                seq_offset: int = 0, batch: Optional[int] = None, seed: Optional[int] = None):
    """Materialise K, V, Q and cur_len for workload ``w``.

    ``layers`` restricts generation to a subset of layers (the returned tensors
    then hold only those layers, in the given order); each layer is drawn from
    its own stream, so a subset reproduces the same values as the full set.
    ``seq_offset``/``batch`` select sequences the same way (for sharding a
    batch across ranks).  All draws are seeded from ``w.seed`` (or ``seed``).
    """
    base_seed = w.seed if seed is None else seed
    layers = list(range(w.n_layers)) if layers is None else list(layers)
    B = w.batch if batch is None else batch
    seqs = list(range(seq_offset, seq_offset + B))
    cap, D, H, Hq, win = w.cap, w.head_dim, w.n_kv_heads, w.n_q_heads, w.window
    K = torch.zeros((len(layers), B, H, cap, D), dtype=torch.bfloat16, device=device)
    V = torch.zeros_like(K)
    Q = torch.empty((len(layers), B, Hq, win, D), dtype=torch.bfloat16, device=device)
    cur_len = torch.tensor([w.budget_of(b) + w.buffer for b in seqs], dtype=torch.int32)
    for li, l in enumerate(layers):
        for bi, b in enumerate(seqs):
            n = int(cur_len[bi])
            runs = dup_runs(n, w.dup_of(b), seed=base_seed * 1_000_003 + b)
            g = torch.Generator(device=device)
            g.manual_seed((base_seed * 7919 + l) * 104729 + b)
            kf = torch.randn((H, n, D), generator=g, device=device, dtype=torch.float32)
            if w.ar_rho > 0.0:
                kf = _ar1(kf, w.ar_rho)
            vf = torch.randn((H, n, D), generator=g, device=device, dtype=torch.float32)
            _apply_runs(kf, runs, g, 0.01)
            _apply_runs(vf, runs, g, 0.01)
            K[li, bi, :, :n, :] = kf.to(torch.bfloat16)
            V[li, bi, :, :n, :] = vf.to(torch.bfloat16)
            Q[li, bi] = torch.randn((Hq, win, D), generator=g, device=device,
                                    dtype=torch.float32).to(torch.bfloat16)
    return {"K": K, "V": V, "Q": Q, "cur_len": cur_len.to(device)}


def pack_ragged(X: torch.Tensor, caps: Sequence[int]) -> torch.Tensor:
    """[n_layers, batch, H, cap, D] -> [n_layers, sum_b H * caps[b], D]: every
    sequence's first caps[b] rows of each head, the sequences' blocks packed back
    to back in batch order (the per-sequence-capacity pool layout)."""
    L, B, H, _, D = X.shape
    return torch.cat([X[:, b, :, :int(caps[b])].reshape(L, H * int(caps[b]), D)
                      for b in range(B)], dim=1).contiguous()


def unpack_ragged(P: torch.Tensor, caps: Sequence[int], n_kv: int, cap: int) -> torch.Tensor:
    """Inverse of pack_ragged: [n_layers, rows, D] -> [n_layers, batch, H, cap, D]
    (rows past a sequence's capacity are zero)."""
    L, _, D = P.shape
    out = torch.zeros((L, len(caps), n_kv, cap, D), dtype=P.dtype, device=P.device)
    r = 0
    for b, c in enumerate(caps):
        out[:, b, :, :int(c)] = P[:, r:r + n_kv * int(c)].reshape(L, n_kv, int(c), D)
        r += n_kv * int(c)
    return out


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Raw bf16 bit patterns of a tensor as a uint16 numpy array (host copy)."""
    assert t.dtype == torch.bfloat16
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


class DecodeTrace:
    """New tokens of a steady-state decode loop, one chunk at a time, on the device.

    Keys continue a stationary AR(1) process per (layer, sequence, KV head,
    dimension); about ``dup_frac`` of each chunk's tokens are near-duplicate
    runs (4..16 tokens) copied from rows currently in the cache, plus
    N(0, 0.01^2) noise: a reasoning trace repeating context it still holds.
    Values are N(0, 1) except in the copied runs.  Queries of the window are
    fresh N(0, 1) every step.
    """

    def __init__(self, w: Workload, device: str = "cuda", seed: Optional[int] = None):
        self.w = w
        self.dev = device
        s = w.seed if seed is None else seed
        self.gen = torch.Generator(device=device)
        self.gen.manual_seed(s * 7919 + 17)
        self.rng = np.random.default_rng(s * 31 + 7)
        L, B, H, D = w.n_layers, w.batch, w.n_kv_heads, w.head_dim
        self.state = torch.randn((L, B, H, D), generator=self.gen, device=device)

    def chunk(self, n: int, K: torch.Tensor, V: torch.Tensor, cur_len: Sequence[int]):
        """n new tokens [L, B, H, n, D] (bf16) for K and V; copies read the cache K, V."""
        w = self.w
        L, B, H, D = w.n_layers, w.batch, w.n_kv_heads, w.head_dim
        rho = w.ar_rho
        eps = torch.randn((L, B, H, n, D), generator=self.gen, device=self.dev)
        if rho > 0.0:
            pw = torch.pow(torch.tensor(rho, device=self.dev), torch.arange(1, n + 1, device=self.dev,
                                                                             dtype=torch.float32))
            # AR(1) driven by eps from a zero start, plus the decayed previous state
            drive = eps * float(np.sqrt(1.0 - rho * rho))
            k = _ar1_from_zero(drive, rho) + pw[:, None] * self.state[..., None, :]
        else:
            k = eps
        v = torch.randn((L, B, H, n, D), generator=self.gen, device=self.dev)
        for b in range(B):
            avail = int(cur_len[b])
            target = int(round(self.w.dup_of(b) * n))
            t = 0
            covered = 0
            while covered < target and t < n - 4 and avail > 16:
                Lr = int(self.rng.integers(4, 17))
                Lr = min(Lr, n - t, avail)
                src = int(self.rng.integers(0, avail - Lr + 1))
                k[:, b, :, t:t + Lr] = K[:, b, :, src:src + Lr].float() + 0.01 * torch.randn(
                    (L, H, Lr, D), generator=self.gen, device=self.dev)
                v[:, b, :, t:t + Lr] = V[:, b, :, src:src + Lr].float() + 0.01 * torch.randn(
                    (L, H, Lr, D), generator=self.gen, device=self.dev)
                covered += Lr
                t += Lr + int(self.rng.integers(1, max(2, (n - covered) // 3)))
        self.state = k[..., -1, :].clone()
        return k.to(torch.bfloat16).contiguous(), v.to(torch.bfloat16).contiguous()

    def queries(self):
        w = self.w
        return torch.randn((w.n_layers, w.batch, w.n_q_heads, w.window, w.head_dim),
                           generator=self.gen, device=self.dev).to(torch.bfloat16)
