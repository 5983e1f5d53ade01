"""Seeded synthetic inputs for the ALHR inference path (shared by tests and the benchmark).

This module holds no part of the method's arithmetic: it only draws numbers. Every element
is a pure function of (seed, tensor id, flat element index), so any slice of any tensor can be
regenerated on its own, on the CPU or on a GPU, with identical bits.

Generator: SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
generators", OOPSLA 2014; the mixing constants of Vigna's public-domain splitmix64.c).
Element k of a stream with base state s is mix(s + (k+1)*GAMMA mod 2^64). The stream base of
(seed, tensor id) is mix(seed * 2^16 + tensor id). All 64-bit words are held as int64 bit
patterns in torch tensors; right shifts are made logical by masking.

Workloads follow the five shapes of the benchmark table (T = 1K / 4K / 16K prefill, an
associative-recall-shaped prefill and a long-context decode): see WORKLOADS.
"""
from __future__ import annotations

import dataclasses
import math

import torch

MASK64 = (1 << 64) - 1


def _signed64(c: int) -> int:
    c &= MASK64
    return c - (1 << 64) if c >= (1 << 63) else c


GAMMA = 0x9E3779B97F4A7C15
_MIX1 = _signed64(0xBF58476D1CE4E5B9)
_MIX2 = _signed64(0x94D049BB133111EB)

# tensor ids of the streams
TID_Q, TID_K, TID_V, TID_W, TID_PLANT, TID_NOISE = 1, 2, 3, 4, 5, 6

_CHUNK = 1 << 24  # elements generated per step (bounds the int64 temporaries)


def _lsr(z: torch.Tensor, s: int) -> torch.Tensor:
    """Logical right shift of int64 bit patterns."""
    return (z >> s) & ((1 << (64 - s)) - 1)


def _mix_tensor(z: torch.Tensor) -> torch.Tensor:
    z = (z ^ _lsr(z, 30)) * _MIX1
    z = (z ^ _lsr(z, 27)) * _MIX2
    return z ^ _lsr(z, 31)


def mix64(x: int) -> int:
    """SplitMix64 output mix on a Python int (mod 2^64)."""
    z = x & MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
    return z ^ (z >> 31)


def stream_base(seed: int, tid: int) -> int:
    return mix64((seed << 16) + tid)


def raw_words(seed: int, tid: int, start: int, count: int, device) -> torch.Tensor:
    """int64 bit patterns of stream elements [start, start + count)."""
    base = stream_base(seed, tid)
    k = torch.arange(start + 1, start + count + 1, dtype=torch.int64, device=device)
    z = k * _signed64(GAMMA) + _signed64(base)
    return _mix_tensor(z)


def _fill(numel: int, device, dtype, fn) -> torch.Tensor:
    out = torch.empty(numel, dtype=dtype, device=device)
    for s in range(0, numel, _CHUNK):
        c = min(_CHUNK, numel - s)
        out[s:s + c] = fn(s, c)
    return out


def uniform_int8(seed: int, tid: int, shape, lo: int, hi: int, device="cpu",
                 offset: int = 0) -> torch.Tensor:
    """int8 values uniform on [lo, hi]: lo + ((x >> 32) * (hi - lo + 1)) >> 32."""
    assert -128 <= lo <= hi <= 127
    numel = math.prod(shape)
    span = hi - lo + 1

    def fn(s, c):
        x = raw_words(seed, tid, offset + s, c, device)
        return (lo + ((_lsr(x, 32) * span) >> 32)).to(torch.int8)

    return _fill(numel, device, torch.int8, fn).view(*shape)


def normal_bf16(seed: int, tid: int, shape, device="cpu", offset: int = 0) -> torch.Tensor:
    """bf16 N(0,1) by Box-Muller in float64 (element k uses stream words 2k and 2k+1),
    rounded to nearest even. `offset` is the flat index of the first element."""
    numel = math.prod(shape)
    two53 = float(1 << 53)

    def fn(s, c):
        x = raw_words(seed, tid, 2 * (offset + s), 2 * c, device).view(c, 2)
        u1 = (_lsr(x[:, 0], 11).to(torch.float64) + 0.5) / two53
        u2 = _lsr(x[:, 1], 11).to(torch.float64) / two53
        z = torch.sqrt(-2.0 * torch.log(u1)) * torch.cos(2.0 * math.pi * u2)
        return z.to(torch.bfloat16)

    return _fill(numel, device, torch.bfloat16, fn).view(*shape)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    heads: int
    n: int
    d: int
    q_start: int
    nq: int
    window: int = 16
    max_keys: int = 96
    score_bits: int = 0           # 0 = let the library choose
    qk_lo: int = -16
    qk_hi: int = 16
    w_lo: int = -4
    w_hi: int = 4
    predictor: bool = True        # False: budget = min(i + 1, fixed_budget_cap)
    fixed_budget_cap: int = 0
    plant_pairs: int = 0          # associative-recall planting per sequence
    plant_noise: int = 2
    seed: int = 0
    live_classes: int = 32        # predictor rows of classes >= live_classes are zero

    @property
    def bh(self) -> int:
        return self.batch * self.heads

    def dims(self) -> dict:
        return dict(batch=self.batch, heads=self.heads, n=self.n, d=self.d,
                    q_start=self.q_start, nq=self.nq, window=self.window,
                    max_keys=self.max_keys, score_bits=self.score_bits,
                    value_bound=max(-self.qk_lo, self.qk_hi))

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    # T=1K, fixed budget min(i+1, 32), predictor bypassed
    "tiny_prefill_n1024": Workload("tiny_prefill_n1024", 1, 1, 1024, 64, 0, 1024,
                                   predictor=False, fixed_budget_cap=32),
    # T=4K, predicted budgets, W int8 U[-4,4] of shape 32 x 128
    "prefill_b4h8_n4096": Workload("prefill_b4h8_n4096", 4, 8, 4096, 64, 0, 4096),
    # T=16K, same distributions and predictor, exact int32 scores
    "prefill_b2h8_n16384": Workload("prefill_b2h8_n16384", 2, 8, 16384, 64, 0, 16384,
                                    score_bits=32),
    # T=64K, same distributions: the working set (tree 268 MB, keys, values) exceeds L2
    "prefill_b2h8_n65536": Workload("prefill_b2h8_n65536", 2, 8, 65536, 64, 0, 65536,
                                    score_bits=32),
    # T=16K associative-recall shape: 256 planted pairs per sequence, int64 scores
    "recall_b2h4_n16384_d128": Workload("recall_b2h4_n16384_d128", 2, 4, 16384, 128, 0,
                                        16384, score_bits=64, plant_pairs=256),
    # decode: one query at position n-1 per (sequence, head) against n = 256K keys
    "decode_s64h8_n262144_d128": Workload("decode_s64h8_n262144_d128", 64, 8, 262144, 128,
                                          262143, 1, score_bits=64),
}


def plant_positions(wl: Workload, b: int, device="cpu"):
    """Distinct key positions p in [0, n/2) and query positions u in [n/2, n), paired in
    order, for sequence b (shared by all heads of the sequence)."""
    half = wl.n // 2
    keys_p = raw_words(wl.seed, TID_PLANT, (2 * b) * half, half, device)
    keys_u = raw_words(wl.seed, TID_PLANT, (2 * b + 1) * half, half, device)
    p = torch.argsort(keys_p, stable=True)[: wl.plant_pairs]
    u = half + torch.argsort(keys_u, stable=True)[: wl.plant_pairs]
    return p, u


def make_block_inputs(wl: Workload, lo: int, hi: int, device="cpu") -> dict:
    """The inputs of the flat (b,h) blocks [lo, hi) of a workload (block k = b * heads + h), with
    the same bits as the same blocks of make_inputs(wl): every element is drawn at its flat
    index in the whole batch, so a rank of a sharded run generates its own blocks only.

    Q int8 [1, hi-lo, nq, d], K int8 [1, hi-lo, n, d], V bf16 [1, hi-lo, n, d] (reshaped to
    [sequences, heads, ...] by the caller where the range is whole sequences), W int8 [32, 2d]
    (or None), budget_override int32 [1, hi-lo, nq] (or None)."""
    if not 0 <= lo <= hi <= wl.bh:
        raise ValueError(f"blocks [{lo}, {hi}) outside [0, {wl.bh})")
    H, n, d, nb = wl.heads, wl.n, wl.d, hi - lo
    K = uniform_int8(wl.seed, TID_K, (1, nb, n, d), wl.qk_lo, wl.qk_hi, device,
                     offset=lo * n * d)
    Q = uniform_int8(wl.seed, TID_Q, (1, nb, wl.nq, d), wl.qk_lo, wl.qk_hi, device,
                     offset=lo * wl.nq * d)
    V = normal_bf16(wl.seed, TID_V, (1, nb, n, d), device, offset=lo * n * d)
    if wl.plant_pairs and nb:
        assert wl.q_start == 0 and wl.nq == n
        P = wl.plant_pairs
        for b in range(lo // H, (hi - 1) // H + 1):
            p, u = plant_positions(wl, b, device)
            h0, h1 = max(lo, b * H) - b * H, min(hi, (b + 1) * H) - b * H
            # planting noise: one stream slice per sequence, [heads, pairs, d]
            noise = uniform_int8(wl.seed, TID_NOISE, (h1 - h0, P, d), -wl.plant_noise,
                                 wl.plant_noise, device, offset=(b * H + h0) * P * d)
            k0 = b * H + h0 - lo
            planted = K[0, k0:k0 + h1 - h0][:, p, :].to(torch.int16) + noise.to(torch.int16)
            Qs = Q[0, k0:k0 + h1 - h0]  # a view: [heads of this range, nq, d]
            Qs[:, u, :] = planted.clamp(wl.qk_lo, wl.qk_hi).to(torch.int8)
    W = None
    budget = None
    if wl.predictor:
        W = uniform_int8(wl.seed, TID_W, (32, 2 * d), wl.w_lo, wl.w_hi, device)
        if wl.live_classes < 32:
            W[wl.live_classes:] = 0
    else:
        pos = torch.arange(wl.q_start, wl.q_start + wl.nq, dtype=torch.int32, device=device)
        budget = torch.clamp(pos + 1, max=wl.fixed_budget_cap).expand(1, nb, wl.nq).contiguous()
    return dict(Q=Q, K=K, V=V, W=W, budget_override=budget)


def as_sequences(inp: dict, heads: int) -> dict:
    """Block inputs [1, k*heads, ...] viewed as [k, heads, ...] (whole sequences)."""
    out = {}
    for key, t in inp.items():
        if t is None or key == "W":
            out[key] = t
        else:
            assert t.shape[1] % heads == 0
            out[key] = t.view(t.shape[1] // heads, heads, *t.shape[2:])
    return out


def make_inputs(wl: Workload, device="cpu") -> dict:
    """All inputs of a workload as torch tensors on `device`.

    Q int8 [B,H,nq,d], K int8 [B,H,n,d], V bf16 [B,H,n,d], W int8 [32,2d] (or None),
    budget_override int32 [B,H,nq] (or None)."""
    return as_sequences(make_block_inputs(wl, 0, wl.bh, device), wl.heads)
