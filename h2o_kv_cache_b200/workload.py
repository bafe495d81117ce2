"""Seeded synthetic inputs for the H2O chunk step (shared by tests and bench.py).

This module holds only input generation -- no step of the method's arithmetic.
The pages measure on long-context QA datasets ("Learning how to Forget", Tables
1-3: Helmet and LongBench V2 tasks at 64k / 128k tokens, chunk sizes 2048 /
1024 / 128).  Those datasets are not used; seeded Gaussian streams with the same
shapes stand in for them:

  * Q, K, V iid N(0, 1) * 0.5 per element;
  * planted heavy hitters: per (batch, layer, KV head) a fraction of the stream's
    positions is chosen uniformly without replacement, and each chosen key is
    replaced by ||k|| (0.8 u + 0.6 w): u the unit mean direction of that KV
    head's group of query vectors over the whole stream, w a random unit vector
    orthogonal to u (so cos(k, u) = 0.8 and ||k|| is kept);
  * seed = SplitMix64 of (config id, batch index, layer index); values are drawn
    in a fixed order (Q, K, V, then the planted positions and directions).
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

MASK64 = (1 << 64) - 1


def splitmix64(x: int) -> int:
    """One output of the SplitMix64 generator (Steele, Lea, Flood 2014) for state x."""
    x = (x + 0x9E3779B97F4A7C15) & MASK64
    z = x
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
    return z ^ (z >> 31)


def stream_seed(config_id: int, b: int, layer: int) -> int:
    s = splitmix64(config_id)
    s = splitmix64(s ^ b)
    s = splitmix64(s ^ (layer << 32))
    return s & ((1 << 63) - 1)


@dataclass(frozen=True)
class Config:
    cid: int
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    M: int
    R: int
    T: int            # stream length per sequence
    P: int            # prefill length
    S: int            # chunk length
    dtype: torch.dtype
    planted: float    # fraction of positions with planted heavy-hitter keys
    layers: int = 1

    @property
    def G(self):
        return self.Hq // self.Hkv

    @property
    def n_chunks(self):
        return (self.T - self.P + self.S - 1) // self.S

    def bounds(self):
        """[(t0, t1)] of the prefill followed by every chunk."""
        out = [(0, self.P)]
        t = self.P
        while t < self.T:
            out.append((t, min(self.T, t + self.S)))
            t += self.S
        return out

    def describe(self):
        return (f"B={self.B} Hq={self.Hq} Hkv={self.Hkv} d={self.d} M={self.M} R={self.R} "
                f"stream={self.T} prefill={self.P} S={self.S} layers={self.layers} "
                f"{str(self.dtype).replace('torch.', '')}")


CONFIGS = {
    0: Config(0, "tiny-fp32", 1, 4, 2, 64, 256, 32, 256 + 4 * 32, 256, 32, torch.float32, 0.0),
    1: Config(1, "m2k-s1k", 1, 32, 8, 128, 2048, 256, 16384, 2048, 1024, torch.bfloat16, 0.01),
    2: Config(2, "m16k-s1k", 1, 32, 8, 128, 16384, 1024, 65536, 16384, 1024, torch.bfloat16, 0.01),
    3: Config(3, "m32k-s2k", 1, 32, 8, 128, 32768, 2048, 131072, 32768, 2048, torch.bfloat16, 0.005),
    4: Config(4, "b4-28layer-m8k-s1k", 4, 32, 8, 128, 8192, 512, 32768, 8192, 1024, torch.bfloat16,
              0.01, layers=28),
}


def gen_sequence(cfg: Config, b: int = 0, layer: int = 0, device="cpu", T: int | None = None):
    """One sequence's stream: Q [Hq, T, d], K, V [Hkv, T, d] in cfg.dtype on `device`.
    A shorter T (a prefix of the workload's stream recipe) may be asked for."""
    T = cfg.T if T is None else T
    g = torch.Generator(device=device)
    g.manual_seed(stream_seed(cfg.cid, b, layer))
    Q = torch.randn(cfg.Hq, T, cfg.d, generator=g, device=device) * 0.5
    K = torch.randn(cfg.Hkv, T, cfg.d, generator=g, device=device) * 0.5
    V = torch.randn(cfg.Hkv, T, cfg.d, generator=g, device=device) * 0.5
    n_plant = int(round(cfg.planted * T))
    if n_plant > 0:
        for h in range(cfg.Hkv):
            u = Q[h * cfg.G:(h + 1) * cfg.G].reshape(-1, cfg.d).mean(dim=0)
            u = u / u.norm()
            idx = torch.randperm(T, generator=g, device=device)[:n_plant]
            w = torch.randn(n_plant, cfg.d, generator=g, device=device)
            w = w - (w @ u)[:, None] * u[None, :]
            w = w / w.norm(dim=1, keepdim=True)
            norms = K[h, idx].norm(dim=1, keepdim=True)
            K[h, idx] = norms * (0.8 * u[None, :] + 0.6 * w)
    return Q.to(cfg.dtype), K.to(cfg.dtype), V.to(cfg.dtype)


def gen_batch(cfg: Config, layer: int = 0, device="cpu", T: int | None = None):
    """Q [B, Hq, T, d], K, V [B, Hkv, T, d] for all sequences of one layer."""
    seqs = [gen_sequence(cfg, b, layer, device, T) for b in range(cfg.B)]
    return tuple(torch.stack([s[i] for s in seqs]) for i in range(3))


def split_chunks(Q, K, V, bounds):
    """Contiguous per-chunk tensors [(q, k, v)] for the given (t0, t1) bounds."""
    return [(Q[:, :, a:b].contiguous(), K[:, :, a:b].contiguous(), V[:, :, a:b].contiguous())
            for a, b in bounds]
