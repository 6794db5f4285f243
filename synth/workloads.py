"""Workload table and seeded input generator for the MISA indexer path.

The shapes follow the indexer workloads the MISA pages evaluate on
(DeepSeek-V3.2 with H^I = 64 indexer heads and GLM-5 with H^I = 32, head dim
128, token budget k = 2048; "MISA: Mixture of Indexer Sparse Attention",
Introduction and Empirical Validation).  No dataset, model weights or real
activations are used: every tensor is drawn from a seeded numpy Generator.

Input recipe (per sequence):
  q[t, j, :] ~ N(0, 1) / sqrt(d)                         (bf16, round-to-nearest-even)
  k[s, :]    ~ N(0, 1) / sqrt(d) + drift[s // B, :]       (bf16)
               drift[b, :] ~ N(0, (0.5 / sqrt(d))^2) per element, shared by the
               B tokens of block b, so block statistics carry signal
  needles:   `needles` tokens at random positions; each is re-pointed so that its
             cosine with one routed-candidate head's query is 0.8:
             k_s <- |k_s| * (0.8 * q_hat + 0.6 * u),  u a random unit vector
             orthogonal to q_hat.  For decode rows the head is one of 4 heads
             drawn per sequence; for causal prefill each needle picks a random
             head and a random query t >= s.
  w[t, j]    ~ N(0, 1 / H)                                (fp32)
  pos[t]     decode/tail: the last T positions L-T .. L-1; causal prefill: pos[t] = t

The tiny parity workload uses plain N(0, 1)/sqrt(d) keys (no drift, no needles).
bf16 values are produced here, on the host, as uint16 bit patterns; both the
oracle and the CUDA path receive the same bits.
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    nseq: int          # independent sequences (batch)
    T: int             # queries per sequence
    L: int             # keys per sequence
    H: int             # indexer heads H^I
    d: int             # head dim
    h: int             # routed heads
    B: int             # router block size
    topk: int          # final token budget k
    kprime: int        # MISA-dagger candidate budget k'
    pos_mode: str      # "tail" (queries at the last T positions) or "causal" (pos[t] = t)
    drift: bool        # add per-block drift vectors to keys
    needles: int       # planted needle tokens per sequence

    @property
    def rows(self) -> int:
        return self.nseq * self.T

    def positions(self) -> np.ndarray:
        if self.pos_mode == "tail":
            p = np.arange(self.L - self.T, self.L, dtype=np.int32)
        elif self.pos_mode == "causal":
            assert self.T <= self.L
            p = np.arange(self.T, dtype=np.int32)
        else:
            raise ValueError(self.pos_mode)
        return np.broadcast_to(p, (self.nseq, self.T)).copy()

    def query_prefix_tokens(self) -> int:
        """Number of scored (query t, key s <= pos[t]) pairs in one call."""
        return int((self.positions().astype(np.int64) + 1).sum())

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    # tiny decode-style parity case: 16 queries at the last 16 positions of a 2K prefix
    "tiny_2k": Workload("tiny_2k", nseq=1, T=16, L=2048, H=64, d=128, h=8, B=64,
                        topk=256, kprime=512, pos_mode="tail", drift=False, needles=0),
    # DeepSeek-V3.2-shaped decode: 32 sequences x 1 query over a 32K prefix
    "dsv32_decode_32k": Workload("dsv32_decode_32k", nseq=32, T=1, L=32768, H=64, d=128,
                                 h=8, B=64, topk=2048, kprime=8192, pos_mode="tail",
                                 drift=True, needles=8),
    # DeepSeek-V3.2-shaped causal prefill: T = L = 16384 in one sequence
    "dsv32_prefill_16k": Workload("dsv32_prefill_16k", nseq=1, T=16384, L=16384, H=64,
                                  d=128, h=8, B=64, topk=2048, kprime=8192,
                                  pos_mode="causal", drift=True, needles=8),
    # GLM-5-shaped long decode: 8 sequences x 1 query over 128K, 32 heads, B = 128
    "glm5_decode_128k": Workload("glm5_decode_128k", nseq=8, T=1, L=131072, H=32, d=128,
                                 h=8, B=128, topk=2048, kprime=8192, pos_mode="tail",
                                 drift=True, needles=8),
    # multi-token decode (several draft positions per step): 32 sequences x 4 queries at
    # the last 4 positions of a 32K prefix
    "dsv32_mtp_32k": Workload("dsv32_mtp_32k", nseq=32, T=4, L=32768, H=64, d=128, h=8,
                              B=64, topk=2048, kprime=8192, pos_mode="tail", drift=True,
                              needles=8),
    # 16 queries per sequence over a 32K prefix (a speculative draft of 16 positions)
    "dsv32_draft16_32k": Workload("dsv32_draft16_32k", nseq=32, T=16, L=32768, H=64, d=128,
                                  h=8, B=64, topk=2048, kprime=8192, pos_mode="tail",
                                  drift=True, needles=8),
    # MISA-dagger re-rank against dense DSA at 128K: 16 sequences x 1 query, k' = 8192
    "dagger_128k": Workload("dagger_128k", nseq=16, T=1, L=131072, H=64, d=128, h=8,
                            B=64, topk=2048, kprime=8192, pos_mode="tail", drift=True,
                            needles=8),
}


@dataclasses.dataclass
class IndexerInputs:
    wl: Workload
    q_bits: np.ndarray   # uint16 [nseq, T, H, d], bf16 bit patterns
    w: np.ndarray        # float32 [nseq, T, H]
    k_bits: np.ndarray   # uint16 [nseq, L, d], bf16 bit patterns
    pos: np.ndarray      # int32 [nseq, T]
    needle_pos: np.ndarray  # int64 [nseq, needles] planted positions (for reporting)


def fp32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even); return uint16 bits.

    Inputs are finite by construction, so the NaN case is not handled.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def _bf16_bits_to_fp32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def make_inputs(wl: Workload, seed: int = 0) -> IndexerInputs:
    rng = np.random.default_rng(seed)
    nseq, T, L, H, d, B = wl.nseq, wl.T, wl.L, wl.H, wl.d, wl.B
    inv_sqrt_d = np.float32(1.0 / math.sqrt(d))

    q32 = rng.standard_normal((nseq, T, H, d), dtype=np.float32) * inv_sqrt_d
    q_bits = fp32_to_bf16_bits(q32)
    del q32
    w = (rng.standard_normal((nseq, T, H), dtype=np.float32)
         * np.float32(1.0 / math.sqrt(H))).astype(np.float32)
    pos = wl.positions()

    k_bits = np.empty((nseq, L, d), dtype=np.uint16)
    needle_pos = np.zeros((nseq, wl.needles), dtype=np.int64)
    q_seq = _bf16_bits_to_fp32(q_bits).astype(np.float64)  # needle directions (input shaping only)
    for n in range(nseq):
        ks = rng.standard_normal((L, d), dtype=np.float32) * inv_sqrt_d
        if wl.drift:
            nblk = -(-L // B)
            drift = rng.standard_normal((nblk, d), dtype=np.float32) * np.float32(0.5) * inv_sqrt_d
            ks += np.repeat(drift, B, axis=0)[:L]
        if wl.needles:
            lo = 0
            hi = int(pos[n].max()) + 1
            npos = rng.choice(hi - lo, size=wl.needles, replace=False) + lo
            needle_pos[n] = np.sort(npos)
            heads4 = rng.choice(H, size=min(4, H), replace=False)
            for i, s in enumerate(needle_pos[n]):
                if wl.pos_mode == "causal":
                    # a query that can see this token, and a random head of it
                    t = int(rng.integers(int(s), T)) if s < T else T - 1
                    j = int(rng.integers(0, H))
                else:
                    t = int(rng.integers(0, T))
                    j = int(heads4[i % len(heads4)])
                qv = q_seq[n, t, j]
                qhat = qv / np.linalg.norm(qv)
                g = rng.standard_normal(d)
                u = g - (g @ qhat) * qhat
                u /= np.linalg.norm(u)
                norm = float(np.linalg.norm(ks[s].astype(np.float64)))
                ks[s] = (norm * (0.8 * qhat + 0.6 * u)).astype(np.float32)
        k_bits[n] = fp32_to_bf16_bits(ks)
        del ks
    return IndexerInputs(wl=wl, q_bits=q_bits, w=w, k_bits=k_bits, pos=pos,
                         needle_pos=needle_pos)


def sample_rows(wl: Workload, n: int = 256, seed: int = 0) -> np.ndarray:
    """Seeded sample of (seq, t) query rows, as flat row ids seq * T + t, sorted.

    Workloads with at most n rows return every row.
    """
    if wl.rows <= n:
        return np.arange(wl.rows, dtype=np.int64)
    rng = np.random.default_rng(seed + 7919)
    return np.sort(rng.choice(wl.rows, size=n, replace=False)).astype(np.int64)
