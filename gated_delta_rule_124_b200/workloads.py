"""Seeded synthetic inputs for KDA prefill and decode.

This module only draws random numbers and shapes them into the input
distributions of the benchmark configurations; it contains none of KDA's
arithmetic.  It is the one module shared by the oracle-side tests and the GPU
side (tests, ``bench.py``, ``smoke()``).

Distributions (per configuration):
  q, k   ~ N(0, 1), then L2-normalised over the key dimension per (token, head)
  v      ~ N(0, 1)
  beta   = sigmoid(N(0, 1))
  g      = log(alpha) = -softplus(N(mu_g, 1)) per channel (mu_g = 0, or -2 for
           the long-prefill configuration, "slow decay")
  initial state ~ N(0, 0.02^2)  (standard deviation 0.02), or zeros
  varlen lengths: integers uniform in [lo, hi] inclusive.

Values are drawn in float32 on the host from numpy PCG64 streams keyed by
``(seed, tensor id, block)``, so the result does not depend on the thread
count; q, k, v are then cast to the input dtype.  The oracle reads exactly the
cast values.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np
import torch

_BLOCK = 1 << 22
_THREADS = max(1, min(16, os.cpu_count() or 1))

# Stable ids of the drawn tensors (part of the stream key).
_ID = dict(q=1, k=2, v=3, g=4, beta=5, h0=6, lengths=7)


def _normal(seed: int, tid: int, n: int, mu: float = 0.0, sigma: float = 1.0) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    nblk = (n + _BLOCK - 1) // _BLOCK

    def blk(i):
        lo, hi = i * _BLOCK, min(n, (i + 1) * _BLOCK)
        r = np.random.default_rng([seed, tid, i])
        out[lo:hi] = r.standard_normal(hi - lo, dtype=np.float32)

    if nblk <= 1:
        for i in range(nblk):
            blk(i)
    else:
        with ThreadPoolExecutor(min(_THREADS, nblk)) as ex:
            list(ex.map(blk, range(nblk)))
    if sigma != 1.0:
        out *= np.float32(sigma)
    if mu != 0.0:
        out += np.float32(mu)
    return out


def _blockwise(f, x: np.ndarray, rows: int = 1) -> np.ndarray:
    """f applied to x in blocks of whole rows (the last axis when rows > 1),
    on a thread pool; the same values as f(x) in one piece."""
    out = np.empty(x.shape, dtype=np.float32)
    if rows > 1:
        xf, of = x.reshape(-1, rows), out.reshape(-1, rows)
    else:
        xf, of = x.reshape(-1), out.reshape(-1)
    n = xf.shape[0]
    step = max(1, _BLOCK // max(1, rows))
    nblk = (n + step - 1) // step

    def blk(i):
        lo, hi = i * step, min(n, (i + 1) * step)
        of[lo:hi] = f(xf[lo:hi])

    if nblk <= 1:
        for i in range(nblk):
            blk(i)
    else:
        with ThreadPoolExecutor(min(_THREADS, nblk)) as ex:
            list(ex.map(blk, range(nblk)))
    return out


def _l2norm_rows(x: np.ndarray) -> np.ndarray:
    def f(b):
        n = np.sqrt((b.astype(np.float64) ** 2).sum(-1, keepdims=True))
        return (b / np.maximum(n, 1e-30)).astype(np.float32)
    return _blockwise(f, x, rows=x.shape[-1])


def _neg_softplus(x: np.ndarray) -> np.ndarray:
    def f(b):
        b64 = b.astype(np.float64)
        return (-(np.maximum(b64, 0.0) + np.log1p(np.exp(-np.abs(b64))))).astype(np.float32)
    return _blockwise(f, x)


def _sigmoid(x: np.ndarray) -> np.ndarray:
    return _blockwise(lambda b: (1.0 / (1.0 + np.exp(-b.astype(np.float64)))).astype(np.float32),
                      x)


_TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


@dataclass
class PrefillCase:
    """One prefill problem.  Token-major, flat over packed sequences.

    q, k [total, H, dk] (dtype); v [total, H, dv] (dtype); g [total, H, dk] fp32;
    beta [total, H] fp32; initial_state [N, H, dk, dv] fp32 or None;
    cu_seqlens int32 [N + 1] or None (then B equal sequences of T tokens).
    """
    name: str
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    g: torch.Tensor
    beta: torch.Tensor
    initial_state: torch.Tensor | None
    cu_seqlens: torch.Tensor | None
    B: int
    T: int
    H: int
    dk: int
    dv: int
    chunk: int
    dtype: str
    lengths: list = field(default_factory=list)

    @property
    def N(self) -> int:
        return len(self.lengths)

    @property
    def total(self) -> int:
        return int(self.q.shape[0])

    def cu_host(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.lengths)]).astype(np.int32)

    def to(self, device) -> "PrefillCase":
        mv = lambda t: None if t is None else t.to(device, non_blocking=False).contiguous()
        return PrefillCase(self.name, mv(self.q), mv(self.k), mv(self.v), mv(self.g),
                           mv(self.beta), mv(self.initial_state), mv(self.cu_seqlens), self.B,
                           self.T, self.H, self.dk, self.dv, self.chunk, self.dtype,
                           list(self.lengths))


def make_prefill(seed: int, lengths, H: int, dk: int, dv: int, chunk: int, dtype: str,
                 g_mu: float = 0.0, init_std: float | None = 0.02, varlen: bool = False,
                 name: str = "custom") -> PrefillCase:
    """Draw one prefill problem with the given sequence lengths.

    ``varlen`` selects a ``cu_seqlens`` call; otherwise all lengths must be
    equal and the call is a plain batch of B sequences.
    """
    lengths = [int(x) for x in lengths]
    total = int(sum(lengths))
    N = len(lengths)
    if not varlen and len(set(lengths)) > 1:
        raise ValueError("equal lengths required without varlen")
    q = _l2norm_rows(_normal(seed, _ID["q"], total * H * dk).reshape(total, H, dk))
    k = _l2norm_rows(_normal(seed, _ID["k"], total * H * dk).reshape(total, H, dk))
    v = _normal(seed, _ID["v"], total * H * dv).reshape(total, H, dv)
    g = _neg_softplus(_normal(seed, _ID["g"], total * H * dk, mu=g_mu)).reshape(total, H, dk)
    beta = _sigmoid(_normal(seed, _ID["beta"], total * H)).reshape(total, H)
    h0 = None
    if init_std:
        h0 = torch.from_numpy(
            _normal(seed, _ID["h0"], N * H * dk * dv, sigma=init_std).reshape(N, H, dk, dv))
    tdt = _TORCH_DT[dtype]
    cu = None
    if varlen:
        cu = torch.from_numpy(np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32))
    return PrefillCase(name=name, q=torch.from_numpy(q).to(tdt), k=torch.from_numpy(k).to(tdt),
                       v=torch.from_numpy(v).to(tdt), g=torch.from_numpy(g),
                       beta=torch.from_numpy(beta), initial_state=h0, cu_seqlens=cu,
                       B=1 if varlen else N, T=total if varlen else lengths[0], H=H, dk=dk,
                       dv=dv, chunk=chunk, dtype=dtype, lengths=lengths)


def varlen_lengths(seed: int, n: int, lo: int, hi: int) -> list:
    r = np.random.default_rng([seed, _ID["lengths"]])
    return [int(x) for x in r.integers(lo, hi + 1, size=n)]


# The five benchmark configurations, by what they are.
PREFILL_CONFIGS = {
    0: dict(name="tiny fp32: B=1 H=1 T=64 d=32 C=16", B=1, T=64, H=1, d=32, chunk=16,
            dtype="f32", g_mu=0.0, init_std=None),
    1: dict(name="prefill: B=2 H=32 T=2048 d=128 C=64 bf16", B=2, T=2048, H=32, d=128,
            chunk=64, dtype="bf16", g_mu=0.0, init_std=0.02),
    2: dict(name="long prefill: B=1 H=32 T=65536 d=128 C=64 bf16 slow decay", B=1, T=65536,
            H=32, d=128, chunk=64, dtype="bf16", g_mu=-2.0, init_std=0.02),
    3: dict(name="varlen prefill: 16 seqs U[1024,16384] H=32 d=128 C=64 bf16", nseq=16,
            lo=1024, hi=16384, H=32, d=128, chunk=64, dtype="bf16", g_mu=0.0, init_std=0.02),
}


def prefill_config(index: int) -> PrefillCase:
    c = PREFILL_CONFIGS[index]
    seed = 1000 + index
    if "nseq" in c:
        lengths = varlen_lengths(seed, c["nseq"], c["lo"], c["hi"])
        return make_prefill(seed, lengths, c["H"], c["d"], c["d"], c["chunk"], c["dtype"],
                            g_mu=c["g_mu"], init_std=c["init_std"], varlen=True, name=c["name"])
    return make_prefill(seed, [c["T"]] * c["B"], c["H"], c["d"], c["d"], c["chunk"], c["dtype"],
                        g_mu=c["g_mu"], init_std=c["init_std"], varlen=False, name=c["name"])


@dataclass
class DecodeCase:
    """Recurrent decode problem: ``sets`` distinct one-token input sets, cycled.

    Each set: q, k [N, H, dk] (dtype); v [N, H, dv]; g [N, H, dk] fp32;
    beta [N, H] fp32.  state0 [N, H, dk, dv] fp32.
    """
    name: str
    steps: list
    state0: torch.Tensor
    N: int
    H: int
    dk: int
    dv: int
    dtype: str


DECODE_CONFIG = dict(name="decode: N=256 H=32 d=128 bf16, fp32 state, 8 input sets cycled",
                     N=256, H=32, d=128, dtype="bf16", sets=8, steps=1000)


def make_decode(seed: int, N: int, H: int, dk: int, dv: int, dtype: str, sets: int = 8,
                g_mu: float = 0.0, init_std: float = 0.02, name: str = "custom") -> DecodeCase:
    tdt = _TORCH_DT[dtype]
    steps = []
    for i in range(sets):
        s = seed * 1000 + i
        q = _l2norm_rows(_normal(s, _ID["q"], N * H * dk).reshape(N, H, dk))
        k = _l2norm_rows(_normal(s, _ID["k"], N * H * dk).reshape(N, H, dk))
        v = _normal(s, _ID["v"], N * H * dv).reshape(N, H, dv)
        g = _neg_softplus(_normal(s, _ID["g"], N * H * dk, mu=g_mu)).reshape(N, H, dk)
        beta = _sigmoid(_normal(s, _ID["beta"], N * H)).reshape(N, H)
        steps.append(dict(q=torch.from_numpy(q).to(tdt), k=torch.from_numpy(k).to(tdt),
                          v=torch.from_numpy(v).to(tdt), g=torch.from_numpy(g),
                          beta=torch.from_numpy(beta)))
    state0 = torch.from_numpy(_normal(seed, _ID["h0"], N * H * dk * dv,
                                      sigma=init_std).reshape(N, H, dk, dv))
    return DecodeCase(name, steps, state0, N, H, dk, dv, dtype)


def decode_config() -> DecodeCase:
    c = DECODE_CONFIG
    return make_decode(1004, c["N"], c["H"], c["d"], c["d"], c["dtype"], c["sets"],
                       name=c["name"])
