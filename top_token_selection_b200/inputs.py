"""Seeded synthetic inputs for the PIVOT indexer.

This module only draws inputs.  It holds none of the method's arithmetic
(no scoring, no averaging, no selection); both the CUDA path and the CPU
oracle are fed from it.  Everything is drawn on the host CPU from one seeded
``torch.Generator`` in fp32 and then rounded to the stored format.

Workloads (the pages benchmark on DeepSeek-V3.2 / GLM-5.1 with LongBench and
RULER; no weights or datasets are used here, these synthetic inputs stand in):

* ``int``  -- the exact-arithmetic case: q, k integers uniform in [-3, 3],
  head weights integers uniform in [1, 4], stored as fp32.  Every score is an
  integer far below 2^24, so fp32 arithmetic is exact and results compare
  bit for bit, ties included (ReLU produces many zero scores).
* ``dsa``  -- DSA-shaped: keys N(0,1) per component, a random 2% of "heavy"
  keys scaled by 4 (long-tailed scores along the key axis); queries follow an
  AR(1) walk along position per head, q[t] = 0.95 q[t-1] + 0.31 N(0,1), so
  neighbouring queries pick largely the same keys; w[t,h] = softplus(N(0,1)).
  Stored as bf16 (round to nearest even) or as FP8 e4m3 with one fp32 scale
  per token (amax / 448, round to nearest even, saturating).
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

F32, BF16, E4M3 = 0, 1, 2
DTYPE_NAMES = {F32: "f32", BF16: "bf16", E4M3: "e4m3"}

AR_DECAY = 0.95
AR_NOISE = 0.31
HEAVY_FRACTION = 0.02
HEAVY_SCALE = 4.0
E4M3_MAX = 448.0


@dataclasses.dataclass
class Prefill:
    """One sequence of indexer inputs (host tensors, stored formats)."""
    dtype: int
    q: torch.Tensor                 # [L, H, D]: float32 / bfloat16 / float8_e4m3fn
    q_scale: torch.Tensor | None    # [L] float32 (e4m3 only)
    w: torch.Tensor                 # [L, H] float32
    k: torch.Tensor                 # [L, D]
    k_scale: torch.Tensor | None    # [L] float32 (e4m3 only)

    @property
    def L(self):
        return self.q.shape[0]

    @property
    def H(self):
        return self.q.shape[1]

    @property
    def D(self):
        return self.q.shape[2]

    def codes(self):
        """numpy views of the stored codes, as the oracle wants them."""
        return (codes_of(self.q, self.dtype),
                None if self.q_scale is None else self.q_scale.numpy(),
                self.w.numpy(),
                codes_of(self.k, self.dtype),
                None if self.k_scale is None else self.k_scale.numpy())


@dataclasses.dataclass
class Decode:
    """One MTP decode step for a batch of cached sequences (host tensors)."""
    dtype: int
    q: torch.Tensor                 # [B, Gm, H, D]
    q_scale: torch.Tensor | None    # [B, Gm]
    w: torch.Tensor                 # [B, Gm, H]
    kc: torch.Tensor                # [B, maxlen, D]
    kc_scale: torch.Tensor | None   # [B, maxlen]
    cache_len: torch.Tensor         # [B] int32, counts the Gm new tokens

    def codes(self):
        return (codes_of(self.q, self.dtype),
                None if self.q_scale is None else self.q_scale.numpy(),
                self.w.numpy(),
                codes_of(self.kc, self.dtype),
                None if self.kc_scale is None else self.kc_scale.numpy(),
                self.cache_len.numpy())


def codes_of(t: torch.Tensor, dtype: int) -> np.ndarray:
    """Raw storage codes: float32 values, uint16 bf16 bits or uint8 e4m3 bits."""
    t = t.contiguous()
    if dtype == F32:
        return t.numpy()
    if dtype == BF16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.view(torch.uint8).numpy()


def _store(x: torch.Tensor, dtype: int):
    """Round fp32 rows (last dims flattened per leading index) to the format."""
    if dtype == F32:
        return x.contiguous(), None
    if dtype == BF16:
        return x.to(torch.bfloat16).contiguous(), None
    lead = x.shape[0]
    flat = x.reshape(lead, -1)
    amax = flat.abs().amax(dim=1)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    y = (flat / scale[:, None]).clamp_(-E4M3_MAX, E4M3_MAX)
    return y.to(torch.float8_e4m3fn).reshape(x.shape).contiguous(), scale.float().contiguous()


def _dsa_keys(n: int, D: int, gen: torch.Generator) -> torch.Tensor:
    k = torch.randn(n, D, generator=gen, dtype=torch.float32)
    nheavy = int(round(HEAVY_FRACTION * n))
    if nheavy:
        heavy = torch.randperm(n, generator=gen)[:nheavy]
        k[heavy] *= HEAVY_SCALE
    return k


def _ar1_queries(n: int, H: int, D: int, gen: torch.Generator, chunk: int = 4096,
                 out_dtype: int = F32, start: torch.Tensor | None = None):
    """AR(1) walk along position, generated and stored chunk by chunk."""
    qs, scales = [], []
    prev = start
    for c0 in range(0, n, chunk):
        c = min(chunk, n - c0)
        z = torch.randn(c, H, D, generator=gen, dtype=torch.float32)
        buf = torch.empty(c, H, D, dtype=torch.float32)
        for i in range(c):
            if prev is None:
                buf[i] = z[i]
            else:
                torch.add(prev * AR_DECAY, z[i], alpha=AR_NOISE, out=buf[i])
            prev = buf[i]
        prev = prev.clone()
        stored, sc = _store(buf, out_dtype)
        qs.append(stored)
        if sc is not None:
            scales.append(sc)
    q = torch.cat(qs) if len(qs) > 1 else qs[0]
    return q, (torch.cat(scales) if scales else None)


def make_prefill(L: int, H: int, D: int, dtype: int, kind: str = "dsa", seed: int = 0) -> Prefill:
    gen = torch.Generator().manual_seed(seed)
    if kind == "int":
        q = torch.randint(-3, 4, (L, H, D), generator=gen).float()
        k = torch.randint(-3, 4, (L, D), generator=gen).float()
        w = torch.randint(1, 5, (L, H), generator=gen).float()
        if dtype != F32:
            # small integers are exact in bf16; e4m3 keeps them exact with scale 1
            qs, ks = _store_exact_int(q, dtype), _store_exact_int(k, dtype)
            return Prefill(dtype, qs[0], qs[1], w.contiguous(), ks[0], ks[1])
        return Prefill(dtype, q.contiguous(), None, w.contiguous(), k.contiguous(), None)
    if kind != "dsa":
        raise ValueError(kind)
    k = _dsa_keys(L, D, gen)
    q, q_scale = _ar1_queries(L, H, D, gen, out_dtype=dtype)
    w = torch.nn.functional.softplus(torch.randn(L, H, generator=gen, dtype=torch.float32))
    k_st, k_scale = _store(k, dtype)
    return Prefill(dtype, q, q_scale, w.contiguous(), k_st, k_scale)


def _store_exact_int(x: torch.Tensor, dtype: int):
    if dtype == BF16:
        return x.to(torch.bfloat16).contiguous(), None
    lead = x.shape[0]
    return (x.to(torch.float8_e4m3fn).contiguous(),
            torch.ones(lead, dtype=torch.float32))


def make_decode(B: int, Gm: int, H: int, D: int, dtype: int, len_lo: int, len_hi: int,
                maxlen: int | None = None, seed: int = 0) -> Decode:
    """Cached keys per sequence (cfg-2 generator), lengths uniform in
    [len_lo, len_hi]; the Gm new queries continue the AR(1) walk: the first
    starts from the stationary N(0,1), each next one is one AR step."""
    gen = torch.Generator().manual_seed(seed)
    cache_len = torch.randint(len_lo, len_hi + 1, (B,), generator=gen, dtype=torch.int64)
    if maxlen is None:
        maxlen = len_hi
    maxlen = max(maxlen, int(cache_len.max()))
    esz_dtype = {F32: torch.float32, BF16: torch.bfloat16, E4M3: torch.float8_e4m3fn}[dtype]
    kc = torch.zeros(B, maxlen, D, dtype=esz_dtype)
    kc_scale = torch.ones(B, maxlen, dtype=torch.float32) if dtype == E4M3 else None
    qs, q_scales, ws = [], [], []
    for b in range(B):
        n = int(cache_len[b])
        k = _dsa_keys(n, D, gen)
        k_st, k_sc = _store(k, dtype)
        kc[b, :n] = k_st
        if kc_scale is not None:
            kc_scale[b, :n] = k_sc
        q, q_sc = _ar1_queries(Gm, H, D, gen, out_dtype=dtype)
        qs.append(q)
        if q_sc is not None:
            q_scales.append(q_sc)
        ws.append(torch.nn.functional.softplus(torch.randn(Gm, H, generator=gen)))
    return Decode(dtype, torch.stack(qs).contiguous(),
                  torch.stack(q_scales).contiguous() if q_scales else None,
                  torch.stack(ws).float().contiguous(), kc.contiguous(), kc_scale,
                  cache_len.to(torch.int32))


def make_layers(nlayers: int, L: int, H: int, D: int, dtype: int, rho: float,
                seed: int = 0) -> list[Prefill]:
    """Indexer inputs of `nlayers` consecutive layers over one sequence, with
    layer-to-layer correlation rho: layer 0 from the DSA-shaped generator;
    layer l + 1's queries, keys and weight logits are rho * layer l's plus
    sqrt(1 - rho^2) * an independent draw of the same generator, so each layer
    keeps the generator's marginals while neighbouring layers' selections
    overlap more as rho grows.  (A synthetic stand-in: the pages give no
    cross-layer statistics.)"""
    gen = torch.Generator().manual_seed(seed)
    mix = float(np.sqrt(max(0.0, 1.0 - rho * rho)))
    k = _dsa_keys(L, D, gen)
    q, _ = _ar1_queries(L, H, D, gen, out_dtype=F32)
    z = torch.randn(L, H, generator=gen, dtype=torch.float32)
    out = []
    for layer in range(nlayers):
        if layer:
            k = rho * k + mix * _dsa_keys(L, D, gen)
            q = rho * q + mix * _ar1_queries(L, H, D, gen, out_dtype=F32)[0]
            z = rho * z + mix * torch.randn(L, H, generator=gen, dtype=torch.float32)
        qs, q_scale = _store(q, dtype)
        ks, k_scale = _store(k, dtype)
        w = torch.nn.functional.softplus(z).contiguous()
        out.append(Prefill(dtype, qs, q_scale, w, ks, k_scale))
    return out


# Named workloads (sizes as the benchmark and the parity tests use them).
WORKLOADS = {
    "tiny_int_prefill": dict(L=1024, H=4, D=32, dtype=F32, kind="int", topk=64, g=4, C=256),
    "dsa_prefill_16k": dict(L=16384, H=64, D=128, dtype=BF16, kind="dsa", topk=2048, g=8, C=4096),
    "dsa_prefill_64k": dict(L=65536, H=64, D=128, dtype=BF16, kind="dsa", topk=2048, g=8, C=4096),
    "long_prefill_128k_fp8": dict(L=131072, H=64, D=128, dtype=E4M3, kind="dsa", topk=2048, g=8,
                                  C=4096),
    # the long_prefill_128k_fp8 configuration at L=16384: small enough for
    # full profiler captures, scores still far larger than L2
    "fp8_prefill_16k": dict(L=16384, H=64, D=128, dtype=E4M3, kind="dsa", topk=2048, g=8, C=4096),
    "mtp_decode_b32": dict(B=32, Gm=2, H=64, D=128, dtype=E4M3, len_lo=32768, len_hi=131072,
                           topk=2048, C=4096),
}
