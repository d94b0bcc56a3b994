"""Seeded synthetic inputs shaped like the MSA pages' workloads.

This module only draws random numbers and arranges them into the tensors both
sides consume (the CUDA library and the fp64 oracle).  It contains none of the
method's arithmetic: no RoPE, no pooling, no cosine, no selection, no attention.

Every tensor comes from its own ``torch.Generator`` seeded from
(seed, tensor name, layer, slab), values are drawn in fp32 and converted to the
working dtype with round-to-nearest-even.  The same call on the same device
gives the same bytes; CPU and CUDA generators give different (equally valid)
values, so a test draws on one device and copies the bytes to the other side.

Shapes follow the workloads in the README of "MSA: Memory Sparse Attention"
("Results" setup: Qwen3-4B backbone, memory banks from 277K to 10M tokens, and
the 16K -> 100M scaling curve of Figure 1).  The recipe per configuration:

  tiny     fp32, 64 docs x 512 tokens, P=64, Hkv=Hr=2, Hq=4, d=dr=64, Tq=Lloc=32,
           k=2.  All tensors N(0,1); doc 17's router keys all equal query token 5.
  1m       bf16, 2048 docs x 512, Hq=32, Hkv=Hr=8, d=dr=128, Tq=Lloc=512, k=16.
           K, V, Q, local K/V ~ 0.5 N(0,1); router keys = one of 64 N(0,1) centres
           per document + 0.3 N(0,1) per token; Qr token t = centre (t mod 4) of 4
           randomly chosen centres + 0.3 N(0,1).
  decode16m bf16, 32768 docs x 512, 64 queries of 1 token, 4096 local tokens;
           256 centres; query b is near document j_b's centre (+ 0.05 N(0,1)).
  100m     bf16, 195,312 docs x 512 + one 256-token doc = 100,000,000 tokens
           (1,562,500 chunks), Tq=Lloc=64; 1024 centres; query tokens 0..7 are
           N(0,1) and planted (all router keys of 8 random documents equal one of
           them); tokens 8..63 are near random centres.
  stack10m bf16, 20,000 docs x 500 tokens (chunks 7 x 64 + 52), Tq=Lloc=4096,
           16 layers with independently seeded queries; 64 centres as in 1m.
"""
from __future__ import annotations

import dataclasses
import hashlib
from typing import Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    dtype: str              # "f32" or "bf16"
    D: int                  # documents
    L: int                  # tokens per document
    last_len: Optional[int]  # length of the final document if it differs from L
    P: int                  # chunk size
    Hkv: int
    Hr: int
    Hq: int
    d: int
    dr: int
    B: int
    Tq: int
    Lloc: int
    k: int
    theta: float = 1e6
    n_centres: int = 0      # 0: router keys are plain N(0,1)
    query_mode: str = "normal"   # normal | centres4 | near_doc | planted8
    kv_scale: float = 1.0
    sigma: float = 0.3
    layers: int = 1
    docs_per_slab: int = 0  # raw tokens are drawn per slab of documents (0 = all at once)
    planted_doc: int = -1   # tiny: document whose router keys equal query token planted_tok
    planted_tok: int = 5

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def ntok(self) -> int:
        return int(doc_tok_offsets(self)[-1])

    @property
    def chunks_per_doc_max(self) -> int:
        return -(-max(self.L, self.last_len or 0) // self.P)

    @property
    def C(self) -> int:
        n = -(-self.L // self.P) * (self.D - (1 if self.last_len else 0))
        if self.last_len:
            n += -(-self.last_len // self.P)
        return n

    @property
    def Mmax(self) -> int:
        return self.k * self.chunks_per_doc_max

    def scaled(self, **kw) -> "Config":
        """A copy with some fields replaced (smaller test cases of the same shape)."""
        return dataclasses.replace(self, **kw)


CONFIGS = {
    "tiny": Config("tiny", "f32", D=64, L=512, last_len=None, P=64, Hkv=2, Hr=2, Hq=4, d=64, dr=64,
                   B=1, Tq=32, Lloc=32, k=2, planted_doc=17),
    "1m": Config("1m", "bf16", D=2048, L=512, last_len=None, P=64, Hkv=8, Hr=8, Hq=32, d=128, dr=128,
                 B=1, Tq=512, Lloc=512, k=16, n_centres=64, query_mode="centres4", kv_scale=0.5),
    "decode16m": Config("decode16m", "bf16", D=32768, L=512, last_len=None, P=64, Hkv=8, Hr=8, Hq=32,
                        d=128, dr=128, B=64, Tq=1, Lloc=4096, k=16, n_centres=256,
                        query_mode="near_doc", kv_scale=0.5, docs_per_slab=2048),
    "100m": Config("100m", "bf16", D=195313, L=512, last_len=256, P=64, Hkv=8, Hr=8, Hq=32, d=128,
                   dr=128, B=1, Tq=64, Lloc=64, k=16, n_centres=1024, query_mode="planted8",
                   kv_scale=0.5, docs_per_slab=2048),
    "stack10m": Config("stack10m", "bf16", D=20000, L=500, last_len=None, P=64, Hkv=8, Hr=8, Hq=32,
                       d=128, dr=128, B=1, Tq=4096, Lloc=4096, k=16, n_centres=64,
                       query_mode="centres4", kv_scale=0.5, layers=16, docs_per_slab=2000),
}


def get_config(name: str) -> Config:
    return CONFIGS[name]


# ----------------------------------------------------------------------------
def _seed(*parts) -> int:
    h = hashlib.sha256(repr(parts).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def _gen(device, *parts) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_seed(*parts))
    return g


def _randn(shape, device, *parts) -> torch.Tensor:
    return torch.randn(shape, generator=_gen(device, *parts), device=device, dtype=torch.float32)


def doc_tok_offsets(cfg: Config) -> np.ndarray:
    """Token offsets [D+1] (int64): document j holds tokens [off[j], off[j+1])."""
    lens = np.full(cfg.D, cfg.L, dtype=np.int64)
    if cfg.last_len:
        lens[-1] = cfg.last_len
    return np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)


def _centres(cfg: Config, device, seed: int):
    c = _randn((cfg.n_centres, cfg.Hr, cfg.dr), device, seed, "centres")
    g = _gen("cpu", seed, "doc_centre")
    doc_c = torch.randint(cfg.n_centres, (cfg.D,), generator=g).to(device)
    return c, doc_c


def planted_docs(cfg: Config, seed: int = 0) -> np.ndarray:
    """Documents whose router keys are planted equal to a query token (tiny: one, 100m: eight)."""
    if cfg.query_mode == "planted8":
        rng = np.random.default_rng(_seed(seed, "planted"))
        return np.sort(rng.choice(cfg.D - 1, size=8, replace=False)).astype(np.int64)
    if cfg.planted_doc >= 0:
        return np.array([cfg.planted_doc], dtype=np.int64)
    return np.zeros(0, dtype=np.int64)


def gen_query(cfg: Config, layer: int = 0, device="cpu", seed: int = 0):
    """Query-side tensors of one layer: Qr [B,Tq,Hr,dr], Q [B,Tq,Hq,d], Kloc/Vloc [B,Lloc,Hkv,d]."""
    s = (seed, "layer", layer)
    B, Tq = cfg.B, cfg.Tq
    Q = _randn((B, Tq, cfg.Hq, cfg.d), device, *s, "Q") * cfg.kv_scale
    Kl = _randn((B, cfg.Lloc, cfg.Hkv, cfg.d), device, *s, "Kloc") * cfg.kv_scale
    Vl = _randn((B, cfg.Lloc, cfg.Hkv, cfg.d), device, *s, "Vloc") * cfg.kv_scale
    noise = _randn((B, Tq, cfg.Hr, cfg.dr), device, *s, "Qr")
    if cfg.query_mode == "normal":
        Qr = noise
    else:
        cen, doc_c = _centres(cfg, device, seed)
        g = _gen("cpu", *s, "pick")
        if cfg.query_mode == "centres4":
            pick = torch.randint(cfg.n_centres, (4,), generator=g).to(device)
            which = pick[torch.arange(Tq, device=device) % 4]
            Qr = cen[which][None] + cfg.sigma * noise
        elif cfg.query_mode == "near_doc":
            docs = torch.randint(cfg.D, (B,), generator=g).to(device)
            Qr = cen[doc_c[docs]][:, None] + 0.05 * noise
        elif cfg.query_mode == "planted8":
            pick = torch.randint(cfg.n_centres, (Tq,), generator=g).to(device)
            Qr = cen[pick][None] + cfg.sigma * noise
            Qr[:, :8] = noise[:, :8]
        else:
            raise ValueError(cfg.query_mode)
    dt = cfg.torch_dtype
    return dict(Qr=Qr.to(dt), Q=Q.to(dt), Kloc=Kl.to(dt), Vloc=Vl.to(dt))


def slab_bounds(cfg: Config):
    """Document ranges [(lo, hi)] in which raw tokens are drawn."""
    step = cfg.docs_per_slab or cfg.D
    return [(lo, min(lo + step, cfg.D)) for lo in range(0, cfg.D, step)]


def gen_raw_slab(cfg: Config, doc_lo: int, doc_hi: int, device="cpu", seed: int = 0, Qr0=None):
    """Raw per-token K, V [n, Hkv, d] and Kr [n, Hr, dr] for documents [doc_lo, doc_hi).

    doc_lo must start a slab (see slab_bounds) so any slab can be redrawn alone.
    Qr0 ([Tq, Hr, dr], query 0's router projections of layer 0) is needed to plant
    exact matches; when omitted it is drawn here with gen_query.
    """
    off = doc_tok_offsets(cfg)
    t0, t1 = int(off[doc_lo]), int(off[doc_hi])
    n = t1 - t0
    s = (seed, "slab", doc_lo)
    K = _randn((n, cfg.Hkv, cfg.d), device, *s, "K") * cfg.kv_scale
    V = _randn((n, cfg.Hkv, cfg.d), device, *s, "V") * cfg.kv_scale
    noise = _randn((n, cfg.Hr, cfg.dr), device, *s, "Kr")
    if cfg.n_centres:
        cen, doc_c = _centres(cfg, device, seed)
        lens = torch.from_numpy(np.diff(off[doc_lo : doc_hi + 1])).to(device)
        tok_doc = torch.repeat_interleave(torch.arange(doc_lo, doc_hi, device=device), lens)
        Kr = cen[doc_c[tok_doc]] + cfg.sigma * noise
    else:
        Kr = noise
    pl = planted_docs(cfg, seed)
    if len(pl):
        if Qr0 is None:
            Qr0 = gen_query(cfg, 0, device, seed)["Qr"][0]
        Qr0 = Qr0.to(device=device, dtype=torch.float32)
        for i, j in enumerate(pl.tolist()):
            if doc_lo <= j < doc_hi:
                tok = cfg.planted_tok if cfg.query_mode != "planted8" else i
                Kr[int(off[j]) - t0 : int(off[j + 1]) - t0] = Qr0[tok]
    dt = cfg.torch_dtype
    return K.to(dt), V.to(dt), Kr.to(dt)


def gen_bank_bf16(C: int, H: int, dim: int, device="cpu", seed: int = 0, name: str = "bank"):
    """A directly drawn bank tensor [C, H, dim] in bf16 (for step tests that skip pooling)."""
    return _randn((C, H, dim), device, seed, name).to(torch.bfloat16)
