"""Seeded synthetic inputs for the multi-LoRA delta, shared by the oracle tests,
the CUDA parity tests and the benchmark.

This module only draws numbers: token -> adapter assignments, adapter ranks,
activations x, base outputs y (which stand for W x) and adapter matrices A, B.
It holds none of the method's arithmetic.

Shapes follow the pages' workloads:
  * the Llama-3-70B projection shapes of the memory table in "Multi-LoRA
    serving: the single translator with a thousand glossaries ..."
    (blog.lo0.es), section "The maths that matters";
  * the 32-request / 250-tenant decode example of the "Multi-LoRA Serving"
    glossary entry (skillsintelligence.tools), paragraph "Example";
  * ranks "typically 8, 16, 32 or 64" from section "The bare mechanism" of the
    blog.lo0.es post.

Value recipe (all drawn in fp32 and rounded to bf16 with round-to-nearest-even):
  x ~ N(0,1)/sqrt(d_in), A ~ N(0,1)/sqrt(d_in), B ~ N(0,1)/sqrt(r), y ~ N(0,1).
Orientation is the one of section "The bare mechanism": A is r x d_in and
B is d_out x r, both row-major.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Tuple

import numpy as np
import torch

LLAMA70B_PROJECTIONS: Tuple[Tuple[str, int, int], ...] = (
    ("q", 8192, 8192),
    ("k", 8192, 1024),
    ("v", 8192, 1024),
    ("o", 8192, 8192),
    ("gate", 8192, 28672),
    ("up", 8192, 28672),
    ("down", 28672, 8192),
)

WORKLOAD_NAMES = ("tiny", "decode_q_proj", "decode_q_proj_12", "mixed_rank_mlp_up", "prefill_long",
                  "llama70b_layer", "llama70b_layer_shared_x")

# projection whose input x each Llama-3-70B projection reads in a real layer: q, k and v the
# attention input, o its own (the attention output), gate and up the MLP input, down its own
LLAMA70B_X_SOURCE = (0, 0, 0, 3, 4, 4, 6)


@dataclasses.dataclass
class Workload:
    """Metadata of one synthetic batch (no tensors)."""

    name: str
    seed: int
    T: int                                   # tokens in the batch
    projections: List[Tuple[str, int, int]]  # (name, d_in, d_out)
    pool_ids: np.ndarray                     # int32 ids of the adapters resident in the pool
    pool_ranks: np.ndarray                   # int32 rank of each resident adapter (same order)
    adapter_ids: np.ndarray                  # int32[T] adapter per token, -1 = no adapter
    scale: float = 1.0
    note: str = ""
    x_source: Optional[List[int]] = None     # projection whose x each projection reads (None: its own)

    def x_of(self, proj: int) -> int:
        return proj if self.x_source is None else int(self.x_source[proj])

    def rank_of(self, adapter_id: int) -> int:
        return int(self.pool_ranks[self._index()[int(adapter_id)]])

    def _index(self) -> Dict[int, int]:
        if not hasattr(self, "_idx_cache"):
            self._idx_cache = {int(a): i for i, a in enumerate(self.pool_ids)}
        return self._idx_cache

    @property
    def distinct_adapters(self) -> int:
        ids = self.adapter_ids[self.adapter_ids >= 0]
        return int(np.unique(ids).size)


def _bounded_zipf(rng: np.random.Generator, s: float, n: int, size: int) -> np.ndarray:
    """Draw `size` values in 0..n-1 with P(k) proportional to 1/(k+1)^s."""
    w = 1.0 / np.arange(1, n + 1, dtype=np.float64) ** s
    w /= w.sum()
    return rng.choice(n, size=size, p=w)


def make(name: str, seed: int = 0, **overrides) -> Workload:
    """Build the metadata of a named workload.

    tiny              T=64, d 512->512, 4 adapters of rank 8, 4 contiguous segments of 16 tokens.
    decode_q_proj     T=32 decode tokens, q_proj 8192->8192, rank 16, adapter per token from a
                      bounded Zipf(s=1.1) over a pool of 250 resident adapters.
    decode_q_proj_12  the same with Zipf(s=1.5): about 12 distinct adapters among the 32
                      requests, the glossary example's "32 requests, 12 tenants".
    mixed_rank_mlp_up T=256, 4096->14336, pool of 512 adapters with ranks uniform over
                      {8,16,32,64}; 64 distinct adapters drawn, tokens assigned uniformly.
    prefill_long      8 requests x 512 tokens, 8 adapters of rank 64, 8192->8192,
                      one contiguous segment per request.
    llama70b_layer    7 projections of a Llama-3-70B layer, T=256 decode tokens each on a
                      distinct adapter drawn from a pool of 2000, rank 16; every projection
                      has its own input x.
    llama70b_layer_shared_x  the same batch with the inputs of a real layer: q, k and v read
                      one x (the attention input), gate and up one x (the MLP input), o and
                      down their own -- 4 distinct x for 7 projections.
    """
    rng = np.random.default_rng(seed)
    if name == "tiny":
        T = overrides.get("T", 64)
        n_ad = 4
        pool_ids = np.arange(n_ad, dtype=np.int32)
        pool_ranks = np.full(n_ad, overrides.get("rank", 8), dtype=np.int32)
        seg = T // n_ad
        ids = np.repeat(pool_ids, seg).astype(np.int32)
        d = overrides.get("d", 512)
        wl = Workload(name, seed, T, [("proj", d, d)], pool_ids, pool_ranks, ids)
    elif name in ("decode_q_proj", "decode_q_proj_12"):
        T = overrides.get("T", 32)
        n_pool = overrides.get("pool", 250)
        s = overrides.get("zipf_s", 1.1 if name == "decode_q_proj" else 1.5)
        d = overrides.get("d", 8192)
        pool_ids = np.arange(n_pool, dtype=np.int32)
        pool_ranks = np.full(n_pool, overrides.get("rank", 16), dtype=np.int32)
        ids = _bounded_zipf(rng, s, n_pool, T).astype(np.int32)
        wl = Workload(name, seed, T, [("q", d, d)], pool_ids, pool_ranks, ids)
    elif name == "mixed_rank_mlp_up":
        T = overrides.get("T", 256)
        n_pool = overrides.get("pool", 512)
        n_active = overrides.get("active", 64)
        d_in = overrides.get("d_in", 4096)
        d_out = overrides.get("d_out", 14336)
        pool_ids = np.arange(n_pool, dtype=np.int32)
        pool_ranks = rng.choice(np.array([8, 16, 32, 64], dtype=np.int32), size=n_pool)
        active = rng.choice(n_pool, size=n_active, replace=False)
        ids = active[rng.integers(0, n_active, size=T)].astype(np.int32)
        wl = Workload(name, seed, T, [("up", d_in, d_out)], pool_ids,
                      pool_ranks.astype(np.int32), ids)
    elif name == "prefill_long":
        n_req = overrides.get("requests", 8)
        L = overrides.get("seq", 512)
        d = overrides.get("d", 8192)
        T = n_req * L
        pool_ids = np.arange(n_req, dtype=np.int32)
        pool_ranks = np.full(n_req, overrides.get("rank", 64), dtype=np.int32)
        ids = np.repeat(pool_ids, L).astype(np.int32)
        wl = Workload(name, seed, T, [("proj", d, d)], pool_ids, pool_ranks, ids)
    elif name in ("llama70b_layer", "llama70b_layer_shared_x"):
        T = overrides.get("T", 256)
        n_pool = overrides.get("pool", 2000)
        projs = overrides.get("projections", list(LLAMA70B_PROJECTIONS))
        pool_ids = np.arange(n_pool, dtype=np.int32)
        pool_ranks = np.full(n_pool, overrides.get("rank", 16), dtype=np.int32)
        ids = rng.choice(n_pool, size=T, replace=False).astype(np.int32)
        wl = Workload(name, seed, T, [tuple(p) for p in projs], pool_ids, pool_ranks, ids,
                      x_source=list(LLAMA70B_X_SOURCE) if name == "llama70b_layer_shared_x" else None)
    else:
        raise KeyError(f"unknown workload {name!r}; known: {WORKLOAD_NAMES}")
    return wl


# ----------------------------------------------------------------------------
# tensors
# ----------------------------------------------------------------------------

def _gen(device, *key: int) -> torch.Generator:
    g = torch.Generator(device=device)
    h = 0x9E3779B97F4A7C15
    for k in key:
        h = (h * 0x100000001B3 + (int(k) & 0xFFFFFFFF) + 0x632BE59BD9B4E019) & 0x7FFFFFFFFFFFFFFF
    g.manual_seed(h)
    return g


def _randn_bf16(shape, std: float, g: torch.Generator, device) -> torch.Tensor:
    t = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(torch.bfloat16)


def activations(wl: Workload, proj: int, device="cpu") -> Tuple[torch.Tensor, torch.Tensor]:
    """x bf16 [T][d_in] and y bf16 [T][d_out] (y stands for the base output W x).  A
    projection that shares its input (wl.x_source) gets the same x values as the
    projection it reads from."""
    _, d_in, d_out = wl.projections[proj]
    src = wl.x_of(proj)
    assert wl.projections[src][1] == d_in, "projections sharing x need the same d_in"
    x = _randn_bf16((wl.T, d_in), 1.0 / math.sqrt(d_in), _gen(device, wl.seed, src, 1), device)
    y = _randn_bf16((wl.T, d_out), 1.0, _gen(device, wl.seed, proj, 2), device)
    return x, y


class AdapterBank:
    """All resident adapters' A and B for every projection, grouped by rank.

    bank.A[p][rho] is bf16 [n_rho][rho][d_in]; bank.B[p][rho] is bf16 [n_rho][d_out][rho].
    """

    def __init__(self, wl: Workload, device="cpu", projections: Optional[List[int]] = None):
        self.wl = wl
        self.device = device
        self.projs = list(range(len(wl.projections))) if projections is None else list(projections)
        self.slot: Dict[int, Tuple[int, int]] = {}
        groups: Dict[int, List[int]] = {}
        for a, r in zip(wl.pool_ids.tolist(), wl.pool_ranks.tolist()):
            groups.setdefault(int(r), []).append(int(a))
        for r, members in groups.items():
            for i, a in enumerate(members):
                self.slot[a] = (r, i)
        self.groups = groups
        self.A: Dict[int, Dict[int, torch.Tensor]] = {}
        self.B: Dict[int, Dict[int, torch.Tensor]] = {}
        for p in self.projs:
            _, d_in, d_out = wl.projections[p]
            self.A[p], self.B[p] = {}, {}
            for r, members in groups.items():
                n = len(members)
                if r == 0:
                    self.A[p][r] = torch.zeros(n, 0, d_in, dtype=torch.bfloat16, device=device)
                    self.B[p][r] = torch.zeros(n, d_out, 0, dtype=torch.bfloat16, device=device)
                    continue
                self.A[p][r] = _randn_bf16((n, r, d_in), 1.0 / math.sqrt(d_in),
                                           _gen(device, wl.seed, p, 3, r), device)
                self.B[p][r] = _randn_bf16((n, d_out, r), 1.0 / math.sqrt(r),
                                           _gen(device, wl.seed, p, 4, r), device)

    def get(self, adapter: int, proj: int) -> Tuple[torch.Tensor, torch.Tensor]:
        """(A [r][d_in], B [d_out][r]) views for one adapter and projection."""
        r, i = self.slot[int(adapter)]
        return self.A[proj][r][i], self.B[proj][r][i]


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact widening of a bf16 (or fp32) tensor to a float64 numpy array."""
    return t.detach().to("cpu").to(torch.float64).numpy()
