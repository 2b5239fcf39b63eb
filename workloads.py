"""Seeded synthetic inputs for exact maximum-inner-product search.

This module only draws numbers: raw candidate vectors, raw user (query)
vectors and exclusion bitmasks. It holds none of the method's arithmetic (no
normalisation, no scoring, no selection), so both the CUDA library and the fp64
oracle can take its output as their common input.

Recipes (the pages publish no dataset for this path; these stand in for a
candidate-tower corpus and a batch of user-tower outputs):

* ``clusters``: Gaussian taste clusters. Centre m is a unit vector with
  components +-1/sqrt(d) (random signs); a row is ``centre + sigma * N(0, I)``.
  Cluster sizes are uniform, or Zipf(1.0) (size of cluster c proportional to
  1/c, largest-remainder rounding to n rows, row order shuffled). Queries pick
  a cluster uniformly. (Toy in mhtirogla.ai "Two-tower retrieval": 8 taste
  groups, d = 16, 400 items, 128 users per batch.)
* ``gaussian``: rows ~ N(0, I).
* ``lognormal_rows``: rows ``N(0, I) * exp(0.5 * z)``, z ~ N(0, 1) per row
  (raw, un-normalised candidate vectors of varied length), stored in bf16.
* exclusion mask: independent Bernoulli(rate) per candidate, packed 32 per
  uint32 word, bit (j & 31) of word (j >> 5) set = candidate j excluded.

In-batch training batches (``Batch``, for the sampled-softmax loss): user and
item vectors ~ N(0, I / d) (length close to 1, as unit-norm tower outputs are;
"Two-Tower Retrieval at Industrial Scale", section 3, (B, 64) unit-norm user
and item towers), stored in bf16. Each column's item id is drawn from a
catalogue with Zipf popularity p(c) proportional to (c + 1)^-s, so popular
items repeat inside a batch (the accidental hits); a repeated id carries the
vector of its first occurrence; log q_j is the log of the drawing probability
of column j's item. A column is padding with probability pad_rate. Columns
b..nc-1 are drawn the same way and act as shared negatives.

Every tensor is drawn with ``torch.Generator`` seeded from the workload seed,
in fixed-size chunks, so the same call gives the same numbers on the same
device type.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

CHUNK_ROWS = 1 << 20
BASE_SEED = 20261202


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    n: int                 # candidates
    d: int                 # embedding width
    b: int                 # queries per batch
    k: int
    tau: float
    raw_dtype: str         # dtype of the raw corpus rows: "f32" | "bf16"
    store: str             # "f32" | "bf16": normalised rows stored; "raw": rows kept raw, norms fused
    query_dtype: str       # dtype the normalised queries are stored in
    recipe: str            # "clusters" | "gaussian" | "lognormal_rows"
    query_recipe: str      # "clusters" | "gaussian"
    n_clusters: int = 0
    sigma: float = 0.0
    zipf: bool = False
    mask_rate: float = 0.0
    oracle_queries: int = 0  # 0: check every query; else a seeded sample of this many
    seed: int = BASE_SEED

    @property
    def masked(self) -> bool:
        return self.mask_rate > 0.0

    @property
    def tolerance(self) -> float:
        """Absolute score tolerance: 1e-5 for an fp32 corpus, 2e-3 for bf16."""
        return 1e-5 if self.store == "f32" else 2e-3

    def describe(self) -> dict:
        return dataclasses.asdict(self)


# The five workloads, at full size.
WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", n=400, d=16, b=128, k=10, tau=1.0, raw_dtype="f32",
                         store="f32", query_dtype="f32", recipe="clusters", query_recipe="clusters",
                         n_clusters=8, sigma=0.3, seed=BASE_SEED + 1),
    "stream_b1": Workload("stream_b1", n=1_000_000, d=128, b=1, k=100, tau=1.0, raw_dtype="f32",
                          store="bf16", query_dtype="f32", recipe="gaussian",
                          query_recipe="gaussian", seed=BASE_SEED + 2),
    "small_batch": Workload("small_batch", n=10_000_000, d=128, b=32, k=500, tau=0.1,
                            raw_dtype="f32", store="bf16", query_dtype="bf16", recipe="clusters",
                            query_recipe="clusters", n_clusters=1024, sigma=0.3, zipf=True,
                            seed=BASE_SEED + 3),
    "large_batch": Workload("large_batch", n=50_000_000, d=128, b=1024, k=1000, tau=1.0,
                            raw_dtype="f32", store="bf16", query_dtype="bf16", recipe="clusters",
                            query_recipe="clusters", n_clusters=1024, sigma=0.3, zipf=True,
                            oracle_queries=16, seed=BASE_SEED + 4),
    "masked_fused": Workload("masked_fused", n=20_000_000, d=256, b=4096, k=256, tau=0.05,
                             raw_dtype="bf16", store="raw", query_dtype="bf16",
                             recipe="lognormal_rows", query_recipe="gaussian", mask_rate=0.05,
                             oracle_queries=16, seed=BASE_SEED + 5),
}


def workload(name: str, **overrides) -> Workload:
    """A named workload, optionally resized (``n=``, ``b=``, ``k=`` ...)."""
    return dataclasses.replace(WORKLOADS[name], **overrides)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _torch_dtype(name: str):
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def zipf_sizes(n: int, n_clusters: int) -> np.ndarray:
    """Cluster sizes proportional to 1/c (c = 1..C), largest-remainder rounding to n."""
    w = 1.0 / np.arange(1, n_clusters + 1, dtype=np.float64)
    exact = w / w.sum() * n
    sizes = np.floor(exact).astype(np.int64)
    short = int(n - sizes.sum())
    order = np.argsort(-(exact - sizes), kind="stable")
    sizes[order[:short]] += 1
    return sizes


def _centres(w: Workload, g: torch.Generator, device) -> torch.Tensor:
    signs = torch.randint(0, 2, (w.n_clusters, w.d), generator=g, device=device)
    return (signs.to(torch.float32) * 2.0 - 1.0) * (1.0 / math.sqrt(w.d))


def _cluster_rows(centres, assign, sigma, d, g, device, out, row0, limit=None):
    """out[row0 + i] = centres[assign[i]] + sigma * N(0, I), for i < limit
    (default: every row). Noise is drawn in whole chunks, so a prefix holds
    the same numbers as the full draw."""
    limit = assign.numel() if limit is None else limit
    for s in range(0, limit, CHUNK_ROWS):
        a = assign[s:s + CHUNK_ROWS]
        noise = torch.randn((a.numel(), d), generator=g, device=device, dtype=torch.float32)
        m = min(a.numel(), limit - s)
        out[row0 + s:row0 + s + m] = (centres[a[:m]] + sigma * noise[:m]).to(out.dtype)


def corpus(w: Workload, device="cpu", rows: int | None = None) -> torch.Tensor:
    """Raw candidate rows [n, d] in ``w.raw_dtype``; with ``rows``, only the
    first ``rows`` of them (the same numbers as the full corpus holds there,
    without drawing the rest)."""
    g = _gen(w.seed, device)
    m_out = w.n if rows is None else max(0, min(int(rows), w.n))
    out = torch.empty((m_out, w.d), dtype=_torch_dtype(w.raw_dtype), device=device)
    if w.recipe == "clusters":
        centres = _centres(w, g, device)
        if w.zipf:
            sizes = torch.from_numpy(zipf_sizes(w.n, w.n_clusters)).to(device)
            assign = torch.repeat_interleave(torch.arange(w.n_clusters, device=device), sizes)
            assign = assign[torch.randperm(w.n, generator=g, device=device)]
        else:
            assign = torch.randint(0, w.n_clusters, (w.n,), generator=g, device=device)
        _cluster_rows(centres, assign, w.sigma, w.d, g, device, out, 0, limit=m_out)
    elif w.recipe == "gaussian":
        for s in range(0, m_out, CHUNK_ROWS):
            m = min(CHUNK_ROWS, w.n - s)
            x = torch.randn((m, w.d), generator=g, device=device)
            keep = min(m, m_out - s)
            out[s:s + keep] = x[:keep].to(out.dtype)
    elif w.recipe == "lognormal_rows":
        for s in range(0, m_out, CHUNK_ROWS):
            m = min(CHUNK_ROWS, w.n - s)
            x = torch.randn((m, w.d), generator=g, device=device)
            z = torch.randn((m, 1), generator=g, device=device)
            keep = min(m, m_out - s)
            out[s:s + keep] = (x[:keep] * torch.exp(0.5 * z[:keep])).to(out.dtype)
    else:
        raise ValueError(w.recipe)
    return out


def queries(w: Workload, device="cpu") -> torch.Tensor:
    """Raw user vectors [b, d] (fp32)."""
    g = _gen(w.seed + 1_000_003, device)
    out = torch.empty((w.b, w.d), dtype=torch.float32, device=device)
    if w.query_recipe == "clusters":
        # the same centres as the corpus: re-draw them from the corpus seed
        centres = _centres(w, _gen(w.seed, device), device)
        assign = torch.randint(0, w.n_clusters, (w.b,), generator=g, device=device)
        _cluster_rows(centres, assign, w.sigma, w.d, g, device, out, 0)
    elif w.query_recipe == "gaussian":
        out.copy_(torch.randn((w.b, w.d), generator=g, device=device))
    else:
        raise ValueError(w.query_recipe)
    return out


def exclusion_bits(w: Workload, device="cpu") -> torch.Tensor | None:
    """Packed exclusion bitmask (int32 words holding uint32 bit patterns), or None."""
    if not w.masked:
        return None
    g = _gen(w.seed + 2_000_003, device)
    words = (w.n + 31) // 32
    bits = torch.zeros(words * 32, dtype=torch.bool, device=device)
    bits[:w.n] = torch.rand((w.n,), generator=g, device=device) < w.mask_rate
    weights = (torch.ones(32, dtype=torch.int64, device=device) << torch.arange(32, device=device))
    packed = (bits.view(words, 32).to(torch.int64) * weights).sum(dim=1)
    return (packed - ((packed >> 31) << 32)).to(torch.int32)  # same bits, as int32


def oracle_query_ids(w: Workload) -> np.ndarray:
    """Which queries the oracle checks: all, or a seeded sample without replacement."""
    if w.oracle_queries <= 0 or w.oracle_queries >= w.b:
        return np.arange(w.b, dtype=np.int64)
    rng = np.random.Generator(np.random.Philox(w.seed + 3_000_003))
    return np.sort(rng.choice(w.b, size=w.oracle_queries, replace=False)).astype(np.int64)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """A bf16 tensor's bit patterns as a numpy uint16 array (host copy)."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def to_numpy_rows(t: torch.Tensor) -> np.ndarray:
    """Host copy in the oracle's array convention (fp32 as float32, bf16 as uint16 bits)."""
    if t.dtype == torch.bfloat16:
        return bf16_bits(t)
    return t.detach().contiguous().cpu().numpy()


# ---------------------------------------------------------------------------
# in-batch training batches
# ---------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class Batch:
    name: str
    b: int               # users (rows); row i's positive is column i
    nc: int              # candidate columns, nc >= b (columns >= b: shared negatives)
    d: int
    tau: float
    catalogue: int       # items the ids are drawn from
    zipf_s: float        # popularity exponent
    pad_rate: float      # probability that a column (and its row) is padding
    oracle_rows: int = 0  # 0: check every row; else a seeded sample of this many
    seed: int = BASE_SEED + 11

    def describe(self) -> dict:
        return dataclasses.asdict(self)


BATCHES = {
    # the article's batch of 8192 rows with 64-wide towers
    "inbatch_b8192_d64": Batch("inbatch_b8192_d64", b=8192, nc=8192, d=64, tau=0.05, catalogue=1_000_000,
                               zipf_s=1.0, pad_rate=0.01, oracle_rows=64, seed=BASE_SEED + 11),
    # a large global batch: 2^32 logits
    "inbatch_b65536_d64": Batch("inbatch_b65536_d64", b=65536, nc=65536, d=64, tau=0.05, catalogue=1_000_000,
                                zipf_s=1.0, pad_rate=0.01, oracle_rows=32, seed=BASE_SEED + 12),
    # wider towers and as many shared negatives as in-batch ones
    "inbatch_b16384_g16384_d128": Batch("inbatch_b16384_g16384_d128", b=16384, nc=32768, d=128, tau=0.05,
                                        catalogue=1_000_000, zipf_s=1.0, pad_rate=0.01, oracle_rows=32,
                                        seed=BASE_SEED + 13),
}


def batch(name: str, **overrides) -> Batch:
    """A named training batch, optionally resized (``b=``, ``nc=``, ``d=`` ...)."""
    return dataclasses.replace(BATCHES[name], **overrides)


def batch_inputs(w: Batch, device="cpu") -> dict:
    """users bf16 [b, d], items bf16 [nc, d], logq f32 [nc], item_ids int64 [nc],
    valid bool [nc]; drawn on the CPU (the same numbers for every device) and
    then moved to ``device``."""
    g = _gen(w.seed, "cpu")
    users = (torch.randn((w.b, w.d), generator=g) / math.sqrt(w.d)).to(torch.bfloat16)
    weights = torch.arange(1, w.catalogue + 1, dtype=torch.float64) ** (-w.zipf_s)
    prob = weights / weights.sum()
    ids = torch.multinomial(prob, w.nc, replacement=True, generator=g)
    vecs = (torch.randn((w.nc, w.d), generator=g) / math.sqrt(w.d)).to(torch.bfloat16)
    # a repeated item carries the vector of its first occurrence
    _, inverse = torch.unique(ids, return_inverse=True)
    first = torch.full((int(inverse.max()) + 1 if w.nc else 0,), w.nc, dtype=torch.int64)
    first = first.scatter_reduce(0, inverse, torch.arange(w.nc), reduce="amin")
    items = vecs[first[inverse]]
    logq = torch.log(prob[ids]).to(torch.float32)
    valid = torch.rand(w.nc, generator=g) >= w.pad_rate
    return {"users": users.to(device), "items": items.contiguous().to(device), "logq": logq.to(device),
            "item_ids": ids.to(device), "valid": valid.to(device)}


def oracle_row_ids(w: Batch) -> np.ndarray:
    """The rows the oracle checks for a full-size batch (sorted, seeded)."""
    if w.oracle_rows == 0 or w.oracle_rows >= w.b:
        return np.arange(w.b, dtype=np.int64)
    rng = np.random.Generator(np.random.Philox(w.seed + 5_000_011))
    return np.sort(rng.choice(w.b, size=w.oracle_rows, replace=False)).astype(np.int64)
