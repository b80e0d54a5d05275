"""Seeded synthetic decode workloads: request lengths, paged KV caches, block tables.

This module only draws random numbers and lays them out; it holds none of the
attention arithmetic.  Both the CUDA path and the CPU oracle consume what it
returns, which is why it lives in a module of its own.

The shapes follow the kind of traffic described in "Tencent HPC lands in
SGLang, challenging default inference kernels", section "Why Tencent HPC
matters for online model serving": a continuous batch that mixes long
histories (tens of thousands of tokens) with short, just-started requests.

Recipe (all draws in this order, from ``numpy.random.default_rng(seed)`` for
integers and ``torch.Generator().manual_seed(seed)`` for values):
  1. request lengths (config specific);
  2. page assignment: request b needs ceil(L_b / P) pages; 5 % spare pages are
     added; the physical ids are a random permutation of all pages, handed to
     the requests in order; unused block-table entries hold -1;
  3. K rows picked as outliers (Bernoulli per token row, shared by all KV
     heads of that row), when the config asks for them;
  4. q ~ N(0,1) ([B, Hq, d], or [B, q_len, Hq, d] for multi-query decode),
     then K ~ N(0,1) (outlier rows multiplied before rounding),
     then V ~ N(0,1), each rounded to bf16 (round-to-nearest-even);
  5. slots past the end of each request and the spare pages are filled with
     NaN ("poison"), so that any read outside the valid tokens shows up.
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

BF16_NAN = 0x7FC0  # a quiet NaN in bfloat16


@dataclasses.dataclass(frozen=True)
class Problem:
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    page_size: int
    max_pages_per_req: int
    num_pages: int
    scale: float  # an fp32 value; both sides use exactly this number
    q_len: int = 1  # queries per request (the last q_len cached tokens)

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def capacity_tokens(self) -> int:
        return self.max_pages_per_req * self.page_size


@dataclasses.dataclass
class Workload:
    name: str
    problem: Problem
    seq_lens: np.ndarray  # int32 [B]
    block_table: np.ndarray  # int32 [B, max_pages_per_req]
    q: torch.Tensor  # bf16 CPU [B, Hq, d]
    k_cache: torch.Tensor  # bf16 CPU [num_pages, Hkv, P, d]
    v_cache: torch.Tensor  # bf16 CPU [num_pages, Hkv, P, d]
    seed: int
    recipe: str = ""

    @property
    def kv_bytes(self) -> int:
        """Bytes of K and V that one decode step must read: sum_b L_b * Hkv * d * 2 (K,V) * 2 B."""
        p = self.problem
        return int(np.clip(self.seq_lens, 0, None).astype(np.int64).sum()) * p.num_kv_heads * p.head_dim * 4

    def to(self, device) -> "DeviceWorkload":
        return DeviceWorkload(
            problem=self.problem,
            seq_lens=torch.from_numpy(self.seq_lens).to(device),
            block_table=torch.from_numpy(self.block_table).to(device),
            q=self.q.to(device),
            k_cache=self.k_cache.to(device),
            v_cache=self.v_cache.to(device),
        )


@dataclasses.dataclass
class DeviceWorkload:
    problem: Problem
    seq_lens: torch.Tensor
    block_table: torch.Tensor
    q: torch.Tensor
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    k_scale: torch.Tensor | None = None  # FP8 caches only
    v_scale: torch.Tensor | None = None


def _fp32(x: float) -> float:
    return float(np.float32(x))


def _randn_bf16(gen: torch.Generator, shape, row_scale: np.ndarray | None = None, chunk_pages: int = 2048):
    """N(0,1) bf16 tensor; for a KV cache shape, rows may be multiplied first (row_scale [pages, P])."""
    out = torch.empty(shape, dtype=torch.bfloat16)
    if len(shape) != 4:
        out.copy_(torch.randn(shape, generator=gen))
        return out
    n = shape[0]
    for p0 in range(0, n, chunk_pages):
        p1 = min(n, p0 + chunk_pages)
        x = torch.randn((p1 - p0,) + tuple(shape[1:]), generator=gen)
        if row_scale is not None:
            rs = torch.from_numpy(row_scale[p0:p1]).to(torch.float32)  # [pages, P]
            x.mul_(rs[:, None, :, None])
        out[p0:p1].copy_(x)
    return out


def make_workload(name: str, seq_lens, *, num_q_heads: int, num_kv_heads: int, head_dim: int, page_size: int,
                  seed: int, scale: float | None = None, rng: np.random.Generator | None = None,
                  outlier_frac: float = 0.0, outlier_mult: float = 8.0, spare_frac: float = 0.05,
                  shuffle_pages: bool = True, poison: bool = True, max_pages_per_req: int | None = None,
                  extra_pages: int = 0, recipe: str = "", q_len: int = 1) -> Workload:
    """Build a paged workload for given lengths (steps 2-5 of the module recipe)."""
    rng = rng if rng is not None else np.random.default_rng(seed)
    gen = torch.Generator().manual_seed(seed)
    lens = np.asarray(seq_lens, dtype=np.int64)
    B = lens.shape[0]
    P = page_size
    used = [(int(l) + P - 1) // P if l > 0 else 0 for l in lens]
    total_used = int(sum(used))
    num_pages = max(1, total_used + int(math.ceil(spare_frac * total_used)) + extra_pages)
    if max_pages_per_req is None:
        max_pages_per_req = max(1, max(used) if used else 1)
    assert max(used, default=0) <= max_pages_per_req
    phys = rng.permutation(num_pages).astype(np.int32) if shuffle_pages else np.arange(num_pages, dtype=np.int32)
    block_table = np.full((B, max_pages_per_req), -1, dtype=np.int32)
    o = 0
    for b in range(B):
        block_table[b, :used[b]] = phys[o:o + used[b]]
        o += used[b]

    row_scale = None
    if outlier_frac > 0:
        row_scale = np.ones((num_pages, P), dtype=np.float32)
        for b in range(B):
            L = int(lens[b])
            if L <= 0:
                continue
            hit = rng.random(L) < outlier_frac
            t = np.nonzero(hit)[0]
            row_scale[block_table[b, t // P], t % P] = outlier_mult

    scale = _fp32(1.0 / math.sqrt(head_dim)) if scale is None else _fp32(scale)
    q = _randn_bf16(gen, (B, num_q_heads, head_dim) if q_len == 1 else (B, q_len, num_q_heads, head_dim))
    shape = (num_pages, num_kv_heads, P, head_dim)
    k = _randn_bf16(gen, shape, row_scale)
    v = _randn_bf16(gen, shape)

    if poison:
        live = np.zeros((num_pages, P), dtype=bool)
        for b in range(B):
            L = int(lens[b])
            if L <= 0:
                continue
            t = np.arange(L)
            live[block_table[b, t // P], t % P] = True
        dead = torch.from_numpy(~live)
        nan = torch.tensor(BF16_NAN, dtype=torch.int16).view(torch.bfloat16)
        for cache in (k, v):
            cache.permute(0, 2, 1, 3)[dead] = nan

    problem = Problem(batch=B, num_q_heads=num_q_heads, num_kv_heads=num_kv_heads, head_dim=head_dim,
                      page_size=P, max_pages_per_req=max_pages_per_req, num_pages=num_pages, scale=scale,
                      q_len=q_len)
    return Workload(name=name, problem=problem, seq_lens=lens.astype(np.int32), block_table=block_table,
                    q=q, k_cache=k, v_cache=v, seed=seed, recipe=recipe)


# ---------------------------------------------------------------------------------------------
# FP8 (E4M3) caches.


@dataclasses.dataclass
class Fp8Workload:
    """A workload whose K/V caches are FP8 E4M3 codes with one scale per KV head.

    The cached value of KV head g is k_scale[g] * e4m3(k_code) (and likewise V).
    Quantisation recipe: scale = fp32(max |x| over the live tokens of that head /
    448), code = E4M3 rounding (torch, round-to-nearest-even) of x / scale; unused
    slots stay NaN codes.
    """
    base: Workload
    k_code: torch.Tensor  # uint8 [num_pages, Hkv, P, d]
    v_code: torch.Tensor
    k_scale: np.ndarray  # float32 [Hkv]
    v_scale: np.ndarray

    @property
    def problem(self) -> Problem:
        return self.base.problem

    @property
    def kv_bytes(self) -> int:
        """Bytes of K and V one decode step reads: sum_b L_b * Hkv * d * 2 (K,V) * 1 B."""
        p = self.problem
        return int(np.clip(self.base.seq_lens, 0, None).astype(np.int64).sum()) * p.num_kv_heads * p.head_dim * 2

    def to(self, device) -> "DeviceWorkload":
        b = self.base
        return DeviceWorkload(problem=b.problem, seq_lens=torch.from_numpy(b.seq_lens).to(device),
                              block_table=torch.from_numpy(b.block_table).to(device), q=b.q.to(device),
                              k_cache=self.k_code.to(device), v_cache=self.v_code.to(device),
                              k_scale=torch.from_numpy(self.k_scale).to(device),
                              v_scale=torch.from_numpy(self.v_scale).to(device))


def _quantize_cache(cache: torch.Tensor, chunk_pages: int = 2048):
    Hkv = cache.shape[1]
    amax = torch.zeros(Hkv, dtype=torch.float32)
    for p0 in range(0, cache.shape[0], chunk_pages):
        x = cache[p0:p0 + chunk_pages].float().abs().nan_to_num(0.0)
        amax = torch.maximum(amax, x.amax(dim=(0, 2, 3)))
    scale = (amax / 448.0).clamp_min(torch.finfo(torch.float32).tiny).numpy().astype(np.float32)
    sc = torch.from_numpy(scale)[None, :, None, None]
    code = torch.empty(cache.shape, dtype=torch.uint8)
    for p0 in range(0, cache.shape[0], chunk_pages):
        x = cache[p0:p0 + chunk_pages].float() / sc
        code[p0:p0 + chunk_pages] = x.to(torch.float8_e4m3fn).view(torch.uint8)
    return code, scale


def quantize_fp8(w: Workload) -> Fp8Workload:
    """FP8 E4M3 copy of a workload's caches (q, lengths and block table unchanged)."""
    kc, ks = _quantize_cache(w.k_cache)
    vc, vs = _quantize_cache(w.v_cache)
    return Fp8Workload(base=w, k_code=kc, v_code=vc, k_scale=ks, v_scale=vs)


# ---------------------------------------------------------------------------------------------
# The named configurations.


def tiny(seed: int = 0, **kw) -> Workload:
    """Batch 4, lengths {1,7,64,300}, 4 q heads / 1 KV head, d 64, page 16, shuffled page ids."""
    return make_workload("tiny", [1, 7, 64, 300], num_q_heads=4, num_kv_heads=1, head_dim=64, page_size=16,
                         seed=seed, scale=1.0 / 8.0, recipe="lengths {1,7,64,300}; 4q/1kv; d64; P16", **kw)


def mixed(seed: int = 1, batch: int = 32, **kw) -> Workload:
    """Batch 32, lengths uniform-int [1000, 16000], 64q/8kv, d 128, page 64."""
    rng = np.random.default_rng(seed)
    lens = rng.integers(1000, 16001, size=batch)
    return make_workload("mixed", lens, num_q_heads=64, num_kv_heads=8, head_dim=128, page_size=64, seed=seed,
                         rng=rng, recipe=f"B={batch}, L~U[1000,16000]; 64q/8kv; d128; P64", **kw)


def skewed(seed: int = 2, batch: int = 128, **kw) -> Workload:
    """Batch 128: 10 % of lengths in [16384, 65536], the rest in [256, 2048]; 1 % K rows x8."""
    rng = np.random.default_rng(seed)
    n_long = int(round(0.1 * batch))
    pos = rng.permutation(batch)[:n_long]
    long_lens = rng.integers(16384, 65537, size=n_long)
    short_lens = rng.integers(256, 2049, size=batch - n_long)
    lens = np.empty(batch, dtype=np.int64)
    is_long = np.zeros(batch, dtype=bool)
    is_long[pos] = True
    lens[pos] = long_lens
    lens[~is_long] = short_lens
    return make_workload("skewed", lens, num_q_heads=64, num_kv_heads=8, head_dim=128, page_size=64, seed=seed,
                         rng=rng, outlier_frac=0.01, outlier_mult=8.0,
                         recipe=f"B={batch}: {n_long} long U[16384,65536] at permuted positions, rest U[256,2048];"
                                " 1% K rows x8; 64q/8kv; d128; P64", **kw)


def low_conc(seed: int = 3, **kw) -> Workload:
    """Batch 2, lengths {131072, 1000}, 64q/8kv, d 128, page 64."""
    return make_workload("low_conc", [131072, 1000], num_q_heads=64, num_kv_heads=8, head_dim=128, page_size=64,
                         seed=seed, recipe="lengths {131072, 1000}; 64q/8kv; d128; P64", **kw)


def uniform(seed: int = 5, batch: int = 64, length: int = 4096, **kw) -> Workload:
    """Control: every request the same length (little imbalance to fix)."""
    return make_workload("uniform", [length] * batch, num_q_heads=64, num_kv_heads=8, head_dim=128, page_size=64,
                         seed=seed, recipe=f"B={batch}, L={length}; 64q/8kv; d128; P64", **kw)


CONFIGS = {"tiny": tiny, "mixed": mixed, "skewed": skewed, "low_conc": low_conc, "uniform": uniform}


# ---------------------------------------------------------------------------------------------
# The decode trace: a continuous batch evolving over many steps.


class DecodeTrace:
    """Continuous-batch decode trace: B request slots stepping together.

    Start: lengths lognormal(ln median, sigma) rounded and clipped to
    [1, max_len]; pages as in the module recipe, from a host free list (LIFO)
    of a pool with room to grow.  Step 0 decodes the starting batch.  Before
    each later step, in this order: every slot finishes with probability
    p_finish (its pages go back to the free list and a new request of length
    uniform in new_len takes the slot, with fresh N(0,1) K/V); then every slot
    grows by one token (a fresh N(0,1) K/V row at position L, a new page when
    L % P == 0); then a fresh q ~ N(0,1) is drawn.  The host keeps the whole
    cache (the CPU oracle reads it); `advance()` returns what the device copy
    needs to follow.
    """

    def __init__(self, seed: int = 4, batch: int = 256, steps: int = 256, num_q_heads: int = 32,
                 num_kv_heads: int = 4, head_dim: int = 128, page_size: int = 64, median: float = 4096.0,
                 sigma: float = 1.0, max_len: int = 32768, p_finish: float = 0.01, new_len=(500, 2000),
                 spare_pages: int | None = None):
        self.rng = np.random.default_rng(seed)
        self.gen = torch.Generator().manual_seed(seed)
        self.seed, self.steps, self.p_finish, self.new_len = seed, steps, p_finish, new_len
        P = page_size
        lens = np.clip(np.round(self.rng.lognormal(math.log(median), sigma, batch)), 1, max_len).astype(np.int64)
        self.max_pages = -(-(max_len + steps) // P)
        used = int(sum(-(-int(l) // P) for l in lens))
        spare = spare_pages if spare_pages is not None else batch * (-(-steps // P) + 2) + used // 4
        num_pages = used + spare
        self.problem = Problem(batch=batch, num_q_heads=num_q_heads, num_kv_heads=num_kv_heads,
                               head_dim=head_dim, page_size=P, max_pages_per_req=self.max_pages,
                               num_pages=num_pages, scale=_fp32(1.0 / math.sqrt(head_dim)))
        # free list: a random permutation of the pool, taken from the end
        self.free = list(self.rng.permutation(num_pages).astype(np.int64))
        self.block_table = np.full((batch, self.max_pages), -1, dtype=np.int32)
        self.lens = np.zeros(batch, dtype=np.int64)
        shape = (num_pages, num_kv_heads, P, head_dim)
        self.k_cache = torch.full(shape, float("nan"), dtype=torch.bfloat16)  # unused pages stay NaN
        self.v_cache = torch.full(shape, float("nan"), dtype=torch.bfloat16)
        for b in range(batch):
            self._start_request(b, int(lens[b]))
        self.q = _randn_bf16(self.gen, (batch, num_q_heads, head_dim))
        self.step = 0
        self.recipe = (f"B={batch}, L0~lognormal(ln {median:g}, {sigma:g}) clipped [1,{max_len}], {steps} steps: "
                       f"+1 token/step, finish p={p_finish} -> new U[{new_len[0]},{new_len[1]}]; "
                       f"{num_q_heads}q/{num_kv_heads}kv; d{head_dim}; P{P}")

    # -- host-side state changes
    def _take_page(self) -> int:
        if not self.free:
            raise RuntimeError("trace page pool exhausted")
        return int(self.free.pop())

    def _start_request(self, b: int, L: int) -> list[int]:
        P = self.problem.page_size
        n = -(-L // P)
        pages = [self._take_page() for _ in range(n)]
        self.block_table[b, :] = -1
        self.block_table[b, :n] = pages
        self.lens[b] = L
        idx = torch.tensor(pages, dtype=torch.long)
        sub = (n, self.problem.num_kv_heads, P, self.problem.head_dim)
        self.k_cache[idx] = _randn_bf16(self.gen, sub)
        self.v_cache[idx] = _randn_bf16(self.gen, sub)
        return pages

    def _finish_request(self, b: int):
        n = -(-int(self.lens[b]) // self.problem.page_size)
        self.free.extend(int(x) for x in self.block_table[b, :n][::-1])
        self.block_table[b, :] = -1
        self.lens[b] = 0

    def advance(self) -> dict:
        """Move to the next step; returns the changes: restarted slots and their pages, the
        appended K/V rows ([B, Hkv, d] bf16, at position lens-1), the new q."""
        p = self.problem
        B, P = p.batch, p.page_size
        finish = self.rng.random(B) < self.p_finish
        restarted, new_pages = [], []
        for b in np.nonzero(finish)[0]:
            self._finish_request(int(b))
            L = int(self.rng.integers(self.new_len[0], self.new_len[1] + 1))
            new_pages += self._start_request(int(b), L)
            restarted.append(int(b))
        new_k = _randn_bf16(self.gen, (B, p.num_kv_heads, p.head_dim))
        new_v = _randn_bf16(self.gen, (B, p.num_kv_heads, p.head_dim))
        for b in range(B):
            L = int(self.lens[b])
            if L % P == 0:
                self.block_table[b, L // P] = self._take_page()
            page = int(self.block_table[b, L // P])
            self.k_cache[page, :, L % P, :] = new_k[b]
            self.v_cache[page, :, L % P, :] = new_v[b]
            self.lens[b] = L + 1
        self.q = _randn_bf16(self.gen, (B, p.num_q_heads, p.head_dim))
        self.step += 1
        return dict(restarted=restarted, restarted_pages=new_pages, new_k=new_k, new_v=new_v, q=self.q)

    # -- views
    @property
    def seq_lens(self) -> np.ndarray:
        return self.lens.astype(np.int32)

    def workload(self) -> Workload:
        """The current state as a Workload (host tensors shared, not copied)."""
        prob = dataclasses.replace(self.problem)
        return Workload(name=f"trace@{self.step}", problem=prob, seq_lens=self.seq_lens,
                        block_table=self.block_table.copy(), q=self.q, k_cache=self.k_cache,
                        v_cache=self.v_cache, seed=self.seed, recipe=self.recipe)

    def kv_bytes(self) -> int:
        p = self.problem
        return int(self.lens.sum()) * p.num_kv_heads * p.head_dim * 4
