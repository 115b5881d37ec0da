"""Seeded synthetic inputs for the paged decode workloads.

Both sides of every comparison draw their inputs here: the CUDA path (through the
C-ABI library) and the CPU oracle.  This module only draws random numbers, rounds
them to the storage dtype and states the workload shapes.  It holds none of the
paged-attention arithmetic: no slot mapping, no block-table walk, no softmax and no
block allocation.  Each side builds its own block tables from the lengths and the
free-block order drawn here.

Storage dtypes are "f32", "bf16" and "f16".  bf16 values are carried in numpy as
their uint16 bit patterns (numpy has no bfloat16); f16 uses numpy.float16.

Every array comes from numpy's PCG64 generator keyed by ``(seed, stream, chunk)``,
so a value depends only on the seed and its position, never on the thread count.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

DTYPES = ("f32", "bf16", "f16")
STORAGE_NP = {"f32": np.float32, "bf16": np.uint16, "f16": np.float16}
ELEM_BYTES = {"f32": 4, "bf16": 2, "f16": 2}

# stream ids: one independent random stream per kind of input
_S_LENS, _S_ORDER, _S_KPOOL, _S_VPOOL, _S_Q, _S_NEWK, _S_NEWV, _S_PRIV = range(8)
_CHUNK = 1 << 22  # values per independently keyed chunk of a large array


def round_to_storage(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float32 values to the storage dtype with round-to-nearest-even.

    bf16: the upper 16 bits of the float32 pattern after adding 0x7FFF plus the
    lowest kept bit (ties to even).  Inputs here are finite normal draws.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "f32":
        return x
    if dtype == "f16":
        return x.astype(np.float16)
    if dtype == "bf16":
        u = x.view(np.uint32)
        lsb = np.right_shift(u, 16) & np.uint32(1)
        return np.right_shift(u + np.uint32(0x7FFF) + lsb, 16).astype(np.uint16)
    raise ValueError(f"unknown dtype {dtype!r}")


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def normal_fill(shape, dtype: str, std: float, seed: int, stream: int) -> np.ndarray:
    """N(0, std^2) draws of the given shape, rounded to ``dtype`` storage.

    Large arrays are filled in fixed chunks of 2^22 values, each from its own
    generator keyed by (seed, stream, chunk index), on a thread pool; numpy
    releases the GIL while filling, and the result does not depend on the pool.
    """
    n = int(np.prod(shape)) if len(shape) else 1
    out = np.empty(n, dtype=STORAGE_NP[dtype])
    nchunks = max(1, (n + _CHUNK - 1) // _CHUNK)

    def work(c: int) -> None:
        lo, hi = c * _CHUNK, min(n, (c + 1) * _CHUNK)
        g = np.random.default_rng([seed, stream, c])
        x = g.standard_normal(hi - lo, dtype=np.float32)
        if std != 1.0:
            x *= np.float32(std)
        out[lo:hi] = round_to_storage(x, dtype)

    if nchunks == 1:
        work(0)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(work, range(nchunks)))
    return out.reshape(shape)


@dataclass(frozen=True)
class DecodeConfig:
    """Shape and value distribution of one synthetic decode workload (one layer).

    ``lens`` says how the per-sequence cached lengths are drawn (including the
    token written by the decode step itself):
      ("fixed", (l0, l1, ...))          the given lengths
      ("uniform", lo, hi)               integers uniform on [lo, hi]
      ("lognormal", median, sigma, lo, hi)  rint(exp(ln median + sigma*z)), clipped
      ("prefix", groups, samples, prefix_len, private_max)
                                        shared-prefix groups; see ``prefix_layout``
    """

    name: str
    num_seqs: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    dtype: str
    scale: float
    std: float
    lens: tuple
    partition_size: int = 512     # 0: the library's choice for the batch
    description: str = ""

    @property
    def group(self) -> int:
        return self.num_heads // self.num_kv_heads

    @property
    def elem_bytes(self) -> int:
        return ELEM_BYTES[self.dtype]

    def with_(self, **kw) -> "DecodeConfig":
        d = {k: getattr(self, k) for k in self.__dataclass_fields__}
        d.update(kw)
        return DecodeConfig(**d)


CONFIGS: dict[str, DecodeConfig] = {
    "tiny_fp32": DecodeConfig(
        name="tiny_fp32", num_seqs=5, num_heads=4, num_kv_heads=4, head_dim=64,
        block_size=4, num_blocks=32, dtype="f32", scale=1.0 / 8.0, std=1.0,
        lens=("fixed", (5, 13, 7, 18, 10)),
        description="tiny fp32 paged decode: lengths 5,13,7,18,10; block 4; 4 heads; "
                    "head_dim 64; 32-block pool in seeded order; N(0,1); scale 1/8"),
    "7b_bf16": DecodeConfig(
        name="7b_bf16", num_seqs=64, num_heads=32, num_kv_heads=32, head_dim=128,
        block_size=16, num_blocks=8192, dtype="bf16", scale=1.0 / math.sqrt(128.0), std=1.0,
        lens=("uniform", 128, 2048), partition_size=0,
        description="7B-shaped decode, one layer: 32 q = 32 kv heads, head_dim 128, bf16, "
                    "block 16, batch 64, lengths U[128,2048], 8192-block pool"),
    "13b_fp16": DecodeConfig(
        name="13b_fp16", num_seqs=256, num_heads=40, num_kv_heads=40, head_dim=128,
        block_size=16, num_blocks=16384, dtype="f16", scale=1.0 / math.sqrt(128.0), std=1.0,
        lens=("lognormal", 512.0, 1.0, 16, 4096), partition_size=0,
        description="13B-shaped decode, one layer: 40 heads, head_dim 128, fp16, block 16, "
                    "batch 256, lengths lognormal(median 512, sigma 1) clipped to [16,4096]"),
    "gqa_long_bf16": DecodeConfig(
        name="gqa_long_bf16", num_seqs=8, num_heads=64, num_kv_heads=8, head_dim=128,
        block_size=16, num_blocks=65536, dtype="bf16", scale=1.0 / math.sqrt(128.0), std=0.5,
        lens=("uniform", 32768, 131072), partition_size=512,
        description="GQA long-context decode: 64 q / 8 kv heads, head_dim 128, bf16, block 16, "
                    "batch 8, lengths U[32768,131072], 512-token partitions, N(0,0.5^2)"),
    "prefix_cow_bf16": DecodeConfig(
        name="prefix_cow_bf16", num_seqs=256, num_heads=32, num_kv_heads=32, head_dim=128,
        block_size=16, num_blocks=8192, dtype="bf16", scale=1.0 / math.sqrt(128.0), std=1.0,
        lens=("prefix", 32, 8, 1030, 256),
        description="prefix sharing + COW: 32 groups x 8 samples share a 1030-token prefix; "
                    "0..256 private tokens each; 32 heads, head_dim 128, bf16, block 16"),
}

# The config the benchmark's headline number is quoted on.
HEADLINE = "7b_bf16"


@dataclass
class PrefixLayout:
    """Per-sequence prefix/private split for the shared-prefix workload."""

    groups: int
    samples: int
    prefix_len: int
    private_lens: np.ndarray  # int64 [groups*samples]


@dataclass
class DecodeInputs:
    """Everything one decode workload needs, as host arrays in storage dtype.

    ``context_lens[s]`` tokens are cached before the step; the step appends one
    token per sequence (K/V in ``new_k``/``new_v``) and attends with ``q``.  For
    the shared-prefix workload ``prefix`` says how the context was built.
    """

    cfg: DecodeConfig
    seed: int
    context_lens: np.ndarray          # int64 [S]
    free_order: np.ndarray            # int32 [NB], a permutation of the pool
    k_pool: np.ndarray                # [NB, Hkv, bs, D] storage dtype
    v_pool: np.ndarray                # [NB, Hkv, bs, D]
    q: np.ndarray                     # [S, Hq, D]
    new_k: np.ndarray                 # [S, Hkv, D]
    new_v: np.ndarray                 # [S, Hkv, D]
    prefix: PrefixLayout | None = None
    extra: dict = field(default_factory=dict)


def draw_lengths(cfg: DecodeConfig, seed: int) -> tuple[np.ndarray, PrefixLayout | None]:
    """Per-sequence cached lengths after the decode step (context + 1)."""
    g = np.random.default_rng([seed, _S_LENS])
    kind = cfg.lens[0]
    if kind == "fixed":
        lens = np.asarray(cfg.lens[1], dtype=np.int64)
        assert lens.size == cfg.num_seqs
        return lens, None
    if kind == "uniform":
        lo, hi = cfg.lens[1], cfg.lens[2]
        return g.integers(lo, hi, size=cfg.num_seqs, endpoint=True).astype(np.int64), None
    if kind == "lognormal":
        median, sigma, lo, hi = cfg.lens[1:]
        z = g.standard_normal(cfg.num_seqs)
        lens = np.rint(np.exp(math.log(median) + sigma * z))
        return np.clip(lens, lo, hi).astype(np.int64), None
    if kind == "prefix":
        groups, samples, prefix_len, private_max = cfg.lens[1:]
        assert groups * samples == cfg.num_seqs
        gp = np.random.default_rng([seed, _S_PRIV])
        priv = gp.integers(0, private_max, size=cfg.num_seqs, endpoint=True).astype(np.int64)
        layout = PrefixLayout(groups, samples, prefix_len, priv)
        return prefix_len + priv + 1, layout
    raise ValueError(kind)


def fork_step_layout(cfg: DecodeConfig) -> PrefixLayout:
    """Shared-prefix variant in which no sample has a private token yet."""
    groups, samples, prefix_len, _ = cfg.lens[1:]
    return PrefixLayout(groups, samples, prefix_len, np.zeros(groups * samples, np.int64))


def make_inputs(cfg: DecodeConfig, seed: int = 0, *, fork_step: bool = False,
                pool: bool = True) -> DecodeInputs:
    """Draw one workload.  ``pool=False`` skips the (large) K/V pool fill."""
    lens, prefix = draw_lengths(cfg, seed)
    if fork_step:
        prefix = fork_step_layout(cfg)
        lens = prefix.prefix_len + prefix.private_lens + 1
    order = np.random.default_rng([seed, _S_ORDER]).permutation(cfg.num_blocks).astype(np.int32)
    S, Hq, Hkv, D, bs, NB = (cfg.num_seqs, cfg.num_heads, cfg.num_kv_heads, cfg.head_dim,
                             cfg.block_size, cfg.num_blocks)
    if pool:
        k_pool = normal_fill((NB, Hkv, bs, D), cfg.dtype, cfg.std, seed, _S_KPOOL)
        v_pool = normal_fill((NB, Hkv, bs, D), cfg.dtype, cfg.std, seed, _S_VPOOL)
    else:
        k_pool = v_pool = np.empty((0, Hkv, bs, D), STORAGE_NP[cfg.dtype])
    q = normal_fill((S, Hq, D), cfg.dtype, cfg.std, seed, _S_Q)
    new_k = normal_fill((S, Hkv, D), cfg.dtype, cfg.std, seed, _S_NEWK)
    new_v = normal_fill((S, Hkv, D), cfg.dtype, cfg.std, seed, _S_NEWV)
    return DecodeInputs(cfg=cfg, seed=seed, context_lens=lens - 1, free_order=order,
                        k_pool=k_pool, v_pool=v_pool, q=q, new_k=new_k, new_v=new_v,
                        prefix=prefix)


def device_normal_fill(shape, dtype: str, std: float, seed: int, stream: int, device):
    """N(0, std^2) draws made on a CUDA device by torch's generator keyed by (seed,
    stream), rounded to ``dtype`` (a torch tensor).  Same distribution as
    ``normal_fill`` but not the same values: for throughput runs of large pools,
    where drawing gigabytes on the host would dominate the run and the values only
    need the workload's distribution."""
    t = _torch()
    g = t.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + stream) & ((1 << 63) - 1))
    out = t.empty(shape, dtype=TORCH_DTYPES[dtype], device=device)
    flat = out.view(-1)
    step = 1 << 28                      # bounded float32 scratch per chunk
    for lo in range(0, flat.numel(), step):
        n = min(step, flat.numel() - lo)
        x = t.randn(n, generator=g, device=device, dtype=t.float32)
        if std != 1.0:
            x.mul_(std)
        flat[lo:lo + n].copy_(x)
        del x
    return out


def step_tokens(cfg: DecodeConfig, seed: int, step: int):
    """q / new K / new V for decode step ``step`` (>= 1) of a multi-step run."""
    S, Hq, Hkv, D = cfg.num_seqs, cfg.num_heads, cfg.num_kv_heads, cfg.head_dim
    base = 16 + 3 * step
    q = normal_fill((S, Hq, D), cfg.dtype, cfg.std, seed, base)
    nk = normal_fill((S, Hkv, D), cfg.dtype, cfg.std, seed, base + 1)
    nv = normal_fill((S, Hkv, D), cfg.dtype, cfg.std, seed, base + 2)
    return q, nk, nv


# ---------------------------------------------------------------------------
# torch views of storage arrays (device placement is the caller's business)
# ---------------------------------------------------------------------------

def _torch():
    import torch
    return torch


class _TorchDtypes(dict):
    def __missing__(self, key):
        t = _torch()
        self.update({"f32": t.float32, "bf16": t.bfloat16, "f16": t.float16})
        return dict.__getitem__(self, key)


TORCH_DTYPES = _TorchDtypes()


def storage_to_torch(a: np.ndarray, dtype: str):
    """A CPU torch tensor sharing the bits of a storage array (bf16 from uint16)."""
    t = _torch()
    a = np.ascontiguousarray(a)
    if dtype == "bf16":
        return t.from_numpy(a.view(np.int16)).view(t.bfloat16)
    return t.from_numpy(a)
