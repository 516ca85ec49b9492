"""Seeded synthetic workloads for the paged KV-cache decode path.

This module only *generates inputs*: context lengths, the random placement of
each sequence's blocks in the physical pool, and N(0,1) query / cache / new-token
values rounded to fp16 or bf16. It holds none of the arithmetic of the method
(no attention, no cache write, no block copy, no allocator rules). Both the CUDA
path and the CPU oracle are fed from here, so neither depends on the other.

Workload shapes follow the serving workloads described for vLLM /
PagedAttention ("vLLM / PagedAttention — 分页 KV Cache 分析", §3.1 table: page
size 16 tokens; "vLLM" entity page, 是什么: on-demand blocks, refcount sharing
for parallel sampling). The pages name ShareGPT / Alpaca only as workload
names; no dataset is used: lognormal / uniform synthetic lengths stand in.

Draw order for one seed (numpy ``default_rng(seed)``):
  1. context lengths, 2. block-placement permutation, 3. q, 4. cache contents
  (K then V, whole pool; rows that no sequence has written get a NaN canary),
  5. k_new, v_new.
Large workloads draw 3-5 on the GPU with ``torch.Generator(device="cuda")``
seeded with the same seed (a different stream than numpy, stated in the
workload's ``values_on`` field). Lengths and placement always come from numpy.

Lengths are *post-write* lengths: ``context_lens[s]`` counts every token the
decode step attends to, including the token that this step writes at logical
position ``len-1``. History tokens ``[0, len-1)`` hold values; the slot of
position ``len-1`` holds the canary until ``reshape_and_cache`` writes it.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

F16 = 0
BF16 = 1
DTYPE_NAMES = {F16: "f16", BF16: "bf16"}

# NaN canary bit patterns for slots that were never written.
CANARY = {F16: 0x7E00, BF16: 0x7FC0}


# ----------------------------------------------------------------------------
# rounding of generated fp32 draws to the storage dtype (input generation only)
# ----------------------------------------------------------------------------
def round_to_bits(x: np.ndarray, dtype: int) -> np.ndarray:
    """Round float32 draws to fp16 / bf16 with round-to-nearest-even; uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == F16:
        return x.astype(np.float16).view(np.uint16)
    u = x.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    r[np.isnan(x)] = CANARY[BF16]
    return r


# ----------------------------------------------------------------------------
# workload specs
# ----------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class Spec:
    name: str
    seed: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    dtype: int
    num_layers: int
    lens: tuple = ()              # explicit post-write lengths (tiny)
    dist: tuple = ()              # ("lognormal", median, sigma, lo, hi) | ("uniform", lo, hi)
    batch: int = 0
    pool_blocks: int = 0          # explicit pool size (tiny), else pool_factor * need
    pool_factor: float = 1.2
    pool_extra: int = 0           # blocks added to the pool (room for tokens appended later)
    max_len: int = 0              # length bound used for max_blocks_per_seq
    prompts: int = 0              # shared prefix: prompts x samples
    samples: int = 0
    prefix: int = 0
    suffix_max: int = 0


SPECS = {
    # 1 layer, lengths {7,16,33,100}, MHA 8/8, d 64, bs 16, fp16, 64-block pool.
    "tiny": Spec("tiny", 1, 8, 8, 64, 16, F16, 1, lens=(7, 16, 33, 100),
                 pool_blocks=64, max_len=128),
    # Llama-7B shaped MHA decode: B 64, 32/32 heads, d 128, fp16, 32 layers.
    "llama7b_mha": Spec("llama7b_mha", 2, 32, 32, 128, 16, F16, 32,
                        dist=("lognormal", 512, 1.0, 16, 2048), batch=64, max_len=2048),
    # Llama-3-8B shaped GQA decode: B 256, 32q/8kv, d 128, bf16, 1 layer.
    "llama3_8b_gqa": Spec("llama3_8b_gqa", 3, 32, 8, 128, 16, BF16, 1,
                          dist=("lognormal", 1024, 1.0, 8, 8192), batch=256, max_len=8192),
    # Shared-prefix parallel sampling: 16 prompts x 8 samples, prefix 1024.
    "shared_prefix": Spec("shared_prefix", 4, 32, 8, 128, 16, BF16, 1,
                          prompts=16, samples=8, prefix=1024, suffix_max=256,
                          max_len=1024 + 256 + 1),
    # Long-context decode: B 8, U[32768, 131072], 64q/8kv, d 128, bf16.
    "long_context": Spec("long_context", 5, 64, 8, 128, 16, BF16, 1,
                         dist=("uniform", 32768, 131072), batch=8, max_len=131072),
}


def spec(name: str, **overrides) -> Spec:
    return dataclasses.replace(SPECS[name], **overrides)


def draw_lengths(sp: Spec, rng: np.random.Generator) -> np.ndarray:
    if sp.lens:
        return np.array(sp.lens, dtype=np.int32)
    if sp.prompts:
        u = rng.integers(0, sp.suffix_max + 1, size=sp.prompts * sp.samples)
        return (sp.prefix + u + 1).astype(np.int32)
    kind = sp.dist[0]
    if kind == "lognormal":
        _, median, sigma, lo, hi = sp.dist
        x = rng.lognormal(math.log(median), sigma, size=sp.batch)
        return np.clip(np.rint(x), lo, hi).astype(np.int32)
    if kind == "uniform":
        _, lo, hi = sp.dist
        return rng.integers(lo, hi + 1, size=sp.batch).astype(np.int32)
    raise ValueError(kind)


def cdiv(a, b):
    return -(-a // b)


# ----------------------------------------------------------------------------
# the synthetic state
# ----------------------------------------------------------------------------
@dataclasses.dataclass
class Workload:
    spec: Spec
    context_lens: np.ndarray      # int32 [B], post-write lengths
    perm: np.ndarray              # int32 [NB], placement order of physical blocks
    block_tables: np.ndarray      # int32 [B, MB], -1 padded
    slot_mapping: np.ndarray      # int64 [B], slot of this step's token (position len-1)
    written_rows: np.ndarray      # int32 [NB], rows [0, n) of each block hold history
    num_blocks: int
    max_blocks_per_seq: int
    values_on: str                # "numpy" | "cuda"
    q: object = None              # [L, B, Hq, d]
    k_cache: object = None        # [L, NB, Hkv, bs, d]
    v_cache: object = None
    k_new: object = None          # [L, B, Hkv, d]
    v_new: object = None

    @property
    def num_seqs(self):
        return int(self.context_lens.shape[0])

    @property
    def scale(self):
        return 1.0 / math.sqrt(self.spec.head_dim)

    def kv_bytes(self) -> int:
        """Algorithmic K+V bytes one decode step reads in one layer."""
        s = self.spec
        return int(self.context_lens.astype(np.int64).sum()) * s.num_kv_heads * s.head_dim * 2 * 2


def _placement(sp: Spec, lens: np.ndarray, rng: np.random.Generator):
    """Block tables built by handing out a seeded permutation of the pool in order.

    Sequence s takes the next ceil(len_s / bs) entries of the permutation. Shared
    prefix: per prompt, the prefix's blocks are handed out once (every sample of the
    prompt points at them), then each sample's private suffix blocks in sample order."""
    bs = sp.block_size
    mb = cdiv(sp.max_len, bs)
    if sp.prompts:
        pre_blocks = sp.prefix // bs
        own = [cdiv(int(n) - sp.prefix, bs) for n in lens]
        need = sp.prompts * pre_blocks + sum(own)
    else:
        need = int(sum(cdiv(int(n), bs) for n in lens))
    nb = (sp.pool_blocks or int(math.ceil(sp.pool_factor * need))) + sp.pool_extra
    perm = rng.permutation(nb).astype(np.int32)
    bt = np.full((len(lens), mb), -1, dtype=np.int32)
    off = 0
    if sp.prompts:
        # per prompt: its prefix blocks, then each of its samples' private blocks
        for p in range(sp.prompts):
            prefix_ids = perm[off:off + pre_blocks]
            off += pre_blocks
            for i in range(p * sp.samples, (p + 1) * sp.samples):
                bt[i, :pre_blocks] = prefix_ids
                k = own[i]
                bt[i, pre_blocks:pre_blocks + k] = perm[off:off + k]
                off += k
    else:
        for i, n in enumerate(lens):
            k = cdiv(int(n), bs)
            bt[i, :k] = perm[off:off + k]
            off += k
    # rows written before the step: history positions [0, len-1)
    written = np.zeros(nb, dtype=np.int32)
    for i, n in enumerate(lens):
        hist = int(n) - 1
        for j in range(cdiv(int(n), bs)):
            b = bt[i, j]
            written[b] = max(written[b], min(bs, max(0, hist - j * bs)))
    last = np.maximum(lens.astype(np.int64) - 1, 0)
    slots = np.where(
        lens > 0,
        bt[np.arange(len(lens)), last // bs].astype(np.int64) * bs + last % bs,
        -1,
    ).astype(np.int64)
    return perm, bt, slots, written, nb, mb


def make_workload(name: str, values_on: str = "numpy", num_layers: Optional[int] = None,
                  device: str = "cuda", **overrides) -> Workload:
    """Build the seeded workload ``name`` (a key of SPECS) with optional overrides.

    values_on="numpy": all values as uint16 bit arrays (small workloads).
    values_on="cuda":  values as torch tensors on ``device`` drawn from a seeded
                       CUDA generator (large workloads); dtype torch.float16/bfloat16.
    values_on="none":  lengths and placement only.
    """
    sp = spec(name, **overrides)
    if num_layers is not None:
        sp = dataclasses.replace(sp, num_layers=num_layers)
    rng = np.random.default_rng(sp.seed)
    lens = draw_lengths(sp, rng)
    perm, bt, slots, written, nb, mb = _placement(sp, lens, rng)
    wl = Workload(sp, lens, perm, bt, slots, written, nb, mb, values_on)
    if values_on == "numpy":
        _values_numpy(wl, rng)
    elif values_on == "cuda":
        _values_torch(wl, device)
    return wl


def _canary_rows_mask(wl: Workload) -> np.ndarray:
    bs = wl.spec.block_size
    return np.arange(bs)[None, :] >= wl.written_rows[:, None]      # [NB, bs] True = canary


def _values_numpy(wl: Workload, rng: np.random.Generator):
    sp = wl.spec
    L, B, Hq, Hkv, d, bs = sp.num_layers, wl.num_seqs, sp.num_heads, sp.num_kv_heads, sp.head_dim, sp.block_size
    nb = wl.num_blocks

    def draw(shape):
        return round_to_bits(rng.standard_normal(shape, dtype=np.float32), sp.dtype)

    wl.q = draw((L, B, Hq, d))
    mask = _canary_rows_mask(wl)
    caches = []
    for _ in range(2):
        c = draw((L, nb, Hkv, bs, d))
        c.transpose(0, 1, 3, 2, 4)[:, mask] = CANARY[sp.dtype]
        caches.append(c)
    wl.k_cache, wl.v_cache = caches
    wl.k_new = draw((L, B, Hkv, d))
    wl.v_new = draw((L, B, Hkv, d))


def torch_dtype(dtype: int):
    import torch
    return torch.float16 if dtype == F16 else torch.bfloat16


def _values_torch(wl: Workload, device: str):
    import torch
    sp = wl.spec
    L, B, Hq, Hkv, d, bs = sp.num_layers, wl.num_seqs, sp.num_heads, sp.num_kv_heads, sp.head_dim, sp.block_size
    nb = wl.num_blocks
    td = torch_dtype(sp.dtype)
    gen = torch.Generator(device=device)
    gen.manual_seed(sp.seed)

    def draw(shape):
        out = torch.empty(shape, dtype=td, device=device)
        flat = out.view(-1)
        chunk = 1 << 26
        for i in range(0, flat.numel(), chunk):
            n = min(chunk, flat.numel() - i)
            flat[i:i + n] = torch.randn(n, generator=gen, device=device, dtype=torch.float32).to(td)
        return out

    wl.q = draw((L, B, Hq, d))
    mask = torch.from_numpy(_canary_rows_mask(wl)).to(device)         # [NB, bs]
    canary = CANARY[sp.dtype]          # < 0x8000, fits an int16 fill value
    k_layers, v_layers = [], []
    for which in (k_layers, v_layers):
        for _ in range(L):
            c = draw((nb, Hkv, bs, d))
            cv = c.view(torch.int16)
            cv.masked_fill_(mask[:, None, :, None], canary)
            which.append(c)
    wl.k_cache, wl.v_cache = k_layers, v_layers
    wl.k_new = draw((L, B, Hkv, d))
    wl.v_new = draw((L, B, Hkv, d))


def sample_sequences(wl: Workload, n: int, seed: int = 0) -> np.ndarray:
    """Indices of n sequences to check at full size: the longest, the shortest and
    a seeded random remainder (never derived from any output)."""
    B = wl.num_seqs
    if n >= B:
        return np.arange(B)
    order = np.argsort(wl.context_lens, kind="stable")
    pick = {int(order[-1]), int(order[0])}
    rng = np.random.default_rng(1000 + seed)
    for s in rng.permutation(B):
        if len(pick) >= n:
            break
        pick.add(int(s))
    return np.array(sorted(pick))


# ----------------------------------------------------------------------------
# copy-on-write step of the shared-prefix workload
# ----------------------------------------------------------------------------
@dataclasses.dataclass
class CowStep:
    """Inputs of one parallel-sampling step whose last prefix block is shared.

    Each of ``prompts`` parents has ``parent_lens[p] = prefix + u_p`` tokens,
    u_p uniform in [1, 255] and not a multiple of 16, so its last block is partly
    filled; it is forked into ``samples`` sequences and every sample then appends
    one token. Which blocks hold what is decided by the block manager under test
    (seeded with ``initial_order``); the values here are the whole pool's contents."""
    spec: Spec
    parent_lens: np.ndarray
    initial_order: np.ndarray
    num_blocks: int
    max_blocks_per_seq: int
    num_layers: int
    q: np.ndarray            # [B, Hq, d] bits
    k_cache: np.ndarray      # [L, NB, Hkv, bs, d] bits (every row a value; the test masks)
    v_cache: np.ndarray
    k_new: np.ndarray        # [B, Hkv, d] bits
    v_new: np.ndarray


def make_cow_step(num_layers: int = 2, seed: Optional[int] = None) -> CowStep:
    sp = SPECS["shared_prefix"]
    rng = np.random.default_rng(sp.seed if seed is None else seed)
    bs = sp.block_size
    choices = np.array([u for u in range(1, 256) if u % bs != 0])
    u = rng.choice(choices, size=sp.prompts)
    parent_lens = (sp.prefix + u).astype(np.int32)
    need = int(sum(cdiv(int(n), bs) for n in parent_lens)) + sp.prompts * (sp.samples - 1)
    nb = int(math.ceil(sp.pool_factor * need))
    order = rng.permutation(nb).astype(np.int32)
    B = sp.prompts * sp.samples

    def draw(shape):
        return round_to_bits(rng.standard_normal(shape, dtype=np.float32), sp.dtype)

    q = draw((B, sp.num_heads, sp.head_dim))
    kc = draw((num_layers, nb, sp.num_kv_heads, bs, sp.head_dim))
    vc = draw((num_layers, nb, sp.num_kv_heads, bs, sp.head_dim))
    kn = draw((B, sp.num_kv_heads, sp.head_dim))
    vn = draw((B, sp.num_kv_heads, sp.head_dim))
    return CowStep(sp, parent_lens, order, nb, cdiv(sp.max_len, bs), num_layers, q, kc, vc, kn, vn)
