"""Seeded synthetic workloads for the paged KV-cache decode path.

This module builds the inputs that both the CUDA library and the CPU oracle
consume, and nothing else: sequence lengths, a shuffled free list of physical
blocks, per-sequence block tables, the values of q / K / V, and the slot of the
one new token each sequence appends in a decode step.  It holds none of the
method's arithmetic (no scatter, no gather, no attention); those live in the
CUDA library and, independently, in the oracle.

Structure (lengths, permutations) is drawn on the CPU from a
``torch.Generator`` seeded with ``seed``, so it is identical on every device.
Values are drawn i.i.d. N(0, 1) in fp32 from a generator on the target device
seeded with ``seed + 1`` and cast to the storage dtype with round-to-nearest-
even.  The oracle never regenerates values: it reads back these tensors.

Block allocation follows the pages' description of PagedAttention: the KV cache
is cut into fixed-size 16-token blocks that need not be contiguous, a block
table maps a sequence's logical positions to physical blocks, blocks are handed
out from a free list as a sequence grows (no max-length reservation), identical
prompt prefixes point at the same physical blocks, and a shared block that a
sequence must write into is copied first (copy-on-write).  Sources:
"Was ändert PagedAttention an der KV-Speicherzuweisung für LLMs?"
(slavadubrov.com), introduction and §"Gemeinsame Nutzung erfordert mehr als
Speicherzuweisung"; "PagedAttention et vLLM" (aiunderstanding.org),
§"Plongée profonde"; "Внутреннее устройство vLLM" (artificials.ru), paragraph
on the KV-cache manager (16-token blocks).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional, Sequence

import numpy as np
import torch

BLOCK_SIZE = 16
PAD_BLOCK = -1  # table entries past a sequence's last block

# name -> description of the five synthetic workloads
CONFIGS = {
    "tiny": dict(
        desc="4 seqs, lens {35,1,16,17}, Hq=2 over Hkv=1, D=64, fp32, 16-block pool, "
        "permuted tables, scale 1/sqrt(64)",
    ),
    "mha": dict(
        desc="64 seqs, L~U{128..2048}, Hq=Hkv=32, D=128, bf16, pool 1.25x needed "
        "(shuffled free list), cache write of 64 new tokens then one decode step",
    ),
    "gqa": dict(
        desc="256 seqs, L=round(exp(N(ln 1024, 0.8^2))) clipped to [16,8192], Hq=32 over "
        "Hkv=8, D=128, bf16, permuted blocks",
    ),
    "prefix": dict(
        desc="128 seqs sharing one 4096-token prefix (256 shared blocks) plus private "
        "suffixes L_suf~U{64..512}; Hq=32 over Hkv=8, D=128, bf16",
    ),
    "long": dict(
        desc="8 seqs, L~U{32768..131072}, Hq=64 over Hkv=8, D=128, bf16, "
        "32-block partitions + LSE reduce, permuted blocks",
    ),
}


@dataclass
class Workload:
    name: str
    seed: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    dtype: torch.dtype
    scale: float  # float32 value passed to the kernel
    num_blocks: int
    lens_host: list  # python ints, one per sequence
    tables_host: list  # python lists of physical block ids
    seq_lens: torch.Tensor  # int32 [N]
    block_tables: torch.Tensor  # int32 [N, max_blocks], padded with PAD_BLOCK
    q: torch.Tensor  # [N, Hq, D]
    k_cache: torch.Tensor  # [NB, Hkv, B, D]
    v_cache: torch.Tensor  # [NB, Hkv, B, D]
    new_k: torch.Tensor  # [T, Hkv, D]  (T = N: one new token per sequence)
    new_v: torch.Tensor  # [T, Hkv, D]
    slot_mapping: torch.Tensor  # int64 [T]; -1 = padding (nothing written)
    partition_blocks: int = 0  # 0 = let the library choose
    shared_blocks: list = field(default_factory=list)  # physical ids referenced by >1 seq
    shared_prefix_blocks: int = 0  # leading table entries every sequence shares (whole blocks)
    desc: str = ""
    # several prompt groups: group i = sequences group_start_host[i] .. [i+1]-1,
    # sharing their first group_blocks_host[i] table entries (whole blocks)
    group_start_host: list = field(default_factory=list)
    group_blocks_host: list = field(default_factory=list)
    group_start: Optional[torch.Tensor] = None  # int32 [G + 1] on the device
    group_blocks: Optional[torch.Tensor] = None  # int32 [G]

    @property
    def num_seqs(self) -> int:
        return len(self.lens_host)

    @property
    def max_seq_len(self) -> int:
        return max(self.lens_host) if self.lens_host else 0

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def elem_bytes(self) -> int:
        return torch.finfo(self.dtype).bits // 8

    @property
    def device(self) -> torch.device:
        return self.q.device


def scale_for(head_dim: int) -> float:
    """1/sqrt(D) rounded to float32 (the value the kernel receives)."""
    return float(torch.tensor(1.0 / math.sqrt(head_dim), dtype=torch.float32).item())


def _blocks_for(n_tokens: int, block_size: int) -> int:
    # allocation bookkeeping: how many blocks the allocator hands out
    return -(-n_tokens // block_size)


def _draw_lens(name: str, gen: torch.Generator) -> list:
    if name == "tiny":
        return [35, 1, 16, 17]
    if name == "mha":
        return torch.randint(128, 2048 + 1, (64,), generator=gen).tolist()
    if name == "gqa":
        z = torch.randn(256, generator=gen, dtype=torch.float64)
        lens = torch.round(torch.exp(z * 0.8 + math.log(1024.0)))
        return lens.clamp(16, 8192).to(torch.int64).tolist()
    if name == "long":
        return torch.randint(32768, 131072 + 1, (8,), generator=gen).tolist()
    raise KeyError(name)


def _randn(shape, gen: torch.Generator, device, dtype) -> torch.Tensor:
    """N(0,1) drawn in fp32 on `device`, cast (RNE) to `dtype`; chunked so that a
    multi-GB pool never needs a full fp32 temporary."""
    out = torch.empty(shape, dtype=dtype, device=device)
    flat = out.view(-1)
    n = flat.numel()
    chunk = 1 << 28
    for off in range(0, n, chunk):
        m = min(chunk, n - off)
        flat[off : off + m] = torch.randn(m, generator=gen, device=device, dtype=torch.float32).to(dtype)
    return out


@dataclass
class Plan:
    """Structure of a workload: lengths, pool size and block tables (no values)."""
    lens: list
    tables: list
    num_blocks: int
    shared: list  # physical ids of the full shared prefix blocks (all groups)
    cow_pairs: list  # (shared source block, private copy, tokens copied) for a prefix ending mid-block
    prefix_len: int = 0  # one prompt shared by every sequence (0 with several groups)
    group_start: list = field(default_factory=list)  # sequences of group i: [start[i], start[i+1])
    group_blocks: list = field(default_factory=list)  # full blocks group i shares

    @property
    def needed_blocks(self) -> int:
        ids = set(b for t in self.tables for b in t) | set(src for src, _, _ in self.cow_pairs)
        return len(ids)


def plan(
    lens: Sequence[int],
    seed: int = 0,
    num_blocks: Optional[int] = None,
    pool_factor: float = 1.25,
    prefix_len: int = 0,
    groups: Optional[Sequence[tuple]] = None,
) -> Plan:
    """Allocate physical blocks for sequences of the given total lengths.

    The pool holds ``ceil(pool_factor * needed)`` blocks unless ``num_blocks`` is
    given; blocks are taken in order from a seeded random permutation of the pool
    (a shuffled free list).  ``groups`` = [(count, prefix_len), ...] splits the
    sequences, in order, into prompt groups: the ``count`` sequences of a group
    start with the same ``prefix_len`` tokens, whose full blocks are allocated
    once and named by every table of the group; if the prefix ends inside a
    block, that block is kept once as a shared source and each sequence of the
    group gets a private copy of it (copy-on-write) into which its own suffix
    continues.  ``prefix_len > 0`` without ``groups`` is one group of every
    sequence.
    """
    B = BLOCK_SIZE
    lens = [int(x) for x in lens]
    if groups is None:
        groups = [(len(lens), prefix_len)]
    assert sum(c for c, _ in groups) == len(lens), "the groups must cover every sequence"
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    needed = 0
    start = 0
    for count, pl in groups:
        assert all(L >= pl for L in lens[start:start + count]), "every sequence must hold its prefix"
        needed += pl // B + (1 if pl % B else 0)
        needed += sum(_blocks_for(L - (pl // B) * B, B) for L in lens[start:start + count])
        start += count
    if num_blocks is None:
        num_blocks = max(1, math.ceil(pool_factor * needed))
    assert num_blocks >= needed, (num_blocks, needed)

    free = torch.randperm(num_blocks, generator=gen).tolist()
    cursor = 0

    def take() -> int:
        nonlocal cursor
        b = free[cursor]
        cursor += 1
        return b

    tables, cow_pairs, shared_all, gstart, gblocks = [], [], [], [0], []
    start = 0
    for count, pl in groups:
        n_full, rem = pl // B, pl % B
        shared = [take() for _ in range(n_full)]
        shared_all += shared
        cow_source = take() if rem else None
        for L in lens[start:start + count]:
            t = list(shared)
            for j in range(_blocks_for(L - n_full * B, B)):
                b = take()
                if j == 0 and rem:
                    cow_pairs.append((cow_source, b, rem))
                t.append(b)
            tables.append(t)
        start += count
        gstart.append(start)
        gblocks.append(n_full)
    one = len(groups) == 1
    return Plan(lens, tables, num_blocks, shared_all, cow_pairs, groups[0][1] if one else 0, gstart, gblocks)


def build(
    lens: Sequence[int],
    num_q_heads: int,
    num_kv_heads: int,
    head_dim: int,
    dtype: torch.dtype,
    seed: int = 0,
    device="cpu",
    num_blocks: Optional[int] = None,
    pool_factor: float = 1.25,
    prefix_len: int = 0,
    poison_unused: bool = False,
    partition_blocks: int = 0,
    name: str = "custom",
    desc: str = "",
    table_width: Optional[int] = None,
    groups: Optional[Sequence[tuple]] = None,
) -> Workload:
    """Build a workload from explicit per-sequence total lengths (see ``plan``).

    ``poison_unused`` fills every slot that no table reaches (unused blocks and
    the tail of each sequence's last block) with NaN, so a kernel that reads
    past a sequence's length produces a visibly wrong result.
    """
    B = BLOCK_SIZE
    assert num_q_heads % num_kv_heads == 0
    p = plan(lens, seed=seed, num_blocks=num_blocks, pool_factor=pool_factor, prefix_len=prefix_len, groups=groups)
    lens, tables, num_blocks = p.lens, p.tables, p.num_blocks

    width = max([len(t) for t in tables] + [1])
    if table_width is not None:
        assert table_width >= width
        width = table_width
    tab = torch.full((len(lens), width), PAD_BLOCK, dtype=torch.int32)
    for s, t in enumerate(tables):
        if t:
            tab[s, : len(t)] = torch.tensor(t, dtype=torch.int32)

    vgen = torch.Generator(device=device)
    vgen.manual_seed(seed + 1)
    N = len(lens)
    q = _randn((N, num_q_heads, head_dim), vgen, device, dtype)
    k_cache = _randn((num_blocks, num_kv_heads, B, head_dim), vgen, device, dtype)
    v_cache = _randn((num_blocks, num_kv_heads, B, head_dim), vgen, device, dtype)
    new_k = _randn((N, num_kv_heads, head_dim), vgen, device, dtype)
    new_v = _randn((N, num_kv_heads, head_dim), vgen, device, dtype)

    # copy-on-write of the partial last prefix block into each private copy
    for src, dst, rem in p.cow_pairs:
        k_cache[dst, :, :rem] = k_cache[src, :, :rem]
        v_cache[dst, :, :rem] = v_cache[src, :, :rem]

    slot_mapping = torch.tensor(new_token_slots(p), dtype=torch.int64)

    if poison_unused:
        used = _used_slots(lens, tables, num_blocks).to(device)[:, None, :, None]
        nan = torch.tensor(float("nan"), dtype=dtype, device=device)
        k_cache = torch.where(used, k_cache, nan)
        v_cache = torch.where(used, v_cache, nan)

    return Workload(
        name=name,
        seed=seed,
        num_q_heads=num_q_heads,
        num_kv_heads=num_kv_heads,
        head_dim=head_dim,
        block_size=B,
        dtype=dtype,
        scale=scale_for(head_dim),
        num_blocks=num_blocks,
        lens_host=lens,
        tables_host=tables,
        seq_lens=torch.tensor(lens, dtype=torch.int32).to(device),
        block_tables=tab.to(device),
        q=q,
        k_cache=k_cache,
        v_cache=v_cache,
        new_k=new_k,
        new_v=new_v,
        slot_mapping=slot_mapping.to(device),
        partition_blocks=partition_blocks,
        shared_blocks=sorted(set(p.shared + [src for src, _, _ in p.cow_pairs])),
        shared_prefix_blocks=p.prefix_len // B if groups is None else 0,
        desc=desc,
        group_start_host=list(p.group_start),
        group_blocks_host=list(p.group_blocks),
        group_start=torch.tensor(p.group_start, dtype=torch.int32).to(device),
        group_blocks=torch.tensor(p.group_blocks, dtype=torch.int32).to(device),
    )


def _used_slots(lens, tables, num_blocks: int) -> torch.Tensor:
    """[num_blocks, 16] bool: the slots some sequence's table reaches."""
    B = BLOCK_SIZE
    used = torch.zeros((num_blocks, B), dtype=torch.bool)
    for L, t in zip(lens, tables):
        for j, b in enumerate(t):
            used[b, : min(B, L - j * B)] = True
    return used


E4M3_NAN = 0x7F  # S.1111.111, the code pa_cache_write_fp8 writes for NaN


def fp8_pools(w: Workload, seed: Optional[int] = None, poison_unused: bool = False) -> tuple:
    """E4M3 KV pools with the structure (pool size, tables) of ``w``.

    Returns (k_codes, v_codes, k_scale, v_scale): uint8 [NB, Hkv, 16, D] codes
    drawn uniformly from the 254 codes that are not NaN (bit patterns only: no
    rounding or conversion here), and one fp32 scale per kv head and pool drawn
    uniformly from [1/160, 1/112], so that decoded values stay within about
    +-4, the range of the N(0, 1) values of the bf16 pools; all on ``w.device``.  Values come from a device
    generator seeded with ``seed + 2`` (``seed`` defaults to ``w.seed``).
    ``poison_unused`` sets every slot no table reaches to the NaN code.
    """
    seed = w.seed if seed is None else seed
    dev = w.device
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed + 2)
    shape = (w.num_blocks, w.num_kv_heads, BLOCK_SIZE, w.head_dim)
    pools = []
    for _ in range(2):
        out = torch.empty(shape, dtype=torch.uint8, device=dev)
        flat = out.view(-1)
        chunk = 1 << 28
        for off in range(0, flat.numel(), chunk):
            m = min(chunk, flat.numel() - off)
            c = torch.randint(0, 254, (m,), generator=gen, device=dev, dtype=torch.uint8)
            flat[off : off + m] = c + (c >= E4M3_NAN).to(torch.uint8)  # 0..126, 128..254: no NaN code
        pools.append(out)
    scales = [1.0 / (112.0 + 48.0 * torch.rand(w.num_kv_heads, generator=gen, device=dev)) for _ in range(2)]
    if poison_unused:
        used = _used_slots(w.lens_host, w.tables_host, w.num_blocks).to(dev)[:, None, :, None]
        nan = torch.tensor(E4M3_NAN, dtype=torch.uint8, device=dev)
        pools = [torch.where(used, p, nan) for p in pools]
    return pools[0], pools[1], scales[0].float(), scales[1].float()


def new_token_slots(p: Plan) -> list:
    """Slot of each sequence's newest token (position L-1), -1 for an empty one.
    This is the slot mapping a serving engine hands to the cache write."""
    B = BLOCK_SIZE
    slots = []
    for L, t in zip(p.lens, p.tables):
        if L == 0:
            slots.append(-1)
        else:
            pos = L - 1
            slots.append(t[pos // B] * B + pos % B)
    return slots


def config_lens(name: str, seed: int = 0) -> tuple:
    """(lens, prefix_len) of a named workload, drawn from the seed."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    if name == "prefix":
        suf = torch.randint(64, 512 + 1, (128,), generator=gen).tolist()
        return [4096 + s for s in suf], 4096
    return _draw_lens(name, gen), 0


def config_plan(name: str, seed: int = 0) -> Plan:
    lens, prefix = config_lens(name, seed)
    return plan(lens, seed=seed, num_blocks=16 if name == "tiny" else None, prefix_len=prefix)


def make(name: str, seed: int = 0, device="cpu", poison_unused: bool = False,
         max_seqs: Optional[int] = None, **kw) -> Workload:
    """One of the five named workloads (see CONFIGS).  ``max_seqs`` keeps only
    the first sequences of the batch (a smaller case of the same shape, for
    profiler captures)."""
    desc = CONFIGS[name]["desc"]
    lens, prefix = config_lens(name, seed)
    if max_seqs is not None:
        lens = lens[:max_seqs]
        desc += f" (first {len(lens)} sequences only)"
    common = dict(seed=seed, device=device, poison_unused=poison_unused, name=name, desc=desc)
    if name == "tiny":
        return build(lens, 2, 1, 64, torch.float32, num_blocks=16, **common, **kw)
    if name == "mha":
        return build(lens, 32, 32, 128, torch.bfloat16, **common, **kw)
    if name == "gqa":
        return build(lens, 32, 8, 128, torch.bfloat16, **common, **kw)
    if name == "prefix":
        prefix = kw.pop("prefix_len", prefix)
        if prefix != 4096:  # variant with a different prefix length, same suffixes
            lens = [L - 4096 + prefix for L in lens]
        ng = kw.pop("prompt_groups", 1)
        if ng > 1:  # variant: ng prompts of the same length, each shared by a consecutive share of the batch
            n = len(lens)
            groups = [(n * (i + 1) // ng - n * i // ng, prefix) for i in range(ng)]
            common["desc"] = desc + f" (variant: {ng} prompts, each shared by {n // ng} sequences)"
            return build(lens, 32, 8, 128, torch.bfloat16, groups=groups, **common, **kw)
        return build(lens, 32, 8, 128, torch.bfloat16, prefix_len=prefix, **common, **kw)
    if name == "long":
        kw.setdefault("partition_blocks", 32)
        return build(lens, 64, 8, 128, torch.bfloat16, **common, **kw)
    raise KeyError(name)


def as_numpy(t: torch.Tensor) -> np.ndarray:
    """Host copy as numpy; bf16 comes back as its raw uint16 bit patterns."""
    t = t.detach().to("cpu").contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()
