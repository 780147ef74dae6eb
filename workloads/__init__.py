"""Seeded synthetic inputs for the attention-prologue operations.

This module only draws inputs: ragged batches, page tables, caches, projections, gammas
and the freqs_cis table.  It holds none of the operations' arithmetic, and both the CUDA
library's callers and the CPU oracle's callers consume what it returns.  Everything lives on
the host (torch CPU tensors) and is reproducible from the seed.

Recipe (the shapes and distributions of the workloads the kernel pages name: Llama-style
GQA prefill and decode, MiniMax-style main + indexer caches):
  * lengths: U[lo, hi] per sequence, or a seeded composition of a fixed total with a cap;
  * cache_lengths: U[lo, hi] per sequence;
  * page tables: pages needed by each sequence, ceil((cache_len + len) / page_size), taken
    in order from a seeded permutation of all pages (a few spare pages stay unreferenced);
    unused page-table entries hold 0xFFFFFFFF;
  * projections: N(0, std^2) rounded to the element type;
  * gammas: N(1, 0.1^2) rounded to the element type;
  * caches and output buffers start as seeded random bit patterns (so that any byte the
    operation must not touch is recognisable), except where an operation reads the cache
    (in-place RoPE, radd), where the rows it reads hold N(0, 1) values;
  * freqs_cis[p, 2i] = cos(p * theta^(-2i/rope_dim)), freqs_cis[p, 2i+1] = sin(same),
    evaluated in float64 and rounded once to the table's element type.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional

import torch

TORCH_DTYPES = {"bf16": torch.bfloat16, "f16": torch.float16, "f32": torch.float32,
                "fp8": torch.float8_e4m3fn}
PAGE_SENTINEL = -1  # 0xFFFFFFFF once viewed as uint32


def generator(seed: int) -> torch.Generator:
    return torch.Generator().manual_seed(seed)


def uniform_ints(gen: torch.Generator, n: int, lo: int, hi: int) -> List[int]:
    """n integers drawn uniformly from [lo, hi] (inclusive)."""
    return torch.randint(lo, hi + 1, (n,), generator=gen).tolist()


def lengths_with_total(gen: torch.Generator, n: int, total: int, cap: int) -> List[int]:
    """n positive lengths summing to `total`, each <= cap: seeded weights U[0.25, 1.75]
    scaled to the total, then the rounding remainder spread one token at a time."""
    assert n * cap >= total >= n
    w = 0.25 + 1.5 * torch.rand(n, generator=gen, dtype=torch.float64)
    raw = [max(1, min(cap, int(x))) for x in (w / w.sum() * total).tolist()]
    i = 0
    while sum(raw) != total:
        j = i % n
        if sum(raw) < total and raw[j] < cap:
            raw[j] += 1
        elif sum(raw) > total and raw[j] > 1:
            raw[j] -= 1
        i += 1
    return raw


def row_offsets(lengths: List[int]) -> torch.Tensor:
    """input_row_offsets [batch + 1] as int32 (read as uint32)."""
    offs = [0]
    for n in lengths:
        offs.append(offs[-1] + n)
    return torch.tensor(offs, dtype=torch.int32)


def normal(gen: torch.Generator, shape, std: float = 1.0, mean: float = 0.0,
           dtype: str = "bf16") -> torch.Tensor:
    x = torch.randn(*shape, generator=gen, dtype=torch.float32)
    return (x * std + mean).to(TORCH_DTYPES[dtype])


def random_bits(gen: torch.Generator, n: int, dtype: str = "bf16",
                block: int = 1 << 22) -> torch.Tensor:
    """n elements of seeded random bit patterns (a random block tiled when n is large)."""
    if dtype == "f32":
        src = torch.randint(-(1 << 31), (1 << 31) - 1, (min(n, block),), generator=gen,
                            dtype=torch.int32)
        view = torch.float32
    elif dtype == "fp8":
        src = torch.randint(0, 256, (min(n, block),), generator=gen, dtype=torch.uint8)
        view = torch.float8_e4m3fn
    else:
        src = torch.randint(-(1 << 15), 1 << 15, (min(n, block),), generator=gen,
                            dtype=torch.int16)
        view = TORCH_DTYPES[dtype]
    if n > block:
        src = src.repeat((n + block - 1) // block)[:n]
    return src.view(view).clone()


def freqs_cis(max_seq_len: int, rope_dim: int, theta: float, dtype: str = "f32") -> torch.Tensor:
    """[max_seq_len, rope_dim]: (cos, sin) of p * theta^(-2i/rope_dim) at columns 2i, 2i+1."""
    i = torch.arange(rope_dim // 2, dtype=torch.float64)
    inv = theta ** (-2.0 * i / rope_dim)
    ang = torch.arange(max_seq_len, dtype=torch.float64)[:, None] * inv[None, :]
    tab = torch.stack([torch.cos(ang), torch.sin(ang)], dim=-1).reshape(max_seq_len, rope_dim)
    return tab.to(TORCH_DTYPES[dtype]).contiguous()


# --------------------------------------------------------------------- paged caches --

@dataclass
class PagedKV:
    """Paged cache storage laid out [page][plane][layer][slot][head][dim] (plane 0 = K,
    plane 1 = V when planes == 2) in one flat tensor, with its page table."""
    storage: torch.Tensor
    planes: int
    num_pages: int
    num_layers: int
    page_size: int
    n_kv_heads: int
    head_dim: int
    page_table: torch.Tensor      # int32 [n_seqs, width], -1 = unused
    cache_lengths: torch.Tensor   # int32 [n_seqs]
    dtype: str = "bf16"
    k_scale: Optional[torch.Tensor] = None   # float32 [1] each, for an fp8 cache
    v_scale: Optional[torch.Tensor] = None

    @property
    def head_stride(self) -> int:
        return self.head_dim

    @property
    def slot_stride(self) -> int:
        return self.n_kv_heads * self.head_dim

    @property
    def layer_stride(self) -> int:
        return self.page_size * self.slot_stride

    @property
    def page_stride(self) -> int:
        return self.planes * self.num_layers * self.layer_stride

    @property
    def k_offset(self) -> int:
        return 0

    @property
    def v_offset(self) -> Optional[int]:
        return self.num_layers * self.layer_stride if self.planes == 2 else None

    @property
    def max_pages_per_seq(self) -> int:
        return self.page_table.shape[1]

    def view6(self, storage: Optional[torch.Tensor] = None) -> torch.Tensor:
        s = self.storage if storage is None else storage
        return s.view(self.num_pages, self.planes, self.num_layers, self.page_size,
                      self.n_kv_heads, self.head_dim)


def paged_cache(gen: torch.Generator, *, cache_lengths: List[int], lengths: List[int],
                page_size: int, n_kv_heads: int, head_dim: int, planes: int = 2,
                num_layers: int = 2, width: Optional[int] = None, spare_pages: int = 2,
                dtype: str = "bf16", fill: str = "bits",
                scales: Optional[tuple] = None) -> PagedKV:
    """A paged cache big enough for every sequence's cache_len + len positions."""
    need = [max(1, math.ceil((c + n) / page_size)) for c, n in zip(cache_lengths, lengths)]
    width = width or max(need)
    need = [min(m, width) for m in need]   # a narrower table leaves late positions unmapped
    num_pages = sum(need) + spare_pages
    perm = torch.randperm(num_pages, generator=gen).to(torch.int32)
    table = torch.full((len(lengths), width), PAGE_SENTINEL, dtype=torch.int32)
    k = 0
    for b, m in enumerate(need):
        table[b, :m] = perm[k:k + m]
        k += m
    n_elem = num_pages * planes * num_layers * page_size * n_kv_heads * head_dim
    if fill == "bits":
        storage = random_bits(gen, n_elem, dtype)
    else:
        storage = normal(gen, (n_elem,), dtype=dtype)
    ks = vs = None
    if dtype == "fp8":  # per-plane float32 scales
        ks, vs = (torch.tensor([x], dtype=torch.float32) for x in (scales or (1.0, 1.0)))
    return PagedKV(storage, planes, num_pages, num_layers, page_size, n_kv_heads, head_dim,
                   table, torch.tensor(cache_lengths, dtype=torch.int32), dtype, ks, vs)


@dataclass
class ContKV:
    """Continuous-batching cache laid out [slot][plane][layer][pos][head][dim]."""
    storage: torch.Tensor
    planes: int
    num_slots: int
    num_layers: int
    max_seq_len: int
    n_kv_heads: int
    head_dim: int
    lookup_table: torch.Tensor    # int32 [n_seqs]
    cache_lengths: torch.Tensor   # int32 [n_seqs]
    dtype: str = "bf16"

    @property
    def head_stride(self) -> int:
        return self.head_dim

    @property
    def pos_stride(self) -> int:
        return self.n_kv_heads * self.head_dim

    @property
    def layer_stride(self) -> int:
        return self.max_seq_len * self.pos_stride

    @property
    def slot_stride(self) -> int:
        return self.planes * self.num_layers * self.layer_stride

    @property
    def k_offset(self) -> int:
        return 0

    @property
    def v_offset(self) -> Optional[int]:
        return self.num_layers * self.layer_stride if self.planes == 2 else None


# ------------------------------------------------------------------------ workloads --

@dataclass
class RopeSpec:
    table: torch.Tensor
    dtype: str
    interleaved: bool
    rope_col_offset: int = -1

    @property
    def rope_dim(self) -> int:
        return self.table.shape[1]


@dataclass
class RaggedStore:
    """Inputs of the ragged paged store (optionally with per-head RMSNorm)."""
    qkv: torch.Tensor             # [T, (Hq + 2 Hk) D]
    offsets: torch.Tensor         # int32 [batch + 1]
    n_q_heads: int
    cache: PagedKV
    rope: RopeSpec
    layer_idx: int
    q_out: torch.Tensor           # [T, Hq D], pre-filled with random bits
    lengths: List[int]
    q_gamma: Optional[torch.Tensor] = None
    k_gamma: Optional[torch.Tensor] = None
    epsilon: float = 1e-6
    weight_offset: float = 0.0
    name: str = ""

    @property
    def total_tokens(self) -> int:
        return self.qkv.shape[0]


def ragged_store(seed: int, *, lengths: List[int], cache_lengths: List[int], n_q_heads: int,
                 n_kv_heads: int, head_dim: int, page_size: int, rope_dim: int, theta: float,
                 interleaved: bool, max_seq_len: int, freq_dtype: str = "f32",
                 x_std: float = 1.0, norm: bool = False, epsilon: float = 1e-6,
                 weight_offset: float = 0.0, num_layers: int = 2, layer_idx: int = 1,
                 width: Optional[int] = None, rope_col_offset: int = -1,
                 dtype: str = "bf16", row_pad: int = 0, q_out_dtype: Optional[str] = None,
                 cache_dtype: Optional[str] = None, kv_scales: tuple = (1.0, 1.0),
                 name: str = "") -> RaggedStore:
    gen = generator(seed)
    T = sum(lengths)
    D = head_dim
    cols = (n_q_heads + 2 * n_kv_heads) * D
    qkv = normal(gen, (T, cols + row_pad), std=x_std, dtype=dtype)
    if row_pad:
        qkv = qkv[:, :cols]
    cache = paged_cache(gen, cache_lengths=cache_lengths, lengths=lengths, page_size=page_size,
                        n_kv_heads=n_kv_heads, head_dim=D, num_layers=num_layers, width=width,
                        dtype=cache_dtype or dtype, scales=kv_scales)
    rope = RopeSpec(freqs_cis(max_seq_len, rope_dim, theta, freq_dtype), freq_dtype,
                    interleaved, rope_col_offset)
    q_out = random_bits(gen, T * n_q_heads * D, q_out_dtype or dtype).view(T, n_q_heads * D)
    w = ragged_store_gammas(gen, D, dtype) if norm else (None, None)
    return RaggedStore(qkv, row_offsets(lengths), n_q_heads, cache, rope, layer_idx, q_out,
                       list(lengths), w[0], w[1], epsilon, weight_offset, name)


def ragged_store_gammas(gen, D, dtype):
    return (normal(gen, (D,), std=0.1, mean=1.0, dtype=dtype),
            normal(gen, (D,), std=0.1, mean=1.0, dtype=dtype))


@dataclass
class DualBand:
    """Inputs of the two-cache launch: one combined input buffer whose column blocks are
    [Q main | K main | V main | Q index | K index]."""
    input: torch.Tensor
    offsets: torch.Tensor
    lengths: List[int]
    rope: RopeSpec
    layer_idx: int
    main_cache: PagedKV
    index_cache: PagedKV
    main_cols: tuple              # (q_col, k_col, v_col)
    index_cols: tuple             # (q_col, k_col, -1)
    main_q_heads: int
    index_q_heads: int
    gammas: tuple                 # (q_main, k_main, q_index, k_index)
    main_eps: float
    index_eps: float
    weight_offset: float
    q_main_out: torch.Tensor
    q_index_out: torch.Tensor
    name: str = ""

    @property
    def total_tokens(self) -> int:
        return self.input.shape[0]

    def cache_lengths_of(self, kv: "PagedKV") -> List[int]:
        return [int(x) for x in kv.cache_lengths]


def dual_band(seed: int, *, lengths: List[int], cache_lengths: List[int], main_q_heads: int,
              main_kv_heads: int, index_q_heads: int, index_kv_heads: int, head_dim: int,
              main_page_size: int, index_page_size: int, rope_dim: int, theta: float,
              interleaved: bool, max_seq_len: int, x_std: float = 1.0,
              main_eps: float = 1e-6, index_eps: float = 1e-6, weight_offset: float = 0.0,
              num_layers: int = 2, layer_idx: int = 1, dtype: str = "bf16",
              k_in_place: bool = False, single: bool = False,
              main_cache_dtype: Optional[str] = None, index_cache_dtype: Optional[str] = None,
              kv_scales: tuple = (1.0, 1.0), name: str = "") -> DualBand:
    """k_in_place: the bands' K heads are not read from the input but from the cache slots
    the tokens map to (which hold N(0, x_std) K rows, as if the projection had stored them),
    and V is not stored (the bands' column triples become (q_col, -1, -1)).  single: the
    main band alone (index_cache, index outputs and the index gammas are None)."""
    gen = generator(seed)
    T, D = sum(lengths), head_dim
    qm, km, vm = 0, main_q_heads * D, (main_q_heads + main_kv_heads) * D
    qi = (main_q_heads + 2 * main_kv_heads) * D
    ki = qi + index_q_heads * D
    cols = ki + index_kv_heads * D
    inp = normal(gen, (T, cols), std=x_std, dtype=dtype)
    main = paged_cache(gen, cache_lengths=cache_lengths, lengths=lengths,
                       page_size=main_page_size, n_kv_heads=main_kv_heads, head_dim=D,
                       num_layers=num_layers, width=max_seq_len // main_page_size,
                       dtype=main_cache_dtype or dtype, scales=kv_scales)
    index = paged_cache(gen, cache_lengths=cache_lengths, lengths=lengths,
                        page_size=index_page_size, n_kv_heads=index_kv_heads, head_dim=D,
                        planes=1, num_layers=num_layers, width=max_seq_len // index_page_size,
                        dtype=index_cache_dtype or dtype, scales=kv_scales)
    rope = RopeSpec(freqs_cis(max_seq_len, rope_dim, theta, "f32"), "f32", interleaved)
    gam = tuple(normal(gen, (D,), std=0.1, mean=1.0, dtype=dtype) for _ in range(4))
    q_main_out = random_bits(gen, T * main_q_heads * D, dtype).view(T, main_q_heads * D)
    q_index_out = random_bits(gen, T * index_q_heads * D, dtype).view(T, index_q_heads * D)
    main_cols, index_cols = (qm, km, vm), (qi, ki, -1)
    if k_in_place:
        main_cols, index_cols = (qm, -1, -1), (qi, -1, -1)
        for kv in (main, index):
            fill_k_rows(gen, kv, cache_lengths, lengths, layer_idx, x_std)
    if single:
        index, index_q_heads, q_index_out = None, 0, None
        gam = (gam[0], gam[1], None, None)
    return DualBand(inp, row_offsets(lengths), list(lengths), rope, layer_idx, main, index,
                    main_cols, index_cols, main_q_heads, index_q_heads, gam, main_eps,
                    index_eps, weight_offset, q_main_out, q_index_out, name)


def token_slots(kv: PagedKV, cache_lengths: List[int], lengths: List[int]):
    """(page, slot) of every new token, in row order (positions past the page table are
    skipped)."""
    out = []
    for b, (c, n) in enumerate(zip(cache_lengths, lengths)):
        for t in range(n):
            pos = c + t
            col = pos // kv.page_size
            if col < kv.page_table.shape[1] and int(kv.page_table[b, col]) >= 0:
                out.append((int(kv.page_table[b, col]), pos % kv.page_size))
    return out


def fill_k_rows(gen: torch.Generator, kv: PagedKV, cache_lengths: List[int],
                lengths: List[int], layer_idx: int, std: float) -> None:
    """Write N(0, std) K rows into the cache slots of the new tokens."""
    slots = token_slots(kv, cache_lengths, lengths)
    if not slots:
        return
    idx = torch.tensor(slots, dtype=torch.long)
    kv.view6()[idx[:, 0], 0, layer_idx, idx[:, 1]] = normal(
        gen, (len(slots), kv.n_kv_heads, kv.head_dim), std=std, dtype=kv.dtype)


@dataclass
class BshdDecode:
    q_proj: torch.Tensor          # [B, S, Hq, D]
    cache: ContKV
    rope: RopeSpec
    layer_idx: int
    valid_lengths: torch.Tensor   # int32 [B]
    output: torch.Tensor          # [B, S, Hq, D], pre-filled with random bits
    name: str = ""


def bshd_decode(seed: int, *, B: int, S: int, n_q_heads: int, n_kv_heads: int, head_dim: int,
                cache_lengths: List[int], valid_lengths: List[int], max_seq_len: int,
                rope_dim: int, theta: float, interleaved: bool, freq_dtype: str = "bf16",
                num_slots: Optional[int] = None, num_layers: int = 1, layer_idx: int = 0,
                planes: int = 1, dtype: str = "bf16", name: str = "") -> BshdDecode:
    gen = generator(seed)
    D = head_dim
    q = normal(gen, (B, S, n_q_heads, D), dtype=dtype)
    num_slots = num_slots or B
    lookup = torch.randperm(num_slots, generator=gen)[:B].to(torch.int32)
    n_elem = num_slots * planes * num_layers * max_seq_len * n_kv_heads * D
    cache = ContKV(random_bits(gen, n_elem, dtype), planes, num_slots, num_layers, max_seq_len,
                   n_kv_heads, D, lookup, torch.tensor(cache_lengths, dtype=torch.int32), dtype)
    # K rows the projection already wrote: positions cache_len + s for s < S (in range)
    k_rows = cache.storage.view(num_slots, planes, num_layers, max_seq_len, n_kv_heads, D)
    for b in range(B):
        lo = cache_lengths[b]
        hi = min(lo + S, max_seq_len)
        if hi > lo:
            k_rows[int(lookup[b]), 0, layer_idx, lo:hi] = normal(gen, (hi - lo, n_kv_heads, D),
                                                                 dtype=dtype)
    rope = RopeSpec(freqs_cis(max_seq_len, rope_dim, theta, freq_dtype), freq_dtype, interleaved)
    out = random_bits(gen, B * S * n_q_heads * D, dtype).view(B, S, n_q_heads, D)
    return BshdDecode(q, cache, rope, layer_idx, torch.tensor(valid_lengths, dtype=torch.int32),
                      out, name)


@dataclass
class Radd:
    a: torch.Tensor               # [T, 2 * Hk * D]
    offsets: torch.Tensor
    lengths: List[int]
    cache: PagedKV
    batch_offset: int
    layer_idx: int
    name: str = ""


def radd(seed: int, *, lengths: List[int], cache_lengths: List[int], n_kv_heads: int,
         head_dim: int, page_size: int, batch_offset: int = 0, n_seqs: Optional[int] = None,
         num_layers: int = 2, layer_idx: int = 1, max_seq_len: int = 8192,
         dtype: str = "bf16", name: str = "") -> Radd:
    """radd into a cache whose sequences batch_offset .. batch_offset + batch - 1 receive
    the rows; the cache holds N(0,1) values (it is read as well as written)."""
    gen = generator(seed)
    batch = len(lengths)
    n_seqs = n_seqs or batch + batch_offset
    all_cl = uniform_ints(gen, n_seqs, 0, 0)
    all_len = [1] * n_seqs
    for b in range(batch):
        all_cl[b + batch_offset] = cache_lengths[b]
        all_len[b + batch_offset] = lengths[b]
    cache = paged_cache(gen, cache_lengths=all_cl, lengths=all_len, page_size=page_size,
                        n_kv_heads=n_kv_heads, head_dim=head_dim, num_layers=num_layers,
                        width=max(1, max_seq_len // page_size), dtype=dtype, fill="normal")
    a = normal(gen, (sum(lengths), 2 * n_kv_heads * head_dim), dtype=dtype)
    return Radd(a, row_offsets(lengths), list(lengths), cache, batch_offset, layer_idx, name)


# ------------------------------------------------------------- the named workloads --

def tiny_ragged(seed: int = 0) -> RaggedStore:
    """batch 2, new lengths [3, 5], cache_lengths [0, 7], 4 Q / 2 KV heads, head_dim 64,
    interleaved RoPE theta 1e4, freqs_cis [64, 64] f32, page_size 16, page table a seeded
    permutation of 8 pages (4 per sequence), bf16 QKV ~ N(0, 1), no norm."""
    gen = generator(seed)
    lengths, cls, P, D = [3, 5], [0, 7], 16, 64
    qkv = normal(gen, (8, (4 + 2 * 2) * D))
    perm = torch.randperm(8, generator=gen).to(torch.int32).view(2, 4)
    storage = random_bits(gen, 8 * 2 * 2 * P * 2 * D)
    cache = PagedKV(storage, 2, 8, 2, P, 2, D, perm.contiguous(),
                    torch.tensor(cls, dtype=torch.int32))
    rope = RopeSpec(freqs_cis(64, 64, 1e4, "f32"), "f32", True)
    q_out = random_bits(gen, 8 * 4 * D).view(8, 4 * D)
    return RaggedStore(qkv, row_offsets(lengths), 4, cache, rope, 1, q_out, lengths,
                       name="tiny ragged store: batch 2, lengths [3,5], 4q/2kv heads, d64")


def llama3_8b_prefill_fp8_cache(seed: int = 0) -> RaggedStore:
    """llama3_8b_prefill storing K and V as E4M3 codes (K scale 0.5, V scale 0.25)."""
    gen = generator(seed)
    lengths = uniform_ints(gen, 8, 256, 2048)
    return ragged_store(seed + 1, lengths=lengths, cache_lengths=[0] * 8, n_q_heads=32,
                        n_kv_heads=8, head_dim=128, page_size=128, rope_dim=128, theta=5e5,
                        interleaved=False, max_seq_len=8192, width=64, cache_dtype="fp8",
                        kv_scales=(0.5, 0.25),
                        name="Llama-3-8B ragged prefill into an FP8 (E4M3) cache: 32q/8kv "
                             "heads, d128, batch 8, page 128, half-split RoPE")


def llama3_8b_prefill(seed: int = 0) -> RaggedStore:
    """32 Q / 8 KV heads, head_dim 128, batch 8 with lengths U[256, 2048] (about 9k tokens),
    cache_lengths 0, page_size 128, shuffled page table, bf16 QKV ~ N(0, 1), freqs_cis
    theta 5e5 over 8192 positions (f32), half-split RoPE over the full head."""
    gen = generator(seed)
    lengths = uniform_ints(gen, 8, 256, 2048)
    return ragged_store(seed + 1, lengths=lengths, cache_lengths=[0] * 8, n_q_heads=32,
                        n_kv_heads=8, head_dim=128, page_size=128, rope_dim=128, theta=5e5,
                        interleaved=False, max_seq_len=8192, width=64,
                        name="Llama-3-8B ragged prefill: 32q/8kv heads, d128, batch 8, "
                             "lengths U[256,2048], page 128, half-split RoPE")


def decode_bshd(seed: int = 0) -> BshdDecode:
    """q_proj [256, 1, 32, 128] bf16 ~ N(0, 1), 8 KV heads, continuous cache of 256 slots x
    8192 positions with K already written at cache_len[b], cache_lengths U[1, 8191],
    valid_lengths all 1, interleaved RoPE theta 5e5 (freqs_cis in the element type)."""
    gen = generator(seed)
    cls = uniform_ints(gen, 256, 1, 8191)
    return bshd_decode(seed + 1, B=256, S=1, n_q_heads=32, n_kv_heads=8, head_dim=128,
                       cache_lengths=cls, valid_lengths=[1] * 256, max_seq_len=8192,
                       rope_dim=128, theta=5e5, interleaved=True, freq_dtype="bf16",
                       name="continuous-batch decode: q_proj [256,1,32,128], 8 kv heads, "
                            "cache 256 x 8192, interleaved RoPE")


def per_head_norm(seed: int = 0) -> RaggedStore:
    """64 Q / 8 KV heads, head_dim 128, eps 1e-6, gamma ~ N(1, 0.1) bf16, weight_offset 0,
    16384 tokens over 32 sequences (each <= 4096), cache_lengths U[0, 4096], page_size 128,
    bf16 QKV ~ N(0, 2^2), half-split RoPE over the full head, theta 1e4."""
    gen = generator(seed)
    lengths = lengths_with_total(gen, 32, 16384, 4096)
    cls = uniform_ints(gen, 32, 0, 4096)
    return ragged_store(seed + 1, lengths=lengths, cache_lengths=cls, n_q_heads=64,
                        n_kv_heads=8, head_dim=128, page_size=128, rope_dim=128, theta=1e4,
                        interleaved=False, max_seq_len=8192, x_std=2.0, norm=True,
                        epsilon=1e-6, weight_offset=0.0, width=64,
                        name="per-head QK RMSNorm + RoPE + paged store: 64q/8kv heads, d128, "
                             "16384 tokens over 32 sequences")


def dual_band_minimax_in_place(seed: int = 0) -> DualBand:
    """dual_band_minimax with both key caches updated in place: K is read from the cache
    slots (which hold N(0,1) K rows), V is not touched."""
    gen = generator(seed)
    lengths = lengths_with_total(gen, 64, 32768, 4096)
    cls = uniform_ints(gen, 64, 0, 4096)
    return dual_band(seed + 1, lengths=lengths, cache_lengths=cls, main_q_heads=64,
                     main_kv_heads=8, index_q_heads=8, index_kv_heads=1, head_dim=128,
                     main_page_size=128, index_page_size=64, rope_dim=64, theta=1e4,
                     interleaved=True, max_seq_len=8192, k_in_place=True,
                     name="dual-band fused launch, key caches updated in place: main "
                          "64q/8kv + index 8q/1k, d128, partial RoPE 64, 32768 tokens")


def dual_band_minimax(seed: int = 0) -> DualBand:
    """main GQA band 64 Q / 8 KV heads + index band 8 IndexQ / 1 K-only head, head_dim 128,
    partial RoPE over 64 columns, eps 1e-6, 32768 tokens over 64 sequences (each <= 4096),
    cache_lengths U[0, 4096], page_size 128 (main, K+V) / 64 (index, K only)."""
    gen = generator(seed)
    lengths = lengths_with_total(gen, 64, 32768, 4096)
    cls = uniform_ints(gen, 64, 0, 4096)
    return dual_band(seed + 1, lengths=lengths, cache_lengths=cls, main_q_heads=64,
                     main_kv_heads=8, index_q_heads=8, index_kv_heads=1, head_dim=128,
                     main_page_size=128, index_page_size=64, rope_dim=64, theta=1e4,
                     interleaved=True, max_seq_len=8192,
                     name="dual-band fused launch: main 64q/8kv + index 8q/1k, d128, "
                          "partial RoPE 64, 32768 tokens over 64 sequences")


def radd_minimax(seed: int = 0) -> Radd:
    """kv_cache_radd of bf16 [32768, 2 * 1024] into the main cache (8 KV heads, head_dim
    128, page_size 128) at the rows of 32768 tokens over 64 sequences, batch_offset 0."""
    gen = generator(seed)
    lengths = lengths_with_total(gen, 64, 32768, 4096)
    cls = uniform_ints(gen, 64, 0, 4096)
    return radd(seed + 1, lengths=lengths, cache_lengths=cls, n_kv_heads=8, head_dim=128,
                page_size=128, batch_offset=0,
                name="kv_cache_radd: bf16 [32768, 2048] into the main cache, page 128")


# ------------------------------------------------------- GEMV + partial RMSNorm inputs --

@dataclass
class GemvNorm:
    """One input row x [k], weight W [n, k] (y = x W^T), gamma [n_normed]; the outputs start
    as random-bit sentinels."""
    x: torch.Tensor
    weight: torch.Tensor
    gamma: torch.Tensor
    epsilon: float
    weight_offset: float
    normed_output: torch.Tensor
    unnormed_output: torch.Tensor
    name: str = ""

    @property
    def n(self) -> int:
        return self.weight.shape[0]

    @property
    def k(self) -> int:
        return self.weight.shape[1]

    @property
    def n_normed(self) -> int:
        return self.normed_output.shape[0]


def gemv_norm(seed: int, *, n: int, k: int, n_normed: int, epsilon: float = 1e-6,
              weight_offset: float = 0.0, dtype: str = "bf16", row_pad: int = 0,
              name: str = "") -> GemvNorm:
    """x ~ N(0,1), W ~ N(0, 1/k) so that y ~ N(0,1), gamma ~ N(1, 0.1)."""
    gen = generator(seed)
    x = normal(gen, (k,), dtype=dtype)
    w = normal(gen, (n, k + row_pad), std=k ** -0.5, dtype=dtype)
    if row_pad:
        w = w[:, :k]
    gamma = normal(gen, (n_normed,), std=0.1, mean=1.0, dtype=dtype)
    normed = random_bits(gen, n_normed, dtype)
    unnormed = random_bits(gen, n - n_normed, dtype)
    return GemvNorm(x, w, gamma, epsilon, weight_offset, normed, unnormed, name)


def mla_kv_a_proj(seed: int = 0) -> GemvNorm:
    """The decode-time producer of a latent-attention KV cache entry: hidden 7168 projected
    to a 512-wide latent (RMS-normalised) and a 64-wide rotary key part (passed through),
    one token."""
    return gemv_norm(seed, n=576, k=7168, n_normed=512, epsilon=1e-6,
                     name="GEMV + partial RMSNorm: x [7168] @ W^T [576, 7168], first 512 "
                          "normed, last 64 passed through")
