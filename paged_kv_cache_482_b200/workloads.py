"""Seeded synthetic inputs for one paged decode-attention step.

This module only draws random numbers and lays out the bookkeeping that an
engine's block manager would hand to the kernels: context lengths, block
tables, the slot of every cached token, and the per-KV-head FP8 scales. It
holds none of the attention arithmetic. Both the CUDA path and the CPU checker
consume exactly what it returns, so neither can see the other's results.

Workload shapes follow the benchmark the pages describe: many sequences with
lengths drawn uniformly at random ("Nano-vLLM：轻量高效的大模型推理框架",
section 五 "使用方法", the ``bench.py`` run over 256 sequences; "DeepSeek复刻vLLM
反超原版", section "性能对决", 256 and 1024 sequences with lengths sampled
between 100 and 1024 tokens). No dataset is involved: Q/K/V are N(0, 1) draws
rounded to bf16, which stands in for real activations.

Layout conventions shared with the C-ABI (they are readings, not page text):

* KV pool ``[num_blocks, num_kv_heads, block_size, head_dim]`` (HND); a token
  in slot ``s`` lives in block ``s // block_size`` at offset
  ``s % block_size``.
* ``context_lens[i]`` counts the new token of step i; it is the last token of
  the sequence and is written by ``store_kvcache`` right before the decode.
* ``slot_mapping == -1`` marks a token that must not be written (its block is
  a shared prefix block that already holds it).
* unused tail entries of a block table row are ``-1``.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

# Pool fill patterns for slots that no token was written to. A bf16 quiet NaN
# and the E4M3 NaN code: any read of such a slot poisons the output.
CANARY_BF16 = 0x7FC0
CANARY_FP8 = 0x7F

CACHE_BF16 = "bf16"
CACHE_FP8 = "fp8_e4m3"  # one fp32 scale per KV head, drawn by the harness
CACHE_FP8_TOKEN = "fp8_e4m3_token"  # one fp32 scale per (token, KV head), written by the store


@dataclass(frozen=True)
class DecodeConfig:
    """Shape of one decode step over a paged KV cache.

    ``ctx_lo``/``ctx_hi`` bound the uniform (inclusive) context length. When
    ``prefix_tokens`` > 0 they bound the private suffix instead, and every
    sequence's context is ``prefix_tokens + suffix``.
    """

    name: str
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    ctx_lo: int
    ctx_hi: int
    cache_dtype: str = CACHE_BF16
    prefix_tokens: int = 0
    pool_blocks: int | None = None  # None: blocks in use plus 10 %
    scale: float | None = None  # None: 1/sqrt(head_dim)

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale is not None else 1.0 / math.sqrt(self.head_dim)

    @property
    def max_context(self) -> int:
        return self.prefix_tokens + self.ctx_hi

    @property
    def max_blocks_per_seq(self) -> int:
        return -(-self.max_context // self.block_size)

    def with_(self, **kw) -> "DecodeConfig":
        d = dict(self.__dict__)
        d.update(kw)
        return DecodeConfig(**d)


# The five workloads of the tier, by what they are.
CONFIGS: dict[str, DecodeConfig] = {
    c.name: c
    for c in (
        DecodeConfig("tiny", 4, 2, 1, 64, 16, 1, 300, pool_blocks=128, scale=1.0 / 8.0),
        DecodeConfig("qwen3_0.6b", 256, 16, 8, 128, 256, 100, 2048),
        DecodeConfig("qwen3_8b", 1024, 32, 8, 128, 256, 100, 2048),
        DecodeConfig("prefix_shared", 512, 32, 8, 128, 256, 0, 512, prefix_tokens=1024),
        DecodeConfig("long_fp8", 64, 32, 8, 128, 16, 16384, 32768, cache_dtype=CACHE_FP8),
        # the same long-context step with one scale per (token, KV head)
        DecodeConfig("long_fp8_token", 64, 32, 8, 128, 16, 16384, 32768, cache_dtype=CACHE_FP8_TOKEN),
    )
}


@dataclass
class Workload:
    """All inputs of one decode step plus the history that fills the pool.

    ``k_hist``/``v_hist``/``slot_hist`` hold every cached token that precedes
    the step (for a shared prefix: once). ``k_new``/``v_new``/``slot_new`` are
    the step's own tokens, one per sequence. ``hist_rows[i]`` lists the rows
    of ``k_hist`` that sequence i's blocks hold, in logical order.
    """

    cfg: DecodeConfig
    seed: int
    num_blocks: int
    q: torch.Tensor  # [S, nq, d] bf16
    k_new: torch.Tensor  # [S, nkv, d] bf16
    v_new: torch.Tensor
    slot_new: torch.Tensor  # [S] int32
    k_hist: torch.Tensor  # [H, nkv, d] bf16
    v_hist: torch.Tensor
    slot_hist: torch.Tensor  # [H] int32
    block_tables: torch.Tensor  # [S, max_blocks] int32, -1 padded
    context_lens: torch.Tensor  # [S] int32
    hist_rows: list = field(default_factory=list)  # per seq: 1-D int64 tensor (CPU)
    k_scale: torch.Tensor | None = None  # [nkv] fp32 (FP8 cache only)
    v_scale: torch.Tensor | None = None
    # sequences group_bounds[j] .. group_bounds[j + 1] - 1 share their first
    # group_prefix[j] tokens (the same physical blocks)
    group_bounds: list | None = None
    group_prefix: list | None = None

    @property
    def is_fp8(self) -> bool:
        return self.cfg.cache_dtype in (CACHE_FP8, CACHE_FP8_TOKEN)

    @property
    def token_scales(self) -> bool:
        return self.cfg.cache_dtype == CACHE_FP8_TOKEN

    def kv_tokens(self) -> int:
        return int(self.context_lens.sum().item())


def _randn_bf16(shape, gen: torch.Generator, device) -> torch.Tensor:
    """N(0,1) fp32 draws rounded to bf16 (round-to-nearest-even), chunked."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    flat = out.view(-1)
    chunk = 1 << 26
    for i in range(0, flat.numel(), chunk):
        n = min(chunk, flat.numel() - i)
        flat[i : i + n] = torch.randn(n, generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)
    return out


def _structure(cfg: DecodeConfig, seed: int, ctx_override=None):
    """Context lengths and physical block ids (device independent, CPU).
    ``ctx_override`` ({sequence: context length}) replaces drawn lengths, e.g.
    to put some sequences exactly on split-K partition edges."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    S, bs = cfg.num_seqs, cfg.block_size
    draws = torch.randint(cfg.ctx_lo, cfg.ctx_hi + 1, (S,), generator=g, dtype=torch.int64)
    ctx = draws + cfg.prefix_tokens
    for i, n in (ctx_override or {}).items():
        if not (max(1, cfg.prefix_tokens) <= int(n) <= cfg.max_context):
            raise ValueError(f"context length {n} outside [{max(1, cfg.prefix_tokens)}, {cfg.max_context}]")
        ctx[int(i)] = int(n)
    if cfg.prefix_tokens % bs:
        raise ValueError("a shared prefix must fill whole blocks")
    shared = cfg.prefix_tokens // bs
    own = [-(-int(c) // bs) - shared for c in ctx]
    in_use = shared + sum(own)
    nblk = cfg.pool_blocks if cfg.pool_blocks is not None else in_use + -(-in_use // 10)
    if nblk < in_use:
        raise ValueError(f"pool of {nblk} blocks cannot hold {in_use}")
    perm = torch.randperm(nblk, generator=g, dtype=torch.int64)
    tables = torch.full((S, cfg.max_blocks_per_seq), -1, dtype=torch.int64)
    tables[:, :shared] = perm[:shared]
    nxt = shared
    for i in range(S):
        tables[i, shared : shared + own[i]] = perm[nxt : nxt + own[i]]
        nxt += own[i]
    return ctx, tables, nblk


def generate(cfg: DecodeConfig, seed: int = 0, device: str | torch.device = "cpu", ctx_override=None) -> Workload:
    """Draw one decode step's inputs for ``cfg``.

    Lengths and block ids come from a CPU generator seeded with ``seed`` and
    are the same on every device (``ctx_override`` replaces chosen lengths).
    Q/K/V come from a generator on ``device`` seeded with ``seed + 1``
    (torch's CPU and CUDA generators give different streams, so data drawn on
    different devices differ; each is reproducible).
    """
    device = torch.device(device)
    ctx, tables, nblk = _structure(cfg, seed, ctx_override)
    S, nkv, d, bs = cfg.num_seqs, cfg.num_kv_heads, cfg.head_dim, cfg.block_size
    P = cfg.prefix_tokens

    # Row lists: the shared prefix once, then each sequence's own cached tokens
    # (every position below its last one).
    hist_rows = []
    own_start = []
    n = P
    for i in range(S):
        own = max(int(ctx[i]) - 1 - P, 0)
        own_start.append(n)
        n += own
    H = n
    pos = torch.empty(H, dtype=torch.int64)
    seq_of = torch.empty(H, dtype=torch.int64)
    pos[:P] = torch.arange(P)
    seq_of[:P] = 0  # prefix rows use any sequence's table (all share it)
    for i in range(S):
        own = max(int(ctx[i]) - 1 - P, 0)
        s0 = own_start[i]
        pos[s0 : s0 + own] = torch.arange(P, P + own)
        seq_of[s0 : s0 + own] = i
        # The shared blocks always hold the whole prefix.
        rows = torch.cat([torch.arange(P), torch.arange(s0, s0 + own)])
        hist_rows.append(rows)
    slot_hist = tables[seq_of, pos // bs] * bs + pos % bs

    last = ctx - 1
    slot_new = tables[torch.arange(S), last // bs] * bs + last % bs
    # The step's token at a position inside the shared prefix is already cached.
    slot_new = torch.where(last < P, torch.full_like(slot_new, -1), slot_new)

    gd = torch.Generator(device=device).manual_seed(seed + 1)
    q = _randn_bf16((S, cfg.num_q_heads, d), gd, device)
    k_hist = _randn_bf16((H, nkv, d), gd, device)
    v_hist = _randn_bf16((H, nkv, d), gd, device)
    k_new = _randn_bf16((S, nkv, d), gd, device)
    v_new = _randn_bf16((S, nkv, d), gd, device)

    wl = Workload(
        cfg=cfg,
        seed=seed,
        num_blocks=nblk,
        q=q,
        k_new=k_new,
        v_new=v_new,
        slot_new=slot_new.to(torch.int32).to(device),
        k_hist=k_hist,
        v_hist=v_hist,
        slot_hist=slot_hist.to(torch.int32).to(device),
        block_tables=tables.to(torch.int32).to(device),
        context_lens=ctx.to(torch.int32).to(device),
        hist_rows=hist_rows,
        group_bounds=[0, S],
        group_prefix=[P],
    )
    if cfg.cache_dtype == CACHE_FP8:
        # One fp32 scale per KV head: the head's absolute maximum over every
        # token of the step, divided by the largest E4M3 magnitude (448).
        written = (slot_new >= 0).to(device)
        kmax = k_hist.abs().amax(dim=(0, 2)) if H else torch.zeros(nkv, dtype=torch.bfloat16, device=device)
        vmax = v_hist.abs().amax(dim=(0, 2)) if H else torch.zeros(nkv, dtype=torch.bfloat16, device=device)
        if bool(written.any()):
            kmax = torch.maximum(kmax, k_new[written].abs().amax(dim=(0, 2)))
            vmax = torch.maximum(vmax, v_new[written].abs().amax(dim=(0, 2)))
        # An all-zero head would give scale 0; any positive scale then encodes it exactly.
        one = torch.ones_like(kmax)
        kmax = torch.where(kmax > 0, kmax, one)
        vmax = torch.where(vmax > 0, vmax, one)
        wl.k_scale = kmax.float() / 448.0
        wl.v_scale = vmax.float() / 448.0
    elif cfg.cache_dtype not in (CACHE_BF16, CACHE_FP8_TOKEN):
        raise ValueError(cfg.cache_dtype)
    return wl


def merge(parts: list[Workload], name: str = "merged") -> Workload:
    """One batch made of several workloads of the same heads, head size, block
    size and cache type: their pools side by side (block ids and slots
    offset), their sequences one after the other. Each part's sequences stay
    a group with the part's shared prefix (``group_bounds``). One scale per
    KV head becomes the largest of the parts' (inputs both sides read)."""
    c0 = parts[0].cfg
    for w in parts:
        c = w.cfg
        if (c.num_q_heads, c.num_kv_heads, c.head_dim, c.block_size, c.cache_dtype) != \
                (c0.num_q_heads, c0.num_kv_heads, c0.head_dim, c0.block_size, c0.cache_dtype):
            raise ValueError("parts must share heads, head size, block size and cache type")
    bs = c0.block_size
    width = max(w.block_tables.shape[1] for w in parts)
    tables, slots_h, slots_n, hist_rows = [], [], [], []
    blk_off, row_off = 0, 0
    for w in parts:
        bt = w.block_tables.cpu().long()
        bt = torch.where(bt >= 0, bt + blk_off, bt)
        pad = torch.full((bt.shape[0], width - bt.shape[1]), -1, dtype=torch.long)
        tables.append(torch.cat([bt, pad], dim=1))
        sh, sn = w.slot_hist.cpu().long(), w.slot_new.cpu().long()
        slots_h.append(torch.where(sh >= 0, sh + blk_off * bs, sh))
        slots_n.append(torch.where(sn >= 0, sn + blk_off * bs, sn))
        hist_rows += [r + row_off for r in w.hist_rows]
        blk_off += w.num_blocks
        row_off += w.k_hist.shape[0]
    ctx = torch.cat([w.context_lens.cpu() for w in parts])
    dev = parts[0].q.device
    cfg = c0.with_(name=name, num_seqs=int(ctx.numel()), ctx_lo=1, ctx_hi=int(ctx.max()), prefix_tokens=0,
                   pool_blocks=blk_off)
    wl = Workload(cfg=cfg, seed=parts[0].seed, num_blocks=blk_off,
                  q=torch.cat([w.q for w in parts]), k_new=torch.cat([w.k_new for w in parts]),
                  v_new=torch.cat([w.v_new for w in parts]), slot_new=torch.cat(slots_n).to(torch.int32).to(dev),
                  k_hist=torch.cat([w.k_hist for w in parts]), v_hist=torch.cat([w.v_hist for w in parts]),
                  slot_hist=torch.cat(slots_h).to(torch.int32).to(dev),
                  block_tables=torch.cat(tables).to(torch.int32).to(dev), context_lens=ctx.to(torch.int32).to(dev),
                  hist_rows=hist_rows)
    if c0.cache_dtype == CACHE_FP8:
        wl.k_scale = torch.stack([w.k_scale for w in parts]).amax(0)
        wl.v_scale = torch.stack([w.v_scale for w in parts]).amax(0)
    sizes = [w.cfg.num_seqs for w in parts]
    wl.group_bounds = [0] + list(torch.tensor(sizes).cumsum(0).tolist())
    wl.group_prefix = [w.cfg.prefix_tokens for w in parts]
    return wl


def scale_pools(num_blocks: int, num_kv_heads: int, block_size: int, device="cpu"):
    """Per-token scale pools [num_blocks, num_kv_heads, block_size] fp32 for
    the E4M3 cache with per-token scales, NaN where no token was stored (any
    read of an unwritten scale poisons the output)."""
    shape = (num_blocks, num_kv_heads, block_size)
    return (torch.full(shape, float("nan"), dtype=torch.float32, device=device),
            torch.full(shape, float("nan"), dtype=torch.float32, device=device))


def subset_for_seqs(wl: Workload, seq_ids) -> dict:
    """The rows one needs to rebuild the pool blocks of ``seq_ids`` only.

    Returns host tensors: the history rows (and their slots) that live in
    those sequences' blocks, plus the sequences' step inputs. Used to check a
    sample of a full-size step on the CPU.
    """
    ids = torch.as_tensor(list(seq_ids), dtype=torch.int64)
    rows = torch.unique(torch.cat([wl.hist_rows[int(i)] for i in ids]))
    dev_rows = rows.to(wl.k_hist.device)
    dev_ids = ids.to(wl.q.device)
    return dict(
        seq_ids=ids,
        k_hist=wl.k_hist[dev_rows].cpu(),
        v_hist=wl.v_hist[dev_rows].cpu(),
        slot_hist=wl.slot_hist[dev_rows].cpu(),
        q=wl.q[dev_ids].cpu(),
        k_new=wl.k_new[dev_ids].cpu(),
        v_new=wl.v_new[dev_ids].cpu(),
        slot_new=wl.slot_new[dev_ids].cpu(),
        block_tables=wl.block_tables[dev_ids].cpu(),
        context_lens=wl.context_lens[dev_ids].cpu(),
    )


def logical_kv(wl: Workload, i: int):
    """Sequence i's K and V rows ``[ctx, nkv, d]`` in logical token order.

    Taken from the drawn rows themselves (not from any pool), so a check built
    on it is independent of the pool layout, the block tables and the slots.
    """
    cfg = wl.cfg
    P = cfg.prefix_tokens
    ctx = int(wl.context_lens[i])
    rows = wl.hist_rows[i].to(wl.k_hist.device)
    k = wl.k_hist[rows]
    v = wl.v_hist[rows]
    if ctx > P:  # the step's own token is the last one
        k = torch.cat([k, wl.k_new[i : i + 1]])
        v = torch.cat([v, wl.v_new[i : i + 1]])
    return k[:ctx], v[:ctx]


# ---------------------------------------------------------------- prefill
#
# Chunked prefill ("nano-vllm-lite：深入理解LLM推理机制的教育级开源项目", section
# 核心技术改进 2 "Chunked Prefill"): a long prompt is prefilled in chunks that
# are scheduled together with decode requests. A sequence's step brings a
# chunk of c new tokens on top of the h tokens it already has in the cache;
# its context is h + c and the chunk is the last c positions. A decode
# request in the same batch is the case c = 1.


@dataclass(frozen=True)
class PrefillConfig:
    """Shape of one chunked-prefill step: per sequence a cached history of
    ``hist_lo..hist_hi`` tokens and a chunk of ``chunk_lo..chunk_hi`` new
    tokens (uniform, inclusive). ``decode_seqs`` more sequences join the same
    batch with one new token each (history ``decode_hist_lo..decode_hist_hi``)."""

    name: str
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    hist_lo: int
    hist_hi: int
    chunk_lo: int
    chunk_hi: int
    cache_dtype: str = CACHE_BF16
    decode_seqs: int = 0
    decode_hist_lo: int = 0
    decode_hist_hi: int = 0
    pool_blocks: int | None = None
    scale: float | None = None

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale is not None else 1.0 / math.sqrt(self.head_dim)

    @property
    def total_seqs(self) -> int:
        return self.num_seqs + self.decode_seqs

    @property
    def max_context(self) -> int:
        return max(self.hist_hi + self.chunk_hi, self.decode_hist_hi + 1)

    @property
    def max_blocks_per_seq(self) -> int:
        return -(-self.max_context // self.block_size)

    def with_(self, **kw) -> "PrefillConfig":
        d = dict(self.__dict__)
        d.update(kw)
        return PrefillConfig(**d)


PREFILL_CONFIGS: dict[str, PrefillConfig] = {
    c.name: c
    for c in (
        PrefillConfig("prefill_tiny", 3, 4, 2, 64, 16, 0, 40, 1, 70, pool_blocks=64, scale=1.0 / 8.0),
        # Qwen3-8B-shaped layer, 16 prompts each advancing by a 512-token chunk
        PrefillConfig("prefill_qwen3_8b", 16, 32, 8, 128, 256, 0, 3584, 512, 512),
        # the same chunks scheduled together with 240 decode requests
        PrefillConfig("prefill_mixed", 4, 32, 8, 128, 256, 0, 3584, 512, 512, decode_seqs=240,
                      decode_hist_lo=100, decode_hist_hi=2047),
        PrefillConfig("prefill_fp8", 8, 32, 8, 128, 16, 1024, 8192, 256, 1024, cache_dtype=CACHE_FP8),
        PrefillConfig("prefill_fp8_token", 8, 32, 8, 128, 16, 1024, 8192, 256, 1024, cache_dtype=CACHE_FP8_TOKEN),
    )
}


@dataclass
class PrefillWorkload:
    """All inputs of one chunked-prefill step plus the history that fills the pool.

    Rows of ``q``/``k_new``/``v_new``/``slot_new`` are the chunk tokens of all
    sequences back to back (sequence i owns rows ``cu_q_lens[i]`` to
    ``cu_q_lens[i+1] - 1``). ``k_hist``/``v_hist``/``slot_hist`` are the cached
    tokens before the chunks; ``hist_rows[i]`` lists sequence i's history rows
    in logical order.
    """

    cfg: PrefillConfig
    seed: int
    num_blocks: int
    q: torch.Tensor  # [T, nq, d] bf16
    k_new: torch.Tensor  # [T, nkv, d] bf16
    v_new: torch.Tensor
    slot_new: torch.Tensor  # [T] int32
    k_hist: torch.Tensor  # [H, nkv, d] bf16
    v_hist: torch.Tensor
    slot_hist: torch.Tensor  # [H] int32
    block_tables: torch.Tensor  # [S, max_blocks] int32, -1 padded
    cu_q_lens: torch.Tensor  # [S + 1] int32
    context_lens: torch.Tensor  # [S] int32
    hist_rows: list = field(default_factory=list)
    k_scale: torch.Tensor | None = None
    v_scale: torch.Tensor | None = None

    @property
    def is_fp8(self) -> bool:
        return self.cfg.cache_dtype in (CACHE_FP8, CACHE_FP8_TOKEN)

    @property
    def token_scales(self) -> bool:
        return self.cfg.cache_dtype == CACHE_FP8_TOKEN

    @property
    def total_q(self) -> int:
        return int(self.q.shape[0])


def generate_prefill(cfg: PrefillConfig, seed: int = 0, device: str | torch.device = "cpu") -> PrefillWorkload:
    """Draw one chunked-prefill step's inputs for ``cfg`` (structure from a CPU
    generator seeded with ``seed``, data from a ``device`` generator seeded
    with ``seed + 1``, as in :func:`generate`)."""
    device = torch.device(device)
    g = torch.Generator(device="cpu").manual_seed(seed)
    S, bs, nkv, d = cfg.total_seqs, cfg.block_size, cfg.num_kv_heads, cfg.head_dim
    P, D = cfg.num_seqs, cfg.decode_seqs
    hist = torch.cat([torch.randint(cfg.hist_lo, cfg.hist_hi + 1, (P,), generator=g, dtype=torch.int64),
                      torch.randint(cfg.decode_hist_lo, cfg.decode_hist_hi + 1, (D,), generator=g,
                                    dtype=torch.int64)])
    chunk = torch.cat([torch.randint(cfg.chunk_lo, cfg.chunk_hi + 1, (P,), generator=g, dtype=torch.int64),
                       torch.ones(D, dtype=torch.int64)])
    ctx = hist + chunk
    nb = [-(-int(c) // bs) for c in ctx]
    in_use = sum(nb)
    nblk = cfg.pool_blocks if cfg.pool_blocks is not None else in_use + -(-in_use // 10)
    if nblk < in_use:
        raise ValueError(f"pool of {nblk} blocks cannot hold {in_use}")
    perm = torch.randperm(nblk, generator=g, dtype=torch.int64)
    tables = torch.full((S, cfg.max_blocks_per_seq), -1, dtype=torch.int64)
    nxt = 0
    for i in range(S):
        tables[i, : nb[i]] = perm[nxt : nxt + nb[i]]
        nxt += nb[i]
    cu = torch.zeros(S + 1, dtype=torch.int64)
    cu[1:] = torch.cumsum(chunk, 0)
    H = int(hist.sum())
    hist_start = torch.zeros(S + 1, dtype=torch.int64)
    hist_start[1:] = torch.cumsum(hist, 0)
    seq_h = torch.repeat_interleave(torch.arange(S), hist)
    pos_h = torch.arange(H) - hist_start[seq_h]
    slot_hist = tables[seq_h, pos_h // bs] * bs + pos_h % bs
    T = int(cu[-1])
    seq_q = torch.repeat_interleave(torch.arange(S), chunk)
    pos_q = hist[seq_q] + torch.arange(T) - cu[seq_q]
    slot_new = tables[seq_q, pos_q // bs] * bs + pos_q % bs
    hist_rows = [torch.arange(int(hist_start[i]), int(hist_start[i + 1])) for i in range(S)]

    gd = torch.Generator(device=device).manual_seed(seed + 1)
    q = _randn_bf16((T, cfg.num_q_heads, d), gd, device)
    k_hist = _randn_bf16((H, nkv, d), gd, device)
    v_hist = _randn_bf16((H, nkv, d), gd, device)
    k_new = _randn_bf16((T, nkv, d), gd, device)
    v_new = _randn_bf16((T, nkv, d), gd, device)
    wl = PrefillWorkload(
        cfg=cfg, seed=seed, num_blocks=nblk, q=q, k_new=k_new, v_new=v_new,
        slot_new=slot_new.to(torch.int32).to(device), k_hist=k_hist, v_hist=v_hist,
        slot_hist=slot_hist.to(torch.int32).to(device), block_tables=tables.to(torch.int32).to(device),
        cu_q_lens=cu.to(torch.int32).to(device), context_lens=ctx.to(torch.int32).to(device), hist_rows=hist_rows,
    )
    if cfg.cache_dtype == CACHE_FP8:
        # per KV head: absolute maximum over every stored token / 448
        kmax = torch.cat([k_hist, k_new]).abs().amax(dim=(0, 2)).float()
        vmax = torch.cat([v_hist, v_new]).abs().amax(dim=(0, 2)).float()
        one = torch.ones_like(kmax)
        wl.k_scale = torch.where(kmax > 0, kmax, one) / 448.0
        wl.v_scale = torch.where(vmax > 0, vmax, one) / 448.0
    elif cfg.cache_dtype not in (CACHE_BF16, CACHE_FP8_TOKEN):
        raise ValueError(cfg.cache_dtype)
    return wl


def prefill_logical_kv(wl: PrefillWorkload, i: int):
    """Sequence i's K and V rows ``[ctx, nkv, d]`` in logical order, from the
    drawn rows (history, then its chunk), not from any pool."""
    rows = wl.hist_rows[i].to(wl.k_hist.device)
    a, b = int(wl.cu_q_lens[i]), int(wl.cu_q_lens[i + 1])
    return torch.cat([wl.k_hist[rows], wl.k_new[a:b]]), torch.cat([wl.v_hist[rows], wl.v_new[a:b]])


# ------------------------------------------------------------ add + RMSNorm
#
# The residual add and RMSNorm around the attention of a layer
# ("nano-vllm-lite：深入理解LLM推理机制的教育级开源项目", section 核心技术改进 1
# "CUDA融合内核：Add+RMSNorm"): rows of hidden states, their residual stream
# and the norm weight.


@dataclass(frozen=True)
class NormConfig:
    name: str
    num_tokens: int
    hidden: int
    eps: float = 1e-6
    residual: bool = True


NORM_CONFIGS: dict[str, NormConfig] = {
    c.name: c
    for c in (
        NormConfig("norm_tiny", 5, 64),
        NormConfig("norm_qwen3_0.6b", 256, 1024),
        # Qwen3-8B hidden size, one decode step of 1024 sequences
        NormConfig("norm_qwen3_8b_decode", 1024, 4096),
        # Qwen3-8B hidden size, a chunked-prefill step of 16 x 512 tokens (larger than L2 in total)
        NormConfig("norm_qwen3_8b", 8192, 4096),
    )
}


@dataclass
class NormWorkload:
    cfg: NormConfig
    seed: int
    x: torch.Tensor  # [T, H] bf16
    residual: torch.Tensor | None  # [T, H] bf16
    weight: torch.Tensor  # [H] bf16


def generate_norm(cfg: NormConfig, seed: int = 0, device: str | torch.device = "cpu") -> NormWorkload:
    """x and the residual are N(0, 1) rounded to bf16; the weight is
    1 + 0.1 N(0, 1) rounded to bf16 (a trained norm weight stays near 1)."""
    device = torch.device(device)
    g = torch.Generator(device=device).manual_seed(seed + 1)
    x = _randn_bf16((cfg.num_tokens, cfg.hidden), g, device)
    r = _randn_bf16((cfg.num_tokens, cfg.hidden), g, device) if cfg.residual else None
    w = (1.0 + 0.1 * torch.randn(cfg.hidden, generator=g, device=device)).to(torch.bfloat16)
    return NormWorkload(cfg, seed, x, r, w)


# ------------------------------------------------- rotary embedding + store
#
# The rotary position embedding of q and k that precedes the cache write
# (the FP8 cache of "nano-vllm-lite：深入理解LLM推理机制的教育级开源项目", section
# 核心技术改进 3, stores the rotated keys). The rotation itself is the RoFormer
# paper's (Su et al., 2021); an engine builds its cos/sin table once.

ROPE_HALF = 0  # pairs (i, i + d/2)
ROPE_INTERLEAVED = 1  # pairs (2i, 2i + 1)


def rope_cache(max_position: int, head_dim: int, base: float = 1_000_000.0, device="cpu") -> torch.Tensor:
    """The table a rotary embedding reads: row m holds cos(m theta_i) for
    i < head_dim / 2, then sin(m theta_i), theta_i = base^(-2i / head_dim),
    evaluated in fp64 and stored as fp32 ``[max_position, head_dim]``."""
    i = torch.arange(head_dim // 2, dtype=torch.float64)
    theta = base ** (-2.0 * i / head_dim)
    ang = torch.arange(max_position, dtype=torch.float64)[:, None] * theta[None, :]
    return torch.cat([torch.cos(ang), torch.sin(ang)], dim=1).to(torch.float32).contiguous().to(device)


@dataclass(frozen=True)
class RopeConfig:
    """One step of rotary embedding + store: num_tokens new tokens (one per
    sequence at decode, or the tokens of prefill chunks) at positions below
    max_position, written into distinct slots of a pool."""

    name: str
    num_tokens: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    max_position: int
    style: int = ROPE_HALF
    cache_dtype: str = CACHE_BF16
    base: float = 1_000_000.0
    pool_blocks: int | None = None  # None: enough for every token, plus 10 %

    @property
    def is_fp8(self) -> bool:
        return self.cache_dtype in (CACHE_FP8, CACHE_FP8_TOKEN)

    @property
    def token_scales(self) -> bool:
        return self.cache_dtype == CACHE_FP8_TOKEN

    def with_(self, **kw) -> "RopeConfig":
        d = dict(self.__dict__)
        d.update(kw)
        return RopeConfig(**d)


ROPE_CONFIGS: dict[str, RopeConfig] = {
    c.name: c
    for c in (
        RopeConfig("rope_tiny", 4, 2, 1, 64, 16, 300),
        # one decode step of the Qwen3-8B-shaped layer: 1024 sequences at positions below 2048
        RopeConfig("rope_qwen3_8b", 1024, 32, 8, 128, 256, 2048),
        RopeConfig("rope_qwen3_8b_fp8", 1024, 32, 8, 128, 256, 2048, cache_dtype=CACHE_FP8_TOKEN),
        # a chunked-prefill step of 16 x 512 tokens (inputs and cache writes above L2 in total)
        RopeConfig("rope_prefill_qwen3_8b", 8192, 32, 8, 128, 256, 32768),
        RopeConfig("rope_prefill_qwen3_8b_fp8", 8192, 32, 8, 128, 256, 32768, cache_dtype=CACHE_FP8_TOKEN),
    )
}


@dataclass
class RopeWorkload:
    cfg: RopeConfig
    seed: int
    num_blocks: int
    q: torch.Tensor  # [N, nq, d] bf16
    k: torch.Tensor  # [N, nkv, d] bf16
    v: torch.Tensor
    positions: torch.Tensor  # [N] int32
    slot_mapping: torch.Tensor  # [N] int32, distinct slots
    cos_sin: torch.Tensor  # [max_position, d] fp32
    k_scale: torch.Tensor | None = None  # [nkv] fp32 (one scale per KV head)
    v_scale: torch.Tensor | None = None

    @property
    def is_fp8(self) -> bool:
        return self.cfg.is_fp8


def generate_rope(cfg: RopeConfig, seed: int = 0, device: str | torch.device = "cpu") -> RopeWorkload:
    """Positions uniform in [0, max_position); slots distinct, from a seeded
    permutation of the pool; q/k/v N(0, 1) rounded to bf16."""
    device = torch.device(device)
    g = torch.Generator(device="cpu").manual_seed(seed)
    N, bs = cfg.num_tokens, cfg.block_size
    need = -(-N // bs)
    nblk = cfg.pool_blocks if cfg.pool_blocks is not None else need + -(-need // 10) + 1
    positions = torch.randint(0, cfg.max_position, (N,), generator=g, dtype=torch.int64)
    slots = torch.randperm(nblk * bs, generator=g)[:N]
    gd = torch.Generator(device=device).manual_seed(seed + 1)
    q = _randn_bf16((N, cfg.num_q_heads, cfg.head_dim), gd, device)
    k = _randn_bf16((N, cfg.num_kv_heads, cfg.head_dim), gd, device)
    v = _randn_bf16((N, cfg.num_kv_heads, cfg.head_dim), gd, device)
    wl = RopeWorkload(cfg, seed, nblk, q, k, v, positions.to(torch.int32).to(device),
                      slots.to(torch.int32).to(device), rope_cache(cfg.max_position, cfg.head_dim, cfg.base, device))
    if cfg.cache_dtype == CACHE_FP8:
        # one scale per KV head over the rows as drawn: rotation keeps each
        # pair's norm, so |rotated| <= sqrt(2) * amax; the scale leaves room
        one = torch.ones(cfg.num_kv_heads, dtype=torch.float32, device=device)
        km = k.float().abs().amax(dim=(0, 2)) if N else one
        vm = v.float().abs().amax(dim=(0, 2)) if N else one
        wl.k_scale = torch.where(km > 0, km, one) * 1.5 / 448.0
        wl.v_scale = torch.where(vm > 0, vm, one) / 448.0
    return wl
