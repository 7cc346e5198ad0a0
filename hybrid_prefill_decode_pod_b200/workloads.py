"""Seeded synthetic hybrid batches (inputs only; no attention arithmetic here).

A hybrid batch, in the sense of the POD-Attention pages ("POD-Attention:
Unlocking Full Prefill-Decode Overlap", §2.1 Large Language Model Inference),
is one or more chunked-prefill requests plus many single-token decodes. Each
prefill request p has ``prior_p`` cached tokens and a chunk of ``chunk_p`` new
tokens; each decode request r has a context of ``ctx_r`` tokens. All K/V that
the call reads are already in the cache (the chunk's own K/V sit at positions
prior..prior+chunk-1).

This module is shared by the tests, the benchmark and the smoke check. Both
the CUDA path and the fp64 oracle consume the tensors it returns. It only
draws numbers and lays them out in memory:

* generator: ``torch.Generator('cpu').manual_seed(seed)``;
* draw order: ranged integer contexts (``torch.randint(a, b + 1)``), prefill
  Q ``[sum chunk, H, d]``, then per prefill request K ``[prior + chunk, Hk, d]``
  and V, then decode Q ``[n_dec, H, d]``, then per decode request K
  ``[ctx, Hk, d]`` and V, then (paged layout only) one ``randperm`` of the
  physical block ids;
* every float draw is ``torch.randn(..., dtype=float32)`` rounded to bfloat16
  (round to nearest even).

Paged layout: the pool holds ``sum over all requests (prefill first, then
decode) of ceil(len / page)`` blocks of ``[page, Hk, d]``. Logical block b of
the i-th request (in that order) lives at physical block
``perm[first_block_i + b]``. Unused slots of a partial last block are zero.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence, Tuple

import torch

PAGE_SIZE = 16


@dataclasses.dataclass(frozen=True)
class HybridConfig:
    """Shape of one synthetic hybrid batch.

    ``decode_ctx`` is either an explicit tuple of contexts or ``None`` with
    ``decode_range=(a, b, n)`` meaning n contexts drawn uniformly from the
    integers a..b inclusive.
    """

    name: str
    num_qo_heads: int
    num_kv_heads: int
    head_dim: int
    prefill: Tuple[Tuple[int, int], ...]  # (prior, chunk) per request
    decode_ctx: Optional[Tuple[int, ...]] = None
    decode_range: Optional[Tuple[int, int, int]] = None
    paged: bool = False
    seed: int = 0

    @property
    def group(self) -> int:
        return self.num_qo_heads // self.num_kv_heads


# The five hybrid batches the benchmark and parity tests are defined on.
CONFIGS = {
    "tiny": HybridConfig(
        "tiny", 4, 2, 64, prefill=((64, 32),), decode_ctx=(40, 77, 128, 200)),
    "llama3_8b": HybridConfig(
        "llama3_8b", 32, 8, 128, prefill=((4096, 512),), decode_ctx=(4096,) * 64),
    "decode_heavy": HybridConfig(
        "decode_heavy", 32, 8, 128, prefill=((1024, 256),),
        decode_range=(512, 8192, 256)),
    "long_context": HybridConfig(
        "long_context", 64, 8, 128, prefill=((16384, 1024),),
        decode_range=(16384, 32768, 16)),
    "paged": HybridConfig(
        "paged", 32, 8, 128, prefill=((2048, 512), (8192, 512)),
        decode_range=(1024, 16384, 128), paged=True),
}

# Smaller batches of the same shape families, for profiler captures (a capture
# replays each launch many times, so it is taken on a reduced case).
PROBE_CONFIGS = {
    "long_context_probe": HybridConfig(
        "long_context_probe", 64, 8, 128, prefill=((4096, 1024),), decode_ctx=(4096,) * 16),
}
# Variants of the pages' model shapes (the summary's §A.2 / §A.3.5 list
# Llama-2-7B, Llama-3-8B and Yi-6B; their attention shapes are those of the
# public model architectures: Llama-2-7B is multi-head, 32 heads of 128;
# Yi-6B groups 32 query heads over 4 KV heads of 128), a head_dim-64 mix, and
# a batch of many small chunks, each beside 64 decodes at context 4096.
VARIANT_CONFIGS = {
    "llama2_7b_mha": HybridConfig(
        "llama2_7b_mha", 32, 32, 128, prefill=((4096, 512),), decode_ctx=(4096,) * 64),
    "yi6b_g8": HybridConfig(
        "yi6b_g8", 32, 4, 128, prefill=((4096, 512),), decode_ctx=(4096,) * 64),
    "d64_mix": HybridConfig(
        "d64_mix", 16, 4, 64, prefill=((4096, 512),), decode_ctx=(4096,) * 64),
    # 16 chunks (the per-call maximum) of 1..40 tokens after 0..8192 cached tokens
    "many_chunks": HybridConfig(
        "many_chunks", 32, 8, 128,
        prefill=tuple(((2749 * i) % 8193, 1 + (37 * i) % 40) for i in range(16)),
        decode_ctx=(4096,) * 64),
}
PROBE_CONFIGS.update(VARIANT_CONFIGS)

# Chunked prefill of a 16K-token prompt in chunks of 512 beside 64 decodes at the
# same context (the paper's per-chunk study of a long prompt, restated on
# synthetic Llama-3-8B-shaped inputs): point i has prior 512 i and decodes at
# context 512 (i + 1), i = 0 .. 31.
for _i in range(32):
    PROBE_CONFIGS["chunked16k_%d" % _i] = HybridConfig(
        "chunked16k_%d" % _i, 32, 8, 128, prefill=((512 * _i, 512),),
        decode_ctx=(512 * (_i + 1),) * 64)

# Human-readable descriptions used in the benchmark's JSON line.
CONFIG_DESCRIPTIONS = {
    "tiny": "tiny hybrid batch: 1 prefill (prior 64 + chunk 32) + 4 decodes (40/77/128/200), 4 q / 2 kv heads, d 64",
    "llama3_8b": "Llama-3-8B-shaped: 32 q / 8 kv heads, d 128; 1 prefill chunk 512 after prior 4096 + 64 decodes at 4096",
    "decode_heavy": "decode-heavy: 32 q / 8 kv heads, d 128; 1 prefill chunk 256 after prior 1024 + 256 decodes U[512, 8192]",
    "long_context": "long-context 70B-like: 64 q / 8 kv heads, d 128; 1 prefill chunk 1024 after prior 16384 + 16 decodes U[16384, 32768]",
    "paged": "paged-KV: 32 q / 8 kv heads, d 128; 2 prefill chunks of 512 (priors 2048, 8192) + 128 decodes U[1024, 16384], 16-token blocks, permuted",
    "long_context_probe": "profiling probe: 64 q / 8 kv heads, d 128; 1 prefill chunk 1024 after prior 4096 + 16 decodes at 4096",
    "llama2_7b_mha": "Llama-2-7B-shaped (multi-head): 32 q / 32 kv heads, d 128; 1 prefill chunk 512 after prior 4096 + 64 decodes at 4096",
    "yi6b_g8": "Yi-6B-shaped: 32 q / 4 kv heads, d 128; 1 prefill chunk 512 after prior 4096 + 64 decodes at 4096",
    "d64_mix": "head_dim 64: 16 q / 4 kv heads, d 64; 1 prefill chunk 512 after prior 4096 + 64 decodes at 4096",
    "many_chunks": "16 prefill chunks of 1-40 tokens after 0-8192 cached tokens + 64 decodes at 4096; 32 q / 8 kv heads, d 128",
    **{"chunked16k_%d" % i: "chunk %d of a 16K prompt: 32 q / 8 kv heads, d 128; prefill chunk 512 after prior %d + 64 decodes at %d" % (i, 512 * i, 512 * (i + 1)) for i in range(32)},
}


def get_config(name: str) -> HybridConfig:
    return CONFIGS[name] if name in CONFIGS else PROBE_CONFIGS[name]


@dataclasses.dataclass
class HybridBatch:
    """Host (CPU) tensors of one hybrid batch, all bfloat16 unless noted."""

    cfg: HybridConfig
    priors: List[int]
    chunks: List[int]
    ctx: List[int]
    q_prefill: torch.Tensor            # [sum chunk, H, d]
    k_prefill: List[torch.Tensor]      # per request [prior + chunk, Hk, d]
    v_prefill: List[torch.Tensor]
    q_decode: torch.Tensor             # [n_dec, H, d]
    k_decode: List[torch.Tensor]       # per request [ctx, Hk, d]
    v_decode: List[torch.Tensor]
    # paged layout (None when contiguous)
    k_pool: Optional[torch.Tensor] = None   # [blocks, page, Hk, d]
    v_pool: Optional[torch.Tensor] = None
    block_table_prefill: Optional[torch.Tensor] = None  # int32 [n_prefill, max_blocks]
    block_table_decode: Optional[torch.Tensor] = None   # int32 [n_dec, max_blocks]

    @property
    def kv_lens_prefill(self) -> List[int]:
        return [p + c for p, c in zip(self.priors, self.chunks)]

    @property
    def total_prefill_tokens(self) -> int:
        return sum(self.chunks)

    @property
    def num_decodes(self) -> int:
        return len(self.ctx)


def _randn_bf16(g: torch.Generator, shape) -> torch.Tensor:
    return torch.randn(*shape, dtype=torch.float32, generator=g).to(torch.bfloat16)


def make_batch(cfg: HybridConfig, seed: Optional[int] = None,
               with_pool: Optional[bool] = None) -> HybridBatch:
    """Draw one batch for ``cfg`` in the documented order (see module doc)."""
    g = torch.Generator("cpu").manual_seed(cfg.seed if seed is None else seed)
    H, Hk, d = cfg.num_qo_heads, cfg.num_kv_heads, cfg.head_dim
    if cfg.decode_ctx is not None:
        ctx = [int(x) for x in cfg.decode_ctx]
    elif cfg.decode_range is not None:
        a, b, n = cfg.decode_range
        ctx = [int(x) for x in torch.randint(a, b + 1, (n,), generator=g)]
    else:
        ctx = []
    priors = [p for p, _ in cfg.prefill]
    chunks = [c for _, c in cfg.prefill]
    q_prefill = _randn_bf16(g, (sum(chunks), H, d))
    k_prefill, v_prefill = [], []
    for p, c in cfg.prefill:
        k_prefill.append(_randn_bf16(g, (p + c, Hk, d)))
        v_prefill.append(_randn_bf16(g, (p + c, Hk, d)))
    q_decode = _randn_bf16(g, (len(ctx), H, d))
    k_decode, v_decode = [], []
    for L in ctx:
        k_decode.append(_randn_bf16(g, (L, Hk, d)))
        v_decode.append(_randn_bf16(g, (L, Hk, d)))
    batch = HybridBatch(cfg, priors, chunks, ctx, q_prefill, k_prefill, v_prefill,
                        q_decode, k_decode, v_decode)
    if cfg.paged if with_pool is None else with_pool:
        build_pool(batch, g)
    return batch


def make_custom(H: int, Hk: int, d: int, prefill: Sequence[Tuple[int, int]],
                ctx: Sequence[int], seed: int = 0, paged: bool = False) -> HybridBatch:
    """A batch of explicit shape (for edge cases and scaled-down parity runs)."""
    cfg = HybridConfig("custom", H, Hk, d, prefill=tuple(tuple(x) for x in prefill),
                       decode_ctx=tuple(ctx), paged=paged, seed=seed)
    return make_batch(cfg)


def build_pool(batch: HybridBatch, g: Optional[torch.Generator] = None) -> None:
    """Lay the batch's K/V out in a permuted 16-token block pool.

    Draws the permutation from ``g`` (continuing the batch's stream) so that
    the contiguous and paged variants hold identical K/V values.
    """
    cfg = batch.cfg
    if g is None:
        g = torch.Generator("cpu").manual_seed(cfg.seed + 1)
    Hk, d = cfg.num_kv_heads, cfg.head_dim
    lens = batch.kv_lens_prefill + list(batch.ctx)
    nblk = [math.ceil(L / PAGE_SIZE) for L in lens]
    total = sum(nblk)
    perm = torch.randperm(total, generator=g).to(torch.int32)
    k_pool = torch.zeros(max(total, 1), PAGE_SIZE, Hk, d, dtype=torch.bfloat16)
    v_pool = torch.zeros_like(k_pool)
    ks = batch.k_prefill + batch.k_decode
    vs = batch.v_prefill + batch.v_decode
    tables = []
    first = 0
    for L, nb, k, v in zip(lens, nblk, ks, vs):
        phys = perm[first:first + nb]
        tables.append(phys)
        full = L // PAGE_SIZE
        if full:
            k_pool[phys[:full].long()] = k[: full * PAGE_SIZE].view(full, PAGE_SIZE, Hk, d)
            v_pool[phys[:full].long()] = v[: full * PAGE_SIZE].view(full, PAGE_SIZE, Hk, d)
        rem = L - full * PAGE_SIZE
        if rem:
            k_pool[int(phys[full]), :rem] = k[full * PAGE_SIZE:]
            v_pool[int(phys[full]), :rem] = v[full * PAGE_SIZE:]
        first += nb
    n_p = len(batch.priors)

    def _pad(ts):
        width = max([t.numel() for t in ts] + [1])
        out = torch.zeros(len(ts), width, dtype=torch.int32)
        for i, t in enumerate(ts):
            out[i, : t.numel()] = t
        return out

    batch.k_pool, batch.v_pool = k_pool, v_pool
    batch.block_table_prefill = _pad(tables[:n_p])
    batch.block_table_decode = _pad(tables[n_p:])


def algorithmic_work(H: int, Hk: int, d: int, priors: Sequence[int], chunks: Sequence[int],
                     ctx: Sequence[int], paged: bool = False):
    """FLOPs and bytes the attention must do (no tile rounding, no masked work).

    FLOPs: 2 for QK^T and 2 for PV per (query row, visible key, query head).
    Bytes: each K and V element once, Q read once, O written once (bf16), LSE
    written once (fp32), plus block-table bytes for the paged layout.
    Returns (flops_prefill, flops_decode, bytes_prefill, bytes_decode).
    """
    f_p = 0
    for p, c in zip(priors, chunks):
        f_p += 4 * d * H * (c * (p + 1) + c * (c - 1) // 2)
    f_d = 4 * d * H * sum(ctx)
    b_p = 0
    for p, c in zip(priors, chunks):
        b_p += (p + c) * Hk * d * 2 * 2 + c * H * d * 2 * 2 + c * H * 4
        if paged:
            b_p += math.ceil((p + c) / PAGE_SIZE) * 4
    b_d = 0
    for L in ctx:
        b_d += L * Hk * d * 2 * 2 + H * d * 2 * 2 + H * 4
        if paged:
            b_d += math.ceil(L / PAGE_SIZE) * 4
    return f_p, f_d, b_p, b_d
