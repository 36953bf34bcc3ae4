"""Seeded synthetic inputs for QSA sparse-attention prefill.

This module only draws inputs (Q, the K/V caches, the selected-slot lists);
it holds none of the attention arithmetic, and it is the one module that both
the CUDA path's callers and the oracle's callers share.

The shapes and index structure follow the QSA workloads: head dim 256, the
local GQA head shapes (16,2), (24,2), (12,1), (6,1), (3,1) (page "Qwen4-Exp
QSA llega al Ascend de Huawei", bullet "Formas de cabeza"), and per-token
lists of physical cache slots that combine a local causal window with
uniformly random earlier positions, padded with -1 (same page, section
"Nueve pruebas que pasaron").  A list for a token at position p of a sequence
starting at slot s_0 is:

* p - s_0 + 1 <= K: every causal slot s_0..p, then -1 (n_valid = p - s_0 + 1);
* otherwise: the L most recent slots p-L+1..p plus K-L distinct slots drawn
  uniformly from [s_0, p-L], sorted or in random order.

Torch generators draw everything, so the same seed yields the same values on
the same device type; CPU and CUDA generators differ from each other.  Every
consumer draws once and hands the same tensors to both sides of a comparison.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch

HEAD_DIM = 256
HEAD_SHAPES = ((3, 1), (6, 1), (12, 1), (16, 2), (24, 2))
CONFIG_SEED_BASE = 20261000


@dataclasses.dataclass
class Workload:
    name: str
    q: torch.Tensor                 # [T, Hq, D] bf16
    k_cache: torch.Tensor           # [S, Hkv, D] bf16 (may be a strided view)
    v_cache: torch.Tensor           # [S, Hkv, D] bf16 (same strides as k_cache)
    topk_idx: torch.Tensor          # [T, Hkv, K] int32, -1 = empty
    n_valid: Optional[torch.Tensor]  # [T, Hkv] int32 or None (= K)
    scale: float                    # 0.0 selects 1/sqrt(D)
    positions: torch.Tensor         # [T] int64: the token's own cache slot
    seq_start: torch.Tensor         # [T] int64: first slot of its sequence
    description: str = ""

    @property
    def shape(self):
        T, Hq, D = self.q.shape
        S, Hkv, _ = self.k_cache.shape
        return dict(T=T, Hq=Hq, Hkv=Hkv, D=D, K=self.topk_idx.shape[2], S=S)

    def to(self, device) -> "Workload":
        def mv(x):
            return None if x is None else x.to(device)
        return dataclasses.replace(
            self, q=mv(self.q), k_cache=mv(self.k_cache), v_cache=mv(self.v_cache),
            topk_idx=mv(self.topk_idx), n_valid=mv(self.n_valid),
            positions=mv(self.positions), seq_start=mv(self.seq_start))


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(int(seed))
    return g


def normal_bf16(shape, gen, device, std: float = 1.0) -> torch.Tensor:
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def normal_fp8(shape, gen, device, std: float = 1.0) -> torch.Tensor:
    """N(0, std^2) values stored as OCP FP8 E4M3 (torch float8_e4m3fn,
    round to nearest): a synthetic FP8 KV cache."""
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.float8_e4m3fn)


def random_subset_rows(lo: torch.Tensor, width: torch.Tensor, count: int, gen,
                       device, max_chunk_elems: int = 1 << 27) -> torch.Tensor:
    """For each row r, `count` distinct integers drawn uniformly from
    [lo[r], lo[r] + width[r]) (width[r] >= count).  Random keys + smallest-k:
    every count-subset is equally likely.  Returns int64 [rows, count]."""
    rows = lo.shape[0]
    out = torch.empty((rows, count), dtype=torch.int64, device=device)
    if rows == 0 or count == 0:
        return out
    wmax = int(width.max().item())
    chunk = max(1, min(rows, max_chunk_elems // max(wmax, 1)))
    ar = torch.arange(wmax, device=device)
    for r0 in range(0, rows, chunk):
        r1 = min(rows, r0 + chunk)
        keys = torch.rand((r1 - r0, wmax), generator=gen, device=device)
        keys.masked_fill_(ar[None, :] >= width[r0:r1, None], 2.0)
        sel = torch.topk(keys, count, dim=1, largest=False, sorted=False).indices
        out[r0:r1] = sel + lo[r0:r1, None]
    return out


def causal_lists(positions: torch.Tensor, seq_start: torch.Tensor, topk: int,
                 local: int, num_heads: int, gen, device, ordered: bool = True,
                 per_head: bool = True):
    """Selected-slot lists with the structure described in the module doc.

    Returns (idx int32 [T, H, K], n_valid int32 [T, H])."""
    T = positions.shape[0]
    H = num_heads if per_head else 1
    K = topk
    pos = positions.to(device=device, dtype=torch.int64)
    s0 = seq_start.to(device=device, dtype=torch.int64)
    n_caus = pos - s0 + 1
    full = n_caus > K                                       # rows with a random part
    idx = torch.full((T, H, K), -1, dtype=torch.int64, device=device)
    ar_k = torch.arange(K, device=device)
    # short rows: every causal slot s0..p, in order
    short_vals = s0[:, None] + ar_k[None, :]
    short_mask = ar_k[None, :] < n_caus[:, None]
    short = torch.where(short_mask, short_vals, torch.full_like(short_vals, -1))
    idx[:] = short[:, None, :]
    L = min(local, K)
    R = K - L
    rows_t = torch.nonzero(full).flatten()
    if rows_t.numel() > 0:
        nt = rows_t.numel()
        lo = s0[rows_t].repeat_interleave(H)
        width = (pos[rows_t] - L - s0[rows_t] + 1).repeat_interleave(H)
        rnd = random_subset_rows(lo, width, R, gen, device).view(nt, H, R)
        loc = (pos[rows_t, None] - L + 1 + torch.arange(L, device=device)[None, :])
        lst = torch.cat([rnd, loc[:, None, :].expand(nt, H, L)], dim=2)
        if ordered:
            lst = torch.sort(lst, dim=2).values
        else:
            perm = torch.argsort(torch.rand((nt, H, K), generator=gen, device=device), dim=2)
            lst = torch.gather(lst, 2, perm)
        idx[rows_t] = lst
    n_valid = torch.minimum(n_caus, torch.full_like(n_caus, K)).to(torch.int32)
    n_valid = n_valid[:, None].expand(T, H).contiguous()
    if not per_head and num_heads > 1:
        idx = idx.expand(T, num_heads, K)
        n_valid = n_valid.expand(T, num_heads)
    return idx.to(torch.int32).contiguous(), n_valid.contiguous()


# --------------------------------------------------------------------------
# The five benchmark/parity configurations
# --------------------------------------------------------------------------

def config_tiny(device="cpu", seed=CONFIG_SEED_BASE + 1) -> Workload:
    """1 seq, 256 query tokens over a 256-slot causal cache, heads (3,1),
    K=64: t and its 15 predecessors plus uniform random earlier slots,
    sorted, -1 padded (no n_valid)."""
    gen = _gen(seed, device)
    T = S = 256
    q = normal_bf16((T, 3, HEAD_DIM), gen, device)
    k = normal_bf16((S, 1, HEAD_DIM), gen, device)
    v = normal_bf16((S, 1, HEAD_DIM), gen, device)
    pos = torch.arange(T, device=device)
    s0 = torch.zeros(T, dtype=torch.int64, device=device)
    idx, _ = causal_lists(pos, s0, 64, 16, 1, gen, device, ordered=True)
    return Workload("tiny", q, k, v, idx, None, 1.0 / 16, pos, s0,
                    "T=256 S=256 (3,1) K=64 local16+random sorted, -1 padded")


def config_c2(device="cpu", seed=CONFIG_SEED_BASE + 2) -> Workload:
    """1 seq, 4096 tokens over a 4096-slot cache, heads (6,1), K=512: last 64
    causal slots + uniform random rest, sorted, ragged for t < 512."""
    gen = _gen(seed, device)
    T = S = 4096
    q = normal_bf16((T, 6, HEAD_DIM), gen, device)
    k = normal_bf16((S, 1, HEAD_DIM), gen, device)
    v = normal_bf16((S, 1, HEAD_DIM), gen, device)
    pos = torch.arange(T, device=device)
    s0 = torch.zeros(T, dtype=torch.int64, device=device)
    idx, nv = causal_lists(pos, s0, 512, 64, 1, gen, device, ordered=True)
    return Workload("c2_4k_g6_k512", q, k, v, idx, nv, 1.0 / 16, pos, s0,
                    "T=4096 S=4096 (6,1) K=512 local64+random sorted, ragged t<512")


def config_c3(device="cpu", seed=CONFIG_SEED_BASE + 3, seq_len=8192) -> Workload:
    """2 seqs x 8192 tokens packed (cu_seqlens [0, 8192, 16384]) over a
    16384-slot cache, heads (12,1), K=1024: 128-slot local window + random
    causal rest within the own sequence.  K ~ N(0, 0.5) times a per-row
    scale ~ U(0.5, 2); Q, V ~ N(0, 1)."""
    gen = _gen(seed, device)
    T = S = 2 * seq_len
    q = normal_bf16((T, 12, HEAD_DIM), gen, device)
    kf = torch.randn((S, 1, HEAD_DIM), generator=gen, device=device) * 0.5
    row_scale = torch.rand((S, 1, 1), generator=gen, device=device) * 1.5 + 0.5
    k = (kf * row_scale).to(torch.bfloat16)
    v = normal_bf16((S, 1, HEAD_DIM), gen, device)
    pos = torch.arange(T, device=device)
    s0 = (pos // seq_len) * seq_len
    idx, nv = causal_lists(pos, s0, 1024, 128, 1, gen, device, ordered=True)
    return Workload("c3_2x8k_g12_k1024", q, k, v, idx, nv, 1.0 / 16, pos, s0,
                    "2x8192 varlen S=16384 (12,1) K=1024 local128+random, K~N(0,.5)*U(.5,2)")


def config_c4(device="cpu", seed=CONFIG_SEED_BASE + 4, T=32768) -> Workload:
    """1 seq, 32768 tokens over a 32768-slot cache, heads (16,2), K=2048, an
    independent list per KV head (local 128 + random causal), sorted."""
    gen = _gen(seed, device)
    S = T
    q = normal_bf16((T, 16, HEAD_DIM), gen, device)
    k = normal_bf16((S, 2, HEAD_DIM), gen, device)
    v = normal_bf16((S, 2, HEAD_DIM), gen, device)
    pos = torch.arange(T, device=device)
    s0 = torch.zeros(T, dtype=torch.int64, device=device)
    idx, nv = causal_lists(pos, s0, 2048, 128, 2, gen, device, ordered=True)
    return Workload("c4_32k_g16x2_k2048", q, k, v, idx, nv, 1.0 / 16, pos, s0,
                    "T=32768 S=32768 (16,2) K=2048 per-head local128+random sorted")


def config_c5(device="cpu", seed=CONFIG_SEED_BASE + 5, T=8192, S=131072) -> Workload:
    """Chunked long prefill: 8192 new tokens at positions 122880..131071 over
    a 131072-slot cache, heads (24,2), K=2048; per KV head 256 local + 1792
    random over the earlier slots, in random (unsorted) order."""
    gen = _gen(seed, device)
    q = normal_bf16((T, 24, HEAD_DIM), gen, device)
    k = normal_bf16((S, 2, HEAD_DIM), gen, device)
    v = normal_bf16((S, 2, HEAD_DIM), gen, device)
    pos = torch.arange(S - T, S, device=device)
    s0 = torch.zeros(T, dtype=torch.int64, device=device)
    idx, nv = causal_lists(pos, s0, 2048, 256, 2, gen, device, ordered=False)
    return Workload("c5_chunk8k_at128k_g24x2_k2048", q, k, v, idx, nv, 1.0 / 16, pos, s0,
                    "T=8192 at 122880..131071, S=131072 (24,2) K=2048 local256+random unsorted")


def config_pages_long(device="cpu", seed=CONFIG_SEED_BASE + 6, heads=(24, 2)) -> Workload:
    """The pages' long-prefill case: 7810 query tokens (the last 7810 slots)
    over a 65536-slot cache with 2051 selected slots per query (2048 + a
    3-token causal tail), heads (24,2), lists in random order."""
    gen = _gen(seed, device)
    T, S, K = 7810, 65536, 2051
    Hq, Hkv = heads
    q = normal_bf16((T, Hq, HEAD_DIM), gen, device)
    k = normal_bf16((S, Hkv, HEAD_DIM), gen, device)
    v = normal_bf16((S, Hkv, HEAD_DIM), gen, device)
    pos = torch.arange(S - T, S, device=device)
    s0 = torch.zeros(T, dtype=torch.int64, device=device)
    idx, nv = causal_lists(pos, s0, K, 3, Hkv, gen, device, ordered=False)
    return Workload("pages_long_7810x65536_k2051", q, k, v, idx, nv, 1.0 / 16, pos, s0,
                    "T=7810 S=65536 (24,2) K=2051 (3-token tail + random), unsorted")


def config_decode(device="cpu", seed=CONFIG_SEED_BASE + 7, B=64, ctx=32768, heads=(24, 2),
                  topk=2048, local=256) -> Workload:
    """Decode step: B sequences of `ctx` cached tokens each (sequence b owns
    slots [b*ctx, (b+1)*ctx)), one new query token per sequence at its last
    slot; per KV head `local` most recent slots + random earlier slots of the
    same sequence, unsorted."""
    gen = _gen(seed, device)
    Hq, Hkv = heads
    S = B * ctx
    q = normal_bf16((B, Hq, HEAD_DIM), gen, device)
    k = normal_bf16((S, Hkv, HEAD_DIM), gen, device)
    v = normal_bf16((S, Hkv, HEAD_DIM), gen, device)
    s0 = torch.arange(B, device=device) * ctx
    pos = s0 + ctx - 1
    idx, nv = causal_lists(pos, s0, topk, local, Hkv, gen, device, ordered=False)
    return Workload(f"decode_b{B}_ctx{ctx}_g{Hq}x{Hkv}_k{topk}", q, k, v, idx, nv, 1.0 / 16, pos, s0,
                    f"decode B={B} ctx={ctx} S={S} ({Hq},{Hkv}) K={topk} local{local}+random unsorted")


def config_c5_block4(device="cpu", seed=CONFIG_SEED_BASE + 8, T=8192, S=131072, heads=(24, 2),
                     blocks=512, local_blocks=64, block_size=4) -> Workload:
    """c5 with microblock lists: 8192 new tokens at positions 122880..131071
    over a 131072-slot cache, heads (24,2); per KV head `blocks` entries of
    `block_size` slots (the `local_blocks` newest blocks + random earlier
    blocks, unsorted).  The newest block reaches past the token's own slot;
    last_slot (= the token's slot) masks that tail.  Lists are drawn like
    token lists, in block units.  The returned Workload carries
    block_size and last_slot as attributes."""
    gen = _gen(seed, device)
    Hq, Hkv = heads
    q = normal_bf16((T, Hq, HEAD_DIM), gen, device)
    k = normal_bf16((S, Hkv, HEAD_DIM), gen, device)
    v = normal_bf16((S, Hkv, HEAD_DIM), gen, device)
    pos = torch.arange(S - T, S, device=device)
    s0 = torch.zeros(T, dtype=torch.int64, device=device)
    idx, nv = causal_lists(pos // block_size, s0 // block_size, blocks, local_blocks, Hkv, gen,
                           device, ordered=False)
    w = Workload(f"c5_block{block_size}_{blocks}blk", q, k, v, idx, nv, 1.0 / 16, pos, s0,
                 f"T={T} at {S - T}..{S - 1}, S={S} ({Hq},{Hkv}) {blocks} blocks of {block_size} "
                 f"(local {local_blocks} + random), unsorted, causal tail masked")
    w.block_size = block_size
    w.last_slot = pos.to(torch.int32)
    return w


@dataclasses.dataclass
class IndexerWorkload:
    name: str
    q_idx: torch.Tensor        # [T, H, 128] bf16
    k_idx: torch.Tensor        # [NB, 128] bf16: one key per microblock
    positions: torch.Tensor    # [T] int32
    seq_start: torch.Tensor    # [T] int32
    block_size: int
    budget: int
    description: str = ""


def config_indexer(device="cpu", seed=CONFIG_SEED_BASE + 9, T=8192, S=131072, heads=4, head_dim=128,
                   block_size=4, budget=2048, seq_starts=None) -> IndexerWorkload:
    """The indexer of the published configuration at the c5 size: 8192 new
    tokens at positions S-T..S-1 of one sequence, 4 heads x dim 128 sharing
    one key per microblock of 4 slots (S/4 keys), budget 2048 blocks.  Values
    are standard normal BF16 (synthetic weights: no checkpoint exists here).
    `seq_starts` (optional list of slot offsets, multiples of block_size) cuts
    the T tokens into sequences of equal length packed at the cache end."""
    gen = _gen(seed, device)
    NB = S // block_size
    q = normal_bf16((T, heads, head_dim), gen, device)
    k = normal_bf16((NB, head_dim), gen, device)
    pos = torch.arange(S - T, S, device=device, dtype=torch.int32)
    s0 = torch.zeros(T, dtype=torch.int32, device=device)
    if seq_starts is not None:
        per = T // len(seq_starts)
        for i, st in enumerate(seq_starts):
            s0[i * per:(i + 1) * per] = int(st)
    return IndexerWorkload(f"indexer_T{T}_S{S}", q, k, pos, s0, block_size, budget,
                           f"T={T} at {S - T}..{S - 1}, {NB} block keys, {heads}x{head_dim} heads, "
                           f"ratio {block_size}, budget {budget}")


CONFIGS = {
    "tiny": config_tiny,
    "c2": config_c2,
    "c3": config_c3,
    "c4": config_c4,
    "c5": config_c5,
    "decode": config_decode,
    "c5_block4": config_c5_block4,
}


def make(name: str, device="cpu", **kw) -> Workload:
    if name == "pages_long":
        return config_pages_long(device, **kw)
    return CONFIGS[name](device, **kw)


# --------------------------------------------------------------------------
# Small generic cases for the edge-case tests
# --------------------------------------------------------------------------

def random_lists(T: int, H: int, K: int, S: int, gen, device, distinct=True) -> torch.Tensor:
    """Unordered lists of physical slots drawn uniformly from [0, S) (distinct
    within a list when `distinct`).  int32 [T, H, K]."""
    if K == 0:
        return torch.empty((T, H, 0), dtype=torch.int32, device=device)
    if distinct:
        keys = torch.rand((T * H, S), generator=gen, device=device)
        sel = torch.topk(keys, K, dim=1, largest=False, sorted=False).indices
        perm = torch.argsort(torch.rand((T * H, K), generator=gen, device=device), dim=1)
        sel = torch.gather(sel, 1, perm)
    else:
        sel = torch.randint(0, S, (T * H, K), generator=gen, device=device)
    return sel.view(T, H, K).to(torch.int32).contiguous()


def generic_case(T: int, S: int, Hq: int, Hkv: int, K: int, seed: int, device="cpu",
                 D: int = HEAD_DIM, scale: float = 0.0, name: str = "generic") -> Workload:
    """Random Q/K/V ~ N(0,1) and unordered distinct random lists over [0, S)."""
    gen = _gen(seed, device)
    q = normal_bf16((T, Hq, D), gen, device)
    k = normal_bf16((S, Hkv, D), gen, device)
    v = normal_bf16((S, Hkv, D), gen, device)
    idx = random_lists(T, Hkv, K, S, gen, device)
    pos = torch.full((T,), S - 1, dtype=torch.int64, device=device)
    s0 = torch.zeros(T, dtype=torch.int64, device=device)
    return Workload(name, q, k, v, idx, None, scale, pos, s0,
                    f"T={T} S={S} ({Hq},{Hkv}) K={K} random distinct unordered")


def two_request_case(prefix: int, len_a: int, len_b: int, K: int, heads=(12, 1),
                     seed: int = 7, device="cpu", local: int = 16) -> Workload:
    """Two requests whose block tables share `prefix` physical slots: request
    A owns slots [prefix, prefix+len_a), request B owns the slots after that.
    Each request's tokens select causal positions of their own logical
    sequence (shared prefix + own suffix), mapped to physical slots."""
    gen = _gen(seed, device)
    Hq, Hkv = heads
    S = prefix + len_a + len_b
    T = len_a + len_b
    q = normal_bf16((T, Hq, HEAD_DIM), gen, device)
    k = normal_bf16((S, Hkv, HEAD_DIM), gen, device)
    v = normal_bf16((S, Hkv, HEAD_DIM), gen, device)
    # logical positions: request A tokens at prefix..prefix+len_a-1, B likewise
    logical = torch.cat([torch.arange(prefix, prefix + len_a), torch.arange(prefix, prefix + len_b)]).to(device)
    zero = torch.zeros(T, dtype=torch.int64, device=device)
    lidx, nv = causal_lists(logical, zero, K, local, Hkv, gen, device, ordered=False)
    # block tables: logical -> physical
    table_a = torch.arange(0, prefix + len_a, device=device)
    table_b = torch.cat([torch.arange(0, prefix, device=device),
                         torch.arange(prefix + len_a, S, device=device)])
    is_b = torch.cat([torch.zeros(len_a, dtype=torch.bool), torch.ones(len_b, dtype=torch.bool)]).to(device)
    lidx64 = lidx.to(torch.int64)
    valid = lidx64 >= 0
    safe = lidx64.clamp(min=0)
    phys_a = table_a[safe.clamp(max=table_a.numel() - 1)]
    phys_b = table_b[safe.clamp(max=table_b.numel() - 1)]
    phys = torch.where(is_b[:, None, None], phys_b, phys_a)
    phys = torch.where(valid, phys, torch.full_like(phys, -1)).to(torch.int32)
    pos = torch.where(is_b, table_b[logical.clamp(max=table_b.numel() - 1)],
                      table_a[logical.clamp(max=table_a.numel() - 1)])
    return Workload("two_request", q, k, v, phys.contiguous(), nv, 0.0, pos, zero,
                    f"two requests sharing {prefix} prefix slots, K={K}")
