"""Context-parallel prefill: one long sequence split by query rows over the ranks of a
process group, one process per GPU.

Why one exchange step is enough.  Each token attends only to the top-k of the tokens
before it, and the indexer picks those positions for each token on its own
([Explainer] "稀疏注意力的隐性开销：indexer").  Row t therefore reads the keys s <= t
(indexer) and the K/V rows it selected among them (attention), and never another row's
result.  Once a rank holds the keys of every earlier row, its own rows are independent
work -- exactly a chunk of chunked prefill, with the chunk's first row as the query
offset.

The plan:

* zig-zag ownership.  The sequence is cut into 2W blocks of ``blk`` rows (the last
  ones clipped at L); rank r owns block r and block 2W-1-r.  Causal work grows with
  the row, so pairing the r-th lightest block with the r-th heaviest gives every rank
  the same share of the triangle to within one block's imbalance.
* Each rank holds its own rows of q_I, w and Q (and writes its rows of O) and its own
  rows of the keys k_I, K and V, in a local buffer of two slots [2, blk, ...]: slot 0 is
  block r, slot 1 is block 2W-1-r.
* One all-gather per key tensor (k_I of each F layer, K and V of each layer) puts the
  whole sequence's keys in every rank's own memory, in sequence order, [1, 2W*blk, ...].
  The transfers go through NCCL into local HBM; no kernel reads a peer's memory.
* Then each rank runs the single-GPU layer group on each of its blocks
  (n_q = block rows, q_pos0 = block start, n_kv = block end).  The indexer, the
  top-k, the index cache and the attention touch local memory only; the index cache
  is per rank and per block.

Only one sequence (batch 1) is split this way; independent sequences go to ranks whole
(replicas, no exchange).
"""

from __future__ import annotations

from dataclasses import dataclass


@dataclass(frozen=True)
class Plan:
    """Row ownership of one rank.

    L       sequence length
    world   ranks sharing the sequence
    rank    this rank
    blk     rows per block; the gathered sequence holds 2*world*blk rows (zero padding past L)
    blocks  (start, end) rows of slot 0 and slot 1 of this rank's local buffers;
            a block past the end of the sequence is (L, L) (empty)
    """

    L: int
    world: int
    rank: int
    blk: int
    blocks: tuple

    @property
    def padded_len(self) -> int:
        return 2 * self.world * self.blk

    @property
    def n_rows(self) -> int:
        return sum(e - s for s, e in self.blocks)


def block_rows(L: int, world: int, align: int = 1) -> int:
    """Rows per block: ceil(L / 2W) rounded up to a multiple of `align`.

    The kernels take any query offset, so no alignment is needed; with align = 1 the
    blocks are equal but for the last, which is short by fewer than 2W rows (that
    block's owner, rank 0, then has at most 2W-1 heavy rows less work than the others,
    whose pairs of blocks cost exactly the same)."""
    if L < 1 or world < 1 or align < 1:
        raise ValueError("L, world and align must be positive")
    per = -(-L // (2 * world))
    return max(align, -(-per // align) * align)


def owned_blocks(world: int, rank: int) -> tuple:
    """Block numbers held in slot 0 and slot 1 of rank `rank`."""
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside [0, {world})")
    return (rank, 2 * world - 1 - rank)


def make_plan(L: int, world: int, rank: int, align: int = 1) -> Plan:
    blk = block_rows(L, world, align)
    blocks = tuple((min(b * blk, L), min((b + 1) * blk, L)) for b in owned_blocks(world, rank))
    return Plan(L, world, rank, blk, blocks)


def indexer_work(plan: Plan) -> int:
    """Causal (query, key) pairs the rank's indexer scores: sum over its rows t of t+1."""
    return sum((e * (e + 1) - s * (s + 1)) // 2 for s, e in plan.blocks)


def attention_work(plan: Plan, topk: int) -> int:
    """K/V rows the rank's attention gathers per head: sum over its rows t of min(topk, t+1)."""
    total = 0
    for s, e in plan.blocks:
        lo = min(e, max(s, topk))          # rows [s, lo) see fewer than topk keys
        total += (lo * (lo + 1) - s * (s + 1)) // 2 if lo > s else 0
        total += (e - max(lo, s)) * topk
    return total


# ------------------------------------------------------------------ buffers
def local_rows(x, plan: Plan):
    """This rank's rows of a full-sequence tensor x [1, L, ...] as a zero-padded local
    buffer [2, blk, ...] (slot order of `plan.blocks`).  Input preparation: in a model
    each rank produces these rows itself."""
    import torch

    if x.shape[0] != 1 or x.shape[1] != plan.L:
        raise ValueError(f"expected [1, {plan.L}, ...], got {tuple(x.shape)}")
    out = torch.zeros((2, plan.blk) + tuple(x.shape[2:]), dtype=x.dtype, device=x.device)
    for slot, (s, e) in enumerate(plan.blocks):
        if e > s:
            out[slot, : e - s].copy_(x[0, s:e])
    return out


def scatter_rows(y_local, plan: Plan, out):
    """Write a local buffer [2, blk, ...] back into this rank's rows of out [1, L, ...]."""
    for slot, (s, e) in enumerate(plan.blocks):
        if e > s:
            out[0, s:e].copy_(y_local[slot, : e - s])
    return out


def slot_view(local, plan: Plan, slot: int):
    """Slot `slot` of a local buffer as a dense [1, rows, ...] view (no copy)."""
    s, e = plan.blocks[slot]
    return local[slot : slot + 1, : e - s]


def allgather_keys(local, plan: Plan, group=None, out=None):
    """All ranks' key rows in sequence order, [1, 2*world*blk, ...], in this rank's memory.

    `local` is this rank's [2, blk, ...] key buffer.  The first half of the sequence
    (blocks 0..W-1, slot 0 of ranks 0..W-1) lands in rank order with one all-gather; the
    second half (slot 1 of rank i is block 2W-1-i) with a second all-gather whose output
    slots are taken in reverse rank order.  With one rank the local buffer already is
    the sequence (blocks 0 and 1) and is returned as a view."""
    import torch
    import torch.distributed as dist

    W = plan.world
    tail = tuple(local.shape[2:])
    if tuple(local.shape[:2]) != (2, plan.blk):
        raise ValueError(f"local buffer must be [2, {plan.blk}, ...], got {tuple(local.shape)}")
    if W == 1:
        return local.view((1, 2 * plan.blk) + tail)
    if out is None:
        out = torch.empty((2 * W, plan.blk) + tail, dtype=local.dtype, device=local.device)
    out = out.view((2 * W, plan.blk) + tail)
    first = out[:W]
    if hasattr(dist, "all_gather_into_tensor") and local.is_cuda:
        dist.all_gather_into_tensor(first, local[0].contiguous(), group=group)
    else:
        dist.all_gather(list(first.unbind(0)), local[0].contiguous(), group=group)
    dist.all_gather([out[2 * W - 1 - i] for i in range(W)], local[1].contiguous(), group=group)
    return out.view((1, 2 * W * plan.blk) + tail)


# ----------------------------------------------------------------- executor
ROW_NAMES = ("q_I", "q_scale", "w", "Q", "O")     # per-query-row tensors: local [2, blk, ...]
KEY_NAMES = ("k_I", "k_scale", "K", "V")         # per-key tensors: gathered [1, 2W*blk, ...]


def workspace_size(plan: Plan, H_I, d_I, Hq, Hkv, d_qk, d_v, topk, idx_dtype=None, scale=0.0,
                   o_dtype=None) -> int:
    """Largest layer-group workspace any of the rank's blocks needs."""
    from . import dsa

    kw = {}
    if idx_dtype is not None:
        kw["idx_dtype"] = idx_dtype
    if o_dtype is not None:
        kw["o_dtype"] = o_dtype
    n = 256
    for s, e in plan.blocks:
        if e > s:
            shape = dsa.group_shape(1, e - s, s, e, H_I, d_I, Hq, Hkv, d_qk, d_v, topk, scale=scale, **kw)
            n = max(n, dsa.layer_group_forward_workspace_size(shape))
    return n


def layer_group_forward(plan: Plan, layers, pattern: str, cache_buf, workspace, H_I, d_I, Hq, Hkv, d_qk, d_v,
                        topk, idx_dtype=None, scale=0.0, o_dtype=None, stream=None):
    """Run a layer group on this rank's rows.

    layers[l] holds the per-row tensors of ROW_NAMES as local buffers [2, blk, ...] and the
    keys of KEY_NAMES as gathered buffers [1, >= L, ...] (see `allgather_keys`); F layers
    carry q_I, w, k_I (+ q_scale, k_scale for e4m3), every layer Q, K, V, O.
    `cache_buf` is the rank's index cache, int32 [2, blk, topk] (one slot per block, like
    the row tensors): after the call it holds each block's last F-layer selection.
    Returns (indexer launches, attention launches)."""
    from . import dsa

    kw = {}
    if idx_dtype is not None:
        kw["idx_dtype"] = idx_dtype
    if o_dtype is not None:
        kw["o_dtype"] = o_dtype
    n_idx = n_attn = 0
    for slot, (s, e) in enumerate(plan.blocks):
        if e <= s:
            continue
        shape = dsa.group_shape(1, e - s, s, e, H_I, d_I, Hq, Hkv, d_qk, d_v, topk, scale=scale, **kw)
        blk_layers = []
        for Lh in layers:
            d = {}
            for name in ROW_NAMES:
                if Lh.get(name) is not None:
                    d[name] = slot_view(Lh[name], plan, slot)
            for name in KEY_NAMES:
                if Lh.get(name) is not None:
                    d[name] = Lh[name][:, :e]
            blk_layers.append(d)
        cache = dsa.IndexCache(slot_view(cache_buf, plan, slot))
        st = dsa.layer_group_forward(shape, blk_layers, pattern, cache, workspace=workspace, stream=stream)
        n_idx += st.indexer_launches
        n_attn += st.attention_launches
    return n_idx, n_attn
