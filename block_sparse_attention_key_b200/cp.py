"""Context-parallel decode: one sequence's blocks spread over several GPUs, one
process per GPU, exchanges through torch.distributed (NCCL over NVLink).

Steps (C ABI in include/qsa.h, "context parallelism"): each rank scores its own
blocks and keeps its local top-k as 64-bit keys; an all-gather of the keys; every
rank merges the same union into the same global selection and keeps its own
blocks; each rank attends them and writes one unnormalised partial per (query,
head); an all-gather of the partials; every rank combines them into the output.
The exactness of both merges (the global top-k lies in the union of the local
top-ks; softmax over a union of token sets is the combination of the sets'
partials) is what makes the split lossless.

Host logic only: every arithmetic step runs in libqsa.so.
"""

from . import qsa as _q


def shard_range(n_blocks, world, rank):
    """Block range [lo, lo + n) of `rank` when `n_blocks` blocks are cut into `world`
    contiguous shards of near-equal size (the first n_blocks % world shards one
    larger)."""
    if world < 1 or not 0 <= rank < world or n_blocks < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(n_blocks, world)
    lo = rank * base + min(rank, extra)
    return lo, base + (1 if rank < extra else 0)


def cp_decode(shard_dims, full_dims, *, q, k_shard, v_shard, q_idx, w, pooled_shard, q_seq, q_pos, n_q, blk_lo,
              out, workspace, group=None, stream=None):
    """The layer's selection and attention for n_q decode queries whose sequences are
    sharded by block range across the ranks of `group`.  `shard_dims` describe this
    rank's caches (kv_capacity = its shard's tokens), `full_dims` the whole layer;
    positions are global.  Pooling of appended blocks is the owning rank's
    qsa_pool_block_keys call.  `stream` (a torch.cuda.Stream or a raw cudaStream_t
    handle; None = the current stream) orders the library calls and the collectives
    alike: it is made torch's current stream for the whole exchange, since the
    process group's collectives follow torch's current stream.  Returns (sel_local,
    cnt_local) of this rank."""
    import torch
    if stream is not None and not isinstance(stream, torch.cuda.Stream):
        stream = torch.cuda.ExternalStream(stream)
    with torch.cuda.stream(stream):
        return _cp_decode(shard_dims, full_dims, q, k_shard, v_shard, q_idx, w, pooled_shard, q_seq, q_pos, n_q,
                          blk_lo, out, workspace, group)


def _cp_decode(shard_dims, full_dims, q, k_shard, v_shard, q_idx, w, pooled_shard, q_seq, q_pos, n_q, blk_lo, out,
               workspace, group):
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    dev = q.device
    keys = torch.empty((n_q, _q.QSA_SEL_CAP), dtype=torch.int64, device=dev)
    cnt = torch.empty((n_q,), dtype=torch.int32, device=dev)
    _q.qsa_cp_select_keys(shard_dims, q_idx, w, pooled_shard, q_seq, q_pos, n_q, blk_lo, keys, cnt, workspace)
    # gathered buffers are the ranks' arrays one after another ([world][n_q]...), shaped
    # as a dim-0 concatenation, which every backend's all-gather accepts
    keys_all = torch.empty((world * n_q, _q.QSA_SEL_CAP), dtype=torch.int64, device=dev)
    cnt_all = torch.empty((world * n_q,), dtype=torch.int32, device=dev)
    dist.all_gather_into_tensor(keys_all, keys, group=group)
    dist.all_gather_into_tensor(cnt_all, cnt, group=group)
    sel_local = torch.empty((n_q, _q.QSA_SEL_CAP), dtype=torch.int32, device=dev)
    cnt_local = torch.empty((n_q,), dtype=torch.int32, device=dev)
    _q.qsa_cp_merge_keys(shard_dims, world, keys_all, cnt_all, n_q, blk_lo, sel_local, cnt_local)
    part = torch.empty((n_q, full_dims.n_q_heads, _q.CP_PART_ROW), dtype=torch.float32, device=dev)
    _q.qsa_cp_attn_partial(shard_dims, q, k_shard, v_shard, q_seq, q_pos, n_q, blk_lo, sel_local, cnt_local, part,
                           workspace)
    parts_all = torch.empty((world * n_q,) + tuple(part.shape[1:]), dtype=torch.float32, device=dev)
    dist.all_gather_into_tensor(parts_all, part, group=group)
    _q.qsa_cp_combine(full_dims, world, parts_all, n_q, out)
    return sel_local, cnt_local
