"""Row-sharded data parallelism for the Lynx layer, one process per GPU.

Each output row of Y = S(X) W^T + bias + (X A^T) B^T depends only on the same
row of X (the 2:4 selection and the norm compensation are per token row), so
the token rows split across ranks with no exchange at all: every rank holds
the same W, bias, A and B and runs lynx_linear on its own rows.  That is how
bench.py --gpus N runs (weak scaling, no data-path collective).

When a caller needs the whole Y on every device, gather_rows() all-gathers the
row blocks over the process group (NCCL on GPUs: 2 * rows * N bytes from each
rank over NVLink / NVSwitch).  Shards are contiguous blocks of
ceil(M / world) rows (the last may be shorter, or empty); the all-gather works
on equal blocks, so a short last block is padded and the padding dropped.
"""


def row_shard(M, world, rank):
    """(first row, number of rows) of rank `rank`'s block of M rows."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank must be in [0, world)")
    per = -(-M // world)
    first = min(M, rank * per)
    return first, max(0, min(M, first + per) - first)


def gather_rows(y_local, M, group=None):
    """All-gather the ranks' row blocks of Y into the full [M, N] on every rank.

    y_local: this rank's rows (row_shard(M, world, rank) of them), same dtype
    and device on every rank.  Returns a new tensor [M, N]."""
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    first, rows = row_shard(M, world, rank)
    if y_local.shape[0] != rows:
        raise ValueError(f"rank {rank} holds {y_local.shape[0]} rows, its block has {rows}")
    per = -(-M // world)
    n = y_local.shape[1]
    block = y_local
    if rows != per:
        block = torch.zeros((per, n), dtype=y_local.dtype, device=y_local.device)
        block[:rows] = y_local
    full = torch.empty((per * world, n), dtype=y_local.dtype, device=y_local.device)
    dist.all_gather_into_tensor(full, block.contiguous(), group=group)
    return full[:M]


def sharded_linear(X_local, W, bias=None, A=None, B=None, M=None, skip_sparsify=False, gather=False,
                   group=None, workspace=None, layer=None):
    """This rank's rows of the layer (lynx_linear on X_local, the rank's block of
    the M token rows); with gather=True the full Y [M, N] on every rank.

    `layer` is the function computing a block of rows (default
    lynx.lynx_linear, the CUDA layer); it takes (X, W, bias, A, B,
    skip_sparsify=..., workspace=...) and returns Y."""
    if layer is None:
        from . import lynx

        layer = lynx.lynx_linear
    y_local = layer(X_local, W, bias, A, B, skip_sparsify=skip_sparsify, workspace=workspace)
    if not gather:
        return y_local
    if M is None:
        raise ValueError("gather=True needs the total row count M")
    return gather_rows(y_local, M, group)
