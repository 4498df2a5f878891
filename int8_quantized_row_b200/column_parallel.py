"""Column-parallel LLM.int8() layer over the ranks of a process group, one GPU
per rank.

Rank r keeps the column block cols_r of the weight: Wq[:, cols_r],
sW[cols_r] and, unless the Wq-only variant is used, W16[:, cols_r].  X is
replicated, so every rank finds the same outlier columns and row scales
(both depend on X alone), and its Y[:, cols_r] carries the same bits as those
columns of the one-GPU result: each output column depends only on X, the
outlier set and its own weight column (the column scale sW[n] is one per
output column, as in the LLM.int8() method's vector-wise quantization).  The
full Y, when the caller needs it, is an all-gather of the column blocks
(NCCL over NVLink / NVSwitch); nothing else crosses GPUs.

Blocks are contiguous and a multiple of 16 columns wide (the layer's N % 16
rule), as even as that allows.
"""

ALIGN = 16


def column_bounds(N, world, rank, align=ALIGN):
    """[start, stop) of rank's column block: N split into blocks of whole
    `align`-column groups, the first N/align % world ranks one group wider."""
    if N % align or world < 1 or not 0 <= rank < world:
        raise ValueError(f"cannot split N={N} over {world} ranks in blocks of {align}")
    groups = N // align
    base, extra = divmod(groups, world)
    start = rank * base + min(rank, extra)
    width = base + (1 if rank < extra else 0)
    return start * align, (start + width) * align


def shard_columns(Wq, sW, W16, world, rank):
    """This rank's (Wq, sW, W16) column block, contiguous (W16 may be None)."""
    a, b = column_bounds(Wq.shape[1], world, rank)
    return (Wq[:, a:b].contiguous(), sW[a:b].contiguous(),
            None if W16 is None else W16[:, a:b].contiguous())


def gather_columns(Y_local, N, world, rank, group=None):
    """All-gather the ranks' column blocks [T, N_r] into the full [T, N]."""
    import torch
    import torch.distributed as dist
    T = Y_local.shape[0]
    widths = [b - a for a, b in (column_bounds(N, world, r) for r in range(world))]
    if Y_local.shape[1] != widths[rank]:
        raise ValueError("Y_local is not this rank's column block")
    wmax = max(widths)
    send = Y_local if Y_local.shape[1] == wmax else torch.nn.functional.pad(Y_local, (0, wmax - Y_local.shape[1]))
    buf = torch.empty((world * T, wmax), dtype=Y_local.dtype, device=Y_local.device)
    dist.all_gather_into_tensor(buf, send.contiguous(), group=group)      # rank r's block at rows r*T ..
    buf = buf.view(world, T, wmax)
    return torch.cat([buf[r, :, :widths[r]] for r in range(world)], dim=1)


def int8_mixed_linear_column_parallel(X, Wq_local, sW_local, W16_local, N, alpha=6.0, world=1, rank=0, group=None,
                                      gather=True, local_fn=None):
    """Y [T, N] (or this rank's block [T, N_r] with gather=False) of the layer
    whose columns are split over the group.  local_fn(X, Wq, sW, W16, alpha)
    computes one block; it is the CUDA layer unless a test supplies another."""
    if local_fn is None:
        import int8_quantized_row_b200 as i8

        def local_fn(X, Wq, sW, W16, alpha):
            if W16 is None:
                return i8.int8_mixed_linear_wq(X, Wq, sW, alpha)
            return i8.int8_mixed_linear(X, Wq, sW, W16, alpha)
    Y_local = local_fn(X, Wq_local, sW_local, W16_local, alpha)
    if not gather or world == 1:
        return Y_local
    return gather_columns(Y_local, N, world, rank, group)
