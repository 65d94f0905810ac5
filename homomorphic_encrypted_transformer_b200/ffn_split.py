"""The FFN1 block product split by output group across ranks, then one
ciphertext AllGather (AEGIS summary, section 2.2, FFN partitioning: each
device keeps the weights of one group of output blocks, computes those
blocks by its local plaintext x ciphertext product, and a single AllGather
of the output ciphertexts gives every device the whole layer output).

One process per GPU.  Every rank holds all input ciphertexts of the layer
(the previous layer's gathered output) and only the weight diagonals of its
own output group; the local product is he_pmult_accum_bsgs on that slice.
The exchange is one torch.distributed.all_gather of equally sized blocks of
ciphertexts into buffers this rank owns (NCCL over NVLink between GPUs, gloo
between host processes), so a kernel that later reads a gathered ciphertext
reads this GPU's own memory; no kernel is handed a peer's memory.

Output blocks go to ranks in contiguous groups whose sizes differ by at most
one (the first n_out % world ranks take one more); the gather pads every
rank's group to the largest size, so that all blocks are equal, and drops the
padding when it puts the blocks back in the unsplit product's order.
"""


def output_group(n_out, world, rank):
    """Output blocks [i0, i1) of `rank` among `world` ranks."""
    if world < 1 or not 0 <= rank < world or n_out < 0:
        raise ValueError("bad partition request: n_out=%d world=%d rank=%d" % (n_out, world, rank))
    base, extra = divmod(n_out, world)
    i0 = rank * base + min(rank, extra)
    return i0, i0 + base + (1 if rank < extra else 0)


def max_group(n_out, world):
    """Size of the largest output group (the gather's block size)."""
    return -(-n_out // world)


def assemble(blocks, n_out, world):
    """Puts gathered blocks back in output order.

    blocks: tensor [world][n_groups][max_group][*ct] (rank r's group in
    blocks[r][:, :size_r]); returns [n_groups][n_out][*ct]."""
    import torch

    parts = []
    for r in range(world):
        i0, i1 = output_group(n_out, world, r)
        parts.append(blocks[r][:, :i1 - i0])
    return torch.cat(parts, dim=1)


def gather_output_groups(local, n_out, world, rank, group=None):
    """The one AllGather of the split product.

    local: tensor [n_groups][n_local][*ct] of this rank's output blocks
    (n_local = its group size), on this rank's device (CUDA with NCCL, host
    with gloo).  Returns [n_groups][n_out][*ct] on every rank, in the order
    of the unsplit product.  With world == 1 it returns `local`."""
    import torch

    i0, i1 = output_group(n_out, world, rank)
    if local.shape[1] != i1 - i0:
        raise ValueError("rank %d holds %d output blocks, its group has %d" % (rank, local.shape[1], i1 - i0))
    if world == 1:
        return local
    import torch.distributed as dist

    m = max_group(n_out, world)
    send = local
    if local.shape[1] < m:  # equal block sizes for the collective
        pad = torch.zeros((local.shape[0], m - local.shape[1]) + tuple(local.shape[2:]), dtype=local.dtype,
                          device=local.device)
        send = torch.cat([local, pad], dim=1)
    send = send.contiguous()
    recv = [torch.empty_like(send) for _ in range(world)]
    dist.all_gather(recv, send, group=group)
    return assemble(torch.stack(recv), n_out, world)


def ffn1_output_group(he, ctx, x, n_in, d_pt_local, pt_scale, n_out, bs, gs, stride, n_groups, world, rank):
    """This rank's share of the split FFN1 product, on its GPU.

    x: the n_groups*n_in input ciphertexts (he.Ciphertext, group-major, one
    level l >= 2); d_pt_local: device tensor [n_local][n_in][gs][bs][l][N]
    of the rank's output group's evaluation-domain diagonals.  Returns a
    device tensor [n_groups][n_local][2][l-1][N] of its output blocks, their
    level l-1 and scale."""
    import torch

    i0, i1 = output_group(n_out, world, rank)
    n_local = i1 - i0
    if d_pt_local.shape[0] != n_local:
        raise ValueError("weights of %d output blocks given, the group has %d" % (d_pt_local.shape[0], n_local))
    level, N = x[0].level, ctx.N
    room = torch.empty((n_groups, n_local, 2 * level * N), dtype=torch.int64, device=x[0].data.device)
    ys = [he.Ciphertext(room[t, i], level, 1.0) for t in range(n_groups) for i in range(n_local)]
    he.he_pmult_accum_bsgs(ctx, x, n_in, d_pt_local, pt_scale, n_local, bs, gs, stride, n_groups, ys)
    out = room[:, :, :2 * (level - 1) * N].reshape(n_groups, n_local, 2, level - 1, N)
    return out, ys[0].level, ys[0].scale


def ffn1_split(he, ctx, x, n_in, d_pt_local, pt_scale, n_out, bs, gs, stride, n_groups, world, rank, group=None):
    """Local product of this rank's output group, then the AllGather: every
    rank returns [n_groups][n_out][2][l-1][N], the whole layer output, with
    its level and scale."""
    local, level, scale = ffn1_output_group(he, ctx, x, n_in, d_pt_local, pt_scale, n_out, bs, gs, stride,
                                            n_groups, world, rank)
    return gather_output_groups(local, n_out, world, rank, group), level, scale
