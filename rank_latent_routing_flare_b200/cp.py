"""Context-parallel FLARE / FLARE++ forward over torch.distributed.

The FLARE++ paper (arXiv 2608.11519, section "Multi-GPU context parallelism",
eq. 13-14) shards the tokens of every sequence across ranks.  The projections
and the decoder are pointwise in the tokens and stay local; each encoder pass
(the query synthesis and the encode for FLARE++, the encode for FLARE) needs
one exchange: every rank computes per-split partial sums of its shard, the
partials of all ranks are all-gathered, and every rank merges them with the
log-sum-exp rule in the same fixed order, so all ranks hold bitwise the same
Q(X) and Z.

All arithmetic runs in the CUDA library (the ``*_cp_*`` entry points of
include/flare.h); this module only allocates the buffers and moves the
partials between ranks (an NCCL all-gather on GPUs).  Without an initialised
process group it runs as a single rank.
"""
from __future__ import annotations

from . import _binding as b


def _group_info(group):
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return 0, 1
    return dist.get_rank(group), dist.get_world_size(group)


def allgather_partials(part, world: int, group=None):
    """Concatenate every rank's partials in rank order: [world * part.numel()]."""
    torch = b._torch()
    if world == 1:
        return part
    import torch.distributed as dist
    out = torch.empty(world * part.numel(), dtype=part.dtype, device=part.device)
    dist.all_gather_into_tensor(out, part, group=group)
    return out


def partials_numel(B: int, H: int, N: int, M: int, D: int) -> int:
    nbytes = b.load_library().flare_cp_partials_bytes(B, H, N, M, D)
    if nbytes == 0:
        raise ValueError("unsupported sizes")
    return nbytes // 4


def _status(st, where):
    if st != 0:
        raise b.FlareError(st, where)


def flarepp_mixer_cp_fwd(X, Wk, Wv, Wk_syn, Wv_syn, Q0, lengths=None, group=None, scale: float = 0.0,
                         Y=None, workspace=None, stream=None, Qx_out=None, Z_out=None):
    """FLARE++ forward of this rank's token shard X [B, N, C] (tokens
    [rank*N, (rank+1)*N) of sequences of world*N tokens; ``lengths`` counts
    tokens of the whole sequences).  Returns Y [B, H, N, D] of the shard."""
    torch = b._torch()
    rank, world = _group_info(group)
    B, N, C = X.shape
    H, M, D = Q0.shape
    lib = b.load_library()
    if Y is None:
        Y = torch.empty((B, H, N, D), dtype=torch.bfloat16, device=X.device)
    nbytes = b.flare_workspace_bytes(b.FLARE_VARIANT_FLAREPP, B, H, N, M, D, C)
    ws = b._workspace(workspace, nbytes, X.device)
    st = b._stream_ptr(stream, X.device)
    part = torch.empty(partials_numel(B, H, N, M, D), dtype=torch.float32, device=X.device)
    common = (B, N, C, H, M, D, b._ptr(lengths), rank, world, float(scale), b._ptr(ws), ws.numel(), st)
    _status(lib.flarepp_cp_begin(b._ptr(X), b._ptr(Wk), b._ptr(Wv), b._ptr(Wk_syn), b._ptr(Wv_syn), b._ptr(Q0),
                                 *common, b._ptr(part)), "flarepp_cp_begin")
    gathered = allgather_partials(part, world, group)
    part2 = torch.empty_like(part)
    _status(lib.flarepp_cp_middle(b._ptr(gathered), *common, b._ptr(part2), b._ptr(Qx_out)), "flarepp_cp_middle")
    gathered = allgather_partials(part2, world, group)
    _status(lib.flarepp_cp_end(b._ptr(gathered), b._ptr(Y), *common, b._ptr(Z_out)), "flarepp_cp_end")
    return Y


def flare_mixer_cp_fwd(K, V, Q, lengths=None, group=None, scale: float = 0.0, Y=None, workspace=None,
                       stream=None, Z_out=None):
    """FLARE forward of this rank's token shard K, V [B, H, N, D] (see
    flarepp_mixer_cp_fwd).  Returns Y [B, H, N, D] of the shard."""
    torch = b._torch()
    rank, world = _group_info(group)
    B, H, N, D = K.shape
    M = Q.shape[1]
    lib = b.load_library()
    if Y is None:
        Y = torch.empty_like(K)
    nbytes = b.flare_workspace_bytes(b.FLARE_VARIANT_FLARE, B, H, N, M, D)
    ws = b._workspace(workspace, nbytes, K.device)
    st = b._stream_ptr(stream, K.device)
    part = torch.empty(partials_numel(B, H, N, M, D), dtype=torch.float32, device=K.device)
    common = (B, H, N, M, D, b._ptr(lengths), rank, world, float(scale), b._ptr(ws), ws.numel(), st)
    _status(lib.flare_cp_begin(b._ptr(K), b._ptr(V), b._ptr(Q), *common, b._ptr(part)), "flare_cp_begin")
    gathered = allgather_partials(part, world, group)
    _status(lib.flare_cp_end(b._ptr(gathered), b._ptr(K), b._ptr(Q), b._ptr(Y), *common, b._ptr(Z_out)),
            "flare_cp_end")
    return Y
