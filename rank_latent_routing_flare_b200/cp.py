"""Context-parallel FLARE / FLARE++ forward (and FLARE++ backward) over
torch.distributed.

The FLARE++ paper (arXiv 2608.11519, section "Multi-GPU context parallelism",
eq. 13-14) shards the tokens of every sequence across ranks.  The projections
and the decoder are pointwise in the tokens and stay local; each encoder pass
(the query synthesis and the encode for FLARE++, the encode for FLARE) needs
one exchange: every rank computes per-split partial sums of its shard, the
partials of all ranks are all-gathered, and every rank merges them with the
log-sum-exp rule in the same fixed order, so all ranks hold bitwise the same
Q(X) and Z.  After each gather a second, small one carries, for the rows
whose fast-path sums may have lost mass to underflow (none, usually), every
rank's exact partial sums of its own tokens, so the merge stays exact for any
split of the tokens.

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


def allgather_partials(part, world: int, group=None, stream=None):
    """Concatenate every rank's partials in rank order: [world * part.numel()].

    The library writes ``part`` and reads the result on ``stream`` (None: the
    current stream), while the collective runs on torch's current stream.
    When the two differ, the collective first waits for ``stream``, ``stream``
    then waits for the collective, and both buffers are recorded as used on
    ``stream`` so that the caching allocator does not hand their memory out
    while a library kernel may still touch it."""
    torch = b._torch()
    cur = torch.cuda.current_stream(part.device) if part.is_cuda else None
    other = part.is_cuda and stream is not None and stream != cur
    if other:
        part.record_stream(stream)
    if world == 1:
        return part
    import torch.distributed as dist
    if other:
        cur.wait_stream(stream)
    out = torch.empty(world * part.numel(), dtype=part.dtype, device=part.device)
    dist.all_gather_into_tensor(out, part, group=group)
    if other:
        stream.wait_stream(cur)
        out.record_stream(stream)
    return out


def partials_numel(B: int, H: int, N: int, M: int, D: int) -> int:
    nbytes = b.load_library().flare_cp_partials_bytes(B, H, N, M, D)
    if nbytes == 0:
        raise ValueError("unsupported sizes")
    return nbytes // 4


def exact_numel(B: int, H: int, M: int, D: int) -> int:
    nbytes = b.load_library().flare_cp_exact_bytes(B, H, M, D)
    if nbytes == 0:
        raise ValueError("unsupported sizes")
    return nbytes // 4


def _status(st, where):
    if st != 0:
        raise b.FlareError(st, where)


def _device_status(device_check, workspace_given, ws, stream, where):
    """After the last phase: read the workspace's device error word (a merged
    row whose sums underflowed, a length outside [1, N], an expired bounded
    wait) and raise FlareError if it is set; synchronises the stream.  Done by
    default when the workspace was allocated here (the caller cannot query
    it)."""
    if device_check is None:
        device_check = not workspace_given
    if device_check:
        st = b.load_library().flare_last_device_status(b._ptr(ws), b._stream_ptr(stream, ws.device))
        if st != 0:
            raise b.FlareError(st, where + " (device status)")


def flarepp_mixer_cp_fwd(X, Wk, Wv, Wk_syn, Wv_syn, Q0, lengths=None, group=None, scale: float = 0.0,
                         Y=None, workspace=None, stream=None, Qx_out=None, Z_out=None, device_check=None):
    """FLARE++ forward of this rank's token shard X [B, N, C] (tokens
    [rank*N, (rank+1)*N) of sequences of world*N tokens; ``lengths`` counts
    tokens of the whole sequences).  Returns Y [B, H, N, D] of the shard.
    ``stream``: a torch stream for the library's kernels (None: the current
    stream).  ``device_check``: see ``_device_status``."""
    torch = b._torch()
    rank, world = _group_info(group)
    B, N, C = X.shape
    H, M, D = Q0.shape
    lib = b.load_library()
    if Y is None:
        Y = torch.empty((B, H, N, D), dtype=torch.bfloat16, device=X.device)
    nbytes = b.flare_workspace_bytes(b.FLARE_VARIANT_FLAREPP, B, H, N, M, D, C)
    ws = b._workspace(workspace, nbytes, X.device)
    if stream is not None and X.is_cuda:
        ws.record_stream(stream)
    st = b._stream_ptr(stream, X.device)
    part = torch.empty(partials_numel(B, H, N, M, D), dtype=torch.float32, device=X.device)
    exact = torch.empty(exact_numel(B, H, M, D), dtype=torch.float32, device=X.device)
    weights = [b._ptr(t) for t in (Wk, Wv, Wk_syn, Wv_syn, Q0)]
    common = (B, N, C, H, M, D, b._ptr(lengths), rank, world, float(scale), b._ptr(ws), ws.numel(), st)
    _status(lib.flarepp_cp_begin(b._ptr(X), *weights, *common, b._ptr(part)), "flarepp_cp_begin")
    gathered = allgather_partials(part, world, group, stream)
    _status(lib.flarepp_cp_exact(0, b._ptr(gathered), *weights, *common, b._ptr(exact)), "flarepp_cp_exact(0)")
    gathered_exact = allgather_partials(exact, world, group, stream)
    part2 = torch.empty_like(part)
    _status(lib.flarepp_cp_middle(b._ptr(gathered), b._ptr(gathered_exact), *common, b._ptr(part2),
                                  b._ptr(Qx_out)), "flarepp_cp_middle")
    gathered = allgather_partials(part2, world, group, stream)
    exact2 = torch.empty_like(exact)
    _status(lib.flarepp_cp_exact(1, b._ptr(gathered), *weights, *common, b._ptr(exact2)), "flarepp_cp_exact(1)")
    gathered_exact = allgather_partials(exact2, world, group, stream)
    _status(lib.flarepp_cp_end(b._ptr(gathered), b._ptr(gathered_exact), b._ptr(Y), *common, b._ptr(Z_out)),
            "flarepp_cp_end")
    _device_status(device_check, workspace is not None, ws, stream, "flarepp_mixer_cp_fwd")
    return Y


def flare_mixer_cp_fwd(K, V, Q, lengths=None, group=None, scale: float = 0.0, Y=None, workspace=None,
                       stream=None, Z_out=None, device_check=None):
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
    if stream is not None and K.is_cuda:
        ws.record_stream(stream)
    st = b._stream_ptr(stream, K.device)
    part = torch.empty(partials_numel(B, H, N, M, D), dtype=torch.float32, device=K.device)
    exact = torch.empty(exact_numel(B, H, M, D), dtype=torch.float32, device=K.device)
    common = (B, H, N, M, D, b._ptr(lengths), rank, world, float(scale), b._ptr(ws), ws.numel(), st)
    _status(lib.flare_cp_begin(b._ptr(K), b._ptr(V), b._ptr(Q), *common, b._ptr(part)), "flare_cp_begin")
    gathered = allgather_partials(part, world, group, stream)
    _status(lib.flare_cp_exact(b._ptr(gathered), b._ptr(K), b._ptr(V), b._ptr(Q), *common, b._ptr(exact)),
            "flare_cp_exact")
    gathered_exact = allgather_partials(exact, world, group, stream)
    _status(lib.flare_cp_end(b._ptr(gathered), b._ptr(gathered_exact), b._ptr(K), b._ptr(Q), b._ptr(Y), *common,
                             b._ptr(Z_out)), "flare_cp_end")
    _device_status(device_check, workspace is not None, ws, stream, "flare_mixer_cp_fwd")
    return Y


FLARE_CP_BWD_PHASES = 7
FLARE_CP_BWD_PHASES_FLARE = 4


def flare_mixer_cp_bwd(K, V, Q, dY, lengths=None, group=None, scale: float = 0.0, workspace=None, stream=None,
                       dK=None, dV=None, dQ=None, device_check=None):
    """FLARE backward of this rank's token shard (the sharding of
    flare_mixer_cp_fwd; K, V, dY [B, H, N, D] hold the shard's rows).
    Returns (dK, dV) of the shard's rows (bf16) and dQ [H, M, D] (fp32,
    bitwise the same on every rank).  Four phases with one all-gather of a
    small fp32 buffer between two of them."""
    torch = b._torch()
    rank, world = _group_info(group)
    B, H, N, D = K.shape
    M = Q.shape[1]
    dev = K.device
    lib = b.load_library()
    dK = torch.empty_like(K) if dK is None else dK
    dV = torch.empty_like(K) if dV is None else dV
    dQ = torch.empty((H, M, D), dtype=torch.float32, device=dev) if dQ is None else dQ
    nbytes = b.flare_workspace_bytes(b.FLARE_VARIANT_FLARE_BWD, B, H, N, M, D)
    ws = b._workspace(workspace, nbytes, dev)
    if stream is not None and K.is_cuda:
        ws.record_stream(stream)
    st = b._stream_ptr(stream, dev)
    ins = [b._ptr(t) for t in (K, V, Q, dY)]
    outs = [b._ptr(t) for t in (dK, dV, dQ)]
    gathered = None
    for phase in range(FLARE_CP_BWD_PHASES_FLARE):
        exch = None
        if phase < FLARE_CP_BWD_PHASES_FLARE - 1:
            nb = lib.flare_cp_bwd_exchange_bytes(phase, B, H, N, M, D)
            if nb == 0:
                raise ValueError("unsupported sizes")
            exch = torch.empty(nb // 4, dtype=torch.float32, device=dev)
        _status(lib.flare_cp_bwd_phase(phase, *ins, b._ptr(gathered), b._ptr(exch), *outs, B, H, N, M, D,
                                       b._ptr(lengths), rank, world, float(scale), b._ptr(ws), ws.numel(), st),
                f"flare_cp_bwd_phase({phase})")
        if exch is not None:
            gathered = allgather_partials(exch, world, group, stream)
    _device_status(device_check, workspace is not None, ws, stream, "flare_mixer_cp_bwd")
    return dK, dV, dQ


def flarepp_mixer_cp_bwd(X, Wk, Wv, Wk_syn, Wv_syn, Q0, dY, lengths=None, group=None, scale: float = 0.0,
                         workspace=None, stream=None, grads=None, device_check=None):
    """FLARE++ backward of this rank's token shard (the same sharding as
    flarepp_mixer_cp_fwd; dY [B, H, N, D] holds the shard's rows).  Returns a
    dict: dX [B, N, C] (the shard's rows), dWk, dWv, dWk_syn, dWv_syn, dQ0
    (bitwise the same on every rank).  Seven phases with one all-gather of a
    small fp32 buffer between two of them."""
    torch = b._torch()
    rank, world = _group_info(group)
    B, N, C = X.shape
    H, M, D = Q0.shape
    dev = X.device
    lib = b.load_library()
    g = dict(grads or {})
    if g.get("dX") is None:
        g["dX"] = torch.empty((B, N, C), dtype=torch.bfloat16, device=dev)
    for nm in ("dWk", "dWv", "dWk_syn", "dWv_syn"):
        if g.get(nm) is None:
            g[nm] = torch.empty((C, C), dtype=torch.float32, device=dev)
    if g.get("dQ0") is None:
        g["dQ0"] = torch.empty((H, M, D), dtype=torch.float32, device=dev)
    nbytes = b.flare_workspace_bytes(b.FLARE_VARIANT_FLAREPP_BWD, B, H, N, M, D, C)
    ws = b._workspace(workspace, nbytes, dev)
    if stream is not None and X.is_cuda:
        ws.record_stream(stream)
    st = b._stream_ptr(stream, dev)
    ins = [b._ptr(t) for t in (X, Wk, Wv, Wk_syn, Wv_syn, Q0, dY)]
    outs = [b._ptr(g[k]) for k in ("dX", "dWk", "dWv", "dWk_syn", "dWv_syn", "dQ0")]
    gathered = None
    for phase in range(FLARE_CP_BWD_PHASES):
        exch = None
        if phase < FLARE_CP_BWD_PHASES - 1:
            nb = lib.flarepp_cp_bwd_exchange_bytes(phase, B, N, C, H, M, D)
            if nb == 0:
                raise ValueError("unsupported sizes")
            exch = torch.empty(nb // 4, dtype=torch.float32, device=dev)
        _status(lib.flarepp_cp_bwd_phase(phase, *ins, b._ptr(gathered), b._ptr(exch), *outs, B, N, C, H, M, D,
                                         b._ptr(lengths), rank, world, float(scale), b._ptr(ws), ws.numel(), st),
                f"flarepp_cp_bwd_phase({phase})")
        if exch is not None:
            gathered = allgather_partials(exch, world, group, stream)
    _device_status(device_check, workspace is not None, ws, stream, "flarepp_mixer_cp_bwd")
    return g
