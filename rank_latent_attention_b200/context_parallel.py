"""Token-sharded (context-parallel) FLARE++ mixer over torch.distributed.

"FLARE++: Low-rank attention with dynamic attention routing", section
"Contributions Clés", multi-GPU context-parallelism item: the input tokens
are split over the devices, the encoder gathers them into latent tokens that
every device holds a copy of, and the devices exchange only latent outputs
and softmax statistics, never the N tokens.

Per rank r, holding tokens [start_r, stop_r) of every head:

1. seed encode on the local shard: (O_r, lse_r) = flare_encode_lse(seeds, K_r, V_r)
2. one all-gather of the B*H*M*(D+1) floats [O_r | lse_r] from every rank
3. Q_dyn = flare_lse_combine(gathered)            (identical on every rank)
4. routing encode on the local shard, all-gather, combine -> Z
5. decode of the local tokens: Y_r = flare_decode(K_r, Q_dyn, Z)

Every rank takes the same two collectives in the same order.  The kernels are
the library's; this module only slices, allocates and calls the collective.
``ops`` lets the CPU tests run the same sequence with other implementations
of the four steps (the library itself has no CPU path).

Training: ``flarepp_mix_cp(..., save=True)`` also keeps the whole cloud's
Q_dyn, Z and the two encodes' log-sum-exps (in flarepp_mix_save's layout),
and ``flarepp_mix_backward_cp`` runs the backward in the library's four
phases with an all-reduce of the exchange buffer between them: the token
reductions dZ, dQ_dyn and d_seeds are summed over the ranks, dK and dV stay
with each rank's tokens.
"""
from __future__ import annotations

__all__ = ["token_range", "shard_tokens", "LibraryOps", "flarepp_mix_cp", "flarepp_mix_backward_cp",
           "exchange_floats", "saved_views"]


def token_range(N: int, world: int, rank: int) -> tuple[int, int]:
    """Rank ``rank``'s contiguous token range [start, stop) of ``N`` tokens
    over ``world`` ranks; sizes differ by at most one, and ranks past N get
    an empty range."""
    if not (0 <= rank < world) or N < 0:
        raise ValueError(f"bad shard request N={N} world={world} rank={rank}")
    return (rank * N) // world, ((rank + 1) * N) // world


def shard_tokens(X, world: int, rank: int):
    """This rank's tokens of X [B, H, N, D], contiguous."""
    a, b = token_range(X.shape[2], world, rank)
    return X[:, :, a:b].contiguous()


def exchange_floats(B: int, H: int, M: int, D: int) -> int:
    """Floats each rank sends per encode: O [B,H,M,D] then lse [B,H,M]."""
    return B * H * M * (D + 1)


def saved_views(saved, B: int, H: int, M: int, D: int, dtype, lse_dtype=None):
    """Views (Q_dyn, Z, lse1, lse2) into a saved-state byte buffer laid out as
    flarepp_mix_save writes it: Q_dyn and Z [B,H,M,D] in dtype, then lse1 and
    lse2 [B,H,M] (fp32 unless lse_dtype says otherwise), each region starting
    on a 256-byte boundary."""
    import torch

    lse_dtype = lse_dtype or torch.float32
    esz = torch.empty((), dtype=dtype).element_size()
    lsz = torch.empty((), dtype=lse_dtype).element_size()
    lat = B * H * M

    def region(off, n, dt, shape):
        return saved[off:off + n * torch.empty((), dtype=dt).element_size()].view(dt).view(shape)

    r = lambda x: (x + 255) // 256 * 256  # noqa: E731
    o1 = r(lat * D * esz)
    o2 = o1 + r(lat * D * esz)
    o3 = o2 + r(lat * lsz)
    return (region(0, lat * D, dtype, (B, H, M, D)), region(o1, lat * D, dtype, (B, H, M, D)),
            region(o2, lat, lse_dtype, (B, H, M)), region(o3, lat, lse_dtype, (B, H, M)))


def all_reduce_sum(t, group=None):
    """Sum of t over the ranks, in place (one rank: nothing to do)."""
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
    return t


def gather_rows(send, group=None):
    """All-gather of one flat tensor per rank into [world, numel] (rank order).
    Without an initialised process group the job is one rank."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()):
        return send.unsqueeze(0)
    world = dist.get_world_size(group)
    recv = torch.empty(world * send.numel(), dtype=send.dtype, device=send.device)
    dist.all_gather_into_tensor(recv, send, group=group)
    return recv.view(world, send.numel())


class LibraryOps:
    """The GPU steps: the library's kernels and a NCCL all-gather."""

    exchange_dtype = "float32"  # what flare_encode_lse writes and flare_lse_combine reads

    def __init__(self, group=None, workspace=None):
        self.group = group
        self.workspace = workspace  # device scratch for flare_encode_lse (None: the library allocates)

    def encode_lse(self, Q, K, V, send):
        import rank_latent_attention_b200 as flare

        B, H, _, D = K.shape
        M = Q.shape[-2]
        n = B * H * M * D
        flare.flare_encode_lse(Q, K, V, O=send[:n].view(B, H, M, D), lse=send[n:].view(B, H, M),
                               workspace=self.workspace)

    def all_gather(self, send):
        return gather_rows(send, self.group)

    def combine(self, recv, B, H, M, D, dtype, out=None, lse_out=None):
        import rank_latent_attention_b200 as flare

        flat = recv.view(-1)
        n = B * H * M * D
        return flare.flare_lse_combine(flat, flat[n:], out=out, lse_out=lse_out, dtype=dtype,
                                       shape=(recv.shape[0], B, H, M, D), part_stride=recv.shape[1])

    def saved_bytes(self, B, H, M, D, dtype):
        import rank_latent_attention_b200 as flare

        return flare.flarepp_saved_bytes(B, H, M, D, dtype)

    def all_reduce(self, t):
        return all_reduce_sum(t, self.group)

    def backward_state(self, seeds, K, M):
        """Exchange buffer and the workspace kept across the four phases."""
        import torch

        import rank_latent_attention_b200 as flare

        B, H, N, D = K.shape
        lib = flare.lib()
        code = flare.BF16 if K.dtype == torch.bfloat16 else flare.F32
        exch = torch.empty(lib.flarepp_backward_shard_exchange_floats(B, H, M, D), dtype=torch.float32,
                           device=K.device)
        ws = torch.empty(max(1, lib.flarepp_backward_shard_workspace_size(B, H, N, M, D, code)), dtype=torch.uint8,
                         device=K.device)
        return exch, ws

    def backward_phase(self, phase, seeds, K, V, dY, saved, exch, ws, grads):
        import rank_latent_attention_b200 as flare

        flare.flarepp_mix_backward_shard(phase, seeds, K, V, dY, saved, exch, *grads, ws)

    def decode(self, K, Q, Z):
        import torch

        import rank_latent_attention_b200 as flare

        if K.shape[2] == 0:  # a rank without tokens has nothing to decode
            return torch.empty_like(K)
        return flare.flare_decode(K, Q, Z)


def flarepp_mix_cp(seeds, K, V, *, group=None, ops=None, return_intermediates=False, save=False):
    """FLARE++ forward of this rank's token shard.

    seeds [H, M, D] (every rank the same); K, V [B, H, N_r, D]: this rank's
    tokens (N_r may be 0).  Returns Y [B, H, N_r, D] for the local tokens,
    and with ``return_intermediates`` also the replicated Q_dyn and Z
    [B, H, M, D]; with ``save`` also the saved state for
    ``flarepp_mix_backward_cp`` (last element).
    """
    import torch

    ops = ops or LibraryOps(group)
    B, H, _, D = K.shape
    M = seeds.shape[-2]
    send = torch.empty(exchange_floats(B, H, M, D), dtype=getattr(torch, ops.exchange_dtype), device=K.device)
    saved = views = None
    if save:
        saved = torch.empty(ops.saved_bytes(B, H, M, D, K.dtype), dtype=torch.uint8, device=K.device)
        views = saved_views(saved, B, H, M, D, K.dtype, getattr(ops, "lse_dtype", None))

    ops.encode_lse(seeds, K, V, send)
    Q_dyn = ops.combine(ops.all_gather(send), B, H, M, D, K.dtype,
                        *((views[0], views[2]) if save else ()))
    ops.encode_lse(Q_dyn, K, V, send)
    Z = ops.combine(ops.all_gather(send), B, H, M, D, K.dtype, *((views[1], views[3]) if save else ()))
    Y = ops.decode(K, Q_dyn, Z)
    out = (Y, Q_dyn, Z) if return_intermediates else (Y,)
    if save:
        out = out + (saved,)
    return out if len(out) > 1 else out[0]


def flarepp_mix_backward_cp(seeds, K, V, dY, saved, *, group=None, ops=None):
    """Gradients (d_seeds, dK, dV) of sum(dY * Y) for the sharded forward:
    d_seeds summed over all ranks' tokens (identical on every rank), dK and dV
    for this rank's tokens.  Three all-reduces of the exchange buffer, the same
    on every rank."""
    import torch

    ops = ops or LibraryOps(group)
    B, H, _, D = K.shape
    M = seeds.shape[-2]
    grads = (torch.empty_like(seeds), torch.empty_like(K), torch.empty_like(V))
    exch, ws = ops.backward_state(seeds, K, M)
    lat = B * H * M * D
    for phase, n in ((0, 2 * lat), (1, lat), (2, H * M * D), (3, 0)):
        ops.backward_phase(phase, seeds, K, V, dY, saved, exch, ws, grads)
        if n:
            ops.all_reduce(exch[:n])
    return grads
