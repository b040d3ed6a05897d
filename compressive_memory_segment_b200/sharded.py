"""Sequence-sharded forward: one long sequence split over the ranks of a
process group, each rank holding a block of consecutive segments.

Only (M, z) crosses a segment boundary ("Hugging Face Infini-Attention
reproduction analysis", section "Infini-Attention mechanism", State Transfer),
and M and z are sums over segments. So the ranks exchange one thing: each
block's totals (B*H*(d*d + d) fp32 values, 528 KB for 8 heads at d = 128), in
one all-gather. Rank r then starts its cross-segment prefix from the caller's
state plus the totals of ranks 0..r-1 and runs its block's attention. Every
step of the layer runs in the library's kernels (infini_attn_state_ws,
infini_attn_exscan_parts, infini_attn_finish_ws); this module only moves the
totals between ranks with torch.distributed (NCCL between GPUs).
"""
from __future__ import annotations

from typing import Optional


class CudaPhases:
    """The three phases through the C ABI, on device tensors."""

    def __init__(self, stream=None):
        from compressive_memory_segment_b200 import binding as bd
        self.bd = bd
        self.stream = stream

    def workspace(self, q, seg_len: int):
        return self.bd.workspace_for(q, seg_len)

    def state(self, k, v, seg_len: int, ws):
        import torch
        bd = self.bd
        B, H, L, d = k.shape
        M_tot = torch.empty((B, H, d, d), dtype=torch.float32, device=k.device)
        z_tot = torch.empty((B, H, d), dtype=torch.float32, device=k.device)
        bd.check(bd.infini_attn_state_ws(bd.shape_of(k), k, v, seg_len, M_tot, z_tot, ws,
                                         ws.numel() * ws.element_size(), bd.INFINI_PATH_AUTO, self.stream))
        return M_tot, z_tot

    def exscan(self, totals_M, totals_z, part: int, M_in, z_in):
        import torch
        bd = self.bd
        n_parts = totals_M.shape[0]
        off_M = torch.empty(totals_M.shape[1:], dtype=torch.float32, device=totals_M.device)
        off_z = torch.empty(totals_z.shape[1:], dtype=torch.float32, device=totals_z.device)
        bd.check(bd.infini_attn_exscan_parts(off_M.numel(), off_z.numel(), n_parts, part, totals_M, totals_z,
                                             M_in, z_in, off_M, off_z, self.stream))
        return off_M, off_z

    def finish(self, q, k, v, beta, M_in, z_in, seg_len: int, ws, out=None):
        import torch
        bd = self.bd
        B, H, L, d = q.shape
        out = torch.empty_like(q) if out is None else out
        M_out = torch.empty((B, H, d, d), dtype=torch.float32, device=q.device)
        z_out = torch.empty((B, H, d), dtype=torch.float32, device=q.device)
        bd.check(bd.infini_attn_finish_ws(bd.shape_of(q), q, k, v, beta, M_in, z_in, seg_len, out, M_out, z_out,
                                          ws, ws.numel() * ws.element_size(), bd.INFINI_PATH_AUTO, self.stream))
        return out, M_out, z_out


def forward_sequence_sharded(q, k, v, beta, seg_len: int, M_in=None, z_in=None, group=None,
                             phases=None, workspace=None, share_final_state: bool = True):
    """This rank's block of the sequence: q, k, v [B, H, L_r, d] with L_r a
    multiple of seg_len; ranks hold consecutive blocks in rank order. M_in, z_in
    (the state before the whole sequence) must be the same on every rank.

    Returns (out [B, H, L_r, d], M_out, z_out). M_out, z_out are the state after
    this rank's block; with share_final_state every rank gets the state after
    the whole sequence (broadcast from the last rank).
    """
    import torch
    import torch.distributed as dist
    ph = phases if phases is not None else CudaPhases()
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    ws = workspace if workspace is not None else ph.workspace(q, seg_len)

    M_tot, z_tot = ph.state(k, v, seg_len, ws)
    n_M, n_z = M_tot.numel(), z_tot.numel()
    packed = torch.cat([M_tot.reshape(-1), z_tot.reshape(-1)])
    parts = [torch.empty_like(packed) for _ in range(world)]
    dist.all_gather(parts, packed, group=group)
    allp = torch.stack(parts)                              # [world, n_M + n_z], rank order
    totals_M = allp[:, :n_M].contiguous().view((world,) + tuple(M_tot.shape))
    totals_z = allp[:, n_M:].contiguous().view((world,) + tuple(z_tot.shape))
    off_M, off_z = ph.exscan(totals_M, totals_z, rank, M_in, z_in)
    out, M_out, z_out = ph.finish(q, k, v, beta, off_M, off_z, seg_len, ws)
    if share_final_state and world > 1:
        last = dist.get_global_rank(group, world - 1) if group is not None else world - 1
        dist.broadcast(M_out, src=last, group=group)
        dist.broadcast(z_out, src=last, group=group)
    return out, M_out, z_out


def forward_blocks_one_device(blocks, beta, seg_len: int, M_in=None, z_in=None,
                              phases: Optional[CudaPhases] = None):
    """The same decomposition run block after block on one device (no
    collective): for tests of the phases, and for callers that process a long
    sequence in pieces. blocks: a list of (q, k, v) for consecutive blocks.
    Returns the per-block outputs and the final state."""
    import torch
    ph = phases if phases is not None else CudaPhases()
    wss = [ph.workspace(q, seg_len) for (q, _, _) in blocks]
    tots = [ph.state(k, v, seg_len, ws) for (q, k, v), ws in zip(blocks, wss)]
    totals_M = torch.stack([t[0] for t in tots])
    totals_z = torch.stack([t[1] for t in tots])
    outs, M_out, z_out = [], None, None
    for r, ((q, k, v), ws) in enumerate(zip(blocks, wss)):
        off_M, off_z = ph.exscan(totals_M, totals_z, r, M_in, z_in)
        o, M_out, z_out = ph.finish(q, k, v, beta, off_M, off_z, seg_len, ws)
        outs.append(o)
    return outs, M_out, z_out
