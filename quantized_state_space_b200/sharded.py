"""Sequence-sharded SSD chunk scan and Mamba-1 selective scan over a
torch.distributed group.

Rank r owns the r-th consecutive slice of the time axis.  The recurrence is
linear in the state, so each rank scans its slice from a zero state (rank 0
from h0) and emits the slice's final state and total log2 decay per (batch,
head), or per (batch, channel, state) for Mamba-1; one all-gather exchanges
these summaries (4 (P N + 1) bytes per (batch, head) and rank; 8 N bytes per
(batch, channel) and rank for Mamba-1); each rank folds its predecessors' summaries into the
start state its slice should have had and adds that state's contribution,
exp(S_t) C_t h_carry (gated like y), to its y; every rank also folds all of
them into the whole sequence's final state.  The scan, the fold and the
carry-in run in the library's kernels; the exchange is the group's
all-gather (NCCL between GPUs, gloo on the host).
"""
import torch
import torch.distributed as dist

from . import api

# keyword arguments that the slice scan and its carry-in both take
_SHARED = ("chunk", "x_group", "x_scale", "se_scale", "se_log2_ratio", "D", "z", "dt_bias",
           "dt_softplus", "workspace", "status")
# keyword arguments of the Mamba-1 slice scan; its carry-in takes the subset
# _SHARED_M1_CARRY
_SHARED_M1 = ("x_group", "x_scale", "se_scale", "se_log2_ratio", "se_lo", "se_hi", "D", "z",
              "dt_bias", "dt_softplus", "status")
_SHARED_M1_CARRY = ("D", "z", "dt_bias", "dt_softplus", "status")


def exchange(h_end, dec, group=None):
    """All-gather of the slice summaries (final state, total log2 decay), in
    rank order."""
    world = dist.get_world_size(group)
    hs = [torch.empty_like(h_end) for _ in range(world)]
    ds = [torch.empty_like(dec) for _ in range(world)]
    dist.all_gather(hs, h_end.contiguous(), group=group)
    dist.all_gather(ds, dec.contiguous(), group=group)
    return hs, ds


def ssd_chunk_scan_sequence_sharded(x, dt, A, B, C, B_scale, C_scale, state_group_size, *,
                                    group=None, h0=None, **kw):
    """This rank's slice (x, dt, B, C, z of its steps) of one sequence batch.
    Returns (y of the slice, final state of the whole sequence); every rank
    takes the same collective steps."""
    unknown = set(kw) - set(_SHARED)
    if unknown:
        raise TypeError("unsupported arguments: %s" % sorted(unknown))
    rank = dist.get_rank(group)
    b, _, H, _ = x.shape
    dec = torch.empty((b, H), dtype=torch.float32, device=x.device)
    y, h_end = api.ssd_chunk_scan(x, dt, A, B, C, B_scale, C_scale, state_group_size,
                                  h0=h0 if rank == 0 else None, dec_final=dec, **kw)
    hs, ds = exchange(h_end, dec, group)
    if rank > 0:
        h_carry = api.state_chain(hs[:rank], ds[:rank])
        api.ssd_carry_in(x, dt, A, B, C, B_scale, C_scale, state_group_size, h_carry, y, **kw)
    return y, api.state_chain(hs, ds)


def selective_scan_sequence_sharded(x, dt, A, B, C, B_scale, C_scale, state_group_size, *,
                                    group=None, h0=None, **kw):
    """Mamba-1 form: this rank's slice (x, dt, z (b, d, L_r); B, C
    (b, G, N, L_r)) of one sequence batch.  Returns (y of the slice, final
    state of the whole sequence); every rank takes the same collective
    steps."""
    unknown = set(kw) - set(_SHARED_M1)
    if unknown:
        raise TypeError("unsupported arguments: %s" % sorted(unknown))
    rank = dist.get_rank(group)
    b, d, _ = x.shape
    Nst = B.shape[2]
    dec = torch.empty((b, d, Nst), dtype=torch.float32, device=x.device)
    y, h_end = api.selective_scan(x, dt, A, B, C, B_scale, C_scale, state_group_size,
                                  h0=h0 if rank == 0 else None, dec_final=dec, **kw)
    hs, ds = exchange(h_end, dec, group)
    if rank > 0:
        h_carry = api.state_chain(hs[:rank], ds[:rank])
        api.selective_scan_carry_in(x, dt, A, B, C, B_scale, C_scale, state_group_size, h_carry,
                                    y, **{k: v for k, v in kw.items() if k in _SHARED_M1_CARRY})
    return y, api.state_chain(hs, ds)
