"""Sequence-parallel prefill across ranks: Chunk Parallelism.

"YOCO 深度技术分析", section 5.3.3: when one sequence is split over devices, gated
retention passes only its state between them (the state has d_k x d_v numbers
per head, however long the slices are).  Rank r of the group holds the r-th
contiguous slice of the same B x H sequences.  The prefill then takes one
exchange step:

1. every rank computes its slice's state increment dS_r and total log-decay
   a_r (``prefill_state``: K, V and the gate only);
2. the ranks all-gather (dS, a) -- d_k x d_v + 1 floats per (batch, head);
3. every rank folds the slices before it into its initial state
   (``state_fold``: S_in(r) = e^{a_{r-1}} S_in(r-1) + dS_{r-1}, S_in(0) = S0);
4. every rank runs the prefill of its slice from S_in(r)
   (``prefill`` with ``S0`` and ``resume``: the decay sums and state pieces
   of step 1 are taken from its workspace, so the slice's K and V are read by
   one state pass, as in a prefill on one device).

The last rank's final state is the state after the whole sequence.  The
collectives are torch.distributed calls (NCCL over NVLink on GPUs); every
computing step runs in libgret.  ``ops`` lets a caller substitute the three
computing steps (the host logic is tested that way on CPU ranks).
"""
from __future__ import annotations


class LibraryOps:
    """The three computing steps as libgret calls (CUDA tensors).  The state
    pass's workspace is kept for the prefill of the same slice."""

    def __init__(self, workspace=None):
        self.workspace = workspace

    def state(self, K, V, z, tau, chunk):
        from .gret import gret_prefill_state_workspace_size, prefill_state, _io_of
        import torch
        B, N, H, dk = K.shape
        need = gret_prefill_state_workspace_size(B, H, N, dk, V.shape[-1], chunk, _io_of(K))
        if self.workspace is None or self.workspace.numel() * self.workspace.element_size() < need:
            self.workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=K.device)
        return prefill_state(K, V, z, tau, chunk, workspace=self.workspace)

    def fold(self, dS_all, decay_all, rank, S0):
        from .gret import state_fold
        return state_fold(dS_all, decay_all, rank, S0=S0)

    def prefill_from(self, Q, K, V, z, G, tau, chunk, eps, S_in):
        from .gret import prefill
        return prefill(Q, K, V, z, G, tau, chunk, eps=eps, S0=S_in, workspace=self.workspace, resume=True)


def prefill_sequence_parallel(Q, K, V, z, G, tau: float, chunk: int, eps: float = 1e-5, S0=None, group=None,
                              ops=None):
    """Prefill of this rank's slice of sequences split across the ranks of ``group``.

    Q, K [B,N_r,H,dk]; V, G [B,N_r,H,dv]; z [B,N_r,H]: this rank's tokens, which
    follow those of every lower rank.  S0 [B,H,dk,dv] (the state before rank 0's
    first token) or None, the same on every rank.  Returns (O of this slice,
    state after this slice)."""
    import torch
    import torch.distributed as dist

    ops = ops or LibraryOps()
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    dS, decay = ops.state(K, V, z, tau, chunk)
    # gathered along the batch dimension, then seen as [world][B]...: rank r's slice first
    dS_all = torch.empty((world * dS.shape[0],) + tuple(dS.shape[1:]), dtype=dS.dtype, device=dS.device)
    decay_all = torch.empty((world * decay.shape[0],) + tuple(decay.shape[1:]), dtype=decay.dtype,
                            device=decay.device)
    dist.all_gather_into_tensor(dS_all, dS.contiguous(), group=group)
    dist.all_gather_into_tensor(decay_all, decay.contiguous(), group=group)
    dS_all = dS_all.view((world,) + tuple(dS.shape))
    decay_all = decay_all.view((world,) + tuple(decay.shape))
    S_in = ops.fold(dS_all, decay_all, rank, S0)
    return ops.prefill_from(Q, K, V, z, G, tau, chunk, eps, S_in)
