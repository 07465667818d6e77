"""A sequence split across devices: the real scan of one long sequence on R ranks.

Rank r holds the r-th slice of consecutive tokens (x, dt, B, C of those tokens;
A and D whole).  The state passing of "Block Anatomy, Numerical Stability &
Scaling" (Numerical Stability, section 4) carries each chunk's end state into
the later chunks through the decay between them; at slice granularity that is
one exchange:

1. every rank scans its slice state-only (``ssd_scan_final_state``), from a zero
   state (rank 0 from the caller's initial state): its end state S_r and total
   log-decay Lam_r;
2. the ranks all-gather (S_r, Lam_r): 4 * P * N bytes per (batch, head) and rank;
3. rank r folds those of the ranks before it (``ssd_fold_states``) into the
   state entering its slice, h_0 = S_0, h_j = exp(Lam_j) h_{j-1} + S_j;
4. rank r scans its slice in full from that state (``ssd_scan_fwd``): its y, and
   the true state at the end of its slice.

Every arithmetic step runs in the library's kernels; torch.distributed moves the
states (NCCL on GPUs).  The received states land in local device memory before
use.  ``ops`` swaps the three steps for another implementation of the same
functions (the CPU tests pass the oracle's, to check the exchange itself).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


class LibraryOps:
    """The three steps on the device, through libssd."""

    def final_state(self, x, dt, A, B, init_state, chunk_size):
        from . import ssd_scan_final_state

        return ssd_scan_final_state(x, dt, A, B, init_state, chunk_size=chunk_size)

    def fold(self, states, log_decay):
        from . import ssd_fold_states

        return ssd_fold_states(states, log_decay)

    def scan(self, x, dt, A, B, C, D, init_state, chunk_size):
        from . import ssd_scan_fwd

        return ssd_scan_fwd(x, dt, A, B, C, D, init_state, chunk_size=chunk_size)


def scan_fwd_sequence_parallel(x, dt, A, B, C, D=None, init_state=None, *, chunk_size=256, group=None,
                               ops=None):
    """The scan of one sequence cut into consecutive slices, one per rank of
    ``group``; each rank passes its own slice (and rank 0 the initial state, if
    any).  Returns (y of this rank's slice, state at the end of this slice); the
    last rank's is the sequence's final state."""
    ops = ops or LibraryOps()
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    if world == 1:
        return ops.scan(x, dt, A, B, C, D, init_state, chunk_size)
    S, lam = ops.final_state(x, dt, A, B, init_state if rank == 0 else None, chunk_size)
    S_all = [torch.empty_like(S) for _ in range(world)]
    lam_all = [torch.empty_like(lam) for _ in range(world)]
    dist.all_gather(S_all, S.contiguous(), group=group)
    dist.all_gather(lam_all, lam.contiguous(), group=group)
    if rank == 0:
        h_in = init_state
    else:
        h_in = ops.fold(torch.stack(S_all[:rank]).contiguous(), torch.stack(lam_all[:rank]).contiguous())
    return ops.scan(x, dt, A, B, C, D, h_in, chunk_size)
