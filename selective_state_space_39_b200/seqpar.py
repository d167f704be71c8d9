"""One sequence split across ranks (sequence parallelism) for the scan.

A contiguous chunk of steps acts on the state as the affine map
h -> exp(A_n sum Delta) h + e, e being the chunk's end state from a zero start
(the discretised recurrence of the page "Mamba 논문 리뷰", §2.2; the maps
compose associatively, as in the parallel scan of the page "맘바(Mamba)와
상태공간모델(SSM) 쉽게 이해하기"). Rank r, holding chunk r of the sequence
in order, therefore needs one exchange: the carries (e, sum Delta) of every
rank, from which it composes its true entering state and scans its chunk
again from there. All compute runs in libssmscan.so's kernels; the exchange
is one all-gather of 4 (N + 1) bytes per (batch row, channel) and rank.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from ._binding import ssm_compose_carries, ssm_delta_sum, ssm_scan_fwd


def chunk_carry(x, delta, A, B, C, D=None, z=None, delta_bias=None, softplus=True):
    """(e, dsum) of this chunk: its end state from a zero start (batch, dim,
    N) and its sum of Delta (batch, dim), both float32. No y is written."""
    _, e = ssm_scan_fwd(x, delta, A, B, C, D=D, z=z, delta_bias=delta_bias, softplus=softplus,
                        h0=None, return_y=False)
    return e, ssm_delta_sum(delta, delta_bias, softplus)


def entering_state(rank, A, hend_all, dsum_all, h0=None):
    """The state entering chunk `rank`, from the gathered carries
    (hend_all (R, batch, dim, N), dsum_all (R, batch, dim)) and the
    sequence's initial state h0 (or zero)."""
    return ssm_compose_carries(rank, A, hend_all, dsum_all, h0=h0)


class CudaOps:
    """The three compute steps of the split, on the CUDA library."""
    chunk_carry = staticmethod(chunk_carry)
    entering_state = staticmethod(entering_state)

    @staticmethod
    def scan(x, delta, A, B, C, D, z, delta_bias, softplus, h0):
        return ssm_scan_fwd(x, delta, A, B, C, D=D, z=z, delta_bias=delta_bias,
                            softplus=softplus, h0=h0)


def seq_parallel_scan(x, delta, A, B, C, D=None, z=None, delta_bias=None, softplus=True,
                      h0=None, group=None, ops=CudaOps):
    """This rank's part of one sequence scanned across the ranks of `group`:
    rank r holds chunk r of x, delta, B, C, z (contiguous, in rank order; the
    chunk lengths may differ; A, D, delta_bias and the sequence's h0 are the
    same on every rank). Returns (y of this chunk, the state after this chunk);
    on the last rank the latter is the sequence's h_last. One all-gather (NCCL
    on GPUs) carries the chunk carries between ranks; every rank does two passes
    over its chunk. `ops` supplies the compute steps (the CUDA library; the
    multi-process tests on CPU substitute the reference implementation)."""
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    e, dsum = ops.chunk_carry(x, delta, A, B, C, D=D, z=z, delta_bias=delta_bias,
                              softplus=softplus)
    hend = [torch.empty_like(e) for _ in range(world)]
    dsums = [torch.empty_like(dsum) for _ in range(world)]
    dist.all_gather(hend, e.contiguous(), group=group)
    dist.all_gather(dsums, dsum.contiguous(), group=group)
    h_in = ops.entering_state(rank, A, torch.stack(hend), torch.stack(dsums), h0=h0)
    return ops.scan(x, delta, A, B, C, D, z, delta_bias, softplus, h_in)
