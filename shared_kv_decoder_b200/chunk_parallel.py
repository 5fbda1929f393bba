"""Chunk-parallel prefill of the YOCO attention core across ranks.

"You Only Cache Once" (paperlayer summary, Appendix A "Chunk Parallelism for
Long-Sequence Training of YOCO"; podcast transcript, the Figure 3
discussion): a long sequence is split into contiguous chunks, one per
device.  The self-decoder depends only on nearby positions, so a device
exchanges with its neighbour only: for sliding-window attention, the window
- 1 keys and values before its chunk (a halo).  The cross-decoder reads the
global K/V of every earlier position; it is gathered once and reused by
every cross layer.

One rank per GPU.  Every function works on the calling rank's chunk and takes
two collaborators:
  * ``comm`` -- the two exchanges (``DistComm``: torch.distributed point-to-
    point sends for the halo, one all-gather for the global K/V);
  * ``ops`` -- the attention call (default: this package's kernels through
    ``attention_prefill``).
Argument marshalling and data movement only; the attention runs in the
library's kernels.
"""
import torch
import torch.distributed as dist


class DistComm:
    """Halo exchange and all-gather over a torch.distributed process group
    (NCCL for CUDA tensors, gloo for CPU tensors)."""

    def __init__(self, group=None):
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def halo(self, k_tail, v_tail):
        """Send this rank's last rows (k_tail, v_tail [B, h, Hkv, D]) to the
        next rank and receive the previous rank's; rank 0 receives nothing
        and gets (None, None)."""
        ops, recv = [], None
        if self.rank > 0:
            recv = (torch.empty_like(k_tail), torch.empty_like(v_tail))
            src = dist.get_global_rank(self.group, self.rank - 1) if self.group else self.rank - 1
            ops += [dist.P2POp(dist.irecv, recv[0], src, self.group), dist.P2POp(dist.irecv, recv[1], src, self.group)]
        if self.rank + 1 < self.world:
            dst = dist.get_global_rank(self.group, self.rank + 1) if self.group else self.rank + 1
            ops += [dist.P2POp(dist.isend, k_tail.contiguous(), dst, self.group),
                    dist.P2POp(dist.isend, v_tail.contiguous(), dst, self.group)]
        if ops:
            for r in dist.batch_isend_irecv(ops):
                r.wait()
        return recv if recv is not None else (None, None)

    def all_gather_rows(self, x):
        """x [B, Tc, ...] of equal chunk length on every rank -> [B, world*Tc, ...]
        in rank order."""
        parts = [torch.empty_like(x) for _ in range(self.world)]
        dist.all_gather(parts, x.contiguous(), group=self.group)
        return torch.cat(parts, dim=1)


class KernelOps:
    """This package's kernels."""

    @staticmethod
    def attention_prefill(q, k, v, q_pos0, window):
        from . import attention_prefill
        return attention_prefill(q.contiguous(), k.contiguous(), v.contiguous(), q_pos0=q_pos0, window=window)


def swa_chunk(q, k, v, window, comm, ops=KernelOps):
    """Sliding-window attention of this rank's chunk.  q [B, Tc, Hq, D]; k, v
    [B, Tc, Hkv, D] (this chunk's rows).  The previous window - 1 keys and
    values come from the rank before; the window may not reach past it
    (window - 1 <= Tc)."""
    Tc = q.shape[1]
    h = window - 1
    if h > Tc:
        raise ValueError(f"window {window} reaches past the previous chunk ({Tc} rows)")
    if h <= 0:
        return ops.attention_prefill(q, k, v, 0, window)
    kp, vp = comm.halo(k[:, Tc - h:], v[:, Tc - h:])
    if kp is None:
        return ops.attention_prefill(q, k, v, 0, window)
    return ops.attention_prefill(q, torch.cat([kp, k], dim=1), torch.cat([vp, v], dim=1), h, window)


def gather_global_kv(k_chunk, v_chunk, comm):
    """The global K/V of every rank's chunk, in sequence order: one gather,
    reused by every cross layer."""
    return comm.all_gather_rows(k_chunk), comm.all_gather_rows(v_chunk)


def cross_chunk(q, k_g, v_g, chunk_start, ops=KernelOps):
    """Causal attention of this rank's query rows (absolute positions
    chunk_start ...) over the gathered global K/V up to the chunk's end."""
    end = chunk_start + q.shape[1]
    return ops.attention_prefill(q, k_g[:, :end], v_g[:, :end], chunk_start, 0)
