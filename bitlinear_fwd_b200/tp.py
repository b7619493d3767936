"""Tensor-parallel K-split (row-parallel) BitLinear over torch.distributed.

Rank r holds the columns K_r of x and of the weight matrix W.  BitLinear
(Falcon-Edge blog, section "Falcon-Edge, a series of universal models")
reduces over whole tensors -- each token's absmax over all of K for s_x,
mean |w| over the whole matrix for s_w -- so the split needs three exact
exchanges, all in integers or max:

  pack_ksplit      all-reduce SUM of the uint64 exponent bins of sum |w| and
                   of the element count; every rank then packs its columns
                   with the same s_w as the unsplit matrix;
  forward_ksplit   all-reduce MAX of the tokens' partial absmax, the int32
                   partial contraction of this rank's columns, all-reduce SUM
                   of those partial sums, and the epilogue on the total.

Every rank ends with the bits of the unsplit forward.  On GPUs the process
group is NCCL; the tensors stay on the device.  ``ops`` supplies the local
steps; by default they are the library's kernels (argument marshalling
only), and a test can substitute a host implementation to check the
exchange logic on CPU ranks.
"""

from __future__ import annotations

from typing import Optional

import torch
import torch.distributed as dist


class LibraryOps:
    """The local steps of a K-split as the library's C entry points."""

    def absmean_bins(self, w):
        from . import bitlinear_absmean_bins
        return bitlinear_absmean_bins(w)

    def pack_from_bins(self, w, bins, n_total):
        from . import bitlinear_pack_weights_from_bins
        return bitlinear_pack_weights_from_bins(w, bins, n_total)

    def act_absmax(self, x):
        from . import bitlinear_act_absmax
        return bitlinear_act_absmax(x)

    def forward_partial(self, x, absmax, packed, flags):
        from . import bitlinear_forward_partial
        return bitlinear_forward_partial(x, absmax, packed, flags=flags)

    def epilogue(self, acc, absmax, w_scale, bias, flags):
        from . import bitlinear_epilogue_sum
        return bitlinear_epilogue_sum(acc, absmax, w_scale, bias, flags=flags)


def pack_ksplit(w_shard: torch.Tensor, group=None, ops=None):
    """Packs this rank's columns W[:, K_r] with the whole matrix's s_w.
    Returns (packed, w_scale, w_mean) of this shard."""
    ops = ops or LibraryOps()
    bins = ops.absmean_bins(w_shard)
    dist.all_reduce(bins, op=dist.ReduceOp.SUM, group=group)       # exact integer bins
    count = torch.tensor([w_shard.numel()], dtype=torch.int64, device=bins.device)
    dist.all_reduce(count, op=dist.ReduceOp.SUM, group=group)
    return ops.pack_from_bins(w_shard, bins, int(count.item()))


def forward_ksplit(x_shard: torch.Tensor, packed_shard: torch.Tensor, w_scale: torch.Tensor,
                   bias: Optional[torch.Tensor] = None, group=None, ops=None, flags: int = 0) -> torch.Tensor:
    """y = BitLinear(x) from this rank's K-columns of x and of the packed
    weights; every rank returns the whole y."""
    ops = ops or LibraryOps()
    absmax = ops.act_absmax(x_shard)
    dist.all_reduce(absmax, op=dist.ReduceOp.MAX, group=group)     # the whole row's absmax
    acc = ops.forward_partial(x_shard, absmax, packed_shard, flags)
    dist.all_reduce(acc, op=dist.ReduceOp.SUM, group=group)        # exact int32 sum over the shards
    return ops.epilogue(acc, absmax, w_scale, bias, flags)
