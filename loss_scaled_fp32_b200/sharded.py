"""The loss-scaled step with the optimizer state split across the ranks of a
data-parallel process group (one GPU per rank; torch.distributed over NCCL
carries the collectives, NVLink/NVSwitch on a B200 node).

Each rank owns one contiguous shard of the flat parameter list (all tensors
concatenated): its FP32 master, FP32 momentum and FP16 copy.  One step:

  1. reduce-scatter of the ranks' FP16 gradients (sum) -> this rank's shard;
  2. the check pass over the shard (library) -> a 32-byte record;
  3. all-gather of the records (32 bytes per rank), in rank order;
  4. combine-and-finish + update of the shard (library): every rank adds the
     records in rank order, so all ranks see the same norm and the same next
     loss scale, bit for bit;
  5. all-gather of the FP16 copies -> the full FP16 weights on every rank.

The library does all arithmetic; this module only moves buffers between the
library and the collectives.
"""
import torch
import torch.distributed as dist

from . import MPT, MPT_PARTIAL_BYTES, shard_len


def exchange_records(out, mine, group=None):
    """All-gather every rank's 32-byte record into ``out`` (world * 32 bytes,
    rank order)."""
    dist.all_gather_into_tensor(out, mine, group=group)
    return out


class ShardedMPT:
    """Optimizer over a flat list of ``total`` parameters split across the
    ranks of ``group``; the loss scale lives on the device (queued steps)."""

    def __init__(self, total, config=None, group=None, device=None):
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.total = int(total)
        self.shard = shard_len(self.total, self.world)
        self.padded = self.shard * self.world
        self.opt = MPT([self.shard], config, device=device)
        dev = self.opt.device
        self.grad_shard = torch.zeros(self.shard, dtype=torch.float16, device=dev)
        self.records = torch.empty(self.world * MPT_PARTIAL_BYTES, dtype=torch.uint8, device=dev)
        self.w16_full = torch.empty(self.padded, dtype=torch.float16, device=dev)

    @property
    def begin(self):
        return self.rank * self.shard

    def load_master(self, flat_master):
        """Copy this rank's slice of the full flat FP32 master (``total``
        elements) into its shard; padding stays zero; refresh the FP16 copy."""
        m = self.opt.master(0)
        m.zero_()
        lo, hi = self.begin, min(self.begin + self.shard, self.total)
        if hi > lo:
            m[: hi - lo].copy_(flat_master[lo:hi])
        self.opt.refresh_half()
        dist.all_gather_into_tensor(self.w16_full, self.opt.w16(0), group=self.group)

    def set_scale(self, scale, clean_run=0):
        self.opt.set_scaler_state(scale, clean_run)

    def device_scale(self):
        return self.opt.device_scale()

    def step(self, flat_grads, lr, momentum, weight_decay, clip=0.0, marks=None):
        """``flat_grads``: this rank's FP16 gradients of the whole list, padded
        to ``padded`` elements (zeros past ``total``).  Returns the full FP16
        weights (a view of ``total`` elements).  ``marks``: optional list of
        six CUDA timing events, recorded on the current stream before the
        reduce-scatter and after each of the five phases (reduce-scatter,
        check pass, record all-gather, finish and update, FP16 all-gather)."""
        if flat_grads.numel() != self.padded or flat_grads.element_size() != 2:
            raise ValueError(f"expected {self.padded} FP16 gradients")
        mark = (lambda i: marks[i].record()) if marks is not None else (lambda i: None)
        mark(0)
        dist.reduce_scatter_tensor(self.grad_shard, flat_grads, op=dist.ReduceOp.SUM,
                                   group=self.group)
        mark(1)
        mine = self.opt.step_partial([self.grad_shard])
        mark(2)
        exchange_records(self.records, mine, self.group)
        mark(3)
        self.opt.step_finish(self.records, self.world, lr, momentum, weight_decay, clip)
        mark(4)
        dist.all_gather_into_tensor(self.w16_full, self.opt.w16(0), group=self.group)
        mark(5)
        return self.w16_full[: self.total]

    def wait(self):
        return self.opt.wait()

    def close(self):
        self.opt.close()
