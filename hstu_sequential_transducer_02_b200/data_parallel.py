"""Data-parallel training of the HSTU layer stack across ranks.

Sequences are sharded across ranks (one process per GPU, as `bench.py` runs
them) and every rank holds the same weights.  The training loss is a sum over
tokens, so after the backward pass each parameter's gradient is the SUM of the
ranks' gradients: the only exchange of a training step is that all-reduce
("Actions Speak Louder than Words" summary, 2.2: the stack is trained end to
end; the relative-bias tables receive gradients too).

The reduction is issued per layer, as soon as that layer's backward has
produced its gradients: the backward runs from the last layer to the first, so
the transfer of layer l overlaps the backward of layers l-1 ... 0.  Each layer's
ten parameter gradients travel as one flat fp32 bucket (one collective per
layer instead of ten).  On GPUs the process group is NCCL (NVLink / NVSwitch);
the same code runs on CPU tensors with gloo.
"""
from typing import Dict, List, Optional

import torch
import torch.distributed as dist

# gradients of the layer's parameters, as returned by binding.Layer.backward
# (the activation gradient "uvqk" is per token and is not reduced)
PARAM_GRADS = ("w1", "b1", "ln1_gamma", "ln1_beta", "ln2_gamma", "ln2_beta", "w2", "b2", "pos_bias", "time_bias")


class GradAllReduce:
    """Sums the parameter gradients of every layer over the ranks of `group`.

    Call `layer_done(grads)` once per layer right after its backward (any order),
    then `wait()` before the optimizer reads the gradients: it completes the
    outstanding reductions and writes the sums back into the given tensors.
    With one rank both calls do nothing."""

    def __init__(self, group: Optional[dist.ProcessGroup] = None):
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1
        self._pending: List[tuple] = []

    def layer_done(self, grads: Dict[str, torch.Tensor]) -> None:
        if self.world == 1:
            return
        tensors = [grads[n] for n in PARAM_GRADS]
        for t in tensors:
            if t.dtype != torch.float32:
                raise TypeError("parameter gradients are fp32")
        flat = torch.cat([t.reshape(-1) for t in tensors])
        work = dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=self.group, async_op=True)
        self._pending.append((work, flat, tensors))

    def wait(self) -> None:
        for work, flat, tensors in self._pending:
            work.wait()
            off = 0
            for t in tensors:
                n = t.numel()
                t.copy_(flat[off:off + n].view_as(t))
                off += n
        self._pending.clear()
