"""Training step of an HSTU layer stack, data-parallel over ranks.

A rank holds the whole stack (the same weights on every rank) and its own
sequences (one shard of the global batch, as `hstu_lpt_partition` deals them
out).  The step is the forward through every layer with its activations saved,
then the backward from the last layer to the first; the loss is a sum over
tokens, so the gradient of each parameter is the SUM of the ranks' gradients
("Actions Speak Louder than Words" summary, 2.2: the stack, relative-bias tables
included, is trained end to end).  Each layer's parameter gradients go into
their all-reduce as soon as that layer's backward has produced them, so the
transfer of layer l overlaps the backward of layers l-1 ... 0; `step` returns
once every reduction has completed.

The layers are `binding.Layer` objects (their forward and backward run in the
library's CUDA kernels); any object with the same `forward` / `backward`
signature works, which is how the multi-rank logic is tested on CPU ranks.
Layers built with one shared `workspaces` dict reuse the attention preparation
(work lists, timestamp tile records) of the step's first forward and first
backward: every layer sees the same batch.
"""
from __future__ import annotations

from typing import List, Optional, Sequence

from .data_parallel import GradAllReduce


class StackTrainer:
    """Runs one training step of `layers` and reduces the parameter gradients
    over the ranks of `reducer`'s group (no reduction with one rank)."""

    def __init__(self, layers: Sequence, reducer: Optional[GradAllReduce] = None, share_prep: bool = False):
        """share_prep: the layers share their workspaces (binding.Layer(...,
        workspaces=one dict)), so every layer after the first reuses the step's
        attention preparation."""
        self.layers = list(layers)
        self.reducer = reducer if reducer is not None else GradAllReduce()
        self.share_prep = share_prep

    def step(self, x, seq_offsets, timestamps, dy, saved: Sequence, acts: Sequence, num_targets=None):
        """Forward from `x` (activations into `acts`, what the backward needs into
        `saved`), backward from the upstream gradient `dy` of the last layer's
        output.  Returns (dx, per-layer gradient dicts); the parameter gradients
        in them are already summed over the ranks."""
        L = len(self.layers)
        h = x
        for li, (ly, sv, a) in enumerate(zip(self.layers, saved, acts)):
            kw = {"reuse_prep": True} if self.share_prep and li > 0 else {}
            h = ly.forward(h, seq_offsets, timestamps, num_targets=num_targets, saved=sv, out=a, **kw)
        ins = [x] + list(acts[:-1])
        grads: List[dict] = [None] * L
        g = dy
        for li in range(L - 1, -1, -1):
            # the parameters' gradients only (no dU|dV|dQ|dK buffer for the caller)
            kw = {"reuse_prep": True} if self.share_prep and li < L - 1 else {}
            g, grads[li] = self.layers[li].backward(ins[li], g, saved[li], seq_offsets, timestamps,
                                                    num_targets=num_targets, keep_duvqk=False, **kw)
            self.reducer.layer_done(grads[li])
        self.reducer.wait()
        return g, grads
