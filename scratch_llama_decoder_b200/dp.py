"""Data-parallel training step: one process per GPU, the batch split across
ranks, one all-reduce of the gradients between the library's backward and its
update.

Every rank holds a context over its share of the batch (the same number of
sequences on every rank) and the same parameters.  A step is:
  1. llm_grad on the rank's share: the gradient of the rank's mean loss;
  2. all-reduce (sum) of the flat float32 gradient buffer -- NCCL over
     NVLink/NVSwitch between B200s, the step's only exchange;
  3. all-reduce (max) of the ranks' int32 error words (a bad token or a
     non-finite loss on any rank makes every rank skip the update);
  4. llm_adamw with grad_scale = 1 / ranks: the summed gradient becomes the
     gradient of the mean loss over the whole batch, then clipping (if on)
     and AdamW, so every rank applies the same update to the same parameters.
The ranks' losses are summed too: the returned tensor holds the sum of the
ranks' mean losses (divided by the rank count it is the batch mean).

The engine is a LlamaStep (or any object with its grad / adamw / flag_out /
flag_in methods, a device and, for CUDA, a stream); collectives are issued on
the engine's stream so that they follow its kernels in order.
"""
import contextlib

import torch
import torch.distributed as dist


class DataParallelStep:
    def __init__(self, engine, group=None):
        self.engine = engine
        self.group = group
        self.world = (dist.get_world_size(group)
                      if dist.is_available() and dist.is_initialized() else 1)
        self.flag = torch.zeros(1, dtype=torch.int32, device=engine.device)

    def _stream(self):
        e = self.engine
        if getattr(e, "device", torch.device("cpu")).type == "cuda":
            return torch.cuda.stream(e.stream)
        return contextlib.nullcontext()

    def step(self, params, grads, m, v, t, tokens, targets, lr, wd, loss):
        e = self.engine
        with self._stream():
            e.grad(params, grads, tokens, targets, loss)
            if self.world > 1:
                dist.all_reduce(grads, op=dist.ReduceOp.SUM, group=self.group)
                e.flag_out(self.flag)
                dist.all_reduce(self.flag, op=dist.ReduceOp.MAX, group=self.group)
                e.flag_in(self.flag)
                dist.all_reduce(loss, op=dist.ReduceOp.SUM, group=self.group)
            e.adamw(params, grads, m, v, t, lr, wd, grad_scale=1.0 / self.world)
        return loss
