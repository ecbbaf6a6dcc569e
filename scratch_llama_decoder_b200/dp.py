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

Dropout masks are indexed over the whole batch: the wrapper sets the engine's
sequence offset to rank * (its batch), so the ranks together draw the masks
one context over the whole batch would draw, and no two ranks share masks.

The engine is a LlamaStep (or any object with its grad / adamw / flag_out /
flag_in methods, a device and, for CUDA, a stream); collectives are issued on
the engine's stream so that they follow its kernels in order.

With overlap=True the gradient is exchanged in buckets while the backward
still runs: the engine records an event per bucket as its backward finishes
it (layers from the last to the first), a communication stream waits for each
bucket's event and all-reduces that bucket, and the engine's stream waits for
the communication stream before the update.  The sums are the same numbers as
one all-reduce of the whole buffer (the reduction of each element is the same
over the same ranks).
"""
import contextlib

import torch
import torch.distributed as dist


class DataParallelStep:
    def __init__(self, engine, group=None, overlap=False):
        self.engine = engine
        self.group = group
        self.world = (dist.get_world_size(group)
                      if dist.is_available() and dist.is_initialized() else 1)
        self.flag = torch.zeros(1, dtype=torch.int32, device=engine.device)
        set_offset = getattr(engine, "set_dropout_offset", None)
        if set_offset is not None and self.world > 1:
            set_offset(dist.get_rank(group) * int(engine.cfg["batch"]))
        self.overlap = bool(overlap) and self.world > 1
        self._comm = None
        if self.overlap:
            engine.set_grad_buckets(True)
            self.buckets = engine.grad_buckets()
            if engine.device.type == "cuda":
                self._comm = torch.cuda.Stream(device=engine.device)

    def _exchange_buckets(self, grads):
        """One all-reduce per bucket, each after the backward has finished it."""
        e = self.engine
        for k, (off, cnt) in enumerate(self.buckets):
            if self._comm is not None:
                e.grad_bucket_wait(k, self._comm)
                with torch.cuda.stream(self._comm):
                    dist.all_reduce(grads[off:off + cnt], op=dist.ReduceOp.SUM, group=self.group)
            else:
                e.grad_bucket_wait(k, None)
                dist.all_reduce(grads[off:off + cnt], op=dist.ReduceOp.SUM, group=self.group)
        if self._comm is not None:
            e.stream.wait_stream(self._comm)

    def _stream(self):
        e = self.engine
        if getattr(e, "device", torch.device("cpu")).type == "cuda":
            return torch.cuda.stream(e.stream)
        return contextlib.nullcontext()

    def _launches(self):
        n = getattr(self.engine, "last_launch_count", None)
        return n() if n else 0

    def step(self, params, grads, m, v, t, tokens, targets, lr, wd, loss):
        e = self.engine
        with self._stream():
            e.grad(params, grads, tokens, targets, loss)
            launches = self._launches()
            if self.world > 1:
                if self.overlap:
                    self._exchange_buckets(grads)
                else:
                    dist.all_reduce(grads, op=dist.ReduceOp.SUM, group=self.group)
                e.flag_out(self.flag)
                dist.all_reduce(self.flag, op=dist.ReduceOp.MAX, group=self.group)
                e.flag_in(self.flag)
                dist.all_reduce(loss, op=dist.ReduceOp.SUM, group=self.group)
            e.adamw(params, grads, m, v, t, lr, wd, grad_scale=1.0 / self.world)
            # the library's kernels of this step (llm_grad and llm_adamw)
            self.last_launches = launches + self._launches()
        return loss


class ShardedDataParallelStep(DataParallelStep):
    """The data-parallel step with the optimiser state sharded across ranks
    (the parameters' Adam moments live only on the rank that updates them):
      1. llm_grad on the rank's share of the batch, into a flat gradient
         buffer padded to ranks x chunk elements (chunk a multiple of 4;
         llm_grad writes the first n_params, the pad stays zero);
      2. reduce-scatter (sum): each rank receives the summed gradient of its
         chunk of the parameters;
      3. the error words are combined (max) as in DataParallelStep;
      4. llm_adamw_range on the rank's chunk with grad_scale = 1 / ranks;
      5. all-gather of the updated chunks into every rank's parameters.
    Per rank that moves a reduce-scatter plus an all-gather of the gradient's
    size (together one all-reduce's traffic) and keeps 1 / ranks of m and v.
    With clipping on (the engine's grad_clip > 0), step 4 becomes: each rank
    scales its chunk by 1 / ranks and reduces it to its part of the norm
    (llm_grad_norm_part: sum of squares in float64, or the largest |g|), one
    all-reduce of that float64 (SUM, or MAX for the L-infinity norm) gives
    every rank the whole gradient's part, and llm_adamw_range_clip clips the
    chunk by the resulting norm and updates it -- the same scale on every
    rank, the one llm_adamw applies to the whole summed gradient.
    buffers() allocates the padded parameter and gradient buffers and the
    chunk-sized m and v.

    With overlap=True the exchange runs per gradient bucket while the
    backward goes on: rank r owns piece r of every bucket (q = the bucket's
    count / ranks rounded up to a multiple of 4; bucket offsets are multiples
    of 4, so every piece is 16-byte aligned), each bucket is reduce-scattered
    on a communication stream as soon as the backward has finished it, and
    after the update each bucket's pieces are all-gathered.  A bucket's last
    piece may reach up to 4 x ranks elements past the bucket: into the bucket
    finished just before it (buckets complete from the end of the buffer
    backwards, so those gradients are final when read, and the all-gathers,
    in the same order, write back values that are already final and the same
    on every rank) or, for the head, into the buffers' padding.  pieces lists
    (bucket offset, q, elements kept, moment offset) of this rank."""

    def __init__(self, engine, n_params, group=None, overlap=False):
        super().__init__(engine, group, overlap)
        self.rank = dist.get_rank(group) if self.world > 1 else 0
        self.n = int(n_params)
        self._gshard = None
        if self.overlap:
            self.pieces, mo = [], 0
            for off, cnt in self.buckets:
                assert off % 4 == 0
                q = ((cnt + self.world - 1) // self.world + 3) // 4 * 4
                self.pieces.append((off, q, max(0, min(q, cnt - self.rank * q)), mo))
                mo += q
            self.chunk = mo  # this rank's moments: one piece per bucket
            end = max(off + self.world * q for off, q, _, _ in self.pieces)
            self.padded = (max(self.n, end) + 3) // 4 * 4
            self.lo, self.count = None, sum(k for _, _, k, _ in self.pieces)
        else:
            self.chunk = ((self.n + self.world - 1) // self.world + 3) // 4 * 4
            self.padded = self.world * self.chunk
            self.lo = self.rank * self.chunk
            self.count = max(0, min(self.chunk, self.n - self.lo))

    def _clipping(self):
        return getattr(self.engine, "grad_clip", 0.0) > 0.0

    def _norm_part(self):
        """One float64 on the engine's device: this rank's part of the norm."""
        if getattr(self, "_part", None) is None:
            self._part = torch.zeros(1, dtype=torch.float64, device=self.engine.device)
        return self._part

    def _combine(self, part):
        """Every rank's part of the norm, combined: the sum of the ranks' sums
        of squares, or the largest of their largest |g|."""
        if self.world > 1:
            linf = getattr(self.engine, "grad_clip_mode", 0) == 1
            dist.all_reduce(part, op=dist.ReduceOp.MAX if linf else dist.ReduceOp.SUM,
                            group=self.group)

    def buffers(self, dtype=torch.float32):
        dev = self.engine.device
        padded = self.padded
        return (torch.zeros(padded, dtype=dtype, device=dev),
                torch.zeros(padded, dtype=dtype, device=dev),
                torch.zeros(self.chunk, dtype=dtype, device=dev),
                torch.zeros(self.chunk, dtype=dtype, device=dev))

    def _step_buckets(self, params, grads, m, v, t, tokens, targets, lr, wd, loss):
        e, W = self.engine, self.world
        if self._gshard is None:
            self._gshard = torch.zeros(self.chunk, dtype=grads.dtype, device=grads.device)
        gs = self._gshard
        e.grad(params, grads, tokens, targets, loss)
        launches = self._launches()
        for k, (off, q, _, mo) in enumerate(self.pieces):
            if self._comm is not None:
                e.grad_bucket_wait(k, self._comm)
                with torch.cuda.stream(self._comm):
                    dist.reduce_scatter_tensor(gs[mo:mo + q], grads[off:off + W * q],
                                               op=dist.ReduceOp.SUM, group=self.group)
            else:
                e.grad_bucket_wait(k, None)
                dist.reduce_scatter_tensor(gs[mo:mo + q], grads[off:off + W * q],
                                           op=dist.ReduceOp.SUM, group=self.group)
        if self._comm is not None:
            e.stream.wait_stream(self._comm)
        e.flag_out(self.flag)
        dist.all_reduce(self.flag, op=dist.ReduceOp.MAX, group=self.group)
        e.flag_in(self.flag)
        dist.all_reduce(loss, op=dist.ReduceOp.SUM, group=self.group)
        if self._clipping():
            part = self._norm_part()
            part.zero_()
            for off, q, keep, mo in self.pieces:
                if keep:
                    e.grad_norm_part(gs[mo:mo + keep], 1.0 / W, part, accumulate=True)
                    launches += self._launches()
            self._combine(part)
        for off, q, keep, mo in self.pieces:
            if keep:
                a = off + self.rank * q
                if self._clipping():
                    e.adamw_range_clip(params[a:a + keep], gs[mo:mo + keep], m[mo:mo + keep],
                                       v[mo:mo + keep], t, lr, wd, part)
                else:
                    e.adamw_range(params[a:a + keep], gs[mo:mo + keep], m[mo:mo + keep],
                                  v[mo:mo + keep], t, lr, wd, grad_scale=1.0 / W)
                launches += self._launches()
        self.last_launches = launches
        nccl = dist.get_backend(self.group) == "nccl"
        for off, q, _, _ in self.pieces:
            a = off + self.rank * q
            src = params[a:a + q] if nccl else params[a:a + q].clone()
            dist.all_gather_into_tensor(params[off:off + W * q], src, group=self.group)

    def step(self, params, grads, m, v, t, tokens, targets, lr, wd, loss):
        e = self.engine
        if self.overlap:
            with self._stream():
                self._step_buckets(params, grads, m, v, t, tokens, targets, lr, wd, loss)
            return loss
        C, lo, cnt = self.chunk, self.lo, self.count
        with self._stream():
            e.grad(params, grads, tokens, targets, loss)
            launches = self._launches()
            if self.world > 1:
                if self._gshard is None:
                    self._gshard = torch.zeros(C, dtype=grads.dtype, device=grads.device)
                dist.reduce_scatter_tensor(self._gshard, grads, op=dist.ReduceOp.SUM,
                                           group=self.group)
                e.flag_out(self.flag)
                dist.all_reduce(self.flag, op=dist.ReduceOp.MAX, group=self.group)
                e.flag_in(self.flag)
                dist.all_reduce(loss, op=dist.ReduceOp.SUM, group=self.group)
                gs = self._gshard
            else:
                gs = grads
            if self._clipping():
                part = self._norm_part()
                e.grad_norm_part(gs[:cnt], 1.0 / self.world, part)
                launches += self._launches()
                self._combine(part)
                e.adamw_range_clip(params[lo:lo + cnt], gs[:cnt], m[:cnt], v[:cnt], t, lr, wd,
                                   part)
            else:
                e.adamw_range(params[lo:lo + cnt], gs[:cnt], m[:cnt], v[:cnt], t, lr, wd,
                              grad_scale=1.0 / self.world)
            self.last_launches = launches + self._launches()
            if self.world > 1:
                src = params[lo:lo + C]
                if dist.get_backend(self.group) != "nccl":
                    src = src.clone()  # in place only where the backend documents it
                dist.all_gather_into_tensor(params, src, group=self.group)
        return loss
