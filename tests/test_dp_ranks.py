"""The data-parallel step's host logic on CPU: two gloo ranks (spawned
processes, rendezvous on 127.0.0.1), each with half of the batch, driven
through DataParallelStep with an engine that computes on the float64 oracle.
Two ranks must give the single-process step on the whole batch (the mean of
the ranks' mean gradients is the batch-mean gradient when the shares are
equal), and an error on one rank must make both skip the update."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


class OracleEngine:
    """grad / adamw / flag_out / flag_in of the C ABI, computed by the oracle
    on float64 CPU tensors."""
    device = torch.device("cpu")

    def __init__(self, cfg, fail_at=None, clip=0.0, clip_mode=0):
        self.cfg = cfg
        self.flag = 0
        self.fail_at = fail_at
        self.calls = 0
        self.grad_clip, self.grad_clip_mode = float(clip), int(clip_mode)
        self.norms = []  # the norm before clipping of every clipped update

    def _kind(self):
        return "linf" if self.grad_clip_mode == 1 else "l2"

    def _clip_whole(self, grads):
        from oracle import train_terms as TT
        if self.grad_clip > 0.0:
            g, n, _ = TT.clip(grads.numpy(), self.grad_clip, self._kind())
            grads.copy_(torch.from_numpy(g))
            self.norms.append(n)

    # the sharded form's clipping: a part of the norm per range, combined by
    # the caller across ranks, then the clipping rule on the combined value
    def grad_norm_part(self, grads, grad_scale, part, accumulate=False):
        grads.mul_(grad_scale)
        g = grads.numpy()
        if self.grad_clip_mode == 1:
            v = float(np.max(np.abs(g))) if g.size else 0.0
            part.fill_(max(float(part.item()), v) if accumulate else v)
        else:
            v = float(np.sum(g * g))
            part.fill_(float(part.item()) + v if accumulate else v)

    def adamw_range_clip(self, params, grads, m, v, t, lr, wd, total):
        from oracle import train_terms as TT
        if self.grad_clip > 0.0:
            tv = float(total.item())
            n = tv if self.grad_clip_mode == 1 else float(np.sqrt(tv))
            grads.mul_(TT.clip_scale(n, self.grad_clip))
            if getattr(self, "_norm_t", None) != t:  # one norm per step, however many ranges
                self.norms.append(n)
                self._norm_t = t
            else:
                assert n == self.norms[-1]  # every range of a step sees the same norm
        self.adamw_range(params, grads, m, v, t, lr, wd)

    def grad(self, params, grads, tokens, targets, loss):
        import oracle as O
        self.calls += 1
        n = O.n_params(self.cfg)  # buffers may be padded past the parameters
        lv, _, g = O.forward_backward(self.cfg, params.numpy()[:n], tokens.numpy(),
                                      targets.numpy(), want_logits=False)
        grads[:n].copy_(torch.from_numpy(g))
        loss.fill_(lv)
        self.flag = 1 if self.calls == self.fail_at else 0

    def flag_out(self, f):
        f.fill_(self.flag)

    # gradient buckets: the library's ranges (host only); the oracle's
    # gradient is complete when grad returns, so waiting is a no-op
    def set_grad_buckets(self, enable):
        self.buckets_on = bool(enable)

    def grad_buckets(self):
        import scratch_llama_decoder_b200 as P
        return P.grad_buckets(self.cfg)

    def grad_bucket_wait(self, k, stream):
        assert self.buckets_on and stream is None

    def flag_in(self, f):
        self.flag |= int(f.item())

    def adamw_range(self, params, grads, m, v, t, lr, wd, grad_scale=1.0):
        import oracle as O
        grads.mul_(grad_scale)
        if self.flag or params.numel() == 0:
            return
        p2, m2, v2 = O.adamw(params.numpy(), grads.numpy(), m.numpy(), v.numpy(), t, lr, wd)
        params.copy_(torch.from_numpy(p2))
        m.copy_(torch.from_numpy(m2))
        v.copy_(torch.from_numpy(v2))

    def adamw(self, params, grads, m, v, t, lr, wd, grad_scale=1.0):
        import oracle as O
        grads.mul_(grad_scale)
        self._clip_whole(grads)
        if self.flag:
            return
        p2, m2, v2 = O.adamw(params.numpy(), grads.numpy(), m.numpy(), v.numpy(), t, lr, wd)
        params.copy_(torch.from_numpy(p2))
        m.copy_(torch.from_numpy(m2))
        v.copy_(torch.from_numpy(v2))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _setup(full_cfg):
    import oracle as O
    from synth import make_batch, make_params
    p = make_params(full_cfg, O.param_layout(full_cfg)).astype(np.float64)
    tok, tgt = make_batch(full_cfg)
    return p, tok.reshape(full_cfg["batch"], -1), tgt.reshape(full_cfg["batch"], -1)


def _run(engine, dp, p, tok, tgt, steps, lr, wd):
    P = torch.tensor(p)
    G, M, V = (torch.zeros_like(P) for _ in range(3))
    loss = torch.zeros(1, dtype=torch.float64)
    losses = []
    for t in range(1, steps + 1):
        dp.step(P, G, M, V, t, torch.tensor(tok), torch.tensor(tgt), lr, wd, loss)
        losses.append(float(loss.item()))
    return P.numpy(), M.numpy(), V.numpy(), losses


def _rank_main_sharded(rank, world, port, full_cfg, steps, q, overlap=False, clip=0.0,
                       clip_mode=0):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle as O
    from scratch_llama_decoder_b200.dp import ShardedDataParallelStep
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        p, tok, tgt = _setup(full_cfg)
        share = full_cfg["batch"] // world
        cfg = dict(full_cfg, batch=share)
        eng = OracleEngine(cfg, clip=clip, clip_mode=clip_mode)
        dp = ShardedDataParallelStep(eng, O.n_params(cfg), overlap=overlap)
        assert dp.overlap == overlap
        P, G, M, V = dp.buffers(torch.float64)
        P[:p.size].copy_(torch.from_numpy(p))
        loss = torch.zeros(1, dtype=torch.float64)
        for t in range(1, steps + 1):
            dp.step(P, G, M, V, t, torch.tensor(tok[rank * share:(rank + 1) * share]),
                    torch.tensor(tgt[rank * share:(rank + 1) * share]), full_cfg["lr"],
                    full_cfg["wd"], loss)
        if overlap:  # the rank's pieces of every bucket, placed in the full layout
            Mf, Vf = np.full(p.size, np.nan), np.full(p.size, np.nan)
            for off, qq, keep, mo in dp.pieces:
                a = off + rank * qq
                Mf[a:a + keep] = M[mo:mo + keep].numpy()
                Vf[a:a + keep] = V[mo:mo + keep].numpy()
            q.put((rank, (P[:p.size].numpy().copy(), Mf, Vf, None, None, eng.norms)))
        else:
            q.put((rank, (P[:p.size].numpy().copy(), M[:dp.count].numpy().copy(),
                          V[:dp.count].numpy().copy(), dp.lo, dp.count, eng.norms)))
    finally:
        dist.destroy_process_group()


def _rank_main(rank, world, port, full_cfg, steps, fail_rank, fail_at, q, overlap=False):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from scratch_llama_decoder_b200.dp import DataParallelStep
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        p, tok, tgt = _setup(full_cfg)
        share = full_cfg["batch"] // world
        cfg = dict(full_cfg, batch=share)
        eng = OracleEngine(cfg, fail_at=fail_at if rank == fail_rank else None)
        dp = DataParallelStep(eng, overlap=overlap)
        assert dp.overlap == overlap
        out = _run(eng, dp, p, tok[rank * share:(rank + 1) * share],
                   tgt[rank * share:(rank + 1) * share], steps, full_cfg["lr"], full_cfg["wd"])
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


def _two_ranks(full_cfg, steps, fail_rank=-1, fail_at=None, overlap=False):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main,
                         args=(r, 2, port, full_cfg, steps, fail_rank, fail_at, q, overlap))
             for r in range(2)]
    for pr in procs:
        pr.start()
    res = dict(q.get(timeout=300) for _ in range(2))
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    return res


class OffsetEngine:
    """Records the dropout sequence offset a wrapper gives it."""
    device = torch.device("cpu")

    def __init__(self, batch):
        self.cfg = {"batch": batch}
        self.drop_b0 = None

    def set_dropout_offset(self, b0):
        self.drop_b0 = b0


def _rank_offsets(rank, world, port, batch, q):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from scratch_llama_decoder_b200.dp import DataParallelStep, ShardedDataParallelStep
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        a, b = OffsetEngine(batch), OffsetEngine(batch)
        DataParallelStep(a)
        ShardedDataParallelStep(b, 100)
        q.put((rank, (a.drop_b0, b.drop_b0)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_ranks_draw_dropout_masks_at_whole_batch_positions(world):
    """Rank r's share starts at sequence r * batch of the whole batch; one
    process (no group) keeps the engine's own offset."""
    from scratch_llama_decoder_b200.dp import DataParallelStep
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_offsets, args=(r, world, port, 3, q)) for r in range(world)]
    for pr in procs:
        pr.start()
    res = dict(q.get(timeout=300) for _ in range(world))
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    assert res == {r: (3 * r, 3 * r) for r in range(world)}
    e = OffsetEngine(3)
    DataParallelStep(e)
    assert e.drop_b0 is None


def test_two_ranks_equal_one_process_on_the_whole_batch():
    from synth import get_config
    from scratch_llama_decoder_b200.dp import DataParallelStep
    full = get_config("c1", vocab=11, d_model=16, n_layer=2, n_head=4, n_kv_head=2, d_ff=42,
                      ctx=5, batch=2, init_std=0.3, name="gqa-small", index=9)
    res = _two_ranks(full, steps=3)
    p, tok, tgt = _setup(full)
    # DataParallelStep with one rank (no process group) is the plain step
    eng = OracleEngine(full)
    ref = _run(eng, DataParallelStep(eng), p, tok, tgt, 3, full["lr"], full["wd"])
    for r in (0, 1):
        P, M, V, losses = res[r]
        np.testing.assert_allclose(P, ref[0], rtol=1e-12, atol=1e-15)
        np.testing.assert_allclose(M, ref[1], rtol=1e-10, atol=1e-18)
        np.testing.assert_allclose(V, ref[2], rtol=1e-10, atol=1e-22)
        # the summed mean losses over 2 ranks = 2 x the batch-mean loss
        np.testing.assert_allclose(np.array(losses) / 2, ref[3], rtol=1e-12)
    np.testing.assert_array_equal(res[0][0], res[1][0])  # the ranks agree bit for bit


def test_an_error_on_one_rank_skips_the_update_on_both():
    from synth import get_config
    full = get_config("c1", batch=2)
    res = _two_ranks(full, steps=2, fail_rank=1, fail_at=2)
    res_ok = _two_ranks(full, steps=1)
    for r in (0, 1):
        # step 2 was skipped everywhere: parameters stay at their step-1 values
        np.testing.assert_array_equal(res[r][0], res_ok[r][0])


def test_sharded_optimiser_two_ranks_equal_one_process():
    """Reduce-scatter, AdamW on each rank's chunk, all-gather: the parameters
    of the one-process step on the whole batch, and the ranks' moment chunks
    are that step's moments."""
    from synth import get_config
    from scratch_llama_decoder_b200.dp import DataParallelStep
    full = get_config("c1", vocab=11, d_model=16, n_layer=2, n_head=4, n_kv_head=2, d_ff=42,
                      ctx=5, batch=2, init_std=0.3, name="gqa-small", index=9)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main_sharded, args=(r, 2, port, full, 3, q))
             for r in range(2)]
    for pr in procs:
        pr.start()
    res = dict(q.get(timeout=300) for _ in range(2))
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    p, tok, tgt = _setup(full)
    eng = OracleEngine(full)
    ref = _run(eng, DataParallelStep(eng), p, tok, tgt, 3, full["lr"], full["wd"])
    for r in (0, 1):
        P, Mc, Vc, lo, cnt, _ = res[r]
        np.testing.assert_allclose(P, ref[0], rtol=1e-12, atol=1e-15)
        np.testing.assert_allclose(Mc, ref[1][lo:lo + cnt], rtol=1e-10, atol=1e-18)
        np.testing.assert_allclose(Vc, ref[2][lo:lo + cnt], rtol=1e-10, atol=1e-22)
    np.testing.assert_array_equal(res[0][0], res[1][0])
    assert res[0][4] + res[1][4] == p.size  # the chunks cover every parameter once


def test_sharded_wrapper_on_one_rank_is_the_plain_wrapper():
    import oracle as O
    from synth import get_config
    from scratch_llama_decoder_b200.dp import DataParallelStep, ShardedDataParallelStep
    cfg = get_config("c1", batch=2)
    p, tok, tgt = _setup(cfg)
    eng = OracleEngine(cfg)
    ref = _run(eng, DataParallelStep(eng), p, tok, tgt, 2, cfg["lr"], cfg["wd"])
    eng = OracleEngine(cfg)
    dp = ShardedDataParallelStep(eng, O.n_params(cfg))
    assert dp.world == 1 and dp.count == p.size and dp.chunk >= p.size and dp.chunk % 4 == 0
    P, G, M, V = dp.buffers(torch.float64)
    P[:p.size].copy_(torch.from_numpy(p))
    loss = torch.zeros(1, dtype=torch.float64)
    for t in (1, 2):
        dp.step(P, G, M, V, t, torch.tensor(tok), torch.tensor(tgt), cfg["lr"], cfg["wd"], loss)
    np.testing.assert_array_equal(P[:p.size].numpy(), ref[0])
    np.testing.assert_array_equal(M[:p.size].numpy(), ref[1])
    assert not G[p.size:].any() and not P[p.size:].any()


def test_bucketed_exchange_equals_the_whole_buffer_exchange():
    """overlap=True: one all-reduce per gradient bucket (the library's ranges)
    gives the same parameters, moments and losses as one all-reduce of the
    whole buffer, bit for bit, and the one-process step on the whole batch."""
    from synth import get_config
    from scratch_llama_decoder_b200.dp import DataParallelStep
    full = get_config("c1", vocab=11, d_model=16, n_layer=2, n_head=4, n_kv_head=2, d_ff=42,
                      ctx=5, batch=2, init_std=0.3, name="gqa-small", index=9)
    whole = _two_ranks(full, steps=2)
    bucketed = _two_ranks(full, steps=2, overlap=True)
    p, tok, tgt = _setup(full)
    eng = OracleEngine(full)
    ref = _run(eng, DataParallelStep(eng), p, tok, tgt, 2, full["lr"], full["wd"])
    for r in (0, 1):
        for a, b in zip(bucketed[r][:3], whole[r][:3]):
            np.testing.assert_array_equal(a, b)
        assert bucketed[r][3] == whole[r][3]
        np.testing.assert_allclose(bucketed[r][0], ref[0], rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("world", [2, 3])
def test_bucketed_sharded_optimiser_equals_one_process(world):
    """ShardedDataParallelStep(overlap=True): per-bucket reduce-scatter (each
    rank owning one piece of every bucket), AdamW on the pieces, per-bucket
    all-gather.  The ranks' parameters agree bit for bit and equal the
    one-process step on the whole batch; the pieces' moments, placed back,
    cover every parameter exactly once and equal that step's moments."""
    from synth import get_config
    from scratch_llama_decoder_b200.dp import DataParallelStep
    full = get_config("c1", vocab=11, d_model=16, n_layer=2, n_head=4, n_kv_head=2, d_ff=42,
                      ctx=5, batch=world, init_std=0.3, name="gqa-small", index=9)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main_sharded, args=(r, world, port, full, 3, q, True))
             for r in range(world)]
    for pr in procs:
        pr.start()
    res = dict(q.get(timeout=300) for _ in range(world))
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    p, tok, tgt = _setup(full)
    eng = OracleEngine(full)
    ref = _run(eng, DataParallelStep(eng), p, tok, tgt, 3, full["lr"], full["wd"])
    Mf = np.full(p.size, np.nan)
    Vf = np.full(p.size, np.nan)
    for r in range(world):
        np.testing.assert_array_equal(res[r][0], res[0][0])
        np.testing.assert_allclose(res[r][0], ref[0], rtol=1e-12, atol=1e-15)
        have = ~np.isnan(res[r][1])
        assert not np.any(~np.isnan(Mf[have]))  # each element owned by one rank
        Mf[have], Vf[have] = res[r][1][have], res[r][2][have]
    assert not np.any(np.isnan(Mf))
    np.testing.assert_allclose(Mf, ref[1], rtol=1e-10, atol=1e-18)
    np.testing.assert_allclose(Vf, ref[2], rtol=1e-10, atol=1e-22)


def _sharded_ranks(full, world, steps, overlap, clip, clip_mode):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main_sharded,
                         args=(r, world, port, full, steps, q, overlap, clip, clip_mode))
             for r in range(world)]
    for pr in procs:
        pr.start()
    res = dict(q.get(timeout=300) for _ in range(world))
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    return res


@pytest.mark.parametrize("world,overlap,clip_mode", [(2, False, 0), (3, True, 0), (2, True, 1),
                                                     (3, False, 1)],
                         ids=["2ranks-whole-l2", "3ranks-buckets-l2", "2ranks-buckets-linf",
                              "3ranks-whole-linf"])
def test_sharded_optimiser_clips_like_the_whole_gradient(world, overlap, clip_mode):
    """Clipping in the sharded forms (MicroGPT in Rust, Gradient Clipping;
    Transformer-In-Rust: by global norm; randyGPT: the L-infinity form): each
    rank's part of the norm, combined across ranks, gives the norm of the
    whole summed gradient, so the ranks clip as the one-process oracle step
    with the same threshold does.  The threshold sits below the norm of every
    step (checked), so every step is clipped."""
    from synth import get_config
    from scratch_llama_decoder_b200.dp import DataParallelStep
    full = get_config("c1", vocab=11, d_model=16, n_layer=2, n_head=4, n_kv_head=2, d_ff=42,
                      ctx=5, batch=world, init_std=0.3, name="gqa-small", index=9)
    clip = 0.05 if clip_mode == 1 else 0.5
    res = _sharded_ranks(full, world, 3, overlap, clip, clip_mode)
    p, tok, tgt = _setup(full)
    eng = OracleEngine(full, clip=clip, clip_mode=clip_mode)
    ref = _run(eng, DataParallelStep(eng), p, tok, tgt, 3, full["lr"], full["wd"])
    assert len(eng.norms) == 3 and min(eng.norms) > clip  # every step clipped
    for r in range(world):
        P, Mr, Vr = res[r][0], res[r][1], res[r][2]
        np.testing.assert_array_equal(P, res[0][0])  # the ranks agree bit for bit
        np.testing.assert_allclose(P, ref[0], rtol=1e-12, atol=1e-15)
        if overlap:
            have = ~np.isnan(Mr)
            np.testing.assert_allclose(Mr[have], ref[1][have], rtol=1e-10, atol=1e-18)
            np.testing.assert_allclose(Vr[have], ref[2][have], rtol=1e-10, atol=1e-22)
        else:
            lo, cnt = res[r][3], res[r][4]
            np.testing.assert_allclose(Mr, ref[1][lo:lo + cnt], rtol=1e-10, atol=1e-18)
            np.testing.assert_allclose(Vr, ref[2][lo:lo + cnt], rtol=1e-10, atol=1e-22)
        # every rank saw the whole gradient's norm
        np.testing.assert_allclose(res[r][5], eng.norms, rtol=1e-12)


def test_sharded_clipping_with_an_unclipping_threshold_is_the_unclipped_step():
    """A threshold above every norm leaves the sharded step unchanged."""
    from synth import get_config
    full = get_config("c1", vocab=11, d_model=16, n_layer=2, n_head=4, n_kv_head=2, d_ff=42,
                      ctx=5, batch=2, init_std=0.3, name="gqa-small", index=9)
    clipped = _sharded_ranks(full, 2, 2, False, 1e9, 0)
    plain = _sharded_ranks(full, 2, 2, False, 0.0, 0)
    for r in (0, 1):
        np.testing.assert_allclose(clipped[r][0], plain[r][0], rtol=1e-15, atol=0)
