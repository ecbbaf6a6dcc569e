"""GPU parity of single hot-path kernels (C ABI, include/llm_kernels.h)
against the float64 oracle's per-operation functions."""
import ctypes as C

import numpy as np
import pytest
import torch

import oracle as O

pytestmark = pytest.mark.gpu

# (M, N, K): tile multiples, ragged tails in every dimension, the step's shapes
SHAPES = [(128, 256, 64), (200, 300, 136), (1, 8, 8), (640, 768, 512), (384, 1408, 1024),
          (256, 2048, 16384 // 8)]


def _bf16(rng, shape):
    x = torch.tensor(rng.standard_normal(shape), dtype=torch.float32).to(torch.bfloat16)
    return x


@pytest.mark.parametrize("a_k,b_k", [(1, 0), (1, 1), (0, 0), (0, 1)])
@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("tc", [1, 0])
def test_gemm_bf16(M, N, K, a_k, b_k, tc):
    import scratch_llama_decoder_b200 as P
    rng = np.random.default_rng(M * 7 + N * 3 + K)
    # operand storage: K-major A is [M,K]; MN-major A is [K,M]; same for B with N
    A = _bf16(rng, (M, K) if a_k else (K, M))
    B = _bf16(rng, (N, K) if b_k else (K, N))
    lda = A.shape[1]
    ldb = B.shape[1]
    if tc and (lda % 8 or ldb % 8):
        pytest.skip("tensor-core path needs leading dimensions that are multiples of 8")
    Ad, Bd = A.cuda().contiguous(), B.cuda().contiguous()
    ldc = (N + 3) // 4 * 4
    Cd = torch.full((M, ldc), float("nan"), device="cuda")
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = P.lib.llm_kernel_gemm_bf16(M, N, K, C.c_void_p(Ad.data_ptr()), lda, a_k,
                                    C.c_void_p(Bd.data_ptr()), ldb, b_k,
                                    C.c_void_p(Cd.data_ptr()), ldc, tc,
                                    C.c_void_p(flag.data_ptr()), None)
    assert rc == 0
    torch.cuda.synchronize()
    assert flag.item() == 0
    got = Cd[:, :N].double().cpu().numpy()
    a64 = A.float().double().numpy()
    b64 = B.float().double().numpy()
    am = a64 if a_k else a64.T  # [M, K]
    bm = b64 if b_k else b64.T  # [N, K]
    ref = O.mm_nt(am, bm)
    err = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    # bf16 products are exact in fp32; only fp32 summation rounding remains
    assert err < 1e-5, err


# float32 GEMM shapes: tile multiples, ragged tails, K not a multiple of 32,
# the float32 workload's (tokens x 384 x 128, weight gradient over tokens)
SHAPES32 = [(128, 128, 32), (200, 300, 136), (1, 8, 8), (640, 768, 500), (16384, 384, 128),
            (128, 500, 16384), (333, 129, 77)]


@pytest.mark.parametrize("a_k,b_k", [(1, 0), (1, 1), (0, 0), (0, 1)])
@pytest.mark.parametrize("M,N,K", SHAPES32)
@pytest.mark.parametrize("tc", [1, 0])
def test_gemm_f32(M, N, K, a_k, b_k, tc):
    """tc = 1: split-precision tensor-core kernel (3xTF32); 0: CUDA cores.
    Gate 1e-5 norm-wise: 3xTF32 keeps about 2^-21 per product and the
    float32 accumulation adds its rounding; a single tf32 product (2^-11) would
    fail it.  (One TMEM accumulation chain over K = 16384 measured 1.1e-4,
    four interleaved chains 2.9e-5: the tensor core's float32 accumulation
    drops low bits per addition, so the kernel drains its accumulator into
    float32 registers every 512 of K.)"""
    import scratch_llama_decoder_b200 as P
    rng = np.random.default_rng(M * 5 + N * 11 + K)
    A = torch.tensor(rng.standard_normal((M, K) if a_k else (K, M)), dtype=torch.float32)
    B = torch.tensor(rng.standard_normal((N, K) if b_k else (K, N)), dtype=torch.float32)
    lda, ldb = A.shape[1], B.shape[1]
    Ad, Bd = A.cuda().contiguous(), B.cuda().contiguous()
    ldc = (N + 3) // 4 * 4
    Cd = torch.full((M, ldc), float("nan"), device="cuda")
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    nf = C.c_int64(0)
    assert P.lib.llm_kernel_gemm_f32_scratch_floats(M, N, K, C.byref(nf)) == 0
    scratch = torch.empty(max(1, nf.value), device="cuda")
    rc = P.lib.llm_kernel_gemm_f32(M, N, K, C.c_void_p(Ad.data_ptr()), lda, a_k,
                                   C.c_void_p(Bd.data_ptr()), ldb, b_k,
                                   C.c_void_p(Cd.data_ptr()), ldc, tc,
                                   C.c_void_p(scratch.data_ptr()), nf.value,
                                   C.c_void_p(flag.data_ptr()), None)
    assert rc == 0
    torch.cuda.synchronize()
    assert flag.item() == 0
    got = Cd[:, :N].double().cpu().numpy()
    a64, b64 = A.double().numpy(), B.double().numpy()
    ref = O.mm_nt(a64 if a_k else a64.T, b64 if b_k else b64.T)
    err = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert err < 1e-5, err
    assert np.abs(got - ref).max() <= 1e-4 * np.abs(ref).max()


def test_gemm_f32_scratch_too_small():
    import scratch_llama_decoder_b200 as P
    A = torch.zeros(64, 64, device="cuda")
    Cd = torch.zeros(64, 64, device="cuda")
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    nf = C.c_int64(0)
    assert P.lib.llm_kernel_gemm_f32_scratch_floats(64, 64, 64, C.byref(nf)) == 0
    scratch = torch.empty(nf.value, device="cuda")
    p = C.c_void_p(A.data_ptr())
    assert P.lib.llm_kernel_gemm_f32(64, 64, 64, p, 64, 1, p, 64, 1, C.c_void_p(Cd.data_ptr()),
                                     64, 1, C.c_void_p(scratch.data_ptr()), nf.value - 4,
                                     C.c_void_p(flag.data_ptr()), None) == P.LLM_ERR_ARG


@pytest.mark.parametrize("N,d,V", [(16, 16, 27), (16384, 1024, 32000), (1000, 64, 500),
                                   (300, 48, 70000)])
def test_embed_bwd_vs_oracle(N, d, V):
    """Scatter-add of the embedding gradient against the oracle; also
    bit-for-bit equal to float32 sums in the kernel's fixed order (a run of
    at most 64 rows in increasing position order; a longer run as 32
    contiguous parts, each summed in order, then added in part order); zero
    rows for absent ids; Zipf ids put thousands of rows on id 0."""
    import scratch_llama_decoder_b200 as P
    from synth import zipf_tokens
    rng = np.random.default_rng(N + V)
    tok = zipf_tokens(rng, N, V)
    dx = rng.standard_normal((N, d)).astype(np.float32)
    nb = C.c_int64(0)
    assert P.lib.llm_kernel_embed_bwd_scratch_bytes(N, V, C.byref(nb)) == 0
    scratch = torch.empty(nb.value, dtype=torch.uint8, device="cuda")
    td = torch.tensor(tok, device="cuda")
    xd = torch.tensor(dx, device="cuda")
    out = torch.full((V, d), float("nan"), device="cuda")
    rc = P.lib.llm_kernel_embed_bwd(C.c_void_p(td.data_ptr()), C.c_void_p(xd.data_ptr()),
                                    C.c_void_p(out.data_ptr()), N, d, V,
                                    C.c_void_p(scratch.data_ptr()), nb.value, None)
    assert rc == 0
    got = out.cpu().numpy()
    # float32 sums in the kernel's order, done on the host
    ref = np.zeros((V, d), np.float32)
    order = np.argsort(tok, kind="stable")
    bounds = np.searchsorted(tok[order], np.arange(V + 1))
    for v in range(V):
        run = order[bounds[v]:bounds[v + 1]]
        c = run.size
        parts = 32 if c > 64 else 1
        for k in range(parts):
            s = np.zeros(d, np.float32)
            for i in run[c * k // parts:c * (k + 1) // parts]:
                s += dx[i]
            ref[v] = s if k == 0 else ref[v] + s
    np.testing.assert_array_equal(got, ref)
    # and the float64 oracle agrees to float32 rounding
    ref64 = O.embed_bwd(tok, dx, V)
    assert np.linalg.norm(got - ref64) <= 1e-6 * max(1e-30, np.linalg.norm(ref64))
    # too-small scratch is rejected on the host
    assert P.lib.llm_kernel_embed_bwd(C.c_void_p(td.data_ptr()), C.c_void_p(xd.data_ptr()),
                                      C.c_void_p(out.data_ptr()), N, d, V,
                                      C.c_void_p(scratch.data_ptr()), nb.value - 4, None) == \
        P.LLM_ERR_ARG


# (batch, ctx, n_head, n_kv_head, head_dim): tile multiples, ragged lengths,
# one position, MHA/GQA/MQA, both head sizes, the longest context
ATTN = [(1, 64, 2, 2, 64), (2, 200, 4, 2, 64), (1, 130, 8, 8, 32), (3, 1, 4, 1, 64),
        (2, 512, 8, 2, 64), (1, 2048, 2, 2, 64), (1, 333, 4, 1, 32), (2, 384, 8, 2, 32),
        (3, 1, 4, 1, 32), (1, 1024, 2, 2, 32)]


@pytest.mark.parametrize("tc", [2, 1, 0])
@pytest.mark.parametrize("B,T,H,Hkv,hd", ATTN)
def test_attention_fwd_bwd_vs_oracle(B, T, H, Hkv, hd, tc):
    """tc: 2 = tcgen05 kernels, 1 = warp-level mma kernels, 0 = CUDA cores."""
    import scratch_llama_decoder_b200 as P
    if not tc and T > 600:
        pytest.skip("CUDA-core reference kernel: long contexts covered by the step tests")
    rng = np.random.default_rng(B * 1000 + T + H + hd)
    d, kvd = H * hd, Hkv * hd
    w = d + 2 * kvd
    qkv = _bf16(rng, (B * T, w))
    dout = _bf16(rng, (B * T, d))
    qd, dd = qkv.cuda(), dout.cuda()
    o = torch.zeros(B * T, d, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(B, H, T, device="cuda")
    Dv = torch.zeros(B, H, T, device="cuda")
    dq = torch.full((B * T, w), float("nan"), dtype=torch.bfloat16, device="cuda")
    p = lambda t: C.c_void_p(t.data_ptr())
    assert P.lib.llm_kernel_attention_fwd_bf16(p(qd), p(o), p(lse), B, T, H, Hkv, hd, tc,
                                               None) == 0
    assert P.lib.llm_kernel_attention_bwd_bf16(p(qd), p(o), p(dd), p(lse), p(Dv), p(dq), B, T, H,
                                               Hkv, hd, tc, None) == 0
    torch.cuda.synchronize()
    q64 = qkv.float().double().numpy().reshape(B, T, w)
    d64 = dout.float().double().numpy().reshape(B, T, d)
    og = o.float().double().cpu().numpy().reshape(B, T, d)
    lg = lse.double().cpu().numpy()
    dg = dq.float().double().cpu().numpy().reshape(B, T, w)
    for b in range(B):
        o_ref, lse_ref, _ = O.attention_fwd(q64[b], d, H, Hkv)
        dq_ref = O.attention_bwd(q64[b], d64[b], d, H, Hkv)
        assert np.linalg.norm(og[b] - o_ref) / np.linalg.norm(o_ref) < 1e-2
        assert np.abs(lg[b] - lse_ref).max() < 2e-3
        # dq, dk, dv; a block whose exact value is ~0 (T = 1: dq = dk = 0 since
        # dS = P (dP - D) vanishes for a single key) is measured against the
        # scale of the sequence's whole gradient instead
        full = np.linalg.norm(dq_ref)
        for lo, hi in ((0, d), (d, d + kvd), (d + kvd, w)):
            ref = dq_ref[:, lo:hi]
            err = np.linalg.norm(dg[b][:, lo:hi] - ref) / max(np.linalg.norm(ref), 1e-3 * full)
            assert err < 2e-2, (b, lo, err)


def test_attention_tc_head32_writes_only_its_head():
    """Head 32 on the tcgen05 kernels moves 64-wide tiles; their upper 32
    columns lie outside the head and must never be written: outputs sit in
    larger buffers whose guard region past the last row and head stays
    untouched, and O, dq|dk|dv equal the warp-level mma kernels' results to
    bf16 rounding."""
    import scratch_llama_decoder_b200 as P
    B, T, H, Hkv, hd = 2, 200, 4, 2, 32
    rng = np.random.default_rng(32)
    d, kvd = H * hd, Hkv * hd
    w = d + 2 * kvd
    qd = _bf16(rng, (B * T, w)).cuda()
    dd = _bf16(rng, (B * T, d)).cuda()
    p = lambda t: C.c_void_p(t.data_ptr())
    guard = 4096
    res = {}
    for tc in (2, 1):
        obuf = torch.full((B * T * d + guard,), 7.0, dtype=torch.bfloat16, device="cuda")
        gbuf = torch.full((B * T * w + guard,), 7.0, dtype=torch.bfloat16, device="cuda")
        o, dq = obuf[:B * T * d].view(B * T, d), gbuf[:B * T * w].view(B * T, w)
        lse = torch.zeros(B, H, T, device="cuda")
        Dv = torch.zeros(B, H, T, device="cuda")
        assert P.lib.llm_kernel_attention_fwd_bf16(p(qd), p(o), p(lse), B, T, H, Hkv, hd, tc,
                                                   None) == 0
        assert P.lib.llm_kernel_attention_bwd_bf16(p(qd), p(o), p(dd), p(lse), p(Dv), p(dq), B, T,
                                                   H, Hkv, hd, tc, None) == 0
        torch.cuda.synchronize()
        assert bool((obuf[B * T * d:] == 7).all()) and bool((gbuf[B * T * w:] == 7).all()), tc
        res[tc] = (o.float().cpu(), dq.float().cpu())
    for a, b in zip(res[2], res[1]):
        assert torch.isfinite(a).all()
        assert (a - b).norm() / b.norm() < 1e-2


# float32 attention (the float32 configurations): head sizes 32 and 64 with
# tile multiples, ragged lengths, one position, GQA and MQA, the C2 shape
ATTN32 = [(1, 64, 2, 2, 32), (2, 200, 4, 2, 32), (1, 130, 2, 2, 64), (3, 1, 4, 1, 64),
          (2, 333, 4, 4, 32), (1, 256, 4, 4, 32), (2, 129, 8, 2, 64)]


@pytest.mark.parametrize("tiled", [1, 0])
@pytest.mark.parametrize("B,T,H,Hkv,hd", ATTN32)
def test_attention_f32_vs_oracle(B, T, H, Hkv, hd, tiled):
    """tiled: 1 = the tiled CUDA-core kernels, 0 = one warp per row; fp32
    gates (the float32 configurations' logits and gradient tolerances)."""
    import scratch_llama_decoder_b200 as P
    rng = np.random.default_rng(7 * B + T + H + hd)
    d, kvd = H * hd, Hkv * hd
    w = d + 2 * kvd
    qkv = torch.tensor(rng.standard_normal((B * T, w)), dtype=torch.float32)
    dout = torch.tensor(rng.standard_normal((B * T, d)), dtype=torch.float32)
    qd, dd = qkv.cuda(), dout.cuda()
    o = torch.zeros(B * T, d, device="cuda")
    lse = torch.zeros(B, H, T, device="cuda")
    Dv = torch.zeros(B, H, T, device="cuda")
    dq = torch.full((B * T, w), float("nan"), device="cuda")
    p = lambda t: C.c_void_p(t.data_ptr())
    assert P.lib.llm_kernel_attention_fwd_f32(p(qd), p(o), p(lse), B, T, H, Hkv, hd, tiled,
                                              None) == 0
    assert P.lib.llm_kernel_attention_bwd_f32(p(qd), p(o), p(dd), p(lse), p(Dv), p(dq), B, T, H,
                                              Hkv, hd, tiled, None) == 0
    torch.cuda.synchronize()
    q64 = qkv.double().numpy().reshape(B, T, w)
    d64 = dout.double().numpy().reshape(B, T, d)
    og = o.double().cpu().numpy().reshape(B, T, d)
    lg = lse.double().cpu().numpy()
    dg = dq.double().cpu().numpy().reshape(B, T, w)
    assert np.isfinite(dg).all()
    for b in range(B):
        o_ref, lse_ref, _ = O.attention_fwd(q64[b], d, H, Hkv)
        dq_ref = O.attention_bwd(q64[b], d64[b], d, H, Hkv)
        assert np.linalg.norm(og[b] - o_ref) / np.linalg.norm(o_ref) < 1e-5
        assert np.abs(lg[b] - lse_ref).max() < 1e-5
        # a block whose exact value vanishes (T = 1) keeps the fp32 rounding of
        # D = dO . O against dP = dO . v (O(hd eps) of dP): its floor is a
        # hundredth of the sequence's gradient scale
        full = np.linalg.norm(dq_ref)
        for lo, hi in ((0, d), (d, d + kvd), (d + kvd, w)):
            ref = dq_ref[:, lo:hi]
            err = np.linalg.norm(dg[b][:, lo:hi] - ref) / max(np.linalg.norm(ref), 1e-2 * full)
            assert err < 1e-4, (b, lo, err)


def test_attention_f32_tiled_rejects_other_head_sizes():
    import scratch_llama_decoder_b200 as P
    x = torch.zeros(64, 3 * 16, device="cuda")
    o = torch.zeros(64, 16, device="cuda")
    lse = torch.zeros(1, 1, 64, device="cuda")
    p = lambda t: C.c_void_p(t.data_ptr())
    assert P.lib.llm_kernel_attention_fwd_f32(p(x), p(o), p(lse), 1, 64, 1, 1, 16, 1, None) == \
        P.LLM_ERR_ARG
