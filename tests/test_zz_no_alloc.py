"""The allocation-free embedding backward (llm_kernel_embed_bwd_noalloc).

It serves callers that cannot allocate device memory when they call the
library (during graph capture, inside allocator hooks, in frameworks that own
all device memory).  Its scratch is a library-owned device array, so this
test checks it against the scratch-taking entry point llm_kernel_embed_bwd
on the same inputs, on two calls in a row with different sizes (the second
call must not see the first call's leftovers), and that sizes beyond its
limits are refused on the host.  This file is collected after every other
test file; it also passes alone in a fresh process, where its first call does
the per-device set-up.
"""
import ctypes as C

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _scratch_entry(P, td, xd, N, d, V):
    nb = C.c_int64(0)
    assert P.lib.llm_kernel_embed_bwd_scratch_bytes(N, V, C.byref(nb)) == 0
    scratch = torch.empty(nb.value, dtype=torch.uint8, device="cuda")
    out = torch.full((V, d), float("nan"), device="cuda")
    rc = P.lib.llm_kernel_embed_bwd(C.c_void_p(td.data_ptr()), C.c_void_p(xd.data_ptr()),
                                    C.c_void_p(out.data_ptr()), N, d, V,
                                    C.c_void_p(scratch.data_ptr()), nb.value, None)
    assert rc == 0
    torch.cuda.synchronize()
    return out.cpu().numpy()


def _noalloc_entry(P, td, xd, N, d, V):
    out = torch.full((V, d), float("nan"), device="cuda")
    rc = P.lib.llm_kernel_embed_bwd_noalloc(C.c_void_p(td.data_ptr()), C.c_void_p(xd.data_ptr()),
                                            C.c_void_p(out.data_ptr()), N, d, V, None)
    assert rc == 0
    torch.cuda.synchronize()
    return out.cpu().numpy()


def test_noalloc_embed_bwd_matches_scratch_entry_twice():
    import scratch_llama_decoder_b200 as P
    from synth import zipf_tokens
    # the largest case first, then a smaller one reusing the shared array
    for N, d, V in ((16384, 1024, 32000), (777, 96, 500)):
        rng = np.random.default_rng(N)
        tok = zipf_tokens(rng, N, V)
        dx = rng.standard_normal((N, d)).astype(np.float32)
        td = torch.tensor(tok, device="cuda")
        xd = torch.tensor(dx, device="cuda")
        ref = _scratch_entry(P, td, xd, N, d, V)
        got = _noalloc_entry(P, td, xd, N, d, V)
        # the same kernels in the same order: identical results (0 tolerance,
        # tighter than the 1e-3 gradient tolerance of the fp32 tests)
        np.testing.assert_array_equal(got, ref)
        assert np.isfinite(got).all()


def test_noalloc_embed_bwd_refuses_sizes_beyond_limits():
    import scratch_llama_decoder_b200 as P
    dummy = torch.zeros(16, device="cuda")
    ptr = C.c_void_p(dummy.data_ptr())
    assert P.lib.llm_kernel_embed_bwd_noalloc(ptr, ptr, ptr, 65537, 4, 100, None) == \
        P.LLM_ERR_ARG
    assert P.lib.llm_kernel_embed_bwd_noalloc(ptr, ptr, ptr, 100, 4, 65537, None) == \
        P.LLM_ERR_ARG
    assert P.lib.llm_kernel_embed_bwd_noalloc(None, ptr, ptr, 100, 4, 100, None) == \
        P.LLM_ERR_ARG
