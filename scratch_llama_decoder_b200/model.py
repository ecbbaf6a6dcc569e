"""LlamaStep: a context of the C ABI bound to torch device memory and stream.

Argument marshalling only: torch tensors are passed to the library by device
pointer; every step of the computation runs in the library's kernels.
"""
import ctypes as C
import functools

import torch

from . import _lib as L


def _ptr(t):
    return C.c_void_p(t.data_ptr()) if t is not None else None


def _on_device(fn):
    """Runs a method with the context's device current: the library refuses
    calls on a context made with another device current."""
    @functools.wraps(fn)
    def call(self, *args, **kwargs):
        with torch.cuda.device(self.device):
            return fn(self, *args, **kwargs)
    return call


class LlamaStep:
    """Owns the workspace (a torch uint8 tensor) and the llm_ctx for one config.

    cfg: mapping with the llm_config field names (vocab, d_model, n_layer,
    n_head, n_kv_head, d_ff, ctx, batch, rope_base, rms_eps, beta1, beta2,
    adam_eps, compute)."""

    def __init__(self, cfg, device="cuda", stream=None):
        if not torch.cuda.is_available():
            raise RuntimeError("LlamaStep needs a CUDA device (B200, sm_100a); no CPU fallback")
        self.cfg = dict(cfg)
        dev = torch.device(device)
        if dev.type != "cuda":
            raise ValueError(f"LlamaStep runs on a CUDA device, not {dev}")
        if dev.index is None:
            dev = torch.device("cuda", torch.cuda.current_device())
        self.device = dev
        self.layout, self.n_params = L.llm_param_layout(cfg)
        self.ws_bytes = L.llm_workspace_bytes(cfg)
        self._c = L.make_config(cfg)
        with torch.cuda.device(self.device):
            self.workspace = torch.empty(self.ws_bytes, dtype=torch.uint8, device=self.device)
            self.stream = stream if stream is not None else torch.cuda.current_stream(self.device)
            ctx = C.c_void_p()
            L.check(L.lib.llm_create(C.byref(self._c), _ptr(self.workspace), self.ws_bytes,
                                     C.c_void_p(self.stream.cuda_stream), C.byref(ctx)),
                    "llm_create")
        self.ctx = ctx
        self.grad_clip, self.grad_clip_mode = 0.0, 0  # as llm_create leaves them

    def close(self):
        if getattr(self, "ctx", None):
            L.lib.llm_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -------------------------------------------------------------- buffers
    def new_params(self):
        return torch.zeros(self.n_params, dtype=torch.float32, device=self.device)

    @_on_device
    def init(self, params, seed, init_std, scale_out_proj):
        L.check(L.lib.llm_init(self.ctx, seed, float(init_std), int(bool(scale_out_proj)),
                               _ptr(params)), "llm_init")

    @_on_device
    def forward(self, params, tokens, logits=None):
        B, T, V = self.cfg["batch"], self.cfg["ctx"], self.cfg["vocab"]
        if logits is None:
            logits = torch.empty(B, T, V, dtype=torch.float32, device=self.device)
        L.check(L.lib.llm_forward(self.ctx, _ptr(params), _ptr(tokens), _ptr(logits)),
                "llm_forward")
        return logits

    @_on_device
    def step(self, params, grads, m, v, t, tokens, targets, lr, wd, loss=None):
        if loss is None:
            loss = torch.empty(1, dtype=torch.float32, device=self.device)
        L.check(L.lib.llm_step(self.ctx, _ptr(params), _ptr(grads), _ptr(m), _ptr(v), int(t),
                               _ptr(tokens), _ptr(targets), float(lr), float(wd), _ptr(loss)),
                "llm_step")
        return loss

    @_on_device
    def sample_ex(self, logits, temperature, top_k, uniforms, top_p=1.0, penalty=1.0,
                  history=None, out=None):
        """llm_sample_ex: repetition penalty over history (int32 [rows, n]),
        temperature, top-k, top-p."""
        rows = logits.shape[0]
        if out is None:
            out = torch.empty(rows, dtype=torch.int32, device=self.device)
        hl = 0 if history is None else history.shape[1]
        hld = 0 if history is None else history.stride(0)
        L.check(L.lib.llm_sample_ex(self.ctx, _ptr(logits), logits.stride(0), rows,
                                    float(temperature), int(top_k), float(top_p), float(penalty),
                                    _ptr(history), hld, hl, _ptr(uniforms), _ptr(out)),
                "llm_sample_ex")
        return out

    @_on_device
    def grad(self, params, grads, tokens, targets, loss=None):
        """Forward, loss and backward without the update (llm_grad)."""
        if loss is None:
            loss = torch.empty(1, dtype=torch.float32, device=self.device)
        L.check(L.lib.llm_grad(self.ctx, _ptr(params), _ptr(grads), _ptr(tokens), _ptr(targets),
                               _ptr(loss)), "llm_grad")
        return loss

    @_on_device
    def adamw(self, params, grads, m, v, t, lr, wd, grad_scale=1.0):
        """grads *= grad_scale, optional clipping, AdamW (llm_adamw)."""
        L.check(L.lib.llm_adamw(self.ctx, _ptr(params), _ptr(grads), _ptr(m), _ptr(v), int(t),
                                float(lr), float(wd), float(grad_scale)), "llm_adamw")

    @_on_device
    def adamw_range(self, params, grads, m, v, t, lr, wd, grad_scale=1.0):
        """AdamW over the elements of 1-D views params, grads, m, v (equal
        lengths; llm_adamw_range)."""
        n = params.numel()
        assert grads.numel() == n and m.numel() == n and v.numel() == n
        L.check(L.lib.llm_adamw_range(self.ctx, _ptr(params), _ptr(grads), _ptr(m), _ptr(v), n,
                                      int(t), float(lr), float(wd), float(grad_scale)),
                "llm_adamw_range")

    @_on_device
    def grad_norm_part(self, grads, grad_scale, part, accumulate=False):
        """grads (1-D view) *= grad_scale, then its part of the clipping norm
        into part (one float64 on the device; llm_grad_norm_part)."""
        L.check(L.lib.llm_grad_norm_part(self.ctx, _ptr(grads), grads.numel(), float(grad_scale),
                                         int(bool(accumulate)), _ptr(part)),
                "llm_grad_norm_part")

    @_on_device
    def adamw_range_clip(self, params, grads, m, v, t, lr, wd, total):
        """Clip by the ranks' combined norm part total, then AdamW over the
        elements of 1-D views params, grads, m, v (llm_adamw_range_clip)."""
        n = params.numel()
        assert grads.numel() == n and m.numel() == n and v.numel() == n
        L.check(L.lib.llm_adamw_range_clip(self.ctx, _ptr(params), _ptr(grads), _ptr(m), _ptr(v),
                                           n, int(t), float(lr), float(wd), _ptr(total)),
                "llm_adamw_range_clip")

    @_on_device
    def flag_out(self, flag):
        """Copy the step's int32 error word to flag (llm_flag_out)."""
        L.check(L.lib.llm_flag_out(self.ctx, _ptr(flag)), "llm_flag_out")

    @_on_device
    def flag_in(self, flag):
        """OR the int32 word flag into the step's error word (llm_flag_in)."""
        L.check(L.lib.llm_flag_in(self.ctx, _ptr(flag)), "llm_flag_in")

    def grad_buckets(self):
        """[(offset, count)] of the gradient buckets, in the order llm_grad's
        backward finishes them."""
        return L.grad_buckets(self.cfg)

    @_on_device
    def set_grad_buckets(self, enable):
        L.check(L.lib.llm_set_grad_buckets(self.ctx, int(bool(enable))), "llm_set_grad_buckets")

    @_on_device
    def grad_bucket_wait(self, k, stream):
        """Makes torch stream `stream` wait until bucket k of the last
        llm_grad is final."""
        L.check(L.lib.llm_grad_bucket_wait(self.ctx, int(k), C.c_void_p(stream.cuda_stream)),
                "llm_grad_bucket_wait")

    @_on_device
    def decode(self, params, tokens, pos, logits=None):
        """Logits [B, V] of position pos (llm_decode); tokens: int32 [B]."""
        B, V = self.cfg["batch"], self.cfg["vocab"]
        if logits is None:
            logits = torch.empty(B, V, dtype=torch.float32, device=self.device)
        L.check(L.lib.llm_decode(self.ctx, _ptr(params), _ptr(tokens), int(pos), _ptr(logits)),
                "llm_decode")
        return logits

    @_on_device
    def sample(self, logits, temperature, top_k, uniforms, out=None):
        """int32 token ids [rows] from float32 logits [rows, ld] (llm_sample)."""
        rows = logits.shape[0]
        if out is None:
            out = torch.empty(rows, dtype=torch.int32, device=self.device)
        L.check(L.lib.llm_sample(self.ctx, _ptr(logits), logits.stride(0), rows,
                                 float(temperature), int(top_k), _ptr(uniforms), _ptr(out)),
                "llm_sample")
        return out

    @_on_device
    def set_rope_scale(self, factor):
        """RoPE position interpolation: positions t / factor (llm_set_rope_scale)."""
        L.check(L.lib.llm_set_rope_scale(self.ctx, float(factor)), "llm_set_rope_scale")

    @_on_device
    def set_dropout(self, p, seed):
        """Inverted dropout in later training calls (llm_set_dropout)."""
        L.check(L.lib.llm_set_dropout(self.ctx, float(p), int(seed)), "llm_set_dropout")

    def dropout_calls(self):
        """The mask counter: the number the next training call draws with."""
        n = C.c_int64(0)
        L.check(L.lib.llm_get_dropout_calls(self.ctx, C.byref(n)), "llm_get_dropout_calls")
        return n.value

    def set_dropout_calls(self, n):
        L.check(L.lib.llm_set_dropout_calls(self.ctx, int(n)), "llm_set_dropout_calls")

    @_on_device
    def set_dropout_offset(self, b0):
        """Index of this context's first sequence in the whole batch: masks are
        drawn at whole-batch positions (llm_set_dropout_offset)."""
        L.check(L.lib.llm_set_dropout_offset(self.ctx, int(b0)), "llm_set_dropout_offset")

    @_on_device
    def set_grad_clip(self, max_norm):
        """Global-norm gradient clipping in later steps (llm_set_grad_clip)."""
        L.check(L.lib.llm_set_grad_clip(self.ctx, float(max_norm)), "llm_set_grad_clip")
        self.grad_clip = float(max_norm)

    @_on_device
    def set_grad_clip_mode(self, mode):
        """0: global L2 norm (default); 1: L-infinity norm (llm_set_grad_clip_mode)."""
        L.check(L.lib.llm_set_grad_clip_mode(self.ctx, int(mode)), "llm_set_grad_clip_mode")
        self.grad_clip_mode = int(mode)

    @_on_device
    def read_grad_norm(self):
        """Gradient norm before clipping of the last clipped step (llm_read_grad_norm)."""
        v = C.c_double(0.0)
        L.check(L.lib.llm_read_grad_norm(self.ctx, C.byref(v)), "llm_read_grad_norm")
        return v.value

    @_on_device
    def status(self):
        return L.lib.llm_status(self.ctx)

    @_on_device
    def last_launch_count(self):
        return L.lib.llm_last_launch_count(self.ctx)

    @_on_device
    def set_kernel_timing(self, enable):
        L.check(L.lib.llm_set_kernel_timing(self.ctx, int(bool(enable))), "llm_set_kernel_timing")

    @_on_device
    def set_graphs(self, enable):
        """Step graphs on/off (llm_set_graphs)."""
        L.check(L.lib.llm_set_graphs(self.ctx, int(bool(enable))), "llm_set_graphs")

    @_on_device
    def read_kernel_class_timing(self):
        """{class name: (device ms, algorithmic work, launches)} since the last
        reset (llm_read_kernel_class_timing); read before read_kernel_timing,
        which resets."""
        out = {}
        for k, (name, _) in enumerate(L.KERNEL_CLASSES):
            ms, w, n = C.c_double(0), C.c_double(0), C.c_int64(0)
            L.check(L.lib.llm_read_kernel_class_timing(self.ctx, k, C.byref(ms), C.byref(w),
                                                       C.byref(n)),
                    "llm_read_kernel_class_timing")
            out[name] = (ms.value, w.value, n.value)
        return out

    @_on_device
    def read_kernel_timing(self):
        """(device ms, algorithmic FLOPs, launches) of the timed GEMM launches."""
        ms, fl, n = C.c_double(0), C.c_double(0), C.c_int64(0)
        L.check(L.lib.llm_read_kernel_timing(self.ctx, C.byref(ms), C.byref(fl), C.byref(n)),
                "llm_read_kernel_timing")
        return ms.value, fl.value, n.value
