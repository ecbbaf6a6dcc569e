"""ctypes binding of libllm.so (include/llm.h): argument marshalling only.

Every computation runs in the library's CUDA kernels.  Importing this module
raises if the library has not been built; there is no fallback.
"""
import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
# LLM_LIB: another build of the library to load (the sanitizer test loads one
# whose host code is built with AddressSanitizer and UBSan)
LIB_PATH = os.environ.get("LLM_LIB") or os.path.join(HERE, "libllm.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python scratch_llama_decoder_b200/build.py` "
        "(nvcc, sm_100a).  There is no CPU fallback.")

lib = C.CDLL(LIB_PATH)

LLM_OK, LLM_ERR_CONFIG, LLM_ERR_ARG, LLM_ERR_TOKEN = 0, -1, -2, -3
LLM_ERR_NONFINITE, LLM_ERR_CUDA, LLM_ERR_TIMEOUT = -4, -5, -6
LLM_FP32, LLM_BF16 = 0, 1


class llm_config(C.Structure):
    _fields_ = [("vocab", C.c_int32), ("d_model", C.c_int32), ("n_layer", C.c_int32),
                ("n_head", C.c_int32), ("n_kv_head", C.c_int32), ("d_ff", C.c_int32),
                ("ctx", C.c_int32), ("batch", C.c_int32), ("rope_base", C.c_float),
                ("rms_eps", C.c_float), ("beta1", C.c_float), ("beta2", C.c_float),
                ("adam_eps", C.c_float), ("compute", C.c_int32), ("recompute", C.c_int32)]


class llm_tensor_info(C.Structure):
    _fields_ = [("name", C.c_char * 32), ("offset", C.c_int64), ("rows", C.c_int64),
                ("cols", C.c_int64)]


LLM_LR_CONSTANT, LLM_LR_COSINE, LLM_LR_LINEAR = 0, 1, 2
LLM_CLIP_L2, LLM_CLIP_LINF = 0, 1
# kernel classes of llm_read_kernel_class_timing (LLM_KT_*), with the unit of
# the work each is credited with
KERNEL_CLASSES = [("gemm", "flop"), ("attention_fwd", "flop"), ("attention_bwd", "flop"),
                  ("rmsnorm_fwd", "byte"), ("rmsnorm_bwd", "byte"), ("swiglu_fwd", "byte"),
                  ("swiglu_bwd", "byte"), ("cross_entropy", "byte"), ("embed_fwd", "byte"),
                  ("embed_bwd", "byte"), ("adamw", "byte"), ("weight_cast", "byte"),
                  ("wgrad_finish", "byte"), ("gemm_cuda_core", "flop"), ("gemm_tf32", "flop")]
LR_SHAPES = {"constant": LLM_LR_CONSTANT, "cosine": LLM_LR_COSINE, "linear": LLM_LR_LINEAR}


class llm_plateau(C.Structure):
    _fields_ = [("best", C.c_double), ("threshold", C.c_double), ("scale", C.c_double),
                ("bad", C.c_int64), ("patience", C.c_int64), ("reductions", C.c_int32),
                ("max_reductions", C.c_int32), ("factor", C.c_float)]


class llm_lr_schedule(C.Structure):
    _fields_ = [("max_lr", C.c_float), ("min_lr", C.c_float), ("warmup_steps", C.c_int64),
                ("decay_start", C.c_int64), ("total_steps", C.c_int64), ("shape", C.c_int32)]


_vp, _i64, _u64, _f, _i = C.c_void_p, C.c_int64, C.c_uint64, C.c_float, C.c_int
_cfgp = C.POINTER(llm_config)

EXPORTS = {
    "llm_param_layout": (_i, [_cfgp, C.POINTER(llm_tensor_info), C.POINTER(_i), C.POINTER(_i64)]),
    "llm_workspace_bytes": (_i, [_cfgp, C.POINTER(_i64)]),
    "llm_create": (_i, [_cfgp, _vp, _i64, _vp, C.POINTER(_vp)]),
    "llm_destroy": (None, [_vp]),
    "llm_init": (_i, [_vp, _u64, _f, _i, _vp]),
    "llm_forward": (_i, [_vp, _vp, _vp, _vp]),
    "llm_step": (_i, [_vp, _vp, _vp, _vp, _vp, _i64, _vp, _vp, _f, _f, _vp]),
    "llm_grad": (_i, [_vp, _vp, _vp, _vp, _vp, _vp]),
    "llm_adamw": (_i, [_vp, _vp, _vp, _vp, _vp, _i64, _f, _f, _f]),
    "llm_adamw_range": (_i, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _f, _f, _f]),
    "llm_grad_norm_part": (_i, [_vp, _vp, _i64, _f, _i, _vp]),
    "llm_adamw_range_clip": (_i, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _f, _f, _vp]),
    "llm_flag_out": (_i, [_vp, _vp]),
    "llm_flag_in": (_i, [_vp, _vp]),
    "llm_grad_bucket_range": (_i, [_cfgp, _i, C.POINTER(_i64), C.POINTER(_i64)]),
    "llm_set_grad_buckets": (_i, [_vp, _i]),
    "llm_get_dropout_calls": (_i, [_vp, C.POINTER(_i64)]),
    "llm_set_dropout_calls": (_i, [_vp, _i64]),
    "llm_set_dropout_offset": (_i, [_vp, _i64]),
    "llm_grad_bucket_wait": (_i, [_vp, _i, _vp]),
    "llm_decode": (_i, [_vp, _vp, _vp, _i, _vp]),
    "llm_sample": (_i, [_vp, _vp, _i64, _i, _f, _i, _vp, _vp]),
    "llm_sample_ex": (_i, [_vp, _vp, _i64, _i, _f, _i, _f, _f, _vp, _i64, _i, _vp, _vp]),
    "llm_set_grad_clip": (_i, [_vp, _f]),
    "llm_set_dropout": (_i, [_vp, _f, _u64]),
    "llm_set_grad_clip_mode": (_i, [_vp, _i]),
    "llm_set_rope_scale": (_i, [_vp, _f]),
    "llm_read_grad_norm": (_i, [_vp, C.POINTER(C.c_double)]),
    "llm_lr_at": (_i, [C.POINTER(llm_lr_schedule), _i64, C.POINTER(_f)]),
    "llm_plateau_init": (_i, [C.POINTER(llm_plateau), _f, _i64, C.c_int32, C.c_double]),
    "llm_plateau_update": (_i, [C.POINTER(llm_plateau), C.c_double, C.POINTER(_f)]),
    "llm_status": (_i, [_vp]),
    "llm_error_string": (C.c_char_p, [_i]),
    "llm_last_launch_count": (_i, [_vp]),
    "llm_set_kernel_timing": (_i, [_vp, _i]),
    "llm_set_graphs": (_i, [_vp, _i]),
    "llm_read_kernel_timing": (_i, [_vp, C.POINTER(C.c_double), C.POINTER(C.c_double),
                                    C.POINTER(_i64)]),
    "llm_read_kernel_class_timing": (_i, [_vp, _i, C.POINTER(C.c_double), C.POINTER(C.c_double),
                                          C.POINTER(_i64)]),
    # include/llm_kernels.h
    "llm_kernel_gemm_bf16": (_i, [_i, _i, _i, _vp, _i64, _i, _vp, _i64, _i, _vp, _i64, _i, _vp,
                                  _vp]),
    "llm_kernel_gemm_f32_scratch_floats": (_i, [_i, _i, _i, C.POINTER(_i64)]),
    "llm_kernel_gemm_f32": (_i, [_i, _i, _i, _vp, _i64, _i, _vp, _i64, _i, _vp, _i64, _i, _vp,
                                 _i64, _vp, _vp]),
    "llm_kernel_attention_fwd_bf16": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp]),
    "llm_kernel_attention_bwd_bf16": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i,
                                           _vp]),
    "llm_kernel_attention_fwd_f32": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp]),
    "llm_kernel_attention_bwd_f32": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i,
                                          _vp]),
    "llm_kernel_embed_bwd_scratch_bytes": (_i, [_i64, _i, C.POINTER(_i64)]),
    "llm_kernel_embed_bwd": (_i, [_vp, _vp, _vp, _i64, _i, _i, _vp, _i64, _vp]),
    "llm_kernel_embed_bwd_noalloc": (_i, [_vp, _vp, _vp, _i64, _i, _i, _vp]),
}
for _name, (_res, _args) in EXPORTS.items():
    _fn = getattr(lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


class LLMError(RuntimeError):
    def __init__(self, code, where):
        super().__init__(f"{where}: {lib.llm_error_string(code).decode()} ({code})")
        self.code = code


def check(code, where):
    if code != LLM_OK:
        raise LLMError(code, where)
    return code


def make_config(cfg) -> llm_config:
    """llm_config from a mapping with the field names of include/llm.h
    (compute given as "fp32"/"bf16" or 0/1)."""
    comp = cfg.get("compute", 0)
    if isinstance(comp, str):
        comp = {"fp32": LLM_FP32, "bf16": LLM_BF16}[comp]
    return llm_config(cfg["vocab"], cfg["d_model"], cfg["n_layer"], cfg["n_head"],
                      cfg["n_kv_head"], cfg["d_ff"], cfg["ctx"], cfg["batch"],
                      float(cfg.get("rope_base", 10000.0)), float(cfg.get("rms_eps", 1e-5)),
                      float(cfg.get("beta1", 0.9)), float(cfg.get("beta2", 0.999)),
                      float(cfg.get("adam_eps", 1e-8)), int(comp),
                      int(cfg.get("recompute", 0)))


def llm_param_layout(cfg):
    """[(name, offset, rows, cols)], n_params."""
    c = make_config(cfg)
    n = C.c_int(0)
    npar = C.c_int64(0)
    check(lib.llm_param_layout(C.byref(c), None, C.byref(n), C.byref(npar)), "llm_param_layout")
    arr = (llm_tensor_info * n.value)()
    check(lib.llm_param_layout(C.byref(c), arr, C.byref(n), C.byref(npar)), "llm_param_layout")
    return [(t.name.decode(), t.offset, t.rows, t.cols) for t in arr], npar.value


def llm_workspace_bytes(cfg) -> int:
    c = make_config(cfg)
    b = C.c_int64(0)
    check(lib.llm_workspace_bytes(C.byref(c), C.byref(b)), "llm_workspace_bytes")
    return b.value


def grad_buckets(cfg):
    """[(offset, count)] of the gradient buckets in the order the backward
    finishes them (llm_grad_bucket_range; host only)."""
    c = make_config(cfg)
    out, k = [], 0
    off, cnt = C.c_int64(0), C.c_int64(0)
    while True:
        rc = lib.llm_grad_bucket_range(C.byref(c), k, C.byref(off), C.byref(cnt))
        if rc == LLM_ERR_ARG and k > 0:
            return out
        check(rc, "llm_grad_bucket_range")
        out.append((off.value, cnt.value))
        k += 1


def lr_at(t, max_lr, min_lr, warmup, decay_start, total, shape="cosine") -> float:
    """Learning rate of 1-based step t (llm_lr_at)."""
    sc = llm_lr_schedule(max_lr, min_lr, warmup, decay_start, total, LR_SHAPES[shape])
    out = C.c_float(0.0)
    check(lib.llm_lr_at(C.byref(sc), int(t), C.byref(out)), "llm_lr_at")
    return out.value


class Plateau:
    """Learning-rate reduction on a plateau (llm_plateau_init / _update)."""

    def __init__(self, factor=0.5, patience=30, max_reductions=3, threshold=0.0):
        self._s = llm_plateau()
        check(lib.llm_plateau_init(C.byref(self._s), float(factor), int(patience),
                                   int(max_reductions), float(threshold)), "llm_plateau_init")

    def update(self, metric) -> float:
        out = C.c_float(1.0)
        check(lib.llm_plateau_update(C.byref(self._s), float(metric), C.byref(out)),
              "llm_plateau_update")
        return out.value
