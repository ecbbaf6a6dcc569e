"""B200-native training step of a bias-free, pre-norm Llama-style decoder.

The compute lives in libllm.so (hand-written sm_100a CUDA kernels behind the
C ABI of include/llm.h).  This package only marshals arguments: PyTorch
provides device memory and the stream.
"""
from ._lib import (LLM_BF16, LLM_ERR_ARG, LLM_ERR_CONFIG, LLM_ERR_CUDA, LLM_ERR_NONFINITE,  # noqa
                   LLM_ERR_TIMEOUT, LLM_ERR_TOKEN, LLM_FP32, LLM_OK, LLMError, check, lib,
                   Plateau, grad_buckets, llm_param_layout, llm_workspace_bytes, lr_at,
                   make_config)
from .model import LlamaStep  # noqa: F401
