"""B200 (sm_100a) implementation of WeDLM Streaming Parallel Decoding.

The decode step runs in libwedlm.so (CUDA kernels behind the C ABI declared in
include/wedlm.h); ``api`` is its Python binding."""
from .api import (Engine, step_params, reorder_window, entropy_select, entropy_select_noalloc, linear_bf16,  # noqa: F401
                  attention_workspace, attention_bf16, attention_error, entropy_select_async)
