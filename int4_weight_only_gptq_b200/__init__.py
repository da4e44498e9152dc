"""B200-native (sm_100a) INT4 GPTQ W4A16 linear layer.

    Y[M, N] = X[M, K] . dequant(qweight[K/8, N], scales[n_groups, N])

The computation lives in libgptq_w4a16.so (hand-written CUDA for sm_100a behind
a C ABI, declared in include/gptq_w4a16.h); ``binding`` marshals torch tensors
to it.  Importing this package does not load the library; the first call does,
and fails loudly if it is missing.
"""
__version__ = "0.1.0"

_BINDING_NAMES = {"gemm", "gemm_grouped", "gemm_asym", "gemm_gidx", "gemm_lora",
                  "gemm_lora_noalloc", "dequant", "select", "device_error", "version", "load",
                  "GptqError", "KERNEL_AUTO", "KERNEL_DECODE", "KERNEL_PREFILL", "DECODE_MAX_M",
                  "LORA_DECODE_MAX_M", "MAX_GROUPED", "MAX_LORA_RANK", "LORA_SCRATCH_BYTES",
                  "GIDX_MAX_GROUPS", "GROUP_SIZES"}


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
