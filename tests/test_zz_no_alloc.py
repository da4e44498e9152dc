"""gptq_w4a16_gemm_lora_noalloc: the LoRA entry point whose T buffer is the
library's static device memory instead of a caller-provided work buffer.

Collected last on purpose: it checks that the static buffer gives the same
results as the caller-buffer entry point on consecutive calls that reuse it.
"""
import ctypes

import numpy as np
import pytest
import torch

from int4_weight_only_gptq_b200 import binding as B
from int4_weight_only_gptq_b200 import workloads as W


def test_oversize_and_bad_arguments_are_rejected_before_launch():
    from int4_weight_only_gptq_b200.build import build
    build()
    lib = B.load()
    v = ctypes.c_void_p
    X, QW, S, Y, LA, LB = 0x10000, 0x200000, 0x400000, 0x800000, 0x1800000, 0x1C00000
    # M * rank * 2 above the static buffer: GPTQ_ERR_SHAPE, nothing enqueued
    M = B.LORA_SCRATCH_BYTES // (2 * 256) + 1
    assert lib.gptq_w4a16_gemm_lora_noalloc(v(X), v(QW), v(S), M, 512, 256, 128, v(LA), v(LB),
                                            256, v(Y), None) == 2
    assert lib.gptq_w4a16_gemm_lora_noalloc(v(X), v(QW), v(S), 4, 512, 256, 128, v(LA), v(LB),
                                            24, v(Y), None) == 2
    assert lib.gptq_w4a16_gemm_lora_noalloc(v(X), v(QW), v(S), 4, 512, 256, 128, None, v(LB),
                                            32, v(Y), None) == 1
    assert lib.gptq_w4a16_gemm_lora_noalloc(v(X), v(QW), v(S), 0, 512, 256, 128, v(LA), v(LB),
                                            32, None, None) == 0


def _inputs(M, K, N, G, r, seed):
    p = W.make_problem(M, K, N, G, seed=seed)
    ad = W.make_adapter(K, N, r, seed=seed)
    t16 = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.float16).cuda()
    return (t16(p.x), torch.from_numpy(p.qweight).cuda(), t16(p.scales), G,
            t16(ad.lora_a), t16(ad.lora_b))


@pytest.mark.gpu
def test_static_buffer_matches_caller_buffer_on_two_calls():
    """Two calls in a row (a larger one, then a smaller one that reuses the
    start of the buffer): each is bit-identical to the caller-buffer entry."""
    for M, K, N, G, r, seed in ((300, 2048, 392, 64, 64, 1), (16, 1024, 264, 32, 32, 2)):
        args = _inputs(M, K, N, G, r, seed)
        y_static = B.gemm_lora_noalloc(*args)
        y_work = B.gemm_lora(*args)
        torch.cuda.synchronize()
        assert B.device_error() == 0
        assert torch.equal(y_static.view(torch.int16), y_work.view(torch.int16))


@pytest.mark.gpu
def test_mis_shaped_tensors_are_refused_before_the_library_is_called():
    """The C ABI cannot see buffer sizes: the binding refuses tensors whose
    shapes do not match the sizes it would pass (out, lora_b, qweight, scales)."""
    x, qw, s, G, a, b = _inputs(4, 512, 256, 128, 32, 3)
    cases = [
        dict(out=torch.empty((4, 248), dtype=torch.float16, device="cuda")),
        dict(lora_b=b[:248]),
        dict(qweight=qw[:56]),
        dict(scales=s[:2]),
    ]
    for kw in cases:
        args = dict(x=x, qweight=qw, scales=s, group=G, lora_a=a, lora_b=b)
        args.update(kw)
        with pytest.raises(ValueError):
            B.gemm_lora_noalloc(**args)
