"""kv1b_attend_noalloc: attention for callers that cannot allocate device memory or pass a
workspace (e.g. a framework whose allocator owns all device memory, or a decode loop where
cudaMalloc / cudaFree would synchronise the device).  The entry point keeps its split partials in
a fixed device array inside the library.  Called through the C ABI with ctypes; its output must
match kv1b_attend's within the parity tolerance, on two calls in a row.  This file sorts last so a
run that stops at the first failure has already run every other test."""
import ctypes
import math

import numpy as np
import pytest
import torch

import long_context_decode_kv1b_b200 as kv
from parity_utils import assert_rows_close

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 4 << 20


def noalloc_fn():
    fn = kv.lib().kv1b_attend_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.POINTER(kv.CacheDesc), ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32, ctypes.c_float,
                   ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p]
    return fn


def call_noalloc(cache, q, scale, engine=kv.ATTEND_TENSOR):
    out = torch.full((q.shape[0], q.shape[1], 128), float("nan"), dtype=torch.float32, device=q.device)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = noalloc_fn()(ctypes.byref(cache.desc), ctypes.c_void_p(q.data_ptr()), kv.DTYPE_BF16 if q.dtype ==
                      torch.bfloat16 else kv.DTYPE_F32, q.shape[1], scale, ctypes.c_void_p(out.data_ptr()), engine,
                      stream)
    return rc, out


def test_noalloc_matches_attend_on_two_calls_in_a_row():
    dev = "cuda"
    g = torch.Generator(device=dev).manual_seed(31)
    B, Hkv, G = 2, 4, 4
    cache = kv.Cache(B, Hkv, 8192, seed=3)
    K = torch.randn((B, 6000, Hkv, 128), generator=g, device=dev).to(torch.bfloat16)
    V = torch.randn((B, 6000, Hkv, 128), generator=g, device=dev).to(torch.bfloat16)
    cache.append(K, V)
    scale = 1.0 / math.sqrt(128)
    for call in range(2):
        q = torch.randn((B, Hkv * G, 128), generator=g, device=dev).to(torch.bfloat16)
        ref = cache.attend(q, scale).cpu().numpy()
        rc, out = call_noalloc(cache, q, scale)
        assert rc == 0, f"call {call}: {kv.lib().kv1b_status_string(rc)}"
        torch.cuda.synchronize()
        assert_rows_close(out.cpu().numpy(), ref, where=f"noalloc call {call}")
        # the CUDA-core engine through the same fixed scratch
        rc, out_c = call_noalloc(cache, q, scale, engine=kv.ATTEND_CUDA_CORE)
        assert rc == 0
        assert_rows_close(out_c.cpu().numpy(), ref, where=f"noalloc cuda-core call {call}")


def test_noalloc_refuses_shapes_beyond_its_scratch():
    # 64 sequences x 128 query heads x 520 bytes of partials > the 4 MiB array even unsplit
    cache = kv.Cache(64, 16, 128, seed=0)
    q = torch.zeros((64, 128, 128), dtype=torch.float32, device="cuda")
    assert 64 * 128 * 520 > SCRATCH_BYTES
    rc, out = call_noalloc(cache, q, 0.1)
    assert rc == -5
    torch.cuda.synchronize()
    assert torch.isnan(out).all()  # nothing was launched or written
