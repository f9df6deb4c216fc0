"""kv1b_attend_noalloc: attention for callers that cannot allocate device memory or pass a
workspace (e.g. a framework whose allocator owns all device memory, or a decode loop where
cudaMalloc / cudaFree would synchronise the device).  The entry point keeps its split partials and
merge counters in a fixed device array inside the library.  Called through the C ABI with ctypes;
its output must match the CPU oracle within the parity tolerance, on two calls in a row, with the
persistent tensor-core kernel (G = 4, equal lengths) and the CUDA-core split engine (G = 8, ragged
lengths, or asked for).  This file sorts last so a run that stops at the first failure has already
run every other test."""
import ctypes
import math

import pytest
import torch

import oracle
import long_context_decode_kv1b_b200 as kv
from parity_utils import HostKV, assert_rows_close, oracle_attend_all

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


@pytest.mark.parametrize("G,appends", [(4, [6000]), (8, [3000]), (4, [2500, 1])])
def test_noalloc_matches_the_oracle_on_two_calls_in_a_row(G, appends):
    dev = "cuda"
    g = torch.Generator(device=dev).manual_seed(31 + G)
    B, Hkv = 2, 4
    total = sum(appends)
    cache = kv.Cache(B, Hkv, (total + 127) // 128 * 128, seed=3)
    host = HostKV(B, Hkv, cache.capacity)
    for n in appends:
        K = torch.randn((B, n, Hkv, 128), generator=g, device=dev).to(torch.bfloat16)
        V = torch.randn((B, n, Hkv, 128), generator=g, device=dev).to(torch.bfloat16)
        cache.append(K, V)
        host.add(K, V)
    scale = 1.0 / math.sqrt(128)
    D = oracle.signs(3)
    for call in range(2):
        q = torch.randn((B, Hkv * G, 128), generator=g, device=dev).to(torch.bfloat16)
        ref = oracle_attend_all(host, q, D, scale, G)
        for engine in (kv.ATTEND_TENSOR, kv.ATTEND_CUDA_CORE):
            rc, out = call_noalloc(cache, q, scale, engine=engine)
            assert rc == 0, f"call {call}: {kv.lib().kv1b_status_string(rc)}"
            torch.cuda.synchronize()
            assert_rows_close(out.cpu().numpy(), ref, where=f"noalloc G{G} engine {engine} call {call}")
    assert cache.status() == 0


def test_noalloc_refuses_shapes_beyond_its_scratch():
    # 64 sequences x 128 query heads x 520 bytes of partials > the 4 MiB array even unsplit
    cache = kv.Cache(64, 16, 128, seed=0)
    q = torch.zeros((64, 128, 128), dtype=torch.float32, device="cuda")
    assert 64 * 128 * 520 > SCRATCH_BYTES
    rc, out = call_noalloc(cache, q, 0.1, engine=kv.ATTEND_CUDA_CORE)
    assert rc == -5
    torch.cuda.synchronize()
    assert torch.isnan(out).all()  # nothing was launched or written
