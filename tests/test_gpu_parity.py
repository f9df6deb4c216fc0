"""GPU parity: every step of the CUDA path, called through the C ABI, against the CPU oracle.

Bit-exact: key bits, N, 1/C, value codes, fp16 scale/min, query planes and grid, popcount
integers, logits, Top-p index sets.  Attention outputs: <= 1e-3 relative per row (max and l2).
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle
import long_context_decode_kv1b_b200 as kv
from parity_utils import (L2E, HostKV, assert_planes_equal, assert_rows_close, check_probe_row, gpu_head_planes,
                          oracle_attend_all, to_np32)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def rand_kv(g, B, n, H, dtype, scale=1.0):
    K = (torch.randn((B, n, H, 128), generator=g, device=DEV) * scale).to(dtype)
    V = (torch.randn((B, n, H, 128), generator=g, device=DEV) * scale).to(dtype)
    return K, V


def build_cache(B, Hkv, appends, dtype, seed=0, data_seed=1, vscale=1.0, cap=None, rounds=1):
    total = sum(appends)
    cap = cap or (total + 127) // 128 * 128
    cache = kv.Cache(B, Hkv, cap, seed=seed, rounds=rounds)
    host = HostKV(B, Hkv, cap)
    g = torch.Generator(device=DEV).manual_seed(data_seed)
    for n in appends:
        K, V = rand_kv(g, B, n, Hkv, dtype)
        V = (V.float() * vscale).to(dtype)
        cache.append(K, V)
        host.add(K, V)
    return cache, host


# ------------------------------------------------------------------------------------- encode
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
def test_encode_bit_exact_ragged_appends(dtype):
    B, H = 2, 3
    appends = [37, 1, 16, 5, 70]
    cache, host = build_cache(B, H, appends, dtype, seed=123)
    torch.cuda.synchronize()
    D = oracle.signs(123)
    assert np.array_equal(cache.planes()["signs"].cpu().numpy(), D)
    assert cache.lengths == [sum(appends)] * B
    assert cache.planes()["lengths"].cpu().tolist() == [sum(appends)] * B
    for b in range(B):
        for h in range(H):
            assert_planes_equal(gpu_head_planes(cache, b, h, host.n), host.encode(b, h, D), f"b{b} h{h}")
    assert cache.status() == 0


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
def test_prefill_encode_bit_exact_ragged_groups(dtype):
    # appends of >= 64 tokens take the prefill form (one warp per 8-token code word): starts and ends
    # inside an 8-token group and inside a 128-token tile, whole tiles, single tokens in between
    B, H = 2, 3
    appends = [100, 200, 64, 1, 65, 300, 7, 129]
    cache, host = build_cache(B, H, appends, dtype, seed=321, data_seed=4)
    torch.cuda.synchronize()
    D = oracle.signs(321)
    assert cache.lengths == [sum(appends)] * B
    for b in range(B):
        for h in range(H):
            assert_planes_equal(gpu_head_planes(cache, b, h, host.n), host.encode(b, h, D), f"prefill b{b} h{h}")
    assert cache.status() == 0


def test_prefill_encode_strided_rows_and_special_values():
    B, H, n = 2, 2, 200
    g = torch.Generator(device=DEV).manual_seed(15)
    wide = torch.randn((B, n, H, 2, 128), generator=g, device=DEV)
    wide[0, 3, 0, 0, :] = 0.0                     # zero key: every sign bit 1, cinv = 1
    wide[1, 77, 1, 0, 5:40] = 0.0                 # exact zeros inside a key
    wide[0, 9, 1, 1, :] = 0.25                    # a constant (binary16-exact) value row
    wide[1, 150, 0, 1, 32:64] = -3.0e4            # large but representable
    K, V = wide[:, :, :, 0, :], wide[:, :, :, 1, :]  # token stride 512, head stride 256 elements
    cache = kv.Cache(B, H, 256, seed=99)
    cache.append(K[:, :5], V[:, :5])                  # decode form first, then prefill from mid-group
    cache.append(K[:, 5:], V[:, 5:])
    host = HostKV(B, H, 256)
    host.add(K, V)
    D = oracle.signs(99)
    for b in range(B):
        for h in range(H):
            assert_planes_equal(gpu_head_planes(cache, b, h, n), host.encode(b, h, D), f"strided prefill b{b} h{h}")
    assert cache.status() == 0
    V2 = V[:, :80].clone()
    V2[1, 70, 0, 3] = float("nan")
    cache2 = kv.Cache(B, H, 128, seed=1)
    cache2.append(K[:, :80].contiguous(), V2.contiguous())
    assert cache2.status() & kv.STATUS_NONFINITE


def edge_value_rows(n: int, seed: int) -> torch.Tensor:
    """[n, 128] fp32 rows whose first 32-channel group is a scale-search edge case, cycling through:
    a range D = fl64(max - min) that fp64 rounds (min = -15 * 2^-24, max = 2^-140), a range of exactly
    15 h (h = 0.5 and a subnormal binary16), the saturation boundary 15 * 65504 and just above it, a
    constant group, and a range of one subnormal binary16 step; the other groups are random."""
    g = torch.Generator().manual_seed(seed)
    rows = torch.randn((n, 128), generator=g)
    cases = [(-15 * 2.0 ** -24, 2.0 ** -140), (0.0, 7.5), (0.0, 15 * 3 * 2.0 ** -24), (0.0, 982560.0),
             (0.0, 982560.0625), (1.25, 1.25), (-2.0 ** -24, 0.0), (-3.0, 2.0 ** -149)]
    for i in range(n):
        lo, hi = cases[i % len(cases)]
        grp = torch.full((32,), lo)
        grp[7] = hi
        rows[i, :32] = grp
    return rows


@pytest.mark.parametrize("n", [5, 100])
def test_value_scale_search_edge_groups(n):
    # n = 5 takes the decode form of the encode, n = 100 the prefill form
    B, H = 1, 2
    V = torch.stack([edge_value_rows(n, 1), edge_value_rows(n, 2)], dim=1).view(B, n, H, 128).to(DEV)
    K = torch.randn((B, n, H, 128), device=DEV, generator=torch.Generator(device=DEV).manual_seed(3))
    cache = kv.Cache(B, H, 128, seed=5)
    cache.append(K, V)
    host = HostKV(B, H, 128)
    host.add(K, V)
    D = oracle.signs(5)
    for h in range(H):
        assert_planes_equal(gpu_head_planes(cache, 0, h, n), host.encode(0, h, D), f"scale edges n{n} h{h}")
    assert cache.status() & kv.STATUS_FP16_SATURATED  # the group just above 15 * 65504


def test_encode_strided_inputs_and_special_values():
    B, H, n = 1, 2, 48
    g = torch.Generator(device=DEV).manual_seed(5)
    big = torch.randn((B, n, H, 256), generator=g, device=DEV)  # padded last dim -> strided view
    K = big[..., :128].clone()
    K[0, 3, 0, :] = 0.0                       # zero key: every sign bit 1, cinv = 1
    K[0, 4, 1, 10:20] = 0.0                   # exact zeros inside a key
    Vb = big.clone()
    Vb[0, 5, 0, :128] = 0.25                  # constant (binary16-exact) group values
    Vb[0, 6, 1, 0:32] = 3.0e4                 # large but representable
    K = K.contiguous()
    V = Vb[..., :128]                         # non-contiguous view, unit channel stride
    Kb = torch.empty_like(Vb)
    Kb[..., :128] = K
    Kv = Kb[..., :128]
    cache = kv.Cache(B, H, 128, seed=9)
    cache.append(Kv, V)
    host = HostKV(B, H, 128)
    host.add(Kv, V)
    D = oracle.signs(9)
    for h in range(H):
        assert_planes_equal(gpu_head_planes(cache, 0, h, n), host.encode(0, h, D), f"h{h}")
    assert cache.status() == 0


def test_encode_status_flags():
    cache = kv.Cache(1, 1, 128, seed=0)
    K = torch.zeros((1, 1, 1, 128), device=DEV)
    V = torch.zeros((1, 1, 1, 128), device=DEV)
    V[0, 0, 0, 5] = 1e7                       # beyond min + 15 * 65504: saturation
    cache.append(K, V)
    assert cache.status() & kv.STATUS_FP16_SATURATED
    V2 = torch.zeros_like(V)
    V2[0, 0, 0, 7] = float("nan")
    cache.append(K, V2)
    assert cache.status() & kv.STATUS_NONFINITE


def test_capacity_and_argument_errors():
    cache = kv.Cache(1, 1, 128, seed=0)
    K = torch.zeros((1, 100, 1, 128), device=DEV)
    cache.append(K, K)
    with pytest.raises(kv.Kv1bError) as e:
        cache.append(K, K)
    assert e.value.code == -3
    assert cache.lengths == [100]
    q = torch.zeros((1, 3, 128), device=DEV)   # 3 % 1 == 0 but G = 3 fine; 9 heads -> G 9 > 8
    with pytest.raises(kv.Kv1bError):
        cache.attend(torch.zeros((1, 9, 128), device=DEV), 0.1)
    with pytest.raises(kv.Kv1bError):
        cache.attend_topp(q, 0.1, 0.0)
    with pytest.raises(kv.Kv1bError):
        cache.attend_topp(q, 0.1, 1.5)


# ------------------------------------------------------------------------------------- query / scores
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_query_prep_and_scores_bit_exact(dtype):
    B, Hkv, G = 2, 3, 2
    cache, host = build_cache(B, Hkv, [300], dtype, seed=77)
    g = torch.Generator(device=DEV).manual_seed(3)
    q = (torch.randn((B, Hkv * G, 128), generator=g, device=DEV) * 2.0).to(dtype)
    q[0, 1] = 0.0                                # flat query: delta = 0, all codes 0
    qp = cache.query_prep(q)
    sc = cache.scores(q, 0.125)
    torch.cuda.synchronize()
    D = oracle.signs(77)
    qn = to_np32(q)
    for b in range(B):
        for hq in range(Hkv * G):
            r = oracle.query_prep(qn[b, hq], D)
            assert np.array_equal(qp["planes"][b, hq].cpu().numpy().view(np.uint32), r["planes"])
            assert qp["vl"][b, hq].item() == r["vl"] and qp["delta"][b, hq].item() == r["delta"]
            assert qp["Sq"][b, hq].item() == r["Sq"]
            enc = host.encode(b, hq // G, D)
            A, Bc = oracle.score_ints(enc["bits"], r["planes"])
            s = oracle.logits(enc, r, 0.125)
            assert np.array_equal(sc["A"][b, hq, :300].cpu().numpy(), A)
            assert np.array_equal(sc["Bc"][b, hq, :300].cpu().numpy(), Bc)
            assert np.array_equal(sc["s"][b, hq, :300].cpu().numpy().view(np.uint32), s.view(np.uint32))


# ------------------------------------------------------------------------------------- attend
@pytest.mark.parametrize("G", [1, 2, 3, 4, 5, 6, 8])
@pytest.mark.parametrize("engine", [kv.ATTEND_TENSOR, kv.ATTEND_CUDA_CORE])
def test_attend_parity_group_sizes(G, engine):
    # the persistent engine serves G > 4 as launches of at most 4 query heads (G = 3, 5, 6: a launch
    # with absent head slots)
    B, Hkv = 2, 2
    cache, host = build_cache(B, Hkv, [700, 3], torch.bfloat16, seed=5, data_seed=G)
    g = torch.Generator(device=DEV).manual_seed(100 + G)
    q = torch.randn((B, Hkv * G, 128), generator=g, device=DEV).to(torch.bfloat16)
    out = cache.attend(q, 1 / math.sqrt(128), engine=engine)
    ref = oracle_attend_all(host, q, oracle.signs(5), 1 / math.sqrt(128), G)
    assert_rows_close(out.cpu().numpy(), ref, where=f"G{G} e{engine}")
    assert cache.status() == 0


@pytest.mark.parametrize("L", [1, 15, 16, 17, 255, 256, 257, 1000, 4099])
@pytest.mark.parametrize("splits", [0, 1, 3, 7])
def test_attend_parity_lengths_and_splits(L, splits):
    B, Hkv, G = 1, 2, 4
    cache, host = build_cache(B, Hkv, [L], torch.float32, seed=11, data_seed=L)
    g = torch.Generator(device=DEV).manual_seed(L)
    q = torch.randn((B, Hkv * G, 128), generator=g, device=DEV)
    ref = oracle_attend_all(host, q, oracle.signs(11), 0.2, G)
    for engine in (kv.ATTEND_TENSOR, kv.ATTEND_CUDA_CORE):
        out = cache.attend(q, 0.2, engine=engine, num_splits=splits)
        assert_rows_close(out.cpu().numpy(), ref, where=f"L{L} s{splits} e{engine}")
    assert cache.status() == 0


def test_attend_empty_cache_gives_zeros():
    cache = kv.Cache(2, 2, 128, seed=0)
    q = torch.randn((2, 8, 128), device=DEV)
    for engine in (kv.ATTEND_TENSOR, kv.ATTEND_CUDA_CORE):
        assert torch.count_nonzero(cache.attend(q, 0.1, engine=engine)).item() == 0
    out, sel, cnt = cache.attend_topp(q, 0.1, 0.9)
    assert torch.count_nonzero(out).item() == 0 and torch.count_nonzero(cnt).item() == 0


@pytest.mark.parametrize("vscale", [1e-4, 1e-2, 30.0, 1e3])
def test_attend_value_magnitudes(vscale):
    B, Hkv, G = 1, 1, 4
    cache, host = build_cache(B, Hkv, [2000], torch.float32, seed=3, data_seed=7, vscale=vscale)
    q = torch.randn((B, G, 128), device=DEV, generator=torch.Generator(device=DEV).manual_seed(1))
    ref = oracle_attend_all(host, q, oracle.signs(3), 0.09, G)
    for engine in (kv.ATTEND_TENSOR, kv.ATTEND_CUDA_CORE):
        assert_rows_close(cache.attend(q, 0.09, engine=engine).cpu().numpy(), ref, where=f"v{vscale} e{engine}")


def test_attend_peaked_softmax():
    # a large softmax scale concentrates the mass on a few tokens (online rescaling exercised)
    B, Hkv, G = 1, 2, 4
    cache, host = build_cache(B, Hkv, [3000], torch.float32, seed=8, data_seed=2)
    q = torch.randn((B, Hkv * G, 128), device=DEV, generator=torch.Generator(device=DEV).manual_seed(4))
    ref = oracle_attend_all(host, q, oracle.signs(8), 3.0, G)
    for engine in (kv.ATTEND_TENSOR, kv.ATTEND_CUDA_CORE):
        for splits in (0, 5):
            out = cache.attend(q, 3.0, engine=engine, num_splits=splits)
            assert_rows_close(out.cpu().numpy(), ref, where=f"peaked e{engine} s{splits}")


def test_attend_deterministic_reruns():
    cache, host = build_cache(1, 2, [5000], torch.bfloat16, seed=1)
    q = torch.randn((1, 8, 128), device=DEV).to(torch.bfloat16)
    a = cache.attend(q, 0.1).clone()
    b = cache.attend(q, 0.1)
    assert torch.equal(a, b)


def test_attend_workspace_counters_left_clean():
    # a workspace with garbage merge counters: the first call (no flag) zeroes them; every call
    # leaves them zero, so later calls may pass KV1B_ATTEND_WS_CLEAN and skip the zeroing
    B, Hkv, G = 2, 2, 4
    cache, host = build_cache(B, Hkv, [2000, 77], torch.bfloat16, seed=6, data_seed=3)
    q = torch.randn((B, Hkv * G, 128), device=DEV, generator=torch.Generator(device=DEV).manual_seed(9))
    ref = oracle_attend_all(host, q, oracle.signs(6), 0.09, G)
    L = kv.lib()
    n = L.kv1b_attend_workspace_bytes(ctypes.byref(cache.desc), Hkv * G, 0)
    ws = torch.full((n,), 0xA5, dtype=torch.uint8, device=DEV)
    outs = []
    for flags in (kv.ATTEND_TENSOR, kv.ATTEND_TENSOR | kv.ATTEND_WS_CLEAN, kv.ATTEND_TENSOR | kv.ATTEND_WS_CLEAN,
                  kv.ATTEND_CUDA_CORE | kv.ATTEND_WS_CLEAN, kv.ATTEND_TENSOR | kv.ATTEND_WS_CLEAN):
        out = torch.empty((B, Hkv * G, 128), dtype=torch.float32, device=DEV)
        rc = L.kv1b_attend(ctypes.byref(cache.desc), ctypes.c_void_p(q.data_ptr()), kv.DTYPE_F32, Hkv * G,
                           ctypes.c_float(0.09), ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(ws.data_ptr()), n,
                           flags, 0, None)
        assert rc == 0
        assert_rows_close(out.cpu().numpy(), ref, where=f"flags {flags}")
        outs.append(out)
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2]) and torch.equal(outs[0], outs[4])
    assert cache.status() == 0


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_decode_step_from_one_pinned_block(dtype):
    # a decode step whose new K/V and query come in one pinned host block (one copy in) against the
    # same step from device tensors, on two caches built alike; and against the oracle
    B, Hkv, G = 2, 2, 4
    c1, host = build_cache(B, Hkv, [900], dtype, seed=12, data_seed=2, cap=1024)
    c2, _ = build_cache(B, Hkv, [900], dtype, seed=12, data_seed=2, cap=1024)
    g = torch.Generator(device=DEV).manual_seed(77)
    k, v = rand_kv(g, B, 1, Hkv, dtype)
    q = torch.randn((B, Hkv * G, 128), generator=g, device=DEV).to(dtype)
    nblk = kv.step_block_bytes(B, Hkv, Hkv * G, dtype)
    hb = torch.empty(nblk, dtype=torch.uint8).pin_memory()
    hk, hv, hq = kv.step_block_views(hb, B, Hkv, Hkv * G, dtype)
    hk.copy_(k.cpu()), hv.copy_(v.cpu()), hq.copy_(q.cpu())
    db = torch.empty(nblk, dtype=torch.uint8, device=DEV)
    outh = torch.empty((B, Hkv * G, 128), dtype=torch.float32).pin_memory()
    kv.attend_from_host_block(c1, hb, db, Hkv * G, dtype, 0.2, outh)
    c2.append(k, v)
    ref_dev = c2.attend(q, 0.2)
    torch.cuda.synchronize()
    assert torch.equal(outh, ref_dev.cpu())
    host.add(k, v)
    ref = oracle_attend_all(host, q, oracle.signs(12), 0.2, G)
    assert_rows_close(outh.numpy(), ref, where="one-block step")
    assert c1.status() == 0


# ------------------------------------------------------------------------------------- Top-p
def topp_check(cache, host, q, scale, p, G, signs, rows=None):
    out, sel, cnt = cache.attend_topp(q, scale, p)
    torch.cuda.synchronize()
    qn = to_np32(q)
    B, Hq, _ = qn.shape
    encs = {}
    for b in range(B):
        for hq in range(Hq):
            if rows is not None and (b, hq) not in rows:
                continue
            kvh = hq // G
            if (b, kvh) not in encs:
                encs[(b, kvh)] = host.encode(b, kvh, signs)
            rs, ro = oracle.attend_topp(encs[(b, kvh)], qn[b, hq], signs, scale, p)
            n = cnt[b, hq].item()
            assert n == len(rs), f"b{b} hq{hq}: count {n} vs {len(rs)}"
            assert np.array_equal(sel[b, hq, :n].cpu().numpy(), rs), f"b{b} hq{hq}: index sets differ"
            assert_rows_close(out[b, hq].cpu().numpy(), ro, where=f"topp b{b} hq{hq}")
    return cnt


@pytest.mark.parametrize("p", [0.05, 0.5, 0.9, 0.999, 1.0])
def test_topp_parity(p):
    B, Hkv, G = 2, 2, 2
    cache, host = build_cache(B, Hkv, [1500, 37], torch.bfloat16, seed=21, data_seed=3)
    q = torch.randn((B, Hkv * G, 128), device=DEV, generator=torch.Generator(device=DEV).manual_seed(9))
    q = q.to(torch.bfloat16)
    topp_check(cache, host, q, 0.5, p, G, oracle.signs(21))


def test_topp_ties_take_lowest_indices():
    # many identical keys -> identical logits; the selection must take them in index order
    B, Hkv, G, L = 1, 1, 1, 600
    cache = kv.Cache(B, Hkv, 640, seed=4)
    host = HostKV(B, Hkv, 640)
    g = torch.Generator(device=DEV).manual_seed(0)
    K = torch.randn((B, L, Hkv, 128), generator=g, device=DEV)
    K[:, 100:500] = K[:, 50:51]                # 401 equal keys (positions 50 and 100..499)
    V = torch.randn((B, L, Hkv, 128), generator=g, device=DEV)
    cache.append(K, V)
    host.add(K, V)
    q = K[:, 50, :, :].clone().view(B, 1, 128) * 0.3
    for p in (0.3, 0.6, 0.95):
        topp_check(cache, host, q, 0.3, p, G, oracle.signs(4))


@pytest.mark.parametrize("scale", [0.005, 0.5, 4.0])
def test_topp_multi_chunk_ragged(scale):
    # 9097 tokens in two appends: several 4096-token chunks and a ragged tail; a tiny scale puts
    # nearly every token in the threshold bucket, a large one leaves most tokens massless
    B, Hkv, G = 2, 1, 4
    cache, host = build_cache(B, Hkv, [5000, 4097], torch.bfloat16, seed=5, data_seed=6)
    q = torch.randn((B, Hkv * G, 128), device=DEV, generator=torch.Generator(device=DEV).manual_seed(2))
    q = q.to(torch.bfloat16)
    for p in (0.5, 0.99):
        topp_check(cache, host, q, scale, p, G, oracle.signs(5))


@pytest.mark.parametrize("G,qdt", [(1, torch.float32), (3, torch.float16), (8, torch.bfloat16)])
def test_topp_group_sizes(G, qdt):
    # one, a non-power-of-two and the largest number of query heads per kv-head (two operand groups)
    B, Hkv = 1, 2
    cache, host = build_cache(B, Hkv, [4500], torch.bfloat16, seed=13, data_seed=8)
    q = torch.randn((B, Hkv * G, 128), device=DEV, generator=torch.Generator(device=DEV).manual_seed(5)).to(qdt)
    for p in (0.3, 0.95):
        topp_check(cache, host, q, 0.4, p, G, oracle.signs(13))


@pytest.mark.parametrize("G", [4, 8])
def test_topp_flat_and_peaked_sequences(G):
    # one call over two very different selections: sequence 0 has flat attention (a large share of
    # the tokens is needed to reach p), sequence 1 a few planted tokens that carry the mass
    B, Hkv, L = 2, 2, 6000
    cap = (L + 127) // 128 * 128
    cache = kv.Cache(B, Hkv, cap, seed=17)
    host = HostKV(B, Hkv, cap)
    g = torch.Generator(device=DEV).manual_seed(31)
    K = torch.randn((B, L, Hkv, 128), generator=g, device=DEV)
    V = torch.randn((B, L, Hkv, 128), generator=g, device=DEV)
    dirs = torch.nn.functional.normalize(torch.randn((Hkv, 128), generator=g, device=DEV), dim=-1)
    heavy = torch.randperm(L, generator=g, device=DEV)[:12]
    for h in range(Hkv):
        K[1, heavy, h, :] = 6.0 * math.sqrt(128.0) * dirs[h] + 0.1 * torch.randn((12, 128), generator=g, device=DEV)
    K, V = K.to(torch.bfloat16), V.to(torch.bfloat16)
    cache.append(K, V)
    host.add(K, V)
    q = torch.randn((B, Hkv * G, 128), generator=g, device=DEV)
    for h in range(Hkv):
        q[1, h * G:(h + 1) * G] = 4.0 * dirs[h] + 0.3 * torch.randn((G, 128), generator=g, device=DEV)
    for p in (0.6, 0.9):
        cnt = topp_check(cache, host, q, 0.05, p, G, oracle.signs(17))  # sequence 0: logits of std ~0.6
        assert int(cnt[0].min().item()) > L // 10, f"p {p}: flat rows select {cnt[0].tolist()}"
        assert int(cnt[1].max().item()) <= 12, f"p {p}: peaked rows select {cnt[1].tolist()}"
    assert cache.status() == 0


# ------------------------------------------------------------------ exact attention over a selected set
def cache_with_exact(B, Hkv, L, dtype, seed, data_seed):
    """A compressed cache plus the exact keys / values it was built from ([B, L, Hkv, 128] on the GPU)."""
    cap = (L + 127) // 128 * 128
    cache = kv.Cache(B, Hkv, cap, seed=seed)
    g = torch.Generator(device=DEV).manual_seed(data_seed)
    K, V = rand_kv(g, B, L, Hkv, dtype)
    cache.append(K, V)
    return cache, K, V


def exact_check(cache, q, scale, K, V, sel, cnt, G, where=""):
    out = cache.attend_selected_exact(q, scale, K, V, sel, cnt)
    torch.cuda.synchronize()
    qn, Kn, Vn = to_np32(q), to_np32(K), to_np32(V)
    B, Hq, _ = qn.shape
    L = min(cache.lengths[0], K.shape[1])
    for b in range(B):
        for hq in range(Hq):
            n = int(cnt[b, hq].item())
            s = sel[b, hq, :n].cpu().numpy().astype(np.int64)
            s = s[(s >= 0) & (s < L)]  # out-of-range entries are skipped
            ref = oracle.attend_exact_selected(qn[b, hq], Kn[b, :, hq // G], Vn[b, :, hq // G], s, scale)
            if s.size == 0:
                assert torch.count_nonzero(out[b, hq]).item() == 0, f"{where} b{b} hq{hq}: empty set"
            else:
                assert_rows_close(out[b, hq].cpu().numpy(), ref, where=f"{where} b{b} hq{hq}")
    return out


@pytest.mark.parametrize("p", [0.5, 0.95])
def test_exact_over_topp_selection(p):
    B, Hkv, G, L = 2, 2, 4, 5000
    cache, K, V = cache_with_exact(B, Hkv, L, torch.bfloat16, seed=31, data_seed=4)
    q = torch.randn((B, Hkv * G, 128), device=DEV, generator=torch.Generator(device=DEV).manual_seed(6))
    q = q.to(torch.bfloat16)
    _, sel, cnt = cache.attend_topp(q, 0.3, p)
    exact_check(cache, q, 0.3, K, V, sel, cnt, G, where=f"p{p}")
    assert cache.status() == 0


def test_exact_hand_made_sets_and_bad_indices():
    B, Hkv, G, L = 1, 1, 4, 700
    cache, K, V = cache_with_exact(B, Hkv, L, torch.bfloat16, seed=2, data_seed=9)
    cap = cache.capacity
    q = torch.randn((B, G, 128), device=DEV, generator=torch.Generator(device=DEV).manual_seed(1))
    sel = torch.zeros((B, G, cap), dtype=torch.int32, device=DEV)
    cnt = torch.zeros((B, G), dtype=torch.int32, device=DEV)
    # head 0: empty; head 1: one token; head 2: every token; head 3: random subset
    sel[0, 1, 0] = 345
    cnt[0, 1] = 1
    sel[0, 2, :L] = torch.arange(L, dtype=torch.int32, device=DEV)
    cnt[0, 2] = L
    sub = torch.randperm(L, generator=torch.Generator().manual_seed(3))[:123].sort().values.to(torch.int32)
    sel[0, 3, :123] = sub.to(DEV)
    cnt[0, 3] = 123
    exact_check(cache, q, 0.2, K, V, sel, cnt, G, where="hand")
    assert cache.status() == 0
    # indices past the sequence are skipped and flagged
    sel[0, 1, 1] = L + 5
    sel[0, 1, 2] = -3
    cnt[0, 1] = 3
    exact_check(cache, q, 0.2, K, V, sel, cnt, G, where="bad")
    assert cache.status() & 8


@pytest.mark.parametrize("dtype", [torch.float32, torch.float16])
def test_exact_kv_dtypes_and_strides(dtype):
    # keys / values as column slices of wider rows (token stride 2 x 2 x 128 elements, head stride 256)
    B, Hkv, G, L = 2, 2, 2, 1800
    cap = (L + 127) // 128 * 128
    cache = kv.Cache(B, Hkv, cap, seed=5)
    g = torch.Generator(device=DEV).manual_seed(12)
    wide = torch.randn((B, L, Hkv, 2, 128), generator=g, device=DEV).to(dtype)
    K, V = wide[:, :, :, 0, :], wide[:, :, :, 1, :]  # equal strides (L: 512, head: 256, channel: 1)
    Kc, Vc = K.contiguous(), V.contiguous()
    cache.append(Kc, Vc)
    q = torch.randn((B, Hkv * G, 128), device=DEV, generator=torch.Generator(device=DEV).manual_seed(2))
    _, sel, cnt = cache.attend_topp(q, 0.25, 0.8)
    exact_check(cache, q, 0.25, K, V, sel, cnt, G, where=f"{dtype} strided")
    exact_check(cache, q, 0.25, Kc, Vc, sel, cnt, G, where=f"{dtype} contiguous")


def device_address_of_host(t: torch.Tensor) -> int:
    """The device address of pinned host memory (0 when the device cannot address it)."""
    from cuda.bindings import runtime as rt

    err, attr = rt.cudaPointerGetAttributes(t.data_ptr())
    if err != rt.cudaError_t.cudaSuccess or attr.type != rt.cudaMemoryType.cudaMemoryTypeHost:
        return 0
    return int(attr.devicePointer)


def test_exact_kv_from_pinned_host_memory():
    # the exact keys / values stay in host memory (RaBitQCache, core idea: full-precision KV kept off
    # the GPU); the kernel reads the selected rows through the device's mapping of pinned memory
    B, Hkv, G, L = 2, 2, 4, 3000
    cache, K, V = cache_with_exact(B, Hkv, L, torch.bfloat16, seed=44, data_seed=8)
    q = torch.randn((B, Hkv * G, 128), device=DEV, generator=torch.Generator(device=DEV).manual_seed(12))
    _, sel, cnt = cache.attend_topp(q, 0.3, 0.9)
    Kh = torch.empty(K.shape, dtype=K.dtype, pin_memory=True)
    Vh = torch.empty(V.shape, dtype=V.dtype, pin_memory=True)
    Kh.copy_(K)
    Vh.copy_(V)
    torch.cuda.synchronize()
    for t in (Kh, Vh):
        if device_address_of_host(t) != t.data_ptr():
            pytest.skip("pinned host memory is not addressable at its host address on this device")
    out_dev = cache.attend_selected_exact(q, 0.3, K, V, sel, cnt)
    out_host = exact_check(cache, q, 0.3, Kh, Vh, sel, cnt, G, where="host KV")
    assert torch.allclose(out_host, out_dev, rtol=0, atol=0)  # the same arithmetic on the same rows
    assert cache.status() == 0


# ------------------------------------------------------------------ Top-k budget and the kept window
def select_check(cache, host, q, scale, G, signs, mode, p=1.0, k=0, sink=0, recent=0, where=""):
    out, sel, cnt = cache.attend_select(q, scale, mode, p=p, k=k, sink=sink, recent=recent)
    torch.cuda.synchronize()
    qn = to_np32(q)
    B, Hq, _ = qn.shape
    encs = {}
    for b in range(B):
        for hq in range(Hq):
            kvh = hq // G
            if (b, kvh) not in encs:
                encs[(b, kvh)] = host.encode(b, kvh, signs)
            rs, ro = oracle.attend_select(encs[(b, kvh)], qn[b, hq], signs, scale, mode, p=p, k=k, sink=sink,
                                          recent=recent)
            n = cnt[b, hq].item()
            assert n == len(rs), f"{where} b{b} hq{hq}: count {n} vs {len(rs)}"
            assert np.array_equal(sel[b, hq, :n].cpu().numpy(), rs), f"{where} b{b} hq{hq}: index sets differ"
            assert_rows_close(out[b, hq].cpu().numpy(), ro, where=f"{where} b{b} hq{hq}")
    return cnt


@pytest.mark.parametrize("k", [0, 1, 37, 5000, 9999])
def test_topk_parity(k):
    # 5097 tokens over two chunks and a ragged tail; k = 0 and k above the length included
    B, Hkv, G = 1, 2, 4
    cache, host = build_cache(B, Hkv, [5000, 97], torch.bfloat16, seed=17, data_seed=4)
    q = torch.randn((B, Hkv * G, 128), device=DEV, generator=torch.Generator(device=DEV).manual_seed(8))
    cnt = select_check(cache, host, q.to(torch.bfloat16), 0.4, G, oracle.signs(17), kv.SELECT_TOPK, k=k,
                       where=f"k{k}")
    assert torch.all(cnt == min(k, 5097)).item()


@pytest.mark.parametrize("mode,p,k", [(0, 0.5, 0), (0, 0.99, 0), (1, 0, 20)])
@pytest.mark.parametrize("sink,recent", [(4, 0), (0, 64), (16, 300), (3000, 3000)])
def test_select_with_kept_window(mode, p, k, sink, recent):
    B, Hkv, G = 2, 1, 2
    cache, host = build_cache(B, Hkv, [4200], torch.bfloat16, seed=23, data_seed=5)
    q = torch.randn((B, Hkv * G, 128), device=DEV, generator=torch.Generator(device=DEV).manual_seed(3))
    select_check(cache, host, q, 0.5, G, oracle.signs(23), mode, p=p, k=k, sink=sink, recent=recent,
                 where=f"m{mode} s{sink} r{recent}")


def test_topk_ties_take_lowest_indices():
    B, Hkv, G, L = 1, 1, 1, 600
    cache = kv.Cache(B, Hkv, 640, seed=4)
    host = HostKV(B, Hkv, 640)
    g = torch.Generator(device=DEV).manual_seed(0)
    K = torch.randn((B, L, Hkv, 128), generator=g, device=DEV)
    K[:, 100:500] = K[:, 50:51]  # 401 equal keys -> equal logits
    V = torch.randn((B, L, Hkv, 128), generator=g, device=DEV)
    cache.append(K, V)
    host.add(K, V)
    q = K[:, 50, :, :].clone().view(B, 1, 128) * 0.3
    for k in (10, 200, 450):
        select_check(cache, host, q, 0.3, G, oracle.signs(4), kv.SELECT_TOPK, k=k, where=f"ties k{k}")


# ------------------------------------------------------------------ stronger rotation (3 rounds of H D)
def test_rotation_rounds_signs_plane():
    c1 = kv.Cache(1, 1, 128, seed=77)
    c3 = kv.Cache(1, 1, 128, seed=77, rounds=3)
    s1 = c1.planes()["signs_rounds"].cpu().numpy()
    s3 = c3.planes()["signs_rounds"].cpu().numpy()
    assert np.array_equal(s1[0], oracle.signs(77)) and np.count_nonzero(s1[1:]) == 0
    assert np.array_equal(s3.reshape(-1), oracle.signs(77, rounds=3))
    with pytest.raises(kv.Kv1bError):
        kv.Cache(1, 1, 128, seed=77, rounds=4)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_three_rounds_encode_bit_exact_and_attend(dtype):
    B, Hkv, G = 2, 2, 4
    cache, host = build_cache(B, Hkv, [700, 1, 33], dtype, seed=41, data_seed=2, rounds=3)
    D = oracle.signs(41, rounds=3)
    L = cache.lengths[0]
    for b in range(B):
        for h in range(Hkv):
            assert_planes_equal(gpu_head_planes(cache, b, h, L), host.encode(b, h, D), where=f"3 rounds b{b} h{h}")
    q = torch.randn((B, Hkv * G, 128), device=DEV, generator=torch.Generator(device=DEV).manual_seed(4)).to(dtype)
    ref = oracle_attend_all(host, q, D, 0.3, G)
    for engine in (kv.ATTEND_TENSOR, kv.ATTEND_CUDA_CORE):
        assert_rows_close(cache.attend(q, 0.3, engine=engine).cpu().numpy(), ref, where=f"3 rounds e{engine}")
    topp_check(cache, host, q, 0.3, 0.9, G, D)
    assert cache.status() == 0


# ------------------------------------------------- score integers of the kernels kv1b_attend / kv1b_attend_topp run
def probe_check(cache, host, q, scale, G, signs, kernel, where=""):
    """Every (b, hq) row of a kv1b_scores_probe result against the oracle (check_probe_row)."""
    pr = cache.scores_probe(q, scale, kernel)
    torch.cuda.synchronize()
    qn = to_np32(q)
    B, Hq, _ = qn.shape
    encs = {}
    for b in range(B):
        for hq in range(Hq):
            kvh = hq // G
            if (b, kvh) not in encs:
                encs[(b, kvh)] = host.encode(b, kvh, signs)
            check_probe_row(pr, b, hq, encs[(b, kvh)], qn[b, hq], signs, scale, kernel, cache.lengths[b], where)
    return pr


@pytest.mark.parametrize("G", [1, 2, 3, 4, 8])
def test_attend_kernel_score_integers_bit_exact(G):
    # a tile-boundary length (4099 = 32 tiles + 3) and two sequences x two kv-heads
    B, Hkv = 2, 2
    cache, host = build_cache(B, Hkv, [4000, 99], torch.bfloat16, seed=19, data_seed=G)
    q = torch.randn((B, Hkv * G, 128), device=DEV, generator=torch.Generator(device=DEV).manual_seed(40 + G))
    pr = probe_check(cache, host, q, 0.3, G, oracle.signs(19), kv.PROBE_ATTEND, where=f"attend G{G}")
    # the probe runs the whole attend: its output is the default engine's
    ref = oracle_attend_all(host, q, oracle.signs(19), 0.3, G)
    assert_rows_close(pr["out"].cpu().numpy(), ref, where=f"probe out G{G}")
    assert cache.status() == 0


@pytest.mark.parametrize("G,L", [(1, 300), (3, 4099), (4, 9000), (8, 2049)])
def test_topp_score_pass_integers_and_logits_bit_exact(G, L):
    B, Hkv = 1, 2
    cache, host = build_cache(B, Hkv, [L], torch.float32, seed=29, data_seed=L)
    q = torch.randn((B, Hkv * G, 128), device=DEV, generator=torch.Generator(device=DEV).manual_seed(G))
    probe_check(cache, host, q, 0.2, G, oracle.signs(29), kv.PROBE_TOPP, where=f"topp G{G} L{L}")


def test_popc_probe_matches_kv1b_scores():
    B, Hkv, G = 1, 1, 4
    cache, host = build_cache(B, Hkv, [777], torch.bfloat16, seed=3, data_seed=3)
    q = torch.randn((B, Hkv * G, 128), device=DEV, generator=torch.Generator(device=DEV).manual_seed(1))
    pr = probe_check(cache, host, q, 0.1, G, oracle.signs(3), kv.PROBE_POPC, where="popc")
    sc = cache.scores(q, 0.1)
    for k in ("A", "Bc", "s"):
        assert torch.equal(pr[k][..., :777], sc[k][..., :777])


# ------------------------------------------------------------------ bounded pipeline waits of the persistent kernel
def test_attend_wait_runs_out_and_reports_timeout():
    # Each CTA's copy producer stops before its stage `stall` (70,000 tokens x 2 kv-heads = 1,094 tiles:
    # 7-8 tiles, i.e. 3 stages, per CTA): the consumers' wait (2 tries of at most 0.5 ms) runs out, the
    # kernel records KV1B_STATUS_TIMEOUT and returns; the next call, which zeroes the merge counters
    # again, matches the oracle.  A fresh cache per case: the status word keeps its bits.
    B, Hkv, G, L = 1, 2, 4, 70000
    for stall in (-1, 0, 1):
        cache, host = build_cache(B, Hkv, [L], torch.bfloat16, seed=14, data_seed=2)
        q = torch.randn((B, Hkv * G, 128), device=DEV, generator=torch.Generator(device=DEV).manual_seed(3))
        if stall == -1:
            ref = oracle_attend_all(host, q, oracle.signs(14), 0.2, G)
        out = cache.attend_wait_probe(q, 0.2, wait_tries=2, stall_stage=stall)
        torch.cuda.synchronize()
        if stall == -1:  # a short limit alone changes nothing
            assert_rows_close(out.cpu().numpy(), ref, where="short limit, no stall")
            assert cache.status() == 0
            continue
        assert cache.status() & kv.STATUS_TIMEOUT, f"stall at stage {stall}: no timeout reported"
        out = cache.attend(q, 0.2)  # the binding drops WS_CLEAN after a stalled run
        torch.cuda.synchronize()
        assert_rows_close(out.cpu().numpy(), ref, where=f"after a stall at stage {stall}")


# ------------------------------------------------------------------ a long tail far below one dominant token
def tail_cache(L: int, gap_lo: float, gap_hi: float, seed: int):
    """One kv-head, 4 query heads, L + 1 tokens.  Every key is a positive multiple a_t of one vector u,
    so all tokens share the sign bits and the estimated logit is linear in a_t; the dominant token
    (position 777, a = 1) sits gap_t log2 units above token t for the head-0 query q = u, with gap_t
    uniform in [gap_lo, gap_hi].  Tail values have mean +1, the dominant value mean -1, so the output
    depends directly on how much of the mass the tail carries."""
    g = torch.Generator(device=DEV).manual_seed(seed)
    u = torch.randn((128,), generator=g, device=DEV)
    n = L + 1
    cache = kv.Cache(1, 1, (n + 127) // 128 * 128, seed=seed)
    host = HostKV(1, 1, cache.capacity)
    # the logit of a key a * u at scale 1 (the oracle's estimate; the same sign bits for every a > 0)
    D = oracle.signs(seed)
    enc1 = oracle.encode(u.cpu().numpy()[None, :], np.zeros((1, 128), np.float32), D)
    s1 = float(oracle.logits(enc1, oracle.query_prep(u.cpu().numpy(), D), 1.0)[0])
    assert s1 > 0
    span = 40.0  # log2-unit logit of the dominant token: gap = (1 - a) * span
    scale = span / (s1 * L2E)
    a = 1.0 - (gap_lo + (gap_hi - gap_lo) * torch.rand((n,), generator=g, device=DEV)) / span
    a[777] = 1.0
    K = (a[:, None] * u[None, :]).view(1, n, 1, 128)
    V = torch.randn((1, n, 1, 128), generator=g, device=DEV) + 1.0
    V[0, 777] -= 2.0
    for t0 in range(0, n, 1 << 18):
        t1 = min(n, t0 + (1 << 18))
        cache.append(K[:, t0:t1].contiguous(), V[:, t0:t1].contiguous())
        host.add(K[:, t0:t1], V[:, t0:t1])
    q = torch.stack([u * f for f in (1.0, 1.05, 0.95, 1.1)]).view(1, 4, 128)
    return cache, host, q, scale, D


@pytest.mark.parametrize("gap_lo,gap_hi", [(20.0, 28.0), (26.6, 27.4)])
def test_attend_long_tail_below_a_dominant_token(gap_lo, gap_hi):
    # 2^20 tail tokens 2^-20 .. 2^-28 below the dominant one carry ~15 % of the mass (head 0); a tail
    # packed at 2^-27 carries ~0.7 %: with 32-bit fixed-point weights these are fractions of a unit,
    # which the dithered rounding keeps unbiased
    cache, host, q, scale, D = tail_cache(1 << 20, gap_lo, gap_hi, seed=61)
    ref = oracle_attend_all(host, q, D, scale, 4)
    enc = host.encode(0, 0, D)
    s = oracle.logits(enc, oracle.query_prep(q[0, 0].cpu().numpy(), D), scale).astype(np.float64)
    w = np.exp2((s - s.max()) * L2E)
    frac = (w.sum() - 1.0) / w.sum()
    assert (0.05 <= frac <= 0.30) if gap_lo < 25 else (0.003 <= frac <= 0.02), frac
    for engine in (kv.ATTEND_TENSOR, kv.ATTEND_CUDA_CORE):
        out = cache.attend(q, scale, engine=engine)
        assert_rows_close(out.cpu().numpy(), ref, where=f"tail {gap_lo}-{gap_hi} e{engine}")
    assert cache.status() == 0


# ------------------------------------------------------------------ a context split: partial rows + merge
@pytest.mark.parametrize("engine", [kv.ATTEND_TENSOR, kv.ATTEND_CUDA_CORE])
def test_context_split_partial_rows_merge_to_the_whole_attention(engine):
    # one sequence's 9,100 tokens in three caches (three ranks of a context split, emulated one after
    # another on this GPU) plus an empty fourth: each cache's log-sum-exp rows, merged by
    # kv1b_merge_partials, equal the oracle's attention over the whole context; every partial row
    # normalised equals the oracle's attention over its own range
    from long_context_decode_kv1b_b200 import context_split as cs

    B, Hkv, G, L, world = 2, 2, 4, 9100, 3
    g = torch.Generator(device=DEV).manual_seed(77)
    K = torch.randn((B, L, Hkv, 128), generator=g, device=DEV).to(torch.bfloat16)
    V = torch.randn((B, L, Hkv, 128), generator=g, device=DEV).to(torch.bfloat16)
    q = torch.randn((B, Hkv * G, 128), generator=g, device=DEV).to(torch.bfloat16)
    D = oracle.signs(8)
    parts, hosts = [], []
    for r in range(world + 1):
        t0, t1 = cs.shard_bounds(L, world, r) if r < world else (L, L)
        cap = max(128, (t1 - t0 + 127) // 128 * 128)
        cache = kv.Cache(B, Hkv, cap, seed=8)
        host = HostKV(B, Hkv, cap)
        if t1 > t0:
            cache.append(K[:, t0:t1].contiguous(), V[:, t0:t1].contiguous())
            host.add(K[:, t0:t1], V[:, t0:t1])
        parts.append(cache.attend(q, 0.3, engine=engine, partial=True))
        hosts.append(host)
    allp = torch.stack(parts)  # [world + 1, B, Hq, 130], the gathered rows
    out = kv.merge_partials(allp)
    torch.cuda.synchronize()
    whole = HostKV(B, Hkv, L)
    whole.add(K, V)
    ref = oracle_attend_all(whole, q, D, 0.3, G)
    assert_rows_close(out.cpu().numpy(), ref, where=f"split merge e{engine}")
    P = allp.cpu().numpy()
    assert np.all(P[world, :, :, 0] == -np.inf) and not P[world, :, :, 1:].any()  # the empty range
    for r in range(world):
        sub = oracle_attend_all(hosts[r], q, D, 0.3, G)
        assert_rows_close(P[r, :, :, 2:] / P[r, :, :, 1:2], sub, where=f"range {r} e{engine}")
