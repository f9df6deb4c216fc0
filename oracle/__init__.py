"""CPU oracle for decode attention over a 1-bit-key / 4-bit-value KV cache.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
``cpu_baseline`` / ``--impl reference`` arm may import this package.  The product path
(``long_context_decode_kv1b_b200``) never imports it, and it imports nothing from there.

The arithmetic lives in ``kv1b_oracle.cpp`` (plain C++, single thread); this module only
compiles it and marshals numpy arrays through ctypes.  Every function cites, in the C++ source,
the web page and section it follows (RaBitQCache; H1B-KV; the H1IB-KV news article).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kv1b_oracle.cpp")
_SO = os.path.join(_HERE, "libkv1b_oracle.so")
_lib = None

CFLAGS = ["-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC"]


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/libkv1b_oracle.so`` (g++, no fp contraction)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < max(
        os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "kv1b_oracle.h"))
    ):
        tmp = _SO + ".tmp.%d" % os.getpid()
        subprocess.check_call(["g++", *CFLAGS, "-o", tmp, _SRC])
        os.replace(tmp, _SO)
    return _SO


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        P = ctypes.c_void_p
        i32, i64, u64, f32 = ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_float
        sig = {
            "ref_splitmix64_next": (u64, [P]),
            "ref_rotation_signs": (None, [u64, ctypes.c_int, P]),
            "ref_rotation_signs_rounds": (None, [u64, ctypes.c_int, ctypes.c_int, P]),
            "ref_fwht": (None, [P, ctypes.c_int]),
            "ref_tree_sum": (f32, [P, ctypes.c_int]),
            "ref_encode_key": (None, [P, P, ctypes.c_int, P, P, P]),
            "ref_encode_value": (ctypes.c_int, [P, ctypes.c_int, P, P]),
            "ref_encode_keys": (None, [P, i64, P, ctypes.c_int, P, P, P]),
            "ref_encode_values": (ctypes.c_int, [P, i64, ctypes.c_int, P, P]),
            "ref_dequant_value": (None, [P, P, ctypes.c_int, P]),
            "ref_half_to_double": (ctypes.c_double, [ctypes.c_uint16]),
            "ref_query_prep": (None, [P, P, ctypes.c_int, P, P, P, P, P, P]),
            "ref_score_ints": (None, [P, P, ctypes.c_int, P, P]),
            "ref_score_ints_n": (None, [P, i64, P, ctypes.c_int, P, P]),
            "ref_logit": (f32, [i32, i32, i32, f32, f32, f32, f32, f32, ctypes.c_int]),
            "ref_logits": (None, [P, P, P, i64, P, f32, f32, i32, f32, ctypes.c_int, P]),
            "ref_attend_head": (None, [P, P, P, P, P, i64, P, P, f32, ctypes.c_int, P]),
            "ref_exp2_coef": (f32, [ctypes.c_int]),
            "ref_topp_weight": (u64, [f32, f32]),
            "ref_topp_select": (i64, [P, i64, f32, P]),
            "ref_attend_topp_head": (i64, [P, P, P, P, P, i64, P, P, f32, f32, ctypes.c_int, P, P]),
            "ref_attend_exact_selected": (ctypes.c_int, [P, P, P, i64, ctypes.c_int, P, i64, f32, P]),
            "ref_select": (i64, [P, i64, ctypes.c_int, f32, i64, i64, i64, P]),
            "ref_attend_select_head": (i64, [P, P, P, P, P, i64, P, P, f32, ctypes.c_int, f32, i64, i64, i64,
                                             ctypes.c_int, P, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _p(a: np.ndarray) -> ctypes.c_void_p:
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


# ----------------------------------------------------------------------------------------------
def splitmix64(seed: int, n: int) -> np.ndarray:
    st = ctypes.c_uint64(seed)
    return np.array([lib().ref_splitmix64_next(ctypes.byref(st)) for _ in range(n)], dtype=np.uint64)


MAX_ROUNDS = 3


def signs(seed: int, d: int = 128, rounds: int = 1) -> np.ndarray:
    """Rotation signs: [d] for one round, else [rounds * d] (round r = the next d draws)."""
    if rounds == 1:
        out = np.empty(d, np.float32)
        lib().ref_rotation_signs(seed, d, _p(out))
        return out
    out = np.empty(MAX_ROUNDS * d, np.float32)
    lib().ref_rotation_signs_rounds(seed, d, rounds, _p(out))
    return out[:rounds * d].copy()


def _sg(sgn, d: int) -> np.ndarray:
    """Signs as the C oracle reads them: MAX_ROUNDS x d entries, rounds after the given ones zero."""
    sgn = _f32(sgn).reshape(-1)
    assert sgn.size % d == 0 and 0 < sgn.size // d <= MAX_ROUNDS
    out = np.zeros(MAX_ROUNDS * d, np.float32)
    out[:sgn.size] = sgn
    return out


def fwht(x) -> np.ndarray:
    y = _f32(x).copy()
    lib().ref_fwht(_p(y), y.shape[-1])
    return y


def tree_sum(a) -> float:
    a = _f32(a)
    return float(lib().ref_tree_sum(_p(a), a.shape[-1]))


def encode(K, V, sgn) -> dict:
    """Encode L tokens: K, V are [L, d] (any float dtype, converted exactly to fp32)."""
    K = _f32(K)
    V = _f32(V)
    L, d = K.shape
    sgn = _sg(sgn, d)
    bits = np.empty((L, d // 32), np.uint32)
    norm = np.empty(L, np.float32)
    cinv = np.empty(L, np.float32)
    codes = np.empty((L, d // 8), np.uint32)
    sm = np.empty((L, d // 32), np.uint32)
    lib().ref_encode_keys(_p(K), L, _p(sgn), d, _p(bits), _p(norm), _p(cinv))
    flags = lib().ref_encode_values(_p(V), L, d, _p(codes), _p(sm))
    return {"bits": bits, "norm": norm, "cinv": cinv, "codes": codes, "sm": sm, "flags": flags}


def dequant(codes, sm) -> np.ndarray:
    codes = np.ascontiguousarray(codes, np.uint32)
    sm = np.ascontiguousarray(sm, np.uint32)
    d = codes.shape[-1] * 8
    flat_c = codes.reshape(-1, d // 8)
    flat_s = sm.reshape(-1, d // 32)
    out = np.empty((flat_c.shape[0], d), np.float64)
    for t in range(flat_c.shape[0]):
        lib().ref_dequant_value(_p(flat_c[t]), _p(flat_s[t]), d, _p(out[t]))
    return out.reshape(codes.shape[:-1] + (d,))


def half_to_double(h: int) -> float:
    return float(lib().ref_half_to_double(int(h)))


def query_prep(q, sgn) -> dict:
    """q: [d] or [H, d].  Returns planes [H, 4, d/32], vl, delta, Sq, codes [H, d], z [H, d]."""
    q = _f32(q)
    single = q.ndim == 1
    q2 = q.reshape(-1, q.shape[-1])
    H, d = q2.shape
    sgn = _sg(sgn, d)
    planes = np.empty((H, 4, d // 32), np.uint32)
    vl = np.empty(H, np.float32)
    dl = np.empty(H, np.float32)
    Sq = np.empty(H, np.int32)
    codes = np.empty((H, d), np.uint8)
    z = np.empty((H, d), np.float32)
    for h in range(H):
        qh = np.ascontiguousarray(q2[h])
        pv = np.empty(4 * (d // 32), np.uint32)
        a_vl, a_dl, a_sq = ctypes.c_float(), ctypes.c_float(), ctypes.c_int32()
        ch = np.empty(d, np.uint8)
        zh = np.empty(d, np.float32)
        lib().ref_query_prep(_p(qh), _p(sgn), d, _p(pv), ctypes.byref(a_vl), ctypes.byref(a_dl),
                             ctypes.byref(a_sq), _p(ch), _p(zh))
        planes[h] = pv.reshape(4, d // 32)
        vl[h], dl[h], Sq[h] = a_vl.value, a_dl.value, a_sq.value
        codes[h], z[h] = ch, zh
    out = {"planes": planes, "vl": vl, "delta": dl, "Sq": Sq, "codes": codes, "z": z}
    if single:
        out = {k: v[0] for k, v in out.items()}
    return out


def score_ints(bits, planes):
    """bits: [L, d/32]; planes: [4, d/32].  Returns (A [L], Bc [L]) int32."""
    bits = np.ascontiguousarray(bits, np.uint32).reshape(-1, np.shape(bits)[-1])
    planes = np.ascontiguousarray(planes, np.uint32)
    d = bits.shape[1] * 32
    A = np.empty(bits.shape[0], np.int32)
    Bc = np.empty(bits.shape[0], np.int32)
    lib().ref_score_ints_n(_p(bits), bits.shape[0], _p(planes), d, _p(A), _p(Bc))
    return A, Bc


def logit(A, Bc, Sq, vl, delta, norm, cinv, scale, d=128) -> float:
    return float(lib().ref_logit(int(A), int(Bc), int(Sq), float(vl), float(delta), float(norm), float(cinv),
                                 float(scale), d))


def logits(enc: dict, qp: dict, scale: float) -> np.ndarray:
    """Logits of all tokens of one (sequence, kv-head) for one prepared query head."""
    bits = np.ascontiguousarray(enc["bits"], np.uint32)
    L, nw = bits.shape
    d = nw * 32
    s = np.empty(L, np.float32)
    planes = np.ascontiguousarray(qp["planes"], np.uint32)
    lib().ref_logits(_p(bits), _p(_f32(enc["norm"])), _p(_f32(enc["cinv"])), L, _p(planes),
                     float(qp["vl"]), float(qp["delta"]), int(qp["Sq"]), float(scale), d, _p(s))
    return s


def _enc_ptrs(enc):
    bits = np.ascontiguousarray(enc["bits"], np.uint32)
    norm = _f32(enc["norm"])
    cinv = _f32(enc["cinv"])
    codes = np.ascontiguousarray(enc["codes"], np.uint32)
    sm = np.ascontiguousarray(enc["sm"], np.uint32)
    keep = (bits, norm, cinv, codes, sm)
    return keep, [_p(bits), _p(norm), _p(cinv), _p(codes), _p(sm)], bits.shape[0], bits.shape[1] * 32


def attend(enc: dict, q, sgn, scale: float) -> np.ndarray:
    """Full attention of one query head (q: [d]) over one encoded (sequence, kv-head); fp64 out."""
    keep, ptrs, L, d = _enc_ptrs(enc)
    q = _f32(q)
    sgn = _sg(sgn, d)
    out = np.empty(d, np.float64)
    lib().ref_attend_head(*ptrs, L, _p(q), _p(sgn), float(scale), d, _p(out))
    return out


def attend_partial(enc: dict, q, sgn, scale: float):
    """The attention sums of one query head over one encoded token range, before normalisation:
    (m, l, o[d]) with m = max_t s_t log2(e), l = sum_t 2^(s_t log2(e) - m), o = sum_t 2^(s_t log2(e) - m)
    vhat_t in fp64 from the fp32 logits (the same logits and dequantised values as `attend`); an empty
    range gives (-inf, 0, 0).  Ranges merge by log-sum-exp: out = sum_k 2^(m_k - M) o_k / sum_k
    2^(m_k - M) l_k, M = max_k m_k -- the split of one context over several devices."""
    L = np.shape(enc["bits"])[0]
    d = np.shape(enc["bits"])[1] * 32
    if L == 0:
        return -math.inf, 0.0, np.zeros(d)
    s = logits(enc, query_prep(q, sgn), scale).astype(np.float64) * (1.0 / math.log(2.0))
    m = float(s.max())
    w = np.exp2(s - m)
    return m, float(w.sum()), w @ dequant(enc["codes"], enc["sm"])


def exp2_coef(k: int) -> float:
    return float(lib().ref_exp2_coef(k))


def topp_weight(s: float, m: float) -> int:
    return int(lib().ref_topp_weight(float(s), float(m)))


def topp_select(s, p: float) -> np.ndarray:
    s = _f32(s)
    sel = np.empty(max(1, s.shape[0]), np.int64)
    n = lib().ref_topp_select(_p(s), s.shape[0], float(p), _p(sel))
    if n < 0:
        raise ValueError("p must be in (0, 1]")
    return sel[:n].copy()


def attend_topp(enc: dict, q, sgn, scale: float, p: float):
    """Top-p attention of one query head; returns (selected indices ascending, fp64 out)."""
    keep, ptrs, L, d = _enc_ptrs(enc)
    q = _f32(q)
    sgn = _sg(sgn, d)
    out = np.empty(d, np.float64)
    sel = np.empty(max(1, L), np.int64)
    n = lib().ref_attend_topp_head(*ptrs, L, _p(q), _p(sgn), float(scale), float(p), d, _p(sel), _p(out))
    if n < 0:
        raise ValueError("invalid Top-p arguments")
    return sel[:n].copy(), out


SELECT_TOPP, SELECT_TOPK = 0, 1


def select(s, mode: int, p: float = 1.0, k: int = 0, sink: int = 0, recent: int = 0) -> np.ndarray:
    """Top-p (mode 0) or Top-k (mode 1) selection plus the always-kept first `sink` / last `recent`
    tokens; ascending indices."""
    s = _f32(s)
    sel = np.empty(max(1, s.shape[0]), np.int64)
    n = lib().ref_select(_p(s), s.shape[0], int(mode), float(p), int(k), int(sink), int(recent), _p(sel))
    if n < 0:
        raise ValueError("invalid selection arguments")
    return sel[:n].copy()


def attend_select(enc: dict, q, sgn, scale: float, mode: int, p: float = 1.0, k: int = 0, sink: int = 0,
                  recent: int = 0):
    """Attention of one query head over a `select` set; returns (indices ascending, fp64 out)."""
    keep, ptrs, L, d = _enc_ptrs(enc)
    q = _f32(q)
    sgn = _sg(sgn, d)
    out = np.empty(d, np.float64)
    sel = np.empty(max(1, L), np.int64)
    n = lib().ref_attend_select_head(*ptrs, L, _p(q), _p(sgn), float(scale), int(mode), float(p), int(k), int(sink),
                                     int(recent), d, _p(sel), _p(out))
    if n < 0:
        raise ValueError("invalid selection arguments")
    return sel[:n].copy(), out


def attend_exact_selected(q, K, V, sel, scale: float) -> np.ndarray:
    """Exact attention of one query head over the selected tokens: q [d]; K, V [L, d] (exact
    values, converted to fp32 without rounding from bf16 / fp16 / fp32); sel: indices into [0, L).
    Returns fp64 [d] (zeros for an empty selection)."""
    q = _f32(q)
    K = _f32(K)
    V = _f32(V)
    L, d = K.shape
    sel = np.ascontiguousarray(np.asarray(sel, dtype=np.int64).reshape(-1))
    out = np.empty(d, np.float64)
    rc = lib().ref_attend_exact_selected(_p(q), _p(K), _p(V), L, d, _p(sel) if sel.size else None, sel.size,
                                         float(scale), _p(out))
    if rc != 0:
        raise ValueError("selected index out of range")
    return out
