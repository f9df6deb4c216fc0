"""A plain numpy model of the default attend engine's value-weight arithmetic, checked against the
fp64 softmax over the same logits and 4-bit values (host only, no GPU).

The engine (long_context_decode_kv1b_b200/csrc/kv1b_attend_ws.cu) forms, per token, head and
32-channel value group, the weight W = rint(p * scale * 2^E) as a 32-bit unsigned integer and sums
W * code exactly in integers; p = 2^(s - m) against a reference maximum m raised only when a
logit passes it by tau = 4 (p <= 2^4), and E = 31 - tau - 2 - floor(log2 smax) per group, smax
the largest scale seen (2 bits of headroom).  value = min + scale * code, so the min term is summed
in floating point beside it (H1B-KV, technical framework: weights from the sketch, then the 4-bit
values).  The model follows those steps tile by tile (128 tokens) and shows why the weights need
32 bits: when a long tail far below the maximum holds a few percent of the softmax mass or more,
a 23-bit fixed point rounds the tail's weights to a unit or none and biases the output beyond the
1e-3 bar, while 32 bits stay near 1e-6.

The engine adds a dither d in [-1/2, 1/2) before rounding, W = rint(p * scale * 2^E + d): tokens
2^-26.6 or more below the reference maximum get weights under half a unit, which plain rounding sends
to zero all together -- a bias that grows with the number of such tokens one reference covers.  d is
the top byte of a Weyl sequence (n * 0x9E3779B9 + lane * 0x6A09E667, n the 32-token slice, lane =
4 (token & 7) + group: the lane that forms the weights of those tokens), so over many tokens every
fractional weight keeps its expected value; the model reproduces that mapping.
"""
import math

import numpy as np

import oracle

TAU, ROOM, TILE = 4, 2, 128


def fp16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(bits, np.uint16).view(np.float16).astype(np.float32)


def decode_values(enc: dict):
    """codes [L, 128] (0..15), scale / min [L, 4] in fp32 from the oracle's packed planes."""
    words = enc["codes"].astype(np.uint64)  # [L, 16], nibble j of word w = channel 8w + j
    shifts = (4 * np.arange(8, dtype=np.uint64))[None, None, :]
    codes = ((words[:, :, None] >> shifts) & 0xF).reshape(words.shape[0], 128).astype(np.int64)
    sm = enc["sm"].astype(np.uint32)
    return codes, fp16_bits_to_f32(sm & 0xFFFF), fp16_bits_to_f32(sm >> 16)


def dither(t0: int, t1: int, group: int) -> np.ndarray:
    """The engine's rounding offsets of tokens t0 .. t1 - 1 (segment positions) for one value group."""
    t = np.arange(t0, t1, dtype=np.uint64)
    n = t >> np.uint64(5)
    lane = (t & np.uint64(7)) * np.uint64(4) + np.uint64(group)
    h = (n * np.uint64(0x9E3779B9) + lane * np.uint64(0x6A09E667)) & np.uint64(0xFFFFFFFF)
    return ((h >> np.uint64(24)).astype(np.float64) / 256.0 - 0.5).astype(np.float32)


def model_attend(s2: np.ndarray, codes, scale, mn, bits: int = 32, dithered: bool = True) -> np.ndarray:
    """One head: s2 log2-unit logits [L] (fp32).  Returns fp64 out [128].  dithered=False rounds the
    weights without the dither (the form the dither replaced)."""
    L = s2.shape[0]
    m = -math.inf
    E = [None] * 4
    smax = [0.0] * 4
    D = np.zeros(128, np.int64)           # exact sum of W * code per channel (group c // 32)
    F = np.zeros(128, np.float32)         # converted sums
    mid = np.zeros(4, np.float64)         # sum of p * min per group
    lsum = 0.0
    drop = 32 - bits                      # fewer bits: a smaller exponent

    def drain(alpha: float):
        nonlocal F, D
        for g in range(4):
            if E[g] is not None:
                sl = slice(32 * g, 32 * g + 32)
                F[sl] = (F[sl] + D[sl].astype(np.float32) * np.float32(2.0 ** -E[g])) * np.float32(alpha)
        D[:] = 0

    for t0 in range(0, L, TILE):
        t1 = min(L, t0 + TILE)
        st = s2[t0:t1]
        mt = float(st.max())
        changed, alpha = False, 1.0
        if mt > m + TAU:
            alpha = 0.0 if m == -math.inf else 2.0 ** (m - mt)
            m, changed = mt, True
        E_new = list(E)
        for g in range(4):
            sg = float(scale[t0:t1, g].max())
            if sg > smax[g]:
                k = math.floor(math.log2(sg))
                smax[g] = 2.0 ** (k + 1 + ROOM)
                E_new[g] = 31 - TAU - ROOM - k - drop
                changed |= E_new[g] != E[g]
        if changed:
            drain(alpha)
            E = E_new
        lsum *= alpha
        mid *= alpha
        p = np.exp2((st - np.float32(m)).astype(np.float32)).astype(np.float32)
        lsum += float(p.astype(np.float64).sum())
        for g in range(4):
            s2g = (scale[t0:t1, g] * np.float32(2.0 ** E[g])).astype(np.float32)
            if dithered:  # one rounding of p * s2g + d (a fused multiply-add), negative results to 0
                x = (p.astype(np.float64) * s2g.astype(np.float64) + dither(t0, t1, g)).astype(np.float32)
            else:
                x = (p * s2g).astype(np.float32)
            W = np.maximum(np.rint(x), 0).astype(np.int64)
            assert W.max(initial=0) < 2 ** bits
            D[32 * g:32 * g + 32] += W @ codes[t0:t1, 32 * g:32 * g + 32]
            mid[g] += float((p.astype(np.float64) * mn[t0:t1, g].astype(np.float64)).sum())
    drain(1.0)
    return (F.astype(np.float64) + np.repeat(mid, 32)) / lsum


def reference(s2: np.ndarray, codes, scale, mn) -> np.ndarray:
    """fp64 softmax over the same logits of the dequantised values min + scale * code."""
    s = s2.astype(np.float64)
    w = np.exp2(s - s.max())
    vhat = np.repeat(mn.astype(np.float64), 32, axis=1) + np.repeat(scale.astype(np.float64), 32, axis=1) * codes
    return (w[:, None] * vhat).sum(0) / w.sum()


def rel_err(a, b) -> float:
    return float(np.abs(a - b).max() / np.abs(b).max())


def long_tail_case(seed: int, L: int = 65536, gap: float = 18.0):
    """Values of a real encode; logits: a bulk N(0, 1) - gap below four maximal tokens near 0 (the
    first of them at position 0, like an attention sink, so the reference maximum is set from the
    start), so the tail holds a few percent of the mass in weights of ~2^(25 - gap) units at 32
    bits and under one unit at 23."""
    rng = np.random.default_rng(seed)
    K = rng.standard_normal((L, 128)).astype(np.float32)
    V = rng.standard_normal((L, 128)).astype(np.float32)
    enc = oracle.encode(K, V, oracle.signs(seed))
    codes, scale, mn = decode_values(enc)
    s2 = (rng.standard_normal(L) - gap).astype(np.float32)
    top = np.concatenate([[0], rng.choice(np.arange(1, L), 3, replace=False)])
    s2[top] = rng.standard_normal(4).astype(np.float32) * 0.5
    return s2, codes, scale, mn


def test_value_planes_decode_like_the_oracle():
    rng = np.random.default_rng(1)
    V = rng.standard_normal((64, 128)).astype(np.float32)
    enc = oracle.encode(rng.standard_normal((64, 128)).astype(np.float32), V, oracle.signs(1))
    codes, scale, mn = decode_values(enc)
    vhat = np.repeat(mn.astype(np.float64), 32, axis=1) + np.repeat(scale.astype(np.float64), 32, axis=1) * codes
    assert np.array_equal(vhat, oracle.dequant(enc["codes"], enc["sm"]))


def test_32_bit_weights_meet_the_bar_on_a_long_tail_and_23_bits_do_not():
    for seed in (3, 4):
        s2, codes, scale, mn = long_tail_case(seed)
        ref = reference(s2, codes, scale, mn)
        tail = np.exp2(s2.astype(np.float64) - s2.max())
        assert tail[s2 < -8].sum() / tail.sum() > 0.03  # the tail holds a few percent of the mass
        e32 = rel_err(model_attend(s2, codes, scale, mn, 32), ref)
        e23 = rel_err(model_attend(s2, codes, scale, mn, 23), ref)
        assert e32 < 2e-5, e32
        assert e23 > 1e-3, e23


def test_32_bit_weights_on_gaussian_logits_with_a_late_maximum():
    # ordinary logits, the largest one last: every earlier stage is rescaled when it arrives
    rng = np.random.default_rng(7)
    L = 8192
    s2, codes, scale, mn = long_tail_case(7, L=L)
    s2 = (rng.standard_normal(L) * 3.0).astype(np.float32)
    s2[-1] = s2.max() + 12.0
    ref = reference(s2, codes, scale, mn)
    assert rel_err(model_attend(s2, codes, scale, mn, 32), ref) < 2e-5


def packed_tail_case(L: int = 1 << 20, vmean: float = 3.0):
    """One dominant token at position 0 and L tail tokens 2^-27.2 .. 2^-28 below it (log2 units) --
    weights of 0.2 .. 0.5 units at 32 bits; tail values of mean +vmean, the dominant value -vmean."""
    rng = np.random.default_rng(11)
    K = rng.standard_normal((L, 128)).astype(np.float32)
    V = (rng.standard_normal((L, 128)) + vmean).astype(np.float32)
    V[0] -= 2 * vmean
    enc = oracle.encode(K, V, oracle.signs(11))
    codes, scale, mn = decode_values(enc)
    s2 = rng.uniform(-28.0, -27.2, L).astype(np.float32)
    s2[0] = 0.0
    return s2, codes, scale, mn


def test_dither_keeps_a_tail_of_sub_unit_weights_unbiased():
    # one reference maximum over 2^20 tokens whose weights are fractions of a unit (as one quad of
    # the engine sees when a very large cache gives it that many tokens): plain rounding drops most
    # of them and misses the bar; the dithered rounding stays far inside it
    s2, codes, scale, mn = packed_tail_case()
    ref = reference(s2, codes, scale, mn)
    w = np.exp2(s2.astype(np.float64))
    assert 3e-3 < (w.sum() - 1.0) / w.sum() < 8e-3
    e_plain = rel_err(model_attend(s2, codes, scale, mn, dithered=False), ref)
    e_dith = rel_err(model_attend(s2, codes, scale, mn), ref)
    assert e_plain > 1e-3, e_plain
    assert e_dith < 1e-4, e_dith


def test_dither_offsets_are_uniform_per_group():
    # the offsets of any 8192 consecutive tokens cover [-1/2, 1/2) evenly for every value group
    for g in range(4):
        d = dither(4096, 4096 + 8192, g).astype(np.float64)
        assert d.min() >= -0.5 and d.max() < 0.5
        assert abs(d.mean()) < 0.01
        hist = np.histogram(d, bins=16, range=(-0.5, 0.5))[0]
        assert hist.min() > 0.8 * 8192 / 16 and hist.max() < 1.2 * 8192 / 16
