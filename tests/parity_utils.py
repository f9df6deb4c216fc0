"""Helpers shared by the GPU parity tests: run the oracle on the same seeded inputs and compare."""
import numpy as np
import torch

import oracle
import long_context_decode_kv1b_b200 as kv

TOL = 1e-3  # the output bar: <= 1e-3 relative error for attention outputs (fp32 accumulation)


def to_np32(t: torch.Tensor) -> np.ndarray:
    return t.detach().to(torch.float32).cpu().numpy()


def oracle_layout_codes(codes_u8: np.ndarray) -> np.ndarray:
    """[L, 128] codes -> [L, 16] words with nibble j of word w = channel 8w + j (oracle layout)."""
    c = codes_u8.astype(np.uint32).reshape(codes_u8.shape[0], 16, 8)
    w = np.zeros(c.shape[:2], np.uint32)
    for j in range(8):
        w |= c[:, :, j] << np.uint32(4 * j)
    return w


def gpu_head_planes(cache: kv.Cache, b: int, h: int, L: int) -> dict:
    P = cache.planes()
    return {
        "bits": P["k_bits"][b, h, :L].cpu().numpy().view(np.uint32),
        "norm": P["k_norm"][b, h, :L].cpu().numpy(),
        "cinv": P["k_cinv"][b, h, :L].cpu().numpy(),
        "codes": oracle_layout_codes(kv.unpack_codes(P["v_codes"][b, h], L).cpu().numpy()),
        "sm": P["v_sm"][b, h, :L].cpu().numpy().view(np.uint32),
    }


def assert_planes_equal(gpu: dict, ref: dict, where=""):
    for k in ("bits", "norm", "cinv", "codes", "sm"):
        g, r = gpu[k], ref[k]
        if k in ("norm", "cinv"):
            g, r = g.view(np.uint32), np.ascontiguousarray(r).view(np.uint32)
        bad = np.argwhere(g != r)
        assert bad.size == 0, f"{where} {k}: {len(bad)} mismatches, first at {bad[:3].tolist()}"


def assert_rows_close(out_gpu: np.ndarray, out_ref: np.ndarray, tol: float = TOL, where=""):
    """Per row: max|d| <= tol * max|ref| and ||d||_2 <= tol * ||ref||_2 (rows of 128 channels)."""
    g = out_gpu.reshape(-1, out_gpu.shape[-1]).astype(np.float64)
    r = out_ref.reshape(-1, out_ref.shape[-1]).astype(np.float64)
    for i in range(g.shape[0]):
        d = g[i] - r[i]
        mr, nr = np.abs(r[i]).max(), np.linalg.norm(r[i])
        assert np.abs(d).max() <= tol * mr + 1e-30, f"{where} row {i}: max err {np.abs(d).max():.3e} vs {tol * mr:.3e}"
        assert np.linalg.norm(d) <= tol * nr + 1e-30, f"{where} row {i}: l2 err {np.linalg.norm(d):.3e} vs {tol * nr:.3e}"


class HostKV:
    """fp32 host copies of K and V per (b, kv-head), accumulated as tokens are appended."""

    def __init__(self, B, Hkv, cap):
        self.K = np.zeros((B, Hkv, cap, 128), np.float32)
        self.V = np.zeros((B, Hkv, cap, 128), np.float32)
        self.n = 0

    def add(self, K: torch.Tensor, V: torch.Tensor):
        k = to_np32(K).transpose(0, 2, 1, 3)  # [B, H, n, 128]
        v = to_np32(V).transpose(0, 2, 1, 3)
        n = k.shape[2]
        self.K[:, :, self.n:self.n + n] = k
        self.V[:, :, self.n:self.n + n] = v
        self.n += n

    def encode(self, b, h, signs):
        return oracle.encode(self.K[b, h, :self.n], self.V[b, h, :self.n], signs)


def oracle_attend_all(host: HostKV, q: torch.Tensor, signs, scale, G, heads=None) -> np.ndarray:
    qn = to_np32(q)
    B, Hq, _ = qn.shape
    out = np.zeros((B, Hq, 128))
    encs = {}
    for b in range(B):
        for hq in range(Hq):
            if heads is not None and (b, hq) not in heads:
                continue
            kvh = hq // G
            if (b, kvh) not in encs:
                encs[(b, kvh)] = host.encode(b, kvh, signs)
            out[b, hq] = oracle.attend(encs[(b, kvh)], qn[b, hq], signs, scale)
    return out


L2E = 1.4426950408889634


def check_probe_row(pr: dict, b: int, hq: int, enc: dict, q_row: np.ndarray, signs, scale: float, kernel: int,
                    n: int, where: str = ""):
    """One (b, hq) row of a kv1b_scores_probe result against the oracle: the integers bit for bit
    (8 A and 8 Bc from the tensor-core kernels, A and Bc from the popcount hook); the fp32 logits bit
    for bit (popcount hook, Top-p score pass); the persistent attend kernel's log2-unit logits within
    16 roundings of the magnitude of their terms (it forms them in its own fused order)."""
    mult = 1 if kernel == kv.PROBE_POPC else 8
    r = oracle.query_prep(q_row, signs)
    A, Bc = oracle.score_ints(enc["bits"][:n], r["planes"])
    gA, gB = pr["A"][b, hq, :n].cpu().numpy(), pr["Bc"][b, hq, :n].cpu().numpy()
    bad = np.flatnonzero((gA != mult * A) | (gB != mult * Bc))
    assert bad.size == 0, f"{where} b{b} hq{hq}: {bad.size} integer mismatches, first at {bad[:4].tolist()}"
    gs = pr["s"][b, hq, :n].cpu().numpy()
    if kernel == kv.PROBE_ATTEND:
        dl, vl, sq = float(r["delta"]), float(r["vl"]), int(r["Sq"])
        nc = enc["norm"][:n].astype(np.float64) * enc["cinv"][:n].astype(np.float64)
        qs = scale / 128.0 * L2E
        exact = (dl * (2.0 * A - sq) + vl * (2.0 * Bc - 128.0)) * nc * qs
        mag = (abs(dl) * (2.0 * A + sq) + abs(vl) * (2.0 * Bc + 128.0)) * np.abs(nc) * qs
        err = np.abs(gs.astype(np.float64) - exact)
        assert (err <= 16 * 2.0 ** -24 * mag + 1e-30).all(), \
            f"{where} b{b} hq{hq}: log2 logit off by {np.max(err / (mag + 1e-30)):.2e} of its terms"
    else:
        enc_n = {k: v[:n] for k, v in enc.items() if k != "flags"}
        s = oracle.logits(enc_n, r, scale)
        assert np.array_equal(gs.view(np.uint32), s.view(np.uint32)), f"{where} b{b} hq{hq}: logits differ"
