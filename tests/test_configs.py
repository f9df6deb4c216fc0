"""GPU parity on the five workload configurations at their full sizes, run the way bench.py runs
them (prefill in 4096-token chunks, then append one token per sequence + attend per decode step,
default tensor-core engine, automatic split).

The oracle re-encodes the sampled (sequence, kv-head) segments from the same seeded inputs (the
encoding is per token, so a segment can be checked on its own) and recomputes the sampled query
heads' outputs over the whole segment.  Bit-exact: key bits, N, 1/C, value codes, fp16 scale and
min of every token of the sampled segments, Top-p index sets and counts.  Outputs: <= 1e-3
relative per row (max and l2).  Unsampled heads are checked for the properties that hold at any
size (finite, deterministic, status word clean).
"""
import numpy as np
import pytest
import torch

import oracle
import long_context_decode_kv1b_b200 as kv
from long_context_decode_kv1b_b200 import workloads as wl
from parity_utils import assert_planes_equal, assert_rows_close, check_probe_row, gpu_head_planes, to_np32

pytestmark = pytest.mark.gpu
DEV = "cuda"


class Run:
    """A configuration's cache built through the C ABI, with fp32 host copies of sampled segments."""

    def __init__(self, cfg: wl.Config, pairs):
        self.cfg = cfg
        self.pairs = list(pairs)
        cap = cfg.capacity
        self.cache = kv.Cache(cfg.B, cfg.Hkv, cap, seed=cfg.rotation_seed)
        self.K = {pr: np.zeros((cap, 128), np.float32) for pr in self.pairs}
        self.V = {pr: np.zeros((cap, 128), np.float32) for pr in self.pairs}
        self.n = 0
        for start, n in wl.prefill_chunks(cfg):
            K, V = wl.prefill_chunk(cfg, start, n, DEV)
            self._append(K, V)
        self.signs = oracle.signs(cfg.rotation_seed)
        self._enc = {}

    def _append(self, K, V):
        self.cache.append(K, V)
        n = K.shape[1]
        for (b, h) in self.pairs:
            self.K[(b, h)][self.n:self.n + n] = to_np32(K[b, :, h])
            self.V[(b, h)][self.n:self.n + n] = to_np32(V[b, :, h])
        self.n += n

    def step(self, i):
        K, V = wl.step_kv(self.cfg, i, DEV)
        self._append(K, V)

    def encoded(self, pr):
        """Oracle encoding of all tokens appended so far (prefixes of it serve earlier steps)."""
        if pr not in self._enc or self._enc[pr]["bits"].shape[0] < self.n:
            self._enc[pr] = oracle.encode(self.K[pr][:self.n], self.V[pr][:self.n], self.signs)
        return self._enc[pr]

    def check_planes(self):
        torch.cuda.synchronize()
        for (b, h) in self.pairs:
            assert_planes_equal(gpu_head_planes(self.cache, b, h, self.n), self.encoded((b, h)),
                                f"{self.cfg.name} b{b} kvh{h}")

    def check_outputs(self, out, q, n_tokens):
        qn, o = to_np32(q), out.cpu().numpy()
        G = self.cfg.G
        for (b, h) in self.pairs:
            enc = {k: v[:n_tokens] for k, v in self.encoded((b, h)).items() if k != "flags"}
            for j in range(G):
                hq = h * G + j
                ref = oracle.attend(enc, qn[b, hq], self.signs, self.cfg.scale)
                assert_rows_close(o[b, hq], ref, where=f"{self.cfg.name} b{b} hq{hq} L{n_tokens}")
        assert np.isfinite(o).all()


def decode(run: Run, check_steps, check_planes_at_end=True):
    cfg = run.cfg
    out = torch.empty((cfg.B, cfg.Hq, 128), dtype=torch.float32, device=DEV)
    for i in range(cfg.steps):
        run.step(i)
        q = wl.queries(cfg, i, DEV)
        run.cache.attend(q, cfg.scale, out=out)
        if i in check_steps:
            torch.cuda.synchronize()
            run.check_outputs(out, q, run.n)
    if check_planes_at_end:
        run.check_planes()
    assert run.cache.status() == 0
    return out


def test_c1_single_head_fp32():
    cfg = wl.CONFIGS["c1"]
    run = Run(cfg, [(0, 0)])
    run.check_planes()
    q = wl.queries(cfg, 0, DEV)
    for engine in (kv.ATTEND_TENSOR, kv.ATTEND_CUDA_CORE):
        out = run.cache.attend(q, cfg.scale, engine=engine)
        torch.cuda.synchronize()
        run.check_outputs(out, q, run.n)
    assert run.cache.status() == 0


def test_c2_mha_outlier_channels():
    cfg = wl.CONFIGS["c2"]
    run = Run(cfg, [(0, h) for h in range(cfg.Hkv)])
    run.check_planes()
    q = wl.queries(cfg, 0, DEV)
    out = run.cache.attend(q, cfg.scale)
    torch.cuda.synchronize()
    run.check_outputs(out, q, run.n)
    assert run.cache.status() == 0


def probe_rows(run: Run, q, kernel, heads_per_pair=None):
    """kv1b_scores_probe of `kernel` on the run's cache; the sampled segments' query heads (all G of
    them, or the first heads_per_pair) checked against the oracle over every token."""
    cfg = run.cfg
    pr = run.cache.scores_probe(q, cfg.scale, kernel)
    torch.cuda.synchronize()
    qn = to_np32(q)
    for (b, h) in run.pairs:
        for j in range(heads_per_pair or cfg.G):
            check_probe_row(pr, b, h * cfg.G + j, run.encoded((b, h)), qn[b, h * cfg.G + j], run.signs, cfg.scale,
                            kernel, run.n, where=cfg.name)
    return pr


def test_c3_gqa_batch8_decode_steps():
    cfg = wl.CONFIGS["c3"]
    run = Run(cfg, [(0, 0), (0, 7), (5, 3), (7, 7)])
    out = decode(run, check_steps={0, cfg.steps - 1})
    # the last step again: identical bits (deterministic split and merge order)
    q = wl.queries(cfg, cfg.steps - 1, DEV)
    again = run.cache.attend(q, cfg.scale)
    assert torch.equal(out, again)
    # the integers of the kernels this workload runs, bit for bit over every token of the sampled segments
    pr = probe_rows(run, q, kv.PROBE_ATTEND)
    assert torch.equal(pr["out"], out)  # the probe instantiation computes the same attention
    probe_rows(run, q, kv.PROBE_TOPP)


def test_c4_topp_heavy_tokens():
    cfg = wl.CONFIGS["c4"]
    run = Run(cfg, [(0, 0), (2, 5), (7, 7)])
    run.check_planes()
    q = wl.queries(cfg, 0, DEV)
    out, sel, cnt = run.cache.attend_topp(q, cfg.scale, cfg.p)
    torch.cuda.synchronize()
    qn, o, sel, cnt = to_np32(q), out.cpu().numpy(), sel.cpu().numpy(), cnt.cpu().numpy()
    heavy = wl.heavy_tokens(cfg, DEV).cpu().numpy()
    for (b, h) in run.pairs:
        enc = {k: v for k, v in run.encoded((b, h)).items() if k != "flags"}
        for j in range(cfg.G):
            hq = h * cfg.G + j
            ref_sel, ref_out = oracle.attend_topp(enc, qn[b, hq], run.signs, cfg.scale, cfg.p)
            n = int(cnt[b, hq])
            assert n == len(ref_sel), f"c4 b{b} hq{hq}: |S| {n} vs {len(ref_sel)}"
            assert np.array_equal(sel[b, hq, :n], ref_sel), f"c4 b{b} hq{hq}: selected sets differ"
            assert_rows_close(o[b, hq], ref_out, where=f"c4 b{b} hq{hq}")
            # the planted tokens carry the query direction: the adaptive budget is a small set of them
            assert n <= cfg.heavy and np.isin(ref_sel, heavy[b, h]).mean() >= 0.9
    assert np.isfinite(o).all()
    assert (cnt >= 1).all() and (cnt <= run.n).all()
    assert run.cache.status() == 0


def test_c5_one_million_tokens():
    cfg = wl.CONFIGS["c5"]
    run = Run(cfg, [(0, 0), (0, 5)])
    out = torch.empty((cfg.B, cfg.Hq, 128), dtype=torch.float32, device=DEV)
    for i in range(cfg.steps):
        run.step(i)
        q = wl.queries(cfg, i, DEV)
        run.cache.attend(q, cfg.scale, out=out)
        if i == 0:
            torch.cuda.synchronize()
            first = out.clone()
            saved = run.pairs
            run.pairs = [(0, 0)]
            run.check_outputs(out, q, run.n)
            run.pairs = saved
    torch.cuda.synchronize()
    run.check_outputs(out, q, run.n)
    run.check_planes()
    assert run.cache.lengths == [cfg.L + cfg.steps]
    assert not torch.equal(first, out)  # the appended tokens and new queries changed the result
    assert run.cache.status() == 0
    # the score integers of both tensor-core kernels over all 1,048,608 tokens of kv-head 0's heads
    saved = run.pairs
    run.pairs = [(0, 0)]
    probe_rows(run, q, kv.PROBE_ATTEND)
    probe_rows(run, q, kv.PROBE_TOPP)
    run.pairs = saved
    # adaptive Top-p (p = 0.9) on the same cache: sampled heads of kv-heads 0 and 5, selected sets and
    # counts bit for bit, outputs at the bar
    out_p, sel, cnt = run.cache.attend_topp(q, cfg.scale, 0.9)
    torch.cuda.synchronize()
    qn, cnt_h = to_np32(q), cnt.cpu().numpy()
    for (b, h), heads in (((0, 0), (0, 3)), ((0, 5), (21, 22))):
        enc = {k: v[:run.n] for k, v in run.encoded((b, h)).items() if k != "flags"}
        for hq in heads:
            ref_sel, ref_out = oracle.attend_topp(enc, qn[b, hq], run.signs, cfg.scale, 0.9)
            n = int(cnt_h[b, hq])
            assert n == len(ref_sel), f"c5 Top-p hq{hq}: |S| {n} vs {len(ref_sel)}"
            assert np.array_equal(sel[b, hq, :n].cpu().numpy(), ref_sel), f"c5 Top-p hq{hq}: selected sets differ"
            assert_rows_close(out_p[b, hq].cpu().numpy(), ref_out, where=f"c5 Top-p hq{hq}")
    assert (cnt_h >= 1).all() and (cnt_h <= run.n).all()
    assert run.cache.status() == 0
