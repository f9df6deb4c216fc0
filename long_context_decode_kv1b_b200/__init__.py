"""Python binding of ``libkv1b.so`` -- decode attention over a 1-bit-key / 4-bit-value KV cache.

Argument marshalling only: every step of the path runs in the CUDA library (``csrc/``) behind the
C ABI of ``include/kv1b.h``; PyTorch provides device memory and streams.  The library must have
been built (``python -m long_context_decode_kv1b_b200.build``); there is no CPU fallback and
importing the binding on a machine without the built library raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkv1b.so")

HEAD_DIM = 128
MAX_BATCH = 64
DTYPE_F32, DTYPE_BF16, DTYPE_F16 = 0, 1, 2
ATTEND_TENSOR, ATTEND_CUDA_CORE = 0, 1
ATTEND_WS_CLEAN = 2  # flag: the workspace's merge counters are zero (left so by the previous attend)
ATTEND_PARTIAL = 4   # flag: log-sum-exp partial rows (m, l, o[128]) instead of the normalised output
PART_ROW = 2 + 128
STATUS_TIMEOUT = 4
PROBE_POPC, PROBE_ATTEND, PROBE_TOPP = 0, 1, 2
STATUS_NONFINITE, STATUS_FP16_SATURATED = 1, 2
ERRORS = {0: "ok", -1: "invalid argument", -2: "unsupported", -3: "capacity", -4: "misaligned",
          -5: "workspace too small", -6: "CUDA error"}

# symbols declared in include/kv1b.h
SYMBOLS = ("kv1b_cache_bytes", "kv1b_cache_init", "kv1b_cache_init_rounds", "kv1b_encode_append", "kv1b_attend_workspace_bytes",
           "kv1b_attend", "kv1b_attend_noalloc", "kv1b_attend_topp", "kv1b_attend_select",
           "kv1b_attend_selected_exact",
           "kv1b_merge_partials", "kv1b_query_prep", "kv1b_scores", "kv1b_scores_probe", "kv1b_attend_wait_probe",
           "kv1b_read_status", "kv1b_status_string", "kv1b_version")


class Kv1bError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what} failed: {ERRORS.get(code, code)} ({code})")
        self.code = code


class CacheDesc(ctypes.Structure):
    """Mirror of ``kv1b_cache_t``."""
    _fields_ = [
        ("batch", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("capacity", ctypes.c_int32), ("rotation_seed", ctypes.c_uint64),
        ("k_bits", ctypes.c_void_p), ("k_norm", ctypes.c_void_p), ("k_cinv", ctypes.c_void_p),
        ("v_codes", ctypes.c_void_p), ("v_sm", ctypes.c_void_p), ("signs", ctypes.c_void_p),
        ("d_lengths", ctypes.c_void_p), ("d_status", ctypes.c_void_p),
        ("h_lengths", ctypes.c_int64 * MAX_BATCH),
        ("rotation_rounds", ctypes.c_int32), ("reserved", ctypes.c_int32),
    ]


_lib = None


def lib() -> ctypes.CDLL:
    """Load the CUDA library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: run `python -m long_context_decode_kv1b_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, i32, i64, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
        D = ctypes.POINTER(CacheDesc)
        sig = {
            "kv1b_cache_bytes": (sz, [i32, i32, i32, i32]),
            "kv1b_cache_init": (ctypes.c_int, [D, P, sz, i32, i32, i32, i32, ctypes.c_uint64, P]),
            "kv1b_cache_init_rounds": (ctypes.c_int, [D, P, sz, i32, i32, i32, i32, ctypes.c_uint64, i32, P]),
            "kv1b_encode_append": (ctypes.c_int, [D, P, P, i32, i32, i64, i64, i64, P]),
            "kv1b_attend_workspace_bytes": (sz, [D, i32, i32]),
            "kv1b_attend": (ctypes.c_int, [D, P, i32, i32, f32, P, P, sz, i32, i32, P]),
            "kv1b_attend_topp": (ctypes.c_int, [D, P, i32, i32, f32, f32, P, P, P, P, sz, P]),
            "kv1b_attend_select": (ctypes.c_int, [D, P, i32, i32, f32, i32, f32, i32, i32, i32, P, P, P, P, sz, P]),
            "kv1b_attend_selected_exact": (ctypes.c_int, [D, P, i32, i32, f32, P, P, i32, i64, i64, i64, i64, P, P,
                                                          P, P, sz, P]),
            "kv1b_merge_partials": (ctypes.c_int, [P, i32, i64, P, P]),
            "kv1b_query_prep": (ctypes.c_int, [D, P, i32, i32, P, P, P, P, P]),
            "kv1b_scores": (ctypes.c_int, [D, P, i32, i32, f32, P, P, P, P]),
            "kv1b_scores_probe": (ctypes.c_int, [D, P, i32, i32, f32, i32, P, P, P, P, P, sz, P]),
            "kv1b_attend_wait_probe": (ctypes.c_int, [D, P, i32, i32, f32, P, P, sz, i32, i32, P]),
            "kv1b_read_status": (ctypes.c_int, [D, P, P]),
            "kv1b_status_string": (ctypes.c_char_p, [ctypes.c_int]),
            "kv1b_version": (ctypes.c_int, []),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(code: int, what: str):
    if code != 0:
        raise Kv1bError(code, what)


def _check_buf(t: torch.Tensor, shape, dtype, name: str):
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {dtype} tensor of shape {tuple(shape)}")


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return DTYPE_F32
    if t.dtype == torch.bfloat16:
        return DTYPE_BF16
    if t.dtype == torch.float16:
        return DTYPE_F16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _stream(stream=None) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


SELECT_TOPP, SELECT_TOPK = 0, 1


class Cache:
    """A compressed KV cache for `batch` sequences x `num_kv_heads` heads, in one device buffer."""

    def __init__(self, batch: int, num_kv_heads: int, capacity: int, seed: int = 0, device="cuda",
                 stream=None, rounds: int = 1):
        """rounds: rotation rounds H * diag(D_r) (1 .. 3; see kv1b_cache_init_rounds)."""
        L = lib()
        self.batch, self.num_kv_heads, self.capacity, self.seed = batch, num_kv_heads, capacity, seed
        self.rounds = rounds
        self.device = torch.device(device)
        nbytes = L.kv1b_cache_bytes(batch, num_kv_heads, HEAD_DIM, capacity)
        if nbytes == 0:
            raise Kv1bError(-1, "kv1b_cache_bytes")
        self.nbytes = nbytes
        self.buffer = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        self.desc = CacheDesc()
        _check(L.kv1b_cache_init_rounds(ctypes.byref(self.desc), _ptr(self.buffer), nbytes, batch, num_kv_heads,
                                        HEAD_DIM, capacity, seed, rounds, _stream(stream)), "kv1b_cache_init_rounds")
        self._ws = {}
        self._ws_clean = {}  # num_q_heads -> the attend workspace's merge counters are known to be zero

    # ---- views of the device planes (for tests / inspection; layout in include/kv1b.h)
    def _view(self, addr, dtype, shape):
        off = addr - self.buffer.data_ptr()
        n = 1
        for s in shape:
            n *= s
        esz = torch.empty((), dtype=dtype).element_size()
        return self.buffer[off:off + n * esz].view(dtype).view(*shape)

    def planes(self) -> dict:
        B, H, C = self.batch, self.num_kv_heads, self.capacity
        d = self.desc
        return {
            "k_bits": self._view(d.k_bits, torch.int32, (B, H, C, 4)),
            "k_norm": self._view(d.k_norm, torch.float32, (B, H, C)),
            "k_cinv": self._view(d.k_cinv, torch.float32, (B, H, C)),
            "v_codes": self._view(d.v_codes, torch.int32, (B, H, C // 128, HEAD_DIM, 16)),
            "v_sm": self._view(d.v_sm, torch.int32, (B, H, C, 4)),
            "signs": self._view(d.signs, torch.float32, (HEAD_DIM,)),  # round 0
            "signs_rounds": self._view(d.signs, torch.float32, (3, HEAD_DIM)),
            "lengths": self._view(d.d_lengths, torch.int32, (B,)),
        }

    @property
    def lengths(self):
        return [int(self.desc.h_lengths[b]) for b in range(self.batch)]

    def append(self, k: torch.Tensor, v: torch.Tensor, stream=None):
        """k, v: [batch, n_new, num_kv_heads, 128] (channel stride 1), same dtype and strides."""
        if k.shape != v.shape or k.stride() != v.stride() or k.dtype != v.dtype:
            raise ValueError("k and v must have equal shapes, strides and dtypes")
        B, n, H, D = k.shape
        if (B, H, D) != (self.batch, self.num_kv_heads, HEAD_DIM) or k.stride(3) != 1:
            raise ValueError("expected [batch, n_new, num_kv_heads, 128] with unit channel stride")
        _check(lib().kv1b_encode_append(ctypes.byref(self.desc), _ptr(k), _ptr(v), _dtype_code(k), n, k.stride(0),
                                        k.stride(1), k.stride(2), _stream(stream)), "kv1b_encode_append")

    def workspace(self, num_q_heads: int, mode: int) -> torch.Tensor:
        key = (num_q_heads, mode)
        if key not in self._ws:
            n = lib().kv1b_attend_workspace_bytes(ctypes.byref(self.desc), num_q_heads, mode)
            if n == 0:
                raise Kv1bError(-1, "kv1b_attend_workspace_bytes")
            self._ws[key] = torch.empty(n, dtype=torch.uint8, device=self.device)
        return self._ws[key]

    def attend(self, q: torch.Tensor, scale: float, out: torch.Tensor | None = None, engine: int = ATTEND_TENSOR,
               num_splits: int = 0, stream=None, partial: bool = False) -> torch.Tensor:
        """q: [batch, num_q_heads, 128] contiguous.  Returns fp32 [batch, num_q_heads, 128], or with
        partial=True the log-sum-exp rows [batch, num_q_heads, 130] = (m, l, o[128]) for merge_partials."""
        B, Hq, D = q.shape
        if not q.is_contiguous():
            raise ValueError("q must be contiguous")
        width = PART_ROW if partial else D
        if out is None:
            out = torch.empty((B, Hq, width), dtype=torch.float32, device=q.device)
        _check_buf(out, (B, Hq, width), torch.float32, "out")
        ws = self.workspace(Hq, 0)
        # after the first call the workspace's merge counters are zero (each attend leaves them so)
        flags = engine | (ATTEND_WS_CLEAN if self._ws_clean.get(Hq, False) else 0) | (ATTEND_PARTIAL if partial else 0)
        _check(lib().kv1b_attend(ctypes.byref(self.desc), _ptr(q), _dtype_code(q), Hq, float(scale), _ptr(out),
                                 _ptr(ws), ws.numel(), flags, num_splits, _stream(stream)), "kv1b_attend")
        self._ws_clean[Hq] = True
        return out

    def attend_topp(self, q: torch.Tensor, scale: float, p: float, out=None, sel=None, cnt=None, stream=None):
        """Returns (out fp32 [B, Hq, 128], sel_idx int32 [B, Hq, capacity], sel_cnt int32 [B, Hq]);
        out / sel / cnt may be passed in (contiguous, those shapes and dtypes) to reuse buffers."""
        B, Hq, D = q.shape
        if out is None:
            out = torch.empty((B, Hq, D), dtype=torch.float32, device=q.device)
        if sel is None:
            sel = torch.empty((B, Hq, self.capacity), dtype=torch.int32, device=q.device)
        if cnt is None:
            cnt = torch.empty((B, Hq), dtype=torch.int32, device=q.device)
        _check_buf(out, (B, Hq, D), torch.float32, "out")
        _check_buf(sel, (B, Hq, self.capacity), torch.int32, "sel")
        _check_buf(cnt, (B, Hq), torch.int32, "cnt")
        ws = self.workspace(Hq, 1)
        _check(lib().kv1b_attend_topp(ctypes.byref(self.desc), _ptr(q), _dtype_code(q), Hq, float(scale), float(p),
                                      _ptr(out), _ptr(sel), _ptr(cnt), _ptr(ws), ws.numel(), _stream(stream)),
               "kv1b_attend_topp")
        return out, sel, cnt

    def attend_select(self, q: torch.Tensor, scale: float, mode: int, p: float = 1.0, k: int = 0, sink: int = 0,
                      recent: int = 0, out=None, sel=None, cnt=None, stream=None):
        """Top-p (mode SELECT_TOPP, fraction p) or Top-k (SELECT_TOPK, budget k) selection plus the
        always-kept first `sink` / last `recent` tokens, then attention over the set.  Returns
        (out fp32 [B, Hq, 128], sel_idx int32 [B, Hq, capacity], sel_cnt int32 [B, Hq])."""
        B, Hq, D = q.shape
        if out is None:
            out = torch.empty((B, Hq, D), dtype=torch.float32, device=q.device)
        if sel is None:
            sel = torch.empty((B, Hq, self.capacity), dtype=torch.int32, device=q.device)
        if cnt is None:
            cnt = torch.empty((B, Hq), dtype=torch.int32, device=q.device)
        _check_buf(out, (B, Hq, D), torch.float32, "out")
        _check_buf(sel, (B, Hq, self.capacity), torch.int32, "sel")
        _check_buf(cnt, (B, Hq), torch.int32, "cnt")
        ws = self.workspace(Hq, 1)
        _check(lib().kv1b_attend_select(ctypes.byref(self.desc), _ptr(q), _dtype_code(q), Hq, float(scale), int(mode),
                                        float(p), int(k), int(sink), int(recent), _ptr(out), _ptr(sel), _ptr(cnt),
                                        _ptr(ws), ws.numel(), _stream(stream)), "kv1b_attend_select")
        return out, sel, cnt

    def attend_selected_exact(self, q: torch.Tensor, scale: float, k: torch.Tensor, v: torch.Tensor,
                              sel: torch.Tensor, cnt: torch.Tensor, out=None, stream=None) -> torch.Tensor:
        """Exact attention over selected tokens (e.g. attend_topp's sel / cnt) with the caller's exact keys
        and values k, v: [batch, tokens, num_kv_heads, 128], equal strides and dtype, unit channel stride
        (device memory, or host memory the device can address).  Returns fp32 [batch, num_q_heads, 128]."""
        B, Hq, D = q.shape
        if not q.is_contiguous():
            raise ValueError("q must be contiguous")
        if k.shape != v.shape or k.stride() != v.stride() or k.dtype != v.dtype:
            raise ValueError("k and v must have equal shapes, strides and dtypes")
        if k.dim() != 4 or (k.shape[0], k.shape[2], k.shape[3]) != (self.batch, self.num_kv_heads, HEAD_DIM) \
                or k.stride(3) != 1:
            raise ValueError("expected k, v of [batch, tokens, num_kv_heads, 128] with unit channel stride")
        _check_buf(sel, (B, Hq, self.capacity), torch.int32, "sel")
        _check_buf(cnt, (B, Hq), torch.int32, "cnt")
        if out is None:
            out = torch.empty((B, Hq, D), dtype=torch.float32, device=q.device)
        _check_buf(out, (B, Hq, D), torch.float32, "out")
        ws = self.workspace(Hq, 2)
        _check(lib().kv1b_attend_selected_exact(ctypes.byref(self.desc), _ptr(q), _dtype_code(q), Hq, float(scale),
                                                _ptr(k), _ptr(v), _dtype_code(k), k.shape[1], k.stride(0),
                                                k.stride(1), k.stride(2), _ptr(sel), _ptr(cnt), _ptr(out), _ptr(ws),
                                                ws.numel(), _stream(stream)), "kv1b_attend_selected_exact")
        return out

    def query_prep(self, q: torch.Tensor, stream=None) -> dict:
        B, Hq, _ = q.shape
        planes = torch.empty((B, Hq, 4, 4), dtype=torch.int32, device=q.device)
        vl = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
        dl = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
        sq = torch.empty((B, Hq), dtype=torch.int32, device=q.device)
        _check(lib().kv1b_query_prep(ctypes.byref(self.desc), _ptr(q), _dtype_code(q), Hq, _ptr(planes), _ptr(vl),
                                     _ptr(dl), _ptr(sq), _stream(stream)), "kv1b_query_prep")
        return {"planes": planes, "vl": vl, "delta": dl, "Sq": sq}

    def scores(self, q: torch.Tensor, scale: float, stream=None) -> dict:
        B, Hq, _ = q.shape
        shape = (B, Hq, self.capacity)
        A = torch.zeros(shape, dtype=torch.int32, device=q.device)
        Bc = torch.zeros(shape, dtype=torch.int32, device=q.device)
        s = torch.zeros(shape, dtype=torch.float32, device=q.device)
        _check(lib().kv1b_scores(ctypes.byref(self.desc), _ptr(q), _dtype_code(q), Hq, float(scale), _ptr(A), _ptr(Bc),
                                 _ptr(s), _stream(stream)), "kv1b_scores")
        return {"A": A, "Bc": Bc, "s": s}

    def scores_probe(self, q: torch.Tensor, scale: float, kernel: int, stream=None) -> dict:
        """The score integers and logits as `kernel` (PROBE_*) forms them (see kv1b_scores_probe):
        {"A", "Bc", "s"} [B, Hq, capacity], plus "out" for PROBE_ATTEND."""
        B, Hq, _ = q.shape
        shape = (B, Hq, self.capacity)
        A = torch.zeros(shape, dtype=torch.int32, device=q.device)
        Bc = torch.zeros(shape, dtype=torch.int32, device=q.device)
        s = torch.zeros(shape, dtype=torch.float32, device=q.device)
        out = torch.zeros((B, Hq, HEAD_DIM), dtype=torch.float32, device=q.device)
        ws = self.workspace(Hq, 1 if kernel == PROBE_TOPP else 0) if kernel != PROBE_POPC else None
        _check(lib().kv1b_scores_probe(ctypes.byref(self.desc), _ptr(q), _dtype_code(q), Hq, float(scale), int(kernel),
                                       _ptr(A), _ptr(Bc), _ptr(s), _ptr(out), _ptr(ws),
                                       ws.numel() if ws is not None else 0, _stream(stream)), "kv1b_scores_probe")
        if kernel == PROBE_ATTEND:  # the probe zeroes the merge counters itself and leaves them zero
            self._ws_clean[Hq] = True
        return {"A": A, "Bc": Bc, "s": s, "out": out}

    def attend_wait_probe(self, q: torch.Tensor, scale: float, wait_tries: int, stall_stage: int,
                          stream=None) -> torch.Tensor:
        """kv1b_attend's persistent kernel with bounded waits of `wait_tries` tries and, for
        stall_stage >= 0, the copies of that stage never issued (see kv1b_attend_wait_probe)."""
        B, Hq, D = q.shape
        out = torch.zeros((B, Hq, D), dtype=torch.float32, device=q.device)
        ws = self.workspace(Hq, 0)
        _check(lib().kv1b_attend_wait_probe(ctypes.byref(self.desc), _ptr(q), _dtype_code(q), Hq, float(scale),
                                            _ptr(out), _ptr(ws), ws.numel(), int(wait_tries), int(stall_stage),
                                            _stream(stream)), "kv1b_attend_wait_probe")
        self._ws_clean[Hq] = stall_stage < 0  # a stalled run may leave the merge counters set
        return out

    def status(self, stream=None) -> int:
        flags = ctypes.c_int32(0)
        _check(lib().kv1b_read_status(ctypes.byref(self.desc), ctypes.byref(flags), _stream(stream)),
               "kv1b_read_status")
        if flags.value & STATUS_TIMEOUT:  # a timed-out attend may leave its merge counters set
            self._ws_clean.clear()
        return flags.value


def merge_partials(parts: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Log-sum-exp merge of partial rows [n, ..., 130] (Cache.attend(partial=True) of n disjoint token
    ranges of the same sequences) into fp32 [..., 128] (kv1b_merge_partials)."""
    if parts.dtype != torch.float32 or not parts.is_contiguous() or parts.shape[-1] != PART_ROW or parts.dim() < 2:
        raise ValueError("parts must be a contiguous fp32 tensor [n, ..., 130]")
    lead = tuple(parts.shape[1:-1])
    rows = 1
    for x in lead:
        rows *= x
    if out is None:
        out = torch.empty(lead + (HEAD_DIM,), dtype=torch.float32, device=parts.device)
    _check_buf(out, lead + (HEAD_DIM,), torch.float32, "out")
    _check(lib().kv1b_merge_partials(_ptr(parts), parts.shape[0], rows, _ptr(out), _stream(stream)),
           "kv1b_merge_partials")
    return out


def attend_from_host(cache: Cache, q_host: torch.Tensor, k_new_host: torch.Tensor | None, v_new_host: torch.Tensor | None,
                     scale: float, out_host: torch.Tensor, q_dev: torch.Tensor, k_dev: torch.Tensor | None,
                     v_dev: torch.Tensor | None, stream=None) -> torch.Tensor:
    """One decode step with HOST buffers: copy the new token's K/V and the query from pinned host
    memory to the device, append, attend, copy the output back (all on one stream).  The copies in
    come first, so that the append and the attend follow each other directly (the attend is then
    scheduled while the append runs)."""
    s = stream if stream is not None else torch.cuda.current_stream()
    with torch.cuda.stream(s):
        if k_new_host is not None:
            k_dev.copy_(k_new_host, non_blocking=True)
            v_dev.copy_(v_new_host, non_blocking=True)
        q_dev.copy_(q_host, non_blocking=True)
        if k_new_host is not None:
            cache.append(k_dev, v_dev, stream=s)
        out = cache.attend(q_dev, scale, stream=s)
        out_host.copy_(out, non_blocking=True)
    return out_host


def step_block_views(block: torch.Tensor, batch: int, num_kv_heads: int, num_q_heads: int, dtype):
    """Views of one decode step's inputs packed in a uint8 block: the new token's K
    [batch, 1, num_kv_heads, 128], then its V, then the query [batch, num_q_heads, 128], all in
    `dtype`, each starting on a 256-byte multiple.  Returns (k, v, q)."""
    esz = torch.empty((), dtype=dtype).element_size()
    nk = batch * num_kv_heads * HEAD_DIM * esz
    nq = batch * num_q_heads * HEAD_DIM * esz
    if block.dtype != torch.uint8 or block.numel() < 2 * nk + nq or not block.is_contiguous():
        raise ValueError("block must be a contiguous uint8 tensor of at least step_block_bytes() bytes")
    k = block[:nk].view(dtype).view(batch, 1, num_kv_heads, HEAD_DIM)
    v = block[nk:2 * nk].view(dtype).view(batch, 1, num_kv_heads, HEAD_DIM)
    q = block[2 * nk:2 * nk + nq].view(dtype).view(batch, num_q_heads, HEAD_DIM)
    return k, v, q


def step_block_bytes(batch: int, num_kv_heads: int, num_q_heads: int, dtype) -> int:
    esz = torch.empty((), dtype=dtype).element_size()
    return (2 * batch * num_kv_heads + batch * num_q_heads) * HEAD_DIM * esz


def attend_from_host_block(cache: Cache, host_block: torch.Tensor, dev_block: torch.Tensor, num_q_heads: int, dtype,
                           scale: float, out_host: torch.Tensor, stream=None) -> torch.Tensor:
    """One decode step whose inputs (the new token's K and V and the query, laid out as
    step_block_views describes) sit in ONE pinned host block: one copy in, append, attend, the
    output copied back -- two copies per step instead of four."""
    s = stream if stream is not None else torch.cuda.current_stream()
    with torch.cuda.stream(s):
        dev_block.copy_(host_block, non_blocking=True)
        k, v, q = step_block_views(dev_block, cache.batch, cache.num_kv_heads, num_q_heads, dtype)
        cache.append(k, v, stream=s)
        out = cache.attend(q, scale, stream=s)
        out_host.copy_(out, non_blocking=True)
    return out_host


def unpack_codes(v_codes: torch.Tensor, length: int) -> torch.Tensor:
    """Logical codes [length, 128] (uint8) of one (sequence, kv-head) from the code plane
    [capacity/128, 128, 16] (128-token tiles, channel-major rows; nibble j of word w of a row is
    token 8w + j of the tile; layout in include/kv1b.h)."""
    w = v_codes.to(torch.int64) & 0xFFFFFFFF                       # [tiles, 128 ch, 16 words]
    ntile = (length + 127) // 128
    w = w[:ntile]
    shifts = torch.arange(8, device=w.device, dtype=torch.int64) * 4
    nib = (w[..., None] >> shifts) & 0xF                             # [tiles, 128 ch, 16 words, 8]
    out = nib.permute(0, 2, 3, 1).reshape(ntile * 128, HEAD_DIM)     # token = 128 tile + 8 word + j
    return out[:length].to(torch.uint8)
