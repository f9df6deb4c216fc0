"""CPU-only checks of the boundary: the C-ABI library loads and exports every symbol that
include/kv1b.h declares; the header compiles as plain C99 and a C program links against the
library; host-only size queries behave; the binding's struct mirrors the header.  No kernel is
launched here."""
import ctypes
import os
import re
import subprocess

import pytest

import long_context_decode_kv1b_b200 as kv
from long_context_decode_kv1b_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kv1b.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kv1b_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return kv.lib()


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(kv.SYMBOLS) == names


def test_version_and_status_strings(lib):
    assert lib.kv1b_version() == 100
    assert lib.kv1b_status_string(0) == b"ok"
    assert b"capacity" in lib.kv1b_status_string(-3)


def test_cache_bytes_host_rules(lib):
    n = lib.kv1b_cache_bytes(1, 8, 128, 1024)
    # 104 bytes per token-kv-head plus small aligned extras
    assert 104 * 8 * 1024 <= n <= 104 * 8 * 1024 + 4096
    assert lib.kv1b_cache_bytes(1, 8, 64, 1024) == 0      # head_dim must be 128
    assert lib.kv1b_cache_bytes(1, 8, 128, 1000) == 0     # capacity multiple of 128
    assert lib.kv1b_cache_bytes(65, 8, 128, 1024) == 0    # batch <= 64


def test_descriptor_layout_matches_header():
    # int32 x4, u64, 8 pointers, int64[64], int32 rotation_rounds + reserved
    assert ctypes.sizeof(kv.CacheDesc) == 16 + 8 + 8 * 8 + 8 * 64 + 8


def test_init_rounds_rejects_bad_round_counts_without_launching(lib):
    d = kv.CacheDesc()
    for rounds in (0, 4, -1):
        assert lib.kv1b_cache_init_rounds(ctypes.byref(d), ctypes.c_void_p(0x10000), 1 << 20, 1, 1, 128, 128, 0, rounds,
                                          None) == -1


def test_init_rejects_bad_arguments_without_launching(lib):
    d = kv.CacheDesc()
    # null buffer / misaligned buffer / short buffer are refused on the host
    assert lib.kv1b_cache_init(ctypes.byref(d), None, 0, 1, 1, 128, 128, 0, None) == -1
    assert lib.kv1b_cache_init(ctypes.byref(d), ctypes.c_void_p(0x1001), 1 << 20, 1, 1, 128, 128, 0, None) == -4
    assert lib.kv1b_cache_init(ctypes.byref(d), ctypes.c_void_p(0x10000), 16, 1, 1, 128, 128, 0, None) == -5
    assert lib.kv1b_cache_init(ctypes.byref(d), ctypes.c_void_p(0x10000), 1 << 20, 1, 1, 96, 128, 0, None) == -2


def test_attend_rejects_unknown_flag_bits_without_launching(lib):
    # a descriptor that passes the host checks (its pointers are never dereferenced on this path)
    d = kv.CacheDesc()
    d.batch, d.num_kv_heads, d.head_dim, d.capacity = 1, 1, 128, 128
    for name in ("k_bits", "k_norm", "k_cinv", "v_codes", "v_sm", "signs", "d_lengths", "d_status"):
        setattr(d, name, 0x10000)
    buf = ctypes.c_void_p(0x20000)
    for flags in (8, 16, 1 << 30, -1):  # bits 0-2 are the engine, KV1B_ATTEND_WS_CLEAN and KV1B_ATTEND_PARTIAL
        assert lib.kv1b_attend(ctypes.byref(d), buf, kv.DTYPE_F32, 4, ctypes.c_float(0.1), buf, buf, 1 << 20,
                               flags, 0, None) == -1


def test_header_is_plain_c_and_links(lib, tmp_path):
    # a C99 program that takes the address of every declared function and calls the host-only ones
    names = declared_functions()
    fns = ", ".join(f"(void (*)(void)){n}" for n in names)
    src = tmp_path / "abi_check.c"
    src.write_text(f"""#include <stdio.h>
#include "kv1b.h"
int main(void) {{
  void (*fns[])(void) = {{{fns}}};
  printf("%d %lu %d\\n", kv1b_version(), (unsigned long)kv1b_cache_bytes(1, 1, 128, 128),
         (int)(sizeof fns / sizeof fns[0]));
  return 0;
}}
""")
    exe = tmp_path / "abi_check"
    pkg = os.path.dirname(kv.LIB_PATH)
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
                           "-o", str(exe), str(src), "-L", pkg, "-lkv1b", "-Wl,-rpath," + pkg])
    out = subprocess.check_output([str(exe)], text=True).split()
    assert int(out[0]) == lib.kv1b_version()
    assert int(out[1]) == lib.kv1b_cache_bytes(1, 1, 128, 128)
    assert int(out[2]) == len(names)


def test_binding_passes_workspace_clean_flag_after_first_attend(monkeypatch):
    # the binding's bookkeeping against a fake library: the first attend on a workspace lets the
    # library zero the merge counters; later calls say they are clean; a timeout status resets that
    import types

    import torch

    calls, status = [], [0]

    class FakeLib:
        def kv1b_attend_workspace_bytes(self, desc, hq, mode):
            return 4096

        def kv1b_attend(self, desc, q, qdt, hq, scale, out, ws, n, flags, splits, stream):
            calls.append(flags)
            return 0

        def kv1b_read_status(self, desc, flags_ref, stream):
            flags_ref._obj.value = status[0]
            return 0

    fake = FakeLib()
    monkeypatch.setattr(kv, "lib", lambda: fake)
    c = kv.Cache.__new__(kv.Cache)
    c.desc, c._ws, c._ws_clean, c.device = kv.CacheDesc(), {}, {}, torch.device("cpu")
    q, out, st = torch.zeros((1, 4, 128)), torch.zeros((1, 4, 128)), types.SimpleNamespace(cuda_stream=0)
    c.attend(q, 0.1, out=out, stream=st)
    c.attend(q, 0.1, out=out, stream=st)
    c.attend(q, 0.1, out=out, engine=kv.ATTEND_CUDA_CORE, stream=st)
    assert calls == [kv.ATTEND_TENSOR, kv.ATTEND_WS_CLEAN, kv.ATTEND_CUDA_CORE | kv.ATTEND_WS_CLEAN]
    status[0] = kv.STATUS_TIMEOUT
    assert c.status(stream=st) == kv.STATUS_TIMEOUT
    c.attend(q, 0.1, out=out, stream=st)
    assert calls[-1] == kv.ATTEND_TENSOR


def test_step_block_views_layout():
    # one decode step's inputs in one block: K, then V, then q, each at a 256-byte multiple, each a
    # view of the block (a write through a view lands at the documented offset)
    import torch

    for dtype, esz in ((torch.bfloat16, 2), (torch.float32, 4)):
        B, Hkv, Hq = 3, 2, 8
        n = kv.step_block_bytes(B, Hkv, Hq, dtype)
        assert n == (2 * B * Hkv + B * Hq) * 128 * esz
        blk = torch.zeros(n, dtype=torch.uint8)
        k, v, q = kv.step_block_views(blk, B, Hkv, Hq, dtype)
        assert k.shape == (B, 1, Hkv, 128) and v.shape == (B, 1, Hkv, 128) and q.shape == (B, Hq, 128)
        nk = B * Hkv * 128 * esz
        assert v.data_ptr() - blk.data_ptr() == nk and q.data_ptr() - blk.data_ptr() == 2 * nk
        assert nk % 256 == 0
        v.fill_(1)
        assert blk[:nk].count_nonzero() == 0 and blk[nk:2 * nk].count_nonzero() > 0
        assert blk[2 * nk:].count_nonzero() == 0
        with pytest.raises(ValueError):
            kv.step_block_views(blk[:-1], B, Hkv, Hq, dtype)
