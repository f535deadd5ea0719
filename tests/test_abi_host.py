"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every
entry point include/cvq.h declares, reports sizes, and rejects bad arguments with a
status before launching anything.  Every call below carries at least one invalid
argument or has nothing to do (t_cap = 0), so none of them reaches a kernel launch."""
import ctypes
import math
import os
import re

import pytest

from compressed_attention_cvq_b200 import _binding as b

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "cvq.h")

FAKE = 0x10000          # an aligned, non-null address that is never dereferenced
MISALIGNED = 0x10008


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"CVQ_API\s+[\w\s\*]*?\b(cvq_\w+)\s*\(", src)))


def _shape(**kw):
    d = dict(batch=1, n_q_heads=32, n_kv_heads=8, R=2, t_cap=1024, rope_base=500000.0)
    d.update(kw)
    head_dim = d.pop("head_dim", 128)
    group_dim = d.pop("group_dim", 8)
    return b.make_shape(d["batch"], d["n_q_heads"], d["n_kv_heads"], d["R"], d["t_cap"],
                        d["rope_base"], head_dim, group_dim)


def test_every_declared_symbol_is_exported():
    names = _declared()
    assert len(names) >= 10
    lib = ctypes.CDLL(b.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(b.EXPORTED)


def test_abi_version_matches_header():
    v = int(re.search(r"#define CVQ_ABI_VERSION (\d+)", open(HEADER).read()).group(1))
    assert b.lib.cvq_abi_version() == v


def test_status_strings():
    for st, name in b.STATUS_NAMES.items():
        assert b.status_str(st).startswith(name)
    assert "unknown" in b.status_str(99)


def test_sizes():
    s = _shape()
    assert b.lib.cvq_ptable_bytes(ctypes.byref(s)) == 1 * 32 * 16 * 2 * 256 * 8 * 4
    assert b.lib.cvq_partials_bytes(ctypes.byref(s), 5) == 1 * 32 * 5 * 130 * 4
    assert b.lib.cvq_partials_bytes(ctypes.byref(s), 0) == 0
    assert b.lib.cvq_ptable_bytes(ctypes.byref(_shape(head_dim=64))) == 0


@pytest.mark.parametrize("t_cap,n,expect", [(1024, 1, 1024), (1024, 3, 384), (4096, 16, 256),
                                            (131072, 74, 1792), (1, 1, 64), (0, 4, 64),
                                            (100, 7, 64)])
def test_split_tokens(t_cap, n, expect):
    c = b.lib.cvq_split_tokens(ctypes.byref(_shape(t_cap=t_cap)), n)
    assert c == expect
    assert c % 64 == 0 and c * n >= t_cap


def test_suggest_splits_bounds():
    for t in (0, 64, 4096, 131072):
        n = b.lib.cvq_suggest_splits(ctypes.byref(_shape(t_cap=t)), 148)
        assert 1 <= n <= 4096


def _qtable(shape, q=FAKE, dt=0, kcb=FAKE, stride=0, P=FAKE):
    return b.lib.cvq_qtable(ctypes.byref(shape) if shape is not None else None, q, dt, kcb,
                            stride, P, None)


def test_qtable_errors():
    assert _qtable(None) == 1
    assert _qtable(_shape(), q=None) == 1
    assert _qtable(_shape(), P=MISALIGNED) == 3
    assert _qtable(_shape(), dt=7) == 4
    assert _qtable(_shape(head_dim=64)) == 4
    assert _qtable(_shape(R=3)) == 4
    assert _qtable(_shape(n_q_heads=12, n_kv_heads=8)) == 2
    assert _qtable(_shape(n_q_heads=48, n_kv_heads=3)) == 4       # group of 16
    assert _qtable(_shape(batch=0)) == 2
    assert _qtable(_shape(t_cap=-1)) == 2
    assert _qtable(_shape(rope_base=1.0)) == 2
    assert _qtable(_shape(), stride=-5) == 2
    assert _qtable(_shape(), stride=100) == 2                     # below one head's size
    assert _qtable(_shape(), stride=65536 + 2) == 3               # heads not 16-byte aligned


def _decode(shape, n_splits=4, **kw):
    a = dict(ptab=FAKE, kc=FAKE, vc=FAKE, lens=FAKE, vcb=FAKE, vstride=0, po=FAKE, pm=FAKE, pl=FAKE)
    a.update(kw)
    return b.lib.cvq_decode_attn(ctypes.byref(shape), a["ptab"], a["kc"], a["vc"], a["lens"],
                                 a["vcb"], a["vstride"], n_splits, a["po"], a["pm"], a["pl"], None)


def test_decode_errors():
    s = _shape()
    assert _decode(s, ptab=None) == 1
    assert _decode(s, kc=MISALIGNED) == 3
    assert _decode(s, vc=None) == 1
    assert _decode(s, lens=None) == 1
    assert _decode(s, lens=FAKE + 2) == 3
    assert _decode(s, n_splits=0) == 5
    assert _decode(s, n_splits=5000) == 5
    assert _decode(s, vstride=7) == 2
    assert _decode(s, po=None) == 1
    assert _decode(s, pm=FAKE + 1) == 3
    assert _decode(_shape(head_dim=96)) == 4


def _gqa(shape, n_splits=4, **kw):
    a = dict(q=FAKE, dt=0, kcb=FAKE, kstride=0, kc=FAKE, vc=FAKE, lens=FAKE, vcb=FAKE, vstride=0,
             po=FAKE, pm=FAKE, pl=FAKE)
    a.update(kw)
    return b.lib.cvq_decode_attn_gqa(ctypes.byref(shape), a["q"], a["dt"], a["kcb"], a["kstride"],
                                     a["kc"], a["vc"], a["lens"], a["vcb"], a["vstride"], n_splits,
                                     a["po"], a["pm"], a["pl"], None)


def test_decode_gqa_errors():
    s = _shape()
    assert _gqa(s, q=None) == 1
    assert _gqa(s, dt=2) == 4
    assert _gqa(s, kcb=MISALIGNED) == 3
    assert _gqa(s, kstride=1) == 2
    assert _gqa(s, pl=None) == 1
    assert _gqa(_shape(n_q_heads=64, n_kv_heads=8, R=2)) in (4,)    # group 8 with R = 2
    assert _gqa(s, n_splits=-1) == 5


def test_combine_errors():
    s = _shape()
    f = b.lib.cvq_combine
    assert f(ctypes.byref(s), 0, FAKE, FAKE, FAKE, FAKE, FAKE, None) == 5
    assert f(ctypes.byref(s), 2, None, FAKE, FAKE, FAKE, FAKE, None) == 1
    assert f(ctypes.byref(s), 2, FAKE, FAKE, FAKE, MISALIGNED, FAKE, None) == 3
    assert f(ctypes.byref(s), 2, FAKE, FAKE, FAKE, FAKE, FAKE + 2, None) == 3
    assert f(None, 2, FAKE, FAKE, FAKE, FAKE, FAKE, None) == 1


def test_missing_library_fails_loudly(monkeypatch):
    monkeypatch.setattr(b, "LIB_PATH", os.path.join(ROOT, "no_such_libcvq.so"))
    with pytest.raises(ImportError):
        b._load()


def test_product_never_touches_oracle():
    """Neither the package nor its C/CUDA sources refer to the oracle."""
    pkg = os.path.join(ROOT, "compressed_attention_cvq_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                src = open(os.path.join(dirpath, fn)).read()
                assert not re.search(r"\boracle\b", src), fn


def _encode(shape, **kw):
    a = dict(k=FAKE, v=FAKE, kcb=FAKE, kstride=0, vcb=FAKE, vstride=0, pos=FAKE, kc=FAKE, vc=FAKE)
    a.update(kw)
    return b.lib.cvq_encode_append(ctypes.byref(shape) if shape is not None else None, a["k"],
                                   a["v"], a["kcb"], a["kstride"], a["vcb"], a["vstride"],
                                   a["pos"], a["kc"], a["vc"], None)


def test_encode_append_errors():
    s = _shape()
    assert _encode(None) == 1
    assert _encode(s, k=None) == 1
    assert _encode(s, v=MISALIGNED) == 3
    assert _encode(s, pos=None) == 1
    assert _encode(s, kc=MISALIGNED) == 3
    assert _encode(s, vstride=16) == 2
    assert _encode(s, kstride=65536 + 1) == 3
    assert _encode(_shape(R=3)) == 4
    assert _encode(_shape(t_cap=0)) == 0           # nothing to write, no launch


def test_wide_layout_validation():
    """group_dim 64 (64-entry codebooks over 64-scalar groups): R up to 22, t_cap a
    multiple of 16, 4 query heads per KV head; only the GQA decode, the static entry,
    combine and the size helpers take it."""
    w = dict(group_dim=64, R=11, t_cap=1024)
    assert _gqa(_shape(**w), kcb=None) == 1                          # R = 11 accepted
    assert _gqa(_shape(**dict(w, R=23))) == 4
    assert _gqa(_shape(**dict(w, R=0))) == 4
    assert _gqa(_shape(**dict(w, t_cap=1000))) == 2                  # not a multiple of 16
    assert _gqa(_shape(**dict(w, n_q_heads=16))) == 4                # 2 heads per KV head
    assert _gqa(_shape(**w), kstride=8192 * 11 - 4) == 2             # below one head
    assert _gqa(_shape(**w), kstride=8192 * 11 + 2) == 3
    assert _gqa(_shape(group_dim=32)) == 4
    assert _qtable(_shape(**w)) == 4
    assert _decode(_shape(**w)) == 4
    assert _encode(_shape(**w), kc=None) == 1                        # the encoder takes it
    assert _encode(_shape(**w), vstride=8192 * 11 + 2) == 3
    assert b.lib.cvq_ptable_bytes(ctypes.byref(_shape(**w))) == 0
    assert b.lib.cvq_partials_bytes(ctypes.byref(_shape(**w)), 3) == 32 * 3 * 130 * 4
    assert b.lib.cvq_suggest_splits(ctypes.byref(_shape(**dict(w, t_cap=131072))), 148) == 9
    assert b.lib.cvq_suggest_splits(ctypes.byref(_shape(**dict(w, t_cap=32768, R=21))), 148) == 9


def test_attend_workspace_and_errors():
    s = _shape()
    n = b.lib.cvq_attend_workspace_bytes(ctypes.byref(s), 4)
    assert n == 32 * 4 * 130 * 4 + 32 * 4                          # partials, then counters
    assert b.lib.cvq_attend_workspace_bytes(ctypes.byref(_shape(batch=0)), 4) == 0

    def call(shape, **kw):
        a = dict(q=FAKE, kcb=FAKE, kc=FAKE, vc=FAKE, lens=FAKE, vcb=FAKE, ws=FAKE, out=FAKE,
                 lse=FAKE)
        a.update(kw)
        return b.lib.cvq_attend(ctypes.byref(shape), a["q"], 0, a["kcb"], 0, a["kc"], a["vc"],
                                a["lens"], a["vcb"], 0, 4, a["ws"], a["out"], a["lse"], None)
    assert call(s, ws=None) == 1
    assert call(s, ws=MISALIGNED) == 3
    assert call(s, out=MISALIGNED) == 3
    assert call(s, lse=None) == 1
    assert call(s, kcb=None) == 1
    assert call(_shape(R=3)) == 4


def test_static_entry_reports_shape_errors():
    fake = FAKE
    st = b.lib.cvq_attend_static(ctypes.byref(_shape(R=3)), fake, 0, fake, 0, fake, fake, fake,
                                 fake, 0, 4, fake, fake, None)
    assert st == 4
    st = b.lib.cvq_attend_static(ctypes.byref(_shape(n_q_heads=12)), fake, 0, fake, 0, fake,
                                 fake, fake, fake, 0, 4, fake, fake, None)
    assert st == 2


def test_fault_status_rejects_null():
    # checked before the device is touched
    assert b.lib.cvq_fault_status(None, 0) == 1
    assert b.lib.cvq_fault_status(None, 1) == 1


def test_plain_c_consumer(tmp_path):
    """cvq.h compiles as strict C99 and a C program links libcvq.so and gets the documented
    host-side behaviour (tests/c_abi/abi_check.c; nothing it calls launches a kernel)."""
    import shutil
    import subprocess

    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    lib_dir = os.path.dirname(b.LIB_PATH)
    exe = str(tmp_path / "abi_check")
    src = os.path.join(ROOT, "tests", "c_abi", "abi_check.c")
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(ROOT, "include"), src, "-o", exe, "-L", lib_dir, "-lcvq",
                    f"-Wl,-rpath,{lib_dir}"], check=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    assert "c abi ok" in r.stdout


def test_attend_more_argument_errors():
    """Further cvq_attend argument errors, each caught on the host before the device is
    touched: split count range, alignments, query dtype, RoPE base, group size, batch."""
    def call(shape, n_splits=4, q_dtype=0, **kw):
        a = dict(q=FAKE, kcb=FAKE, kc=FAKE, vc=FAKE, lens=FAKE, vcb=FAKE, ws=FAKE, out=FAKE,
                 lse=FAKE)
        a.update(kw)
        return b.lib.cvq_attend(ctypes.byref(shape), a["q"], q_dtype, a["kcb"], 0, a["kc"],
                                a["vc"], a["lens"], a["vcb"], 0, n_splits, a["ws"], a["out"],
                                a["lse"], None)
    s = _shape()
    assert call(s, n_splits=0) == 5
    assert call(s, n_splits=4097) == 5
    assert call(s, lse=FAKE + 2) == 3
    assert call(s, lens=FAKE + 2) == 3
    assert call(s, q_dtype=7) == 4
    assert call(_shape(rope_base=1.0)) == 2
    assert call(_shape(rope_base=float("nan"))) == 2
    assert call(_shape(n_q_heads=24, n_kv_heads=8)) == 4          # 3 query heads per KV head
    assert call(_shape(n_q_heads=30, n_kv_heads=8)) == 2          # not a multiple
    assert call(_shape(batch=70000)) == 2


def test_debug_build_exports_every_symbol():
    """The debug build (device-side range checks) is the same ABI."""
    path = os.path.join(os.path.dirname(b.LIB_PATH), "libcvq_debug.so")
    if not os.path.exists(path):
        pytest.skip("libcvq_debug.so not built (python -m compressed_attention_cvq_b200.build --debug-bounds)")
    lib = ctypes.CDLL(path)
    for n in _declared():
        assert hasattr(lib, n), n


def test_fault_bits_match_header_and_decode():
    src = open(HEADER).read()
    bits = {m.group(1): int(m.group(2)) for m in re.finditer(r"#define (CVQ_FAULT_\w+) (\d+)u", src)}
    assert bits == {"CVQ_FAULT_COPY_TIMEOUT": b.CVQ_FAULT_COPY_TIMEOUT, "CVQ_FAULT_BOUNDS": b.CVQ_FAULT_BOUNDS}
    assert b.CVQ_FAULT_COPY_TIMEOUT == 1 and b.CVQ_FAULT_BOUNDS == 2
    assert b.fault_names(0) == []
    assert b.fault_names(1) == ["copy_timeout"]
    assert b.fault_names(2) == ["bounds"]
    assert b.fault_names(3) == ["copy_timeout", "bounds"]
    assert b.fault_names(2 | 16) == ["bounds", "0x10"]


def test_packed_code_layout_validation():
    """code_bits: 0 / 8 one byte per code, 6 packed (64-scalar groups only, t_cap a multiple
    of 64); every error is returned before any launch (fake pointers are never touched)."""
    s = _shape(group_dim=64, R=11, t_cap=1024, n_q_heads=8, n_kv_heads=2)
    s.code_bits = 6
    # sizes do not depend on the code storage
    s8 = _shape(group_dim=64, R=11, t_cap=1024, n_q_heads=8, n_kv_heads=2)
    assert b.lib.cvq_partials_bytes(ctypes.byref(s), 4) == b.lib.cvq_partials_bytes(ctypes.byref(s8), 4)
    bad = _shape(group_dim=64, R=11, t_cap=1040, n_q_heads=8, n_kv_heads=2)   # 16 | t_cap, 64 does not
    bad.code_bits = 6
    assert b.lib.cvq_pack_codes6(ctypes.byref(bad), FAKE, FAKE, None) == 2          # CVQ_ERR_SHAPE
    narrow = _shape()
    narrow.code_bits = 6
    assert b.lib.cvq_pack_codes6(ctypes.byref(narrow), FAKE, FAKE, None) == 4       # UNSUPPORTED
    odd = _shape(group_dim=64, R=11, t_cap=1024, n_q_heads=8, n_kv_heads=2)
    odd.code_bits = 7
    assert b.lib.cvq_pack_codes6(ctypes.byref(odd), FAKE, FAKE, None) == 4
    unpacked = _shape(group_dim=64, R=11, t_cap=1024, n_q_heads=8, n_kv_heads=2)  # code_bits 0
    assert b.lib.cvq_pack_codes6(ctypes.byref(unpacked), FAKE, FAKE, None) == 4
    assert b.lib.cvq_pack_codes6(ctypes.byref(s), None, FAKE, None) == 1             # NULL
    assert b.lib.cvq_pack_codes6(ctypes.byref(s), FAKE, MISALIGNED, None) == 3       # ALIGN
    # the decode refuses a packed narrow layout and a packed t_cap off the 64 grid
    st = b.lib.cvq_decode_attn_gqa(ctypes.byref(narrow), FAKE, 0, FAKE, 0, FAKE, FAKE, FAKE, FAKE,
                                   0, 2, FAKE, FAKE, FAKE, None)
    assert st == 4
    st = b.lib.cvq_decode_attn_gqa(ctypes.byref(bad), FAKE, 0, FAKE, 0, FAKE, FAKE, FAKE, FAKE,
                                   0, 2, FAKE, FAKE, FAKE, None)
    assert st == 2


def test_c_attend_loop_compiles(tmp_path):
    """The C driver of cvq_attend (tests/c_abi/attend_loop.c) builds with -Wall -Wextra
    -Werror against cvq.h, libcvq.so and the CUDA runtime; without a GPU it reports the CUDA
    error and exits non-zero instead of crashing."""
    import subprocess
    import sys

    sys.path.insert(0, os.path.join(ROOT, "tests", "c_abi"))
    import build_attend_loop

    try:
        exe = build_attend_loop.build(str(tmp_path / "attend_loop"))
    except RuntimeError as e:
        pytest.skip(str(e))
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 1 and "usage" in r.stderr


def _valid_by_header(b, hq, hkv, hd, R, t_cap, base, gd, cb):
    """The shape rules cvq.h states for cvq_shape, restated."""
    if hd != 128 or gd not in (0, 8, 64) or cb not in (0, 8, 6):
        return False
    if gd == 64:
        if not 1 <= R <= 22 or t_cap % 16 != 0 or (cb == 6 and t_cap % 64 != 0):
            return False
    elif R not in (1, 2) or cb == 6:
        return False
    if not (1 <= b <= 65535 and 1 <= hq <= 65535 and hkv >= 1 and t_cap >= 0):
        return False
    if hq % hkv != 0 or hq // hkv not in (1, 2, 4, 8):
        return False
    return math.isfinite(base) and base > 1.0


def test_shape_rules_match_the_header():
    """Random shapes, many of them invalid in one field: the library accepts exactly the
    shapes the header's rules accept (cvq_partials_bytes > 0), and then sizes the partial
    states as B x Hq x n_splits x 130 floats."""
    import random

    b_ = b
    rng = random.Random(12345)
    pick = lambda *xs: xs[rng.randrange(len(xs))]
    for _ in range(4000):
        bb = pick(1, 2, 7, 0, -1, 65535, 65536)
        hkv = pick(1, 2, 3, 8, 0)
        hq = pick(hkv, 2 * hkv, 4 * hkv, 8 * hkv, 3 * hkv, 16 * hkv, hkv + 1, 0, 70000)
        hd = pick(128, 128, 128, 64)
        R = pick(1, 2, 3, 11, 21, 22, 23, 0)
        gd = pick(0, 8, 64, 64, 16)
        cb = pick(0, 8, 6, 6, 4)
        t_cap = pick(0, 64, 100, 96, 4096, 131072, -1)
        base = pick(500000.0, 10000.0, 1.0, 0.5, float("inf"), float("nan"))
        s = b_.make_shape(bb, hq, hkv, R, t_cap, base, head_dim=hd, group_dim=gd, code_bits=cb)
        n = rng.randrange(1, 40)
        got = b_.lib.cvq_partials_bytes(ctypes.byref(s), n)
        ok = _valid_by_header(bb, hq, hkv, hd, R, t_cap, base, gd, cb)
        assert (got > 0) == ok, (bb, hq, hkv, hd, R, t_cap, base, gd, cb, got)
        if ok:
            assert got == bb * hq * n * 130 * 4
