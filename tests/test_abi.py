"""The C ABI library loads, exports every symbol include/pkv.h declares, and its
host-side argument checks reject bad calls before anything is launched.

No GPU: the checks below return before any CUDA call (pointers are fake but
never dereferenced on the host)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pkv.h")


@pytest.fixture(scope="module")
def lib():
    from paged_kv_cache_439_b200 import build, _native
    build.build()
    return _native.lib()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pkv_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = _declared()
    for required in ("pkv_kv_cache_append", "pkv_paged_attention_decode", "pkv_workspace_size",
                     "pkv_decode_num_splits", "pkv_strerror", "pkv_copy", "pkv_version"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    from paged_kv_cache_439_b200 import _native
    out = subprocess.run(["nm", "-D", "--defined-only", _native.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\s[TW]\s+(pkv_\w+)", out))
    missing = [n for n in _declared() if n not in exported]
    assert not missing, missing
    for n in _declared():
        assert hasattr(lib, n)
    # and the binding's prototype table covers them all
    assert set(_native.SIGNATURES) == set(_declared())


def test_strerror_and_version(lib):
    assert lib.pkv_strerror(0) == b"ok"
    for s in range(-8, 0):
        assert lib.pkv_strerror(s) and lib.pkv_strerror(s) != b"unknown pkv status"
    assert lib.pkv_version() >> 16 == 1


FAKE = 0x10000  # 16-byte aligned, never dereferenced by the host checks


def _decode(lib, **kw):
    a = dict(out=FAKE, q=FAKE, q_dt=1, k=FAKE, v=FAKE, cdt=1, ks=None, vs=None, bt=FAKE,
             maxb=4, cl=FAKE, maxctx=64, B=2, nq=8, nkv=2, d=128, bs=16, nb=10, scale=0.1,
             ws=None, wsb=0, splits=1, err=None, stream=None)
    a.update(kw)
    return lib.pkv_paged_attention_decode(
        a["out"], a["q"], a["q_dt"], a["k"], a["v"], a["cdt"], a["ks"], a["vs"], a["bt"],
        a["maxb"], a["cl"], a["maxctx"], a["B"], a["nq"], a["nkv"], a["d"], a["bs"], a["nb"],
        a["scale"], a["ws"], a["wsb"], a["splits"], a["err"], a["stream"])


def test_decode_argument_errors(lib):
    assert _decode(lib, nq=6, nkv=4) == -1            # n_q % n_kv != 0
    assert _decode(lib, out=None) == -1
    assert _decode(lib, B=-1) == -1
    assert _decode(lib, d=96) == -3                    # head_dim outside {64, 128}
    assert _decode(lib, bs=12) == -3                   # not a power of two
    assert _decode(lib, bs=512) == -3
    assert _decode(lib, nq=34, nkv=2) == -3            # group 17 > 16
    assert _decode(lib, cdt=1, q_dt=0) == -2           # bf16 cache needs bf16 q
    assert _decode(lib, cdt=7) == -2
    assert _decode(lib, cdt=2) == -1                   # int8 without scales
    assert _decode(lib, q=FAKE + 8) == -7              # misaligned
    assert _decode(lib, splits=2, maxctx=64) == -5     # split-K without workspace
    assert _decode(lib, B=0) == 0                      # nothing to do
    assert _decode(lib, scale=float("nan")) == -1
    # each split holds at most 8192 tokens
    assert _decode(lib, maxb=1024, maxctx=16384, splits=1) == -4


def test_fused_decode_append_argument_errors(lib):
    def call(**kw):
        a = dict(out=FAKE, q=FAKE, k=FAKE, v=FAKE, sm=FAKE, idt=1, kc=FAKE, vc=FAKE, cdt=1,
                 ks=None, vs=None, bt=FAKE, maxb=4, cl=FAKE, maxctx=64, B=2, nq=4, nkv=2, d=128,
                 bs=16, nb=8, scale=0.125, ws=None, wsb=0, splits=1, err=None)
        a.update(kw)
        return lib.pkv_paged_attention_decode_append(
            a["out"], a["q"], a["k"], a["v"], a["sm"], a["idt"], a["kc"], a["vc"], a["cdt"],
            a["ks"], a["vs"], a["bt"], a["maxb"], a["cl"], a["maxctx"], a["B"], a["nq"], a["nkv"],
            a["d"], a["bs"], a["nb"], a["scale"], a["ws"], a["wsb"], a["splits"], a["err"], None)
    assert call(k=None) == -1
    assert call(sm=None) == -1
    assert call(cdt=0, idt=0) == -4                    # fp32 caches: append, then decode
    assert call(idt=0) == -2                           # new rows must be bf16
    assert call(k=FAKE + 8) == -7                      # misaligned rows
    assert call(sm=FAKE + 4) == -7                     # misaligned slot mapping
    assert call(cdt=2) == -1                           # int8 without scales
    assert call(nq=6, nkv=4) == -1                     # decode checks apply as well
    assert call(B=0) == 0


def test_fused_shared_prefix_argument_errors(lib):
    def call(**kw):
        a = dict(out=FAKE, q=FAKE, k=FAKE, v=FAKE, sm=FAKE, idt=1, kc=FAKE, vc=FAKE, cdt=1,
                 bt=FAKE, maxb=16, cl=FAKE, maxctx=200, B=2, nq=4, nkv=2, d=128, bs=16, nb=32,
                 scale=0.125, prefix=128, ws=None, wsb=0, splits=1, err=None)
        a.update(kw)
        return lib.pkv_paged_attention_decode_shared_prefix_append(
            a["out"], a["q"], a["k"], a["v"], a["sm"], a["idt"], a["kc"], a["vc"], a["cdt"],
            a["bt"], a["maxb"], a["cl"], a["maxctx"], a["B"], a["nq"], a["nkv"], a["d"],
            a["bs"], a["nb"], a["scale"], a["prefix"], a["ws"], a["wsb"], a["splits"], a["err"],
            None)
    assert call(v=None) == -1
    assert call(cdt=2) == -4                           # bf16 caches only
    assert call(idt=0) == -2
    assert call(sm=FAKE + 4) == -7
    assert call(prefix=-16) == -1
    assert call(prefix=24) == -1                       # not a multiple of block_size
    assert call(B=0) == 0


def test_append_argument_errors(lib):
    def call(**kw):
        a = dict(k=FAKE, v=FAKE, sm=FAKE, T=4, nkv=2, d=64, idt=1, kc=FAKE, vc=FAKE, cdt=1, nb=4,
                 bs=16, ks=None, vs=None, err=None)
        a.update(kw)
        return lib.pkv_kv_cache_append(a["k"], a["v"], a["sm"], a["T"], a["nkv"], a["d"],
                                       a["idt"], a["kc"], a["vc"], a["cdt"], a["nb"], a["bs"],
                                       a["ks"], a["vs"], a["err"], None)
    assert call(T=-1) == -1
    assert call(kc=None) == -1
    assert call(d=80) == -3
    assert call(bs=6) == -3
    assert call(idt=2) == -2                  # int8 input
    assert call(idt=0, cdt=1) == -2           # fp32 -> bf16 cache not supported
    assert call(cdt=2) == -1                  # int8 cache without scales
    assert call(k=FAKE + 4) == -7
    assert call(T=0) == 0                     # empty append is a no-op


def test_shared_prefix_argument_errors(lib):
    def call(**kw):
        a = dict(out=FAKE, q=FAKE, q_dt=1, k=FAKE, v=FAKE, cdt=1, bt=FAKE, maxb=8, cl=FAKE,
                 maxctx=128, B=2, nq=8, nkv=2, d=128, bs=16, nb=20, scale=0.1, prefix=32,
                 ws=None, wsb=0, splits=0, err=None)
        a.update(kw)
        return lib.pkv_paged_attention_decode_shared_prefix(
            a["out"], a["q"], a["q_dt"], a["k"], a["v"], a["cdt"], None, None, a["bt"],
            a["maxb"], a["cl"], a["maxctx"], a["B"], a["nq"], a["nkv"], a["d"], a["bs"], a["nb"],
            a["scale"], a["prefix"], a["ws"], a["wsb"], a["splits"], a["err"], None)
    assert call(prefix=-16) == -1
    assert call(prefix=24) == -1                 # not a multiple of block_size
    assert call(prefix=16 * 9) == -1             # beyond the block-table capacity
    assert call(cdt=2) == -4                     # int8 cache: not supported by this call
    assert call(q_dt=0) == -2
    assert call(nq=6, nkv=4) == -1
    assert call() == -5                          # the prefix pass always needs a workspace
    need = lib.pkv_shared_prefix_workspace_size(2, 8, 2, 128, 128, 32, 1, 0)
    assert need > 0
    assert call(B=0, ws=FAKE, wsb=need) == 0


def test_workspace_sizes(lib):
    # one split -> no workspace; explicit splits -> o and lse per (seq, head, split)
    assert lib.pkv_workspace_size(4, 8, 2, 128, 64, 1, 1) == 0
    rows = 4 * 8 * 3
    o = -(-rows * 128 * 4 // 256) * 256
    lse = -(-rows * 4 // 256) * 256
    assert lib.pkv_workspace_size(4, 8, 2, 128, 4000, 1, 3) == o + lse
    # the automatic choice is consistent with pkv_decode_num_splits
    s = lib.pkv_decode_num_splits(16, 8, 128, 32768, 1)
    assert s >= 4   # 32768 tokens need at least 4 splits of <= 8192
    rows = 16 * 64 * s
    assert lib.pkv_workspace_size(16, 64, 8, 128, 32768, 1, 0) == \
        -(-rows * 128 * 4 // 256) * 256 + -(-rows * 4 // 256) * 256


def _header_prototypes():
    """name -> (return type, [parameter types]) for every declaration in pkv.h."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    protos = {}
    for m in re.finditer(r"([A-Za-z_][\w \*]*?)\b(pkv_[a-z0-9_]+)\s*\(([^;{]*?)\)\s*;", text):
        ret, name, params = m.group(1).strip(), m.group(2), m.group(3).strip()
        types = []
        if params and params != "void":
            for p in params.split(","):
                p = " ".join(p.split())
                # drop the parameter name: the last identifier not followed by '*'
                types.append(re.sub(r"\s*\b\w+$", "", p) if not p.endswith("*") else p)
        protos[name] = (ret, types)
    return protos


def _kind(c_type: str) -> str:
    t = c_type.replace("const ", "").strip()
    if "*" in t or t == "pkv_stream_t":
        return "pointer"
    return {"int": "int", "pkv_dtype": "int", "int32_t": "int", "int64_t": "int64",
            "size_t": "size_t", "float": "float", "void": "void"}[t]


def test_binding_prototypes_match_the_header():
    """Each ctypes prototype has the header's parameter count and, position by
    position, the same kind of type, so no argument is passed in the wrong
    register or width."""
    import ctypes
    from paged_kv_cache_439_b200 import _native
    kind_of = {ctypes.c_void_p: "pointer", ctypes.c_char_p: "pointer", ctypes.c_int: "int",
               ctypes.c_int32: "int", ctypes.c_int64: "int64", ctypes.c_size_t: "size_t",
               ctypes.c_float: "float", None: "void"}

    def ck(t):
        if t in kind_of:
            return kind_of[t]
        return "pointer" if issubclass(t, ctypes._Pointer) else repr(t)

    protos = _header_prototypes()
    assert set(protos) == set(_native.SIGNATURES)
    for name, (res, args) in _native.SIGNATURES.items():
        ret, params = protos[name]
        assert [ck(a) for a in args] == [_kind(p) for p in params], name
        assert ck(res) == _kind(ret), name


@pytest.mark.parametrize("cache_dt", [0, 1, 2, 3])
def test_split_plans_cover_the_context_in_bounded_chunks(lib, cache_dt):
    """For every shape the automatic split count covers max_context_len with
    16-token-aligned chunks of at most 8192 tokens (the block-table slice a CTA
    stages in shared memory), and the workspace size matches that count."""
    def ceil(a, b):
        return -(-a // b)
    for max_ctx in (1, 15, 16, 17, 255, 256, 4096, 8192, 8193, 32768, 100_000, 1 << 20):
        for num_seqs in (1, 2, 16, 64, 512):
            for nkv in (1, 8, 40):
                s = lib.pkv_decode_num_splits(num_seqs, nkv, 128, max_ctx, cache_dt)
                assert s >= max(1, ceil(max_ctx, 8192)), (max_ctx, num_seqs, nkv, s)
                chunk = ceil(ceil(max_ctx, s), 16) * 16
                assert chunk <= 8192 and s * chunk >= max_ctx and (s - 1) * chunk < max_ctx
                rows = num_seqs * nkv * s
                want = 0 if s == 1 else ceil(rows * 128 * 4, 256) * 256 + ceil(rows * 4, 256) * 256
                assert lib.pkv_workspace_size(num_seqs, nkv, nkv, 128, max_ctx, cache_dt, 0) == want


def test_shared_prefix_plan(lib):
    import ctypes
    ps, ss = ctypes.c_int(0), ctypes.c_int(0)

    def plan(*a):
        return lib.pkv_shared_prefix_plan(*a, ctypes.byref(ps), ctypes.byref(ss))

    # 64 sequences x 8 KV heads, 4096 shared tokens, suffixes up to 505 tokens:
    # the (sequence, head) units fill the first wave, and the prefix pass fills
    # the rest, so the automatic suffix plan does not split
    assert plan(64, 32, 8, 128, 4601, 4096, 1, 0) == 0
    assert ss.value == 1 and ps.value >= 1
    # the plan is the one the workspace size is computed from
    slots = ps.value + ss.value
    rows = 64 * 32 * slots
    assert lib.pkv_shared_prefix_workspace_size(64, 32, 8, 128, 4601, 4096, 1, 0) == \
        -(-rows * 128 * 4 // 256) * 256 + -(-rows * 4 // 256) * 256
    # an explicit split count is kept
    assert plan(64, 32, 8, 128, 4601, 4096, 1, 2) == 0 and ss.value == 2
    # few units and a long suffix: the suffix is split to occupy the device
    assert plan(1, 8, 8, 128, 4096 + 20000, 4096, 1, 0) == 0 and ss.value > 1
    # argument errors; NULL outputs are allowed
    assert plan(64, 32, 8, 128, 4601, 0, 1, 0) == -1
    assert plan(64, 30, 8, 128, 4601, 4096, 1, 0) == -1
    assert plan(0, 32, 8, 128, 4601, 4096, 1, 0) == -1
    assert lib.pkv_shared_prefix_plan(64, 32, 8, 128, 4601, 4096, 1, 0, None, None) == 0
