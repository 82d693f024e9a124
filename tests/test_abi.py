"""CPU-only checks of the C-ABI library: it loads without a GPU, exports every symbol the
header declares, and its host-side argument checks and size helpers behave as documented.
No call here reaches a CUDA launch."""
import ctypes
import json
import os
import re

import pytest
import torch

import qwen3_qk_norm_rope_b200 as qa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qwen3_attn.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qwen3_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = qa.lib()
    names = declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(qa.SIGNATURES) == names


def test_version_and_status_strings():
    assert "sm_100a" in qa.version()
    for code in range(6):
        assert qa.status_string(code) and qa.status_string(code) != "unknown status"
    assert qa.status_string(99) == "unknown status"


def test_workspace_and_cache_sizes():
    # K' [B, Hkv, T, d] and Q' (as many elements as q) in bf16
    assert qa.prefill_workspace_size(2, 2048, 16, 8) >= 2 * 2048 * (16 + 8) * 128 * 2
    assert qa.prefill_workspace_size(0, 10, 16, 8) == 0
    ns = -(-32769 // 1024)
    assert qa.decode_workspace_size(64, 32, 32769) >= 64 * 32 * ns * (128 + 1) * 4
    # 2*Hkv*d values per token per layer; 1024 for the wide-GQA block of the worked example
    gold = json.load(open(os.path.join(ROOT, "tests", "golden", "worked_examples.json")))["wide_gqa_block"]
    per_token_bytes = qa.kv_cache_bytes(1, gold["n_kv_heads"], 1, gold["head_dim"])
    assert per_token_bytes // 2 == gold["kv_cache_values_per_token_per_layer"]
    assert qa.kv_cache_bytes(64, 8, 32769, 128) == 2 * 64 * 8 * 32769 * 128 * 2


FAKE = ctypes.c_void_p(1 << 20)  # aligned, never dereferenced: every call below fails its host checks


def _prefill_ex(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, gq=FAKE, gk=FAKE, pos=FAKE, out=FAKE, lse=None, kc=None, vc=None, Tcap=0,
             ws=None, ws_bytes=0, B=1, T=128, Hq=16, Hkv=8, d=128, theta=1e6, eps=1e-6)
    a.update(kw)
    return qa.lib().qwen3_attn_prefill_ex(a["q"], a["k"], a["v"], a["gq"], a["gk"], a["pos"], a["out"], a["lse"],
                                          a["kc"], a["vc"], a["Tcap"], a["ws"], a["ws_bytes"], a["B"], a["T"],
                                          a["Hq"], a["Hkv"], a["d"], a["theta"], a["eps"], None)


def test_prefill_argument_checks():
    assert _prefill_ex(q=None) == qa.ERR_INVALID_ARG
    assert _prefill_ex(out=None) == qa.ERR_INVALID_ARG
    assert _prefill_ex(B=0) == qa.ERR_INVALID_ARG
    assert _prefill_ex(T=-1) == qa.ERR_INVALID_ARG
    assert _prefill_ex(d=64) == qa.ERR_UNSUPPORTED
    assert _prefill_ex(Hq=12, Hkv=8) == qa.ERR_UNSUPPORTED
    assert _prefill_ex(Hq=24, Hkv=8) == qa.ERR_UNSUPPORTED  # G = 3 is not a power of two
    assert _prefill_ex(Hq=256, Hkv=1) == qa.ERR_UNSUPPORTED  # G > 128
    assert _prefill_ex(q=ctypes.c_void_p((1 << 20) + 2)) == qa.ERR_INVALID_ARG  # misaligned
    assert _prefill_ex(kc=FAKE) == qa.ERR_INVALID_ARG  # k_cache without v_cache
    assert _prefill_ex(kc=FAKE, vc=FAKE, Tcap=64) == qa.ERR_INVALID_ARG  # Tcap < T
    assert _prefill_ex(theta=0.0, ws=FAKE, ws_bytes=1 << 30) == qa.ERR_INVALID_ARG
    assert _prefill_ex() == qa.ERR_WORKSPACE
    assert _prefill_ex(ws=FAKE, ws_bytes=100) == qa.ERR_WORKSPACE


def _chunk(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, gq=FAKE, gk=FAKE, pos=FAKE, out=FAKE, lse=None, kc=FAKE, vc=FAKE, start=256,
             Tcap=512, ws=None, ws_bytes=0, B=1, T=128, Hq=16, Hkv=8, d=128, theta=1e6, eps=1e-6)
    a.update(kw)
    return qa.lib().qwen3_attn_prefill_chunk(a["q"], a["k"], a["v"], a["gq"], a["gk"], a["pos"], a["out"],
                                             a["lse"], a["kc"], a["vc"], a["start"], a["Tcap"], a["ws"],
                                             a["ws_bytes"], a["B"], a["T"], a["Hq"], a["Hkv"], a["d"], a["theta"],
                                             a["eps"], None)


def test_chunked_prefill_argument_checks():
    assert _chunk(kc=None, vc=None) == qa.ERR_INVALID_ARG  # the chunk needs the caches
    assert _chunk(vc=None) == qa.ERR_INVALID_ARG
    assert _chunk(start=-1) == qa.ERR_INVALID_ARG
    assert _chunk(start=385) == qa.ERR_INVALID_ARG  # start + T > Tcap
    assert _chunk(Tcap=0, start=0) == qa.ERR_INVALID_ARG
    assert _chunk(Hq=24) == qa.ERR_UNSUPPORTED
    assert _chunk(kc=ctypes.c_void_p((1 << 20) + 8)) == qa.ERR_INVALID_ARG  # misaligned cache
    assert _chunk(start=384) == qa.ERR_WORKSPACE  # start + T == Tcap is valid; no workspace given
    assert _chunk(ws=FAKE, ws_bytes=100) == qa.ERR_WORKSPACE
    # prefill_ex has no start: a cached prefix needs the chunked call
    assert _prefill_ex(kc=FAKE, vc=FAKE, Tcap=128) == qa.ERR_WORKSPACE


def test_variant_argument_checks():
    lib = qa.lib()
    good, _ = qa.make_variant(1e6, None, 1.0, 0)

    def pre(var):
        return lib.qwen3_attn_prefill_variant(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None, 0, 0, None,
                                              0, 1, 128, 16, 8, 128, var, 1e-6, None)

    def dec(var):
        return lib.qwen3_attn_decode_variant(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 4, 32, 8,
                                             128, 1000, var, 1e-6, None, 0, None)

    assert pre(ctypes.byref(good)) == qa.ERR_WORKSPACE  # a valid variant gets as far as the workspace check
    assert dec(ctypes.byref(good)) == qa.ERR_WORKSPACE
    assert pre(None) == qa.ERR_INVALID_ARG
    for theta, inv, sc, win in [(0.0, None, 1.0, 0), (1e6, None, 0.0, 0), (1e6, None, float("nan"), 0),
                                (1e6, None, 1.0, -1), (1e6, [float("inf")] + [1.0] * 63, 1.0, 0)]:
        bad, _keep = qa.make_variant(theta, inv, sc, win)
        assert pre(ctypes.byref(bad)) == qa.ERR_INVALID_ARG, (theta, sc, win)
        assert dec(ctypes.byref(bad)) == qa.ERR_INVALID_ARG, (theta, sc, win)
    # a caller's table stands in for theta
    tab, _keep = qa.make_variant(0.0, [0.5 ** i for i in range(64)], 1.0, 64)
    assert pre(ctypes.byref(tab)) == qa.ERR_WORKSPACE


def test_paged_argument_checks():
    lib = qa.lib()
    var, _ = qa.make_variant()

    def dec(kv):
        return lib.qwen3_attn_decode_paged(FAKE, FAKE, FAKE, FAKE, FAKE, kv, FAKE, FAKE, None, 4, 32, 8, 128,
                                           ctypes.byref(var), 1e-6, None, 0, None)

    def pre(kv, start=0, T=128):
        return lib.qwen3_attn_prefill_paged(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, kv, start, None, 0, 1, T,
                                            16, 8, 128, ctypes.byref(var), 1e-6, None)

    good = qa.PagedKV(1 << 20, 1 << 20, 1 << 20, 100, 64, 40)
    assert dec(ctypes.byref(good)) == qa.ERR_WORKSPACE
    assert pre(ctypes.byref(good)) == qa.ERR_WORKSPACE
    assert pre(ctypes.byref(good), start=40 * 64 - 128) == qa.ERR_WORKSPACE  # start + T == capacity
    assert pre(ctypes.byref(good), start=40 * 64 - 127) == qa.ERR_INVALID_ARG  # past the table's capacity
    assert dec(None) == qa.ERR_INVALID_ARG
    for bad in (qa.PagedKV(0, 1 << 20, 1 << 20, 100, 64, 40),        # no pool
                qa.PagedKV(1 << 20, 1 << 20, 0, 100, 64, 40),        # no table
                qa.PagedKV(1 << 20, 1 << 20, 1 << 20, 100, 48, 40),  # page not a power of two
                qa.PagedKV(1 << 20, 1 << 20, 1 << 20, 100, 8, 40),   # page under 16
                qa.PagedKV(1 << 20, 1 << 20, 1 << 20, 0, 64, 40),    # no pages
                qa.PagedKV((1 << 20) + 2, 1 << 20, 1 << 20, 100, 64, 40)):  # misaligned pool
        assert dec(ctypes.byref(bad)) == qa.ERR_INVALID_ARG
        assert pre(ctypes.byref(bad)) == qa.ERR_INVALID_ARG
    # room to gather the start + T keys and values (pages under 64 keys), and Q'
    assert qa.prefill_paged_workspace_size(2, 100, 300, 16, 8) >= 2 * 2 * 8 * 400 * 256 + 2 * 300 * 16 * 256
    assert qa.prefill_paged_workspace_size(2, -1, 300, 16, 8) == 0


def test_varlen_argument_checks():
    lib = qa.lib()
    var, _ = qa.make_variant()

    def pre(kv=None, ctx=None, key_cap=0, ws=None, ws_bytes=0, B=4, N=1000, Hq=16, Hkv=8, d=128, cu=FAKE, q=FAKE,
            out=FAKE):
        return lib.qwen3_attn_prefill_varlen(q, FAKE, FAKE, FAKE, FAKE, FAKE, cu, out, None, kv, ctx, key_cap, ws,
                                             ws_bytes, B, N, Hq, Hkv, d, ctypes.byref(var), 1e-6, None)

    good = qa.PagedKV(1 << 20, 1 << 20, 1 << 20, 100, 64, 40)
    assert pre() == qa.ERR_WORKSPACE
    assert pre(kv=ctypes.byref(good), key_cap=5000) == qa.ERR_WORKSPACE
    assert pre(kv=ctypes.byref(good), ctx=FAKE, key_cap=5000) == qa.ERR_WORKSPACE
    assert pre(ctx=FAKE) == qa.ERR_INVALID_ARG            # cached keys without a cache
    assert pre(key_cap=10) == qa.ERR_INVALID_ARG          # a key capacity without a cache
    assert pre(kv=ctypes.byref(good)) == qa.ERR_INVALID_ARG  # a cache without a key capacity
    assert pre(cu=None) == qa.ERR_INVALID_ARG
    assert pre(q=None) == qa.ERR_INVALID_ARG
    assert pre(cu=ctypes.c_void_p((1 << 20) + 2)) == qa.ERR_INVALID_ARG  # misaligned offsets
    assert pre(B=0) == qa.ERR_INVALID_ARG and pre(N=0) == qa.ERR_INVALID_ARG
    assert pre(Hq=12) == qa.ERR_UNSUPPORTED and pre(d=64) == qa.ERR_UNSUPPORTED
    # metadata, entry list and level scratch, Q' [N, Hq, d], K' and V [N, Hkv, d] (or key_cap
    # rows, for gathering pages under 64 keys)
    n = qa.prefill_varlen_workspace_size(4, 1000, 16, 8)
    assert n >= 1000 * (16 + 2 * 8) * 128 * 2 + 4 * 16
    m = qa.prefill_varlen_workspace_size(4, 1000, 16, 8, key_cap=5000)
    assert m - n >= 2 * (5000 - 1000) * 8 * 128 * 2
    assert qa.prefill_varlen_workspace_size(0, 1000, 16, 8) == 0
    assert qa.prefill_varlen_workspace_size(4, 1000, 16, 8, key_cap=-1) == 0
    assert qa.prefill_varlen_workspace_size(4, 1000, 16, 8, d=64) == 0
    assert pre(ws=FAKE, ws_bytes=n - 1) == qa.ERR_WORKSPACE


def test_decode_and_prologue_argument_checks():
    lib = qa.lib()

    def dec(**kw):
        a = dict(q=FAKE, kn=FAKE, vn=FAKE, gq=FAKE, gk=FAKE, kc=FAKE, vc=FAKE, lens=FAKE, out=FAKE, lse=None, N=4,
                 Hq=32, Hkv=8, d=128, Lmax=4096, ws=None, ws_bytes=0)
        a.update(kw)
        return lib.qwen3_attn_decode(a["q"], a["kn"], a["vn"], a["gq"], a["gk"], a["kc"], a["vc"], a["lens"],
                                     a["out"], a["lse"], a["N"], a["Hq"], a["Hkv"], a["d"], a["Lmax"], 1e6, 1e-6,
                                     a["ws"], a["ws_bytes"], None)

    assert dec(lens=None) == qa.ERR_INVALID_ARG
    assert dec(N=0) == qa.ERR_INVALID_ARG
    assert dec(Hq=64, Hkv=2) == qa.ERR_UNSUPPORTED  # G = 32 > 16
    assert dec(d=256) == qa.ERR_UNSUPPORTED
    assert dec() == qa.ERR_WORKSPACE
    assert dec(ws=FAKE, ws_bytes=16) == qa.ERR_WORKSPACE
    r = lib.qwen3_qk_norm_rope(FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 4, 8, 128, 4, 0, 1e6, 1e-6, None)
    assert r == qa.ERR_INVALID_ARG  # v_src without v_dst
    r = lib.qwen3_qk_norm_rope(FAKE, FAKE, FAKE, FAKE, None, None, 1, 8, 8, 128, 4, 0, 1e6, 1e-6, None)
    assert r == qa.ERR_INVALID_ARG  # Tcap < T when writing at t
    r = lib.qwen3_qk_norm_rope(FAKE, FAKE, FAKE, FAKE, None, None, 1, 8, 8, 64, 8, 0, 1e6, 1e-6, None)
    assert r == qa.ERR_UNSUPPORTED


def test_size_limits_are_rejected_before_any_launch():
    """Past the 32-bit element ranges the kernels index with, calls return UNSUPPORTED at
    the host checks.  (Only the rejected side of each limit is exercised here: a call just
    inside it would go on to launch kernels on the fake pointers.)"""
    lib = qa.lib()
    # prefill: T * Hq query rows of d elements must stay below 2^31 elements
    T = (1 << 24) // 16 + 1
    need = qa.prefill_workspace_size(1, T, 16, 8)
    assert _prefill_ex(T=T, ws=FAKE, ws_bytes=need) == qa.ERR_UNSUPPORTED
    # decode: N * Hkv * Lmax cache rows must fit a 32-bit row index
    r = lib.qwen3_attn_decode(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 64, 32, 8, 128, 1 << 22,
                              1e6, 1e-6, FAKE, 1 << 40, None)
    assert r == qa.ERR_UNSUPPORTED
    # decode: at most 65535 sequences (a grid dimension)
    r = lib.qwen3_attn_decode(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 65536, 32, 8, 128, 16,
                              1e6, 1e-6, FAKE, 1 << 40, None)
    assert r == qa.ERR_UNSUPPORTED
    # the no-allocation decode refuses requests beyond its fixed region before anything else
    r = lib.qwen3_attn_decode_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 4096, 32, 8, 128,
                                      32769, 1e6, 1e-6, None)
    assert r == qa.ERR_WORKSPACE


def test_binding_refuses_cpu_tensors():
    q = torch.zeros(1, 128, 16, 128, dtype=torch.bfloat16)
    k = torch.zeros(1, 128, 8, 128, dtype=torch.bfloat16)
    w = torch.ones(128)
    pos = torch.arange(128, dtype=torch.int32)[None]
    with pytest.raises(ValueError):
        qa.prefill(q, k, k, w, w, pos)
    with pytest.raises(ValueError, match="together"):
        qa.prefill(q, k, k, w, w, pos, v_cache=torch.zeros(1, 8, 128, 128, dtype=torch.bfloat16))


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """Without the built library the binding raises; there is no fallback implementation."""
    monkeypatch.setattr(qa, "_lib", None)
    monkeypatch.setattr(qa, "LIB_PATH", str(tmp_path / "libqwen3attn.so"))
    with pytest.raises(RuntimeError, match="no fallback"):
        qa.lib()


def test_wait_limit_roundtrip():
    old = qa.set_wait_limit(123456)
    assert qa.set_wait_limit(old) == 123456


def _c_param_kind(decl: str) -> str:
    """The ctypes kind a C parameter declaration marshals as."""
    d = " ".join(decl.replace("const ", "").split())
    if d == "void":
        return "none"
    if "qwen3_attn_variant*" in d.replace(" *", "*"):
        return "variant*"
    if "qwen3_paged_kv*" in d.replace(" *", "*"):
        return "paged*"
    if "*" in d or d.startswith("qwen3_stream_t"):
        return "int*" if d.replace(" *", "*").startswith("int*") else "ptr"
    base = d.rsplit(" ", 1)[0] if " " in d else d
    # size_t and uint64_t are one 64-bit unsigned type here (ctypes aliases them too)
    return {"int": "int", "float": "float", "size_t": "u64", "long long": "longlong",
            "uint64_t": "u64", "double": "double"}[base]


def _ctypes_kind(t) -> str:
    if t is ctypes.POINTER(qa.Variant):
        return "variant*"
    if t is ctypes.POINTER(qa.PagedKV):
        return "paged*"
    if t is ctypes.POINTER(ctypes.c_int):
        return "int*"
    return {ctypes.c_void_p: "ptr", ctypes.c_int: "int", ctypes.c_float: "float", ctypes.c_size_t: "u64",
            ctypes.c_longlong: "longlong", ctypes.c_uint64: "u64", ctypes.c_double: "double"}[t]


def test_binding_signatures_match_the_header():
    """Every argument list the ctypes binding declares has the header's arity and kinds (a
    mismatch would pass garbage across the ABI without any error), and so does every
    return type."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    text = re.sub(r"#[^\n]*", "", text)
    decls = re.findall(r"([\w\s\*]+?)\b(qwen3_\w+)\s*\(([^)]*)\)\s*;", text)
    assert len(decls) == len(qa.SIGNATURES)
    ret_kind = {"int": ctypes.c_int, "size_t": ctypes.c_size_t, "const char*": ctypes.c_char_p,
                "void": None, "uint64_t": ctypes.c_uint64}
    for ret, name, params in decls:
        res, args = qa.SIGNATURES[name]
        ret = " ".join(ret.split()).replace(" *", "*")
        assert res is ret_kind[ret], (name, ret)
        kinds = [_c_param_kind(p) for p in params.split(",")]
        kinds = [k for k in kinds if k != "none"]
        assert kinds == [_ctypes_kind(a) for a in args], name


def test_status_codes_match_the_header():
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    codes = {name: int(val) for name, val in re.findall(r"\b(QWEN3_(?:OK|ERR_\w+))\s*=\s*(\d+)", text)}
    assert codes == {"QWEN3_OK": qa.OK, "QWEN3_ERR_INVALID_ARG": qa.ERR_INVALID_ARG,
                     "QWEN3_ERR_UNSUPPORTED": qa.ERR_UNSUPPORTED, "QWEN3_ERR_CUDA": qa.ERR_CUDA,
                     "QWEN3_ERR_DEVICE_TIMEOUT": qa.ERR_DEVICE_TIMEOUT, "QWEN3_ERR_WORKSPACE": qa.ERR_WORKSPACE}
    # and each has its own message
    assert len({qa.status_string(c) for c in codes.values()}) == len(codes)


def test_noalloc_checks_arguments_before_the_region_lookup():
    """A bad argument gets the status qwen3_attn_decode gives it, whether or not a device is
    there to look the region up on; a call whose lookup failed (no device here) leaves no
    error behind for the next call's checks."""
    f = qa.lib().qwen3_attn_decode_noalloc
    dec = qa.lib().qwen3_attn_decode
    args = [FAKE] * 9 + [None, 8, 32, 8, 128, 4096, 1e6, 1e-6, None]
    bad_ptr = list(args)
    bad_ptr[0] = None
    assert f(*bad_ptr) == qa.ERR_INVALID_ARG
    bad_d = list(args)
    bad_d[13] = 64
    assert f(*bad_d) == qa.ERR_UNSUPPORTED == dec(*(bad_d[:17] + [FAKE, 1 << 30, None]))
    bad_g = list(args)
    bad_g[11] = 24
    assert f(*bad_g) == qa.ERR_UNSUPPORTED
    if not torch.cuda.is_available():
        assert f(*args) == qa.ERR_CUDA  # the lookup itself needs a device
        assert f(*bad_ptr) == qa.ERR_INVALID_ARG
        assert f(*args) == qa.ERR_CUDA


def test_softmax_path_constants_match_the_header():
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    vals = {name: int(val) for name, val in re.findall(r"#define\s+(QWEN3_SOFTMAX_\w+)\s+(\d+)", text)}
    assert vals == {"QWEN3_SOFTMAX_AUTO": qa.SOFTMAX_AUTO, "QWEN3_SOFTMAX_RUNNING_MAX": qa.SOFTMAX_RUNNING_MAX}


def test_softmax_path_hook_returns_the_previous_setting_and_refuses_unknown_values():
    """Host-side only: the hook records the setting for later launches and launches nothing."""
    assert qa.set_softmax_path(qa.SOFTMAX_RUNNING_MAX) == qa.SOFTMAX_AUTO
    try:
        assert qa.set_softmax_path(qa.SOFTMAX_RUNNING_MAX) == qa.SOFTMAX_RUNNING_MAX
        with pytest.raises(ValueError):
            qa.set_softmax_path(7)
        assert qa.lib().qwen3_attn_set_softmax_path(-3) == -1
    finally:
        assert qa.set_softmax_path(qa.SOFTMAX_AUTO) == qa.SOFTMAX_RUNNING_MAX


def test_qkv_projection_argument_checks():
    """Host-side only: every call fails a check made before any device work."""
    var, _ = qa.make_variant()

    def qkv(**kw):
        a = dict(x=FAKE, w=FAKE, gq=FAKE, gk=FAKE, pos=FAKE, qo=FAKE, ko=FAKE, vo=FAKE, M=300, hidden=256, Hq=4,
                 Hkv=2, d=128, var=ctypes.byref(var), eps=1e-6, ws=FAKE, ws_bytes=0)
        a.update(kw)
        return qa.lib().qwen3_qkv_proj_norm_rope(a["x"], a["w"], a["gq"], a["gk"], a["pos"], a["qo"], a["ko"],
                                                  a["vo"], a["M"], a["hidden"], a["Hq"], a["Hkv"], a["d"],
                                                  a["var"], a["eps"], a["ws"], a["ws_bytes"], None)

    need = qa.qkv_proj_workspace_size(300)
    assert need >= ((300 + 127) // 128) * 64 * 128 * 8  # the RoPE table, (cos, sin) per row and frequency
    assert qkv(ws_bytes=need - 1) == qa.ERR_WORKSPACE  # every other argument passes its checks
    assert qkv(ws=None, ws_bytes=need) == qa.ERR_WORKSPACE
    assert qkv(x=None, ws_bytes=need) == qa.ERR_INVALID_ARG
    assert qkv(vo=None, ws_bytes=need) == qa.ERR_INVALID_ARG
    assert qkv(var=None, ws_bytes=need) == qa.ERR_INVALID_ARG
    assert qkv(M=0, ws_bytes=need) == qa.ERR_INVALID_ARG
    assert qkv(Hkv=0, ws_bytes=need) == qa.ERR_INVALID_ARG
    assert qkv(d=64, ws_bytes=need) == qa.ERR_UNSUPPORTED
    assert qkv(hidden=100, ws_bytes=need) == qa.ERR_UNSUPPORTED  # rows must be 16-byte multiples for TMA
    assert qkv(x=ctypes.c_void_p((1 << 20) + 8), ws_bytes=need) == qa.ERR_INVALID_ARG  # misaligned
    assert qkv(eps=-1.0, ws_bytes=need) == qa.ERR_INVALID_ARG
    assert qa.qkv_proj_workspace_size(0) == 0


def test_sm_pairs_constants_match_the_header():
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    vals = {name: int(val) for name, val in re.findall(r"#define\s+(QWEN3_SM_PAIRS_\w+)\s+(\d+)", text)}
    assert vals == {"QWEN3_SM_PAIRS_AUTO": qa.SM_PAIRS_AUTO, "QWEN3_SM_PAIRS_OFF": qa.SM_PAIRS_OFF,
                    "QWEN3_SM_PAIRS_ALWAYS": qa.SM_PAIRS_ALWAYS}


def test_sm_pairs_hook_returns_the_previous_setting_and_refuses_unknown_values():
    """Host-side only: the hook records the setting for later qkv projections."""
    assert qa.set_sm_pairs(qa.SM_PAIRS_OFF) == qa.SM_PAIRS_AUTO
    try:
        assert qa.set_sm_pairs(qa.SM_PAIRS_ALWAYS) == qa.SM_PAIRS_OFF
        with pytest.raises(ValueError):
            qa.set_sm_pairs(3)
        assert qa.lib().qwen3_attn_set_sm_pairs(-1) == -1
    finally:
        assert qa.set_sm_pairs(qa.SM_PAIRS_AUTO) == qa.SM_PAIRS_ALWAYS


def test_noalloc_region_limit():
    """The no-allocation decode's fixed region (48 MiB) holds the split-KV partials of up to
    92 sequences of 32 heads at Lmax 32769, the batched-decode workload's 64 among them."""
    region = 48 << 20
    assert qa.decode_workspace_size(64, 32, 32769) <= region
    assert qa.decode_workspace_size(92, 32, 32769) <= region < qa.decode_workspace_size(93, 32, 32769)
    r = qa.lib().qwen3_attn_decode_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 93, 32, 8,
                                           128, 32769, 1e6, 1e-6, None)
    assert r == qa.ERR_WORKSPACE


def test_chunk_workspace_sizes_hold_the_key_split_partials():
    """The key-axis split's partials are sized on the host from the shapes alone: none for a
    chunk with many work items, fp32 O/l and an LSE per (new row, query head, run of keys)
    for a short chunk over a long prefix (the runs: about 128 items in all, each at least 4
    key tiles, at most 32; a chunk with one query tile per KV head takes two runs per item)."""
    def parts(T, n):
        rows = 1 * T * 32 * n
        return ((rows * 128 * 4 + 255) // 256) * 256 + ((rows * 4 + 255) // 256) * 256

    # 64 new tokens, G = 4: two query tiles, one pair item per KV head, 8 items; 235 key
    # tiles -> 16 runs
    assert qa.prefill_chunk_workspace_size(1, 30000, 64, 32, 8) == qa.prefill_workspace_size(1, 64, 32, 8) + parts(64, 16)
    # 16 new tokens: a single query tile (64 rows), so two runs per item -> 32 runs
    base = qa.prefill_workspace_size(1, 16, 32, 8)
    want = base + parts(16, 32)
    assert qa.prefill_chunk_workspace_size(1, 30000, 16, 32, 8) == want
    # a single query tile over 40 key tiles: runs of at least 4 tiles, an even count -> 10
    assert qa.prefill_chunk_workspace_size(1, 5000, 16, 32, 8) == base + parts(16, 10)
    # 32 KV heads of one query tile each: 2 * 128 / 32 = 8 runs
    assert qa.prefill_chunk_workspace_size(1, 30000, 16, 128, 32) == \
        qa.prefill_workspace_size(1, 16, 128, 32) + ((16 * 128 * 8 * 512 + 255) // 256 * 256) + \
        ((16 * 128 * 8 * 4 + 255) // 256 * 256)
    # many items (the 4B-shaped second chunk): no split, no extra bytes
    assert qa.prefill_chunk_workspace_size(1, 4096, 4096, 32, 8) == qa.prefill_workspace_size(1, 4096, 32, 8)
    # a short prefix: fewer than 8 key tiles, no split
    assert qa.prefill_chunk_workspace_size(1, 500, 16, 32, 8) == qa.prefill_workspace_size(1, 16, 32, 8)
    # the paged prefill's workspace carries the same partials after its gathered K, V and Q'
    def al(x):
        return (x + 255) // 256 * 256
    paged = 2 * al(30016 * 8 * 256) + al(16 * 32 * 256) + 256
    assert qa.prefill_paged_workspace_size(1, 30000, 16, 32, 8) == paged + (want - base)
