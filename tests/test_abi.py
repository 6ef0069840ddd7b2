"""The C ABI on the CPU: the library loads, exports every entry point include/hs2.h declares,
and rejects bad arguments on the host before touching the GPU."""
import ctypes
import os
import re

import pytest
import torch

import token_level_sparse_hs2_b200 as hs2

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from token_level_sparse_hs2_b200 import build
    build.build()
    return hs2.lib()


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(hs2_[a-z0-9_]+)\s*\(", src))
    return names


def test_exports_every_declared_symbol(L):
    names = declared_symbols()
    assert {"hs2_block_decode", "hs2_full_attn_scores", "hs2_topk_select",
            "hs2_sparse_gather_attn", "hs2_workspace_size"} <= names
    for n in sorted(names):
        assert hasattr(L, n), n
    assert L.hs2_version() == 1
    assert L.hs2_status_string(6) == b"HS2_ERR_TIMEOUT"


def cpu_cache(batch=2, n_q=1, H=32, d=128, lens=(300, 500), dtype=torch.bfloat16, **kw):
    rows = sum(lens) + 8
    k = torch.zeros((rows, d), dtype=dtype)
    v = torch.zeros((rows, d), dtype=dtype)
    start = [0]
    for t in lens[:-1]:
        start.append(start[-1] + t)
    ks = vs = None
    if dtype == torch.uint8:
        ks = torch.ones(rows)
        vs = torch.ones(rows)
    c = hs2.KvCache(k, v, start, lens, n_q, H, ks, vs)
    c.view.head_dim = d
    for key, val in kw.items():
        setattr(c.view, key, val)
    return c


def status_of(fn):
    try:
        fn()
    except hs2.HS2Error as e:
        return e.status, str(e)
    return 0, ""


def test_workspace_size_host_only(L):
    c = cpu_cache()
    n = hs2.workspace_size(c)
    assert n > 0 and n % 256 == 0
    assert hs2.workspace_size(cpu_cache(lens=(300, 5000))) >= n


@pytest.mark.parametrize("kw,expect", [
    (dict(head_dim=64), 2),
    (dict(n_heads=8), 2),
    (dict(batch=0), 1),
    (dict(n_q=0), 1),
    (dict(kv_dtype=7), 1),
    (dict(reserved=1), 1),
    (dict(kv_rows=10), 1),
])
def test_view_validation(L, kw, expect):
    c = cpu_cache()
    for key, val in kw.items():
        setattr(c.view, key, val)
    st, msg = status_of(lambda: hs2.workspace_size(c))
    assert st == expect, msg


def test_misaligned_and_null_pointers(L):
    c = cpu_cache()
    c.view.k = c.view.k + 2
    assert status_of(lambda: hs2.workspace_size(c))[0] == 1
    c = cpu_cache()
    c.view.v = None
    assert status_of(lambda: hs2.workspace_size(c))[0] == 1
    c = cpu_cache(dtype=torch.uint8)
    c.view.k_scale = None
    assert status_of(lambda: hs2.workspace_size(c))[0] == 1


def test_sequence_shorter_than_queries(L):
    c = cpu_cache(n_q=400)
    st, msg = status_of(lambda: hs2.workspace_size(c))
    assert st == 1 and "n_q" in msg


def test_budget_limits(L):
    c = cpu_cache()
    assert status_of(lambda: hs2.workspace_size(c, topk=0))[0] == 2
    assert status_of(lambda: hs2.workspace_size(c, topk=4096))[0] == 2
    assert status_of(lambda: hs2.workspace_size(c, window=-1))[0] == 2


def test_call_argument_checks_before_any_launch(L):
    c = cpu_cache()
    H = 32
    q = torch.zeros((2, 1, H, 128), dtype=torch.bfloat16)
    out = torch.zeros_like(q, dtype=torch.float32)
    lse = torch.zeros((2, 1, H))
    scores = torch.zeros((2, 500))
    idx = torch.zeros((2, 500), dtype=torch.int32)
    cnt = torch.zeros(2, dtype=torch.int32)
    def aligned(n):
        buf = torch.zeros(n + 256, dtype=torch.uint8)
        off = (-buf.data_ptr()) % 256
        return buf, buf.data_ptr() + off
    ws_buf, ws_ptr = aligned(hs2.workspace_size(c))
    small_buf, small_ptr = aligned(256)
    raw = hs2.lib().hs2_block_decode
    args = lambda **o: [o.get("view", c.ref()), q.data_ptr(),
                        (ctypes.c_void_p * 1)(q.data_ptr()), o.get("n_sparse", 1), 1024, 128,
                        o.get("scale", 0.088), out.data_ptr(),
                        (ctypes.c_void_p * 1)(out.data_ptr()), 1, lse.data_ptr(),
                        scores.data_ptr(), o.get("score_stride", 500), idx.data_ptr(),
                        o.get("idx_stride", 500), cnt.data_ptr(), o.get("ws", ws_ptr),
                        o.get("ws_bytes", ws_buf.numel() - 256), None]
    st = raw(*args(ws=small_ptr, ws_bytes=256))
    assert st == 3, hs2.lib().hs2_last_error()
    assert raw(*args(score_stride=499)) == 1
    assert raw(*args(idx_stride=100)) == 1
    assert raw(*args(scale=float("nan"))) == 1
    assert raw(*args(scale=0.0)) == 1
    assert raw(*args(n_sparse=-1)) == 1
    assert raw(*args(ws=ws_ptr + 16)) == 1
    st = raw(*args(score_stride=499))
    assert st == 1 and b"score_stride" in hs2.lib().hs2_last_error()


def test_optional_block_outputs_sizes_and_checks(L):
    """scores / idx + count may be NULL in hs2_block_decode: hs2_workspace_size's flags reserve
    room for them (scores: rows x (max p + 1, rounded up to 64) floats; selection: rows x
    min(max p + 1, topk + window) positions plus the counts), and a call that leaves an output
    to a workspace sized without its flag is refused on the host before any launch."""
    c = cpu_cache(lens=(300, 500))
    base = hs2.workspace_size(c)
    with_scores = hs2.workspace_size(c, flags=hs2.WS_SCORES)
    with_sel = hs2.workspace_size(c, flags=hs2.WS_SELECTION)
    both = hs2.workspace_size(c, flags=hs2.WS_SCORES | hs2.WS_SELECTION)
    assert with_scores - base >= 2 * 512 * 4
    assert with_sel - base >= 2 * 500 * 4 + 2 * 4
    assert both - base >= (with_scores - base) + (with_sel - base) - 512
    assert status_of(lambda: hs2.workspace_size(c, flags=4))[0] == 1
    H = 32
    q = torch.zeros((2, 1, H, 128), dtype=torch.bfloat16)
    out = torch.zeros_like(q, dtype=torch.float32)
    idx = torch.zeros((2, 500), dtype=torch.int32)
    cnt = torch.zeros(2, dtype=torch.int32)
    buf = torch.zeros(both + 256, dtype=torch.uint8)
    ws = buf.data_ptr() + (-buf.data_ptr()) % 256
    raw = hs2.lib().hs2_block_decode
    def call(scores_p, idx_p, cnt_p, ws_bytes):
        return raw(c.ref(), q.data_ptr(), (ctypes.c_void_p * 1)(q.data_ptr()), 1, 1024, 128,
                   0.088, out.data_ptr(), (ctypes.c_void_p * 1)(out.data_ptr()), 1, None,
                   scores_p, 0, idx_p, 0, cnt_p, ws, ws_bytes, None)
    # idx without count (or the reverse) is an argument error
    assert call(None, idx.data_ptr(), None, both) == 1
    assert b"both" in hs2.lib().hs2_last_error()
    assert call(None, None, cnt.data_ptr(), both) == 1
    # NULL outputs with a workspace sized for fewer of them: refused with the size
    assert call(None, None, None, with_scores) == 3
    assert call(None, None, None, with_sel) == 3
    assert call(None, idx.data_ptr(), cnt.data_ptr(), base) == 3
    assert b"required" in hs2.lib().hs2_last_error()


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    import importlib
    mod = importlib.import_module("token_level_sparse_hs2_b200")
    monkeypatch.setattr(mod, "LIB_PATH", str(tmp_path / "nope.so"))
    monkeypatch.setattr(mod, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        mod.lib()


def test_noalloc_selection_rejects_oversized_calls(L):
    # 100 rows of 20,000 tokens are split over several CTAs each and need far more than the
    # built-in 4 MiB of scratch: rejected on the host with the size
    c = cpu_cache(batch=100, lens=tuple([20000] * 100))
    scores = torch.zeros((100, 20000))
    idx = torch.zeros((100, 1152), dtype=torch.int32)
    cnt = torch.zeros(100, dtype=torch.int32)
    idx.fill_(-7)
    cnt.fill_(-7)
    st = hs2.lib().hs2_topk_select_noalloc(c.ref(), scores.data_ptr(), 20000, 1024, 128,
                                           idx.data_ptr(), 1152, cnt.data_ptr(), None)
    assert st == 3 and b"scratch" in hs2.lib().hs2_last_error()
    assert (idx == -7).all() and (cnt == -7).all()   # refused before anything was written


def test_selftest_rejects_bad_arguments_without_launching():
    import ctypes
    import token_level_sparse_hs2_b200 as hs2
    L = hs2.lib()
    assert L.hs2_selftest_wait_timeout(1000, None, 64, None) == 3         # HS2_ERR_WORKSPACE
    buf = ctypes.create_string_buffer(1024)
    addr = (ctypes.addressof(buf) + 255) & ~255
    assert L.hs2_selftest_wait_timeout(0, ctypes.c_void_p(addr), 256, None) == 1   # limit 0


def test_block_selection_argument_checks(L):
    c = cpu_cache(lens=(300, 5000))
    n = hs2.topk_select_blocks_workspace_size(c, 64)
    # block scores of both rows: ceil(5000 / 64) = 79 -> stride 80 floats per row
    assert n >= 256 + 2 * 80 * 4 and n % 256 == 0
    for bs, topk, expect in ((48, 1024, 2), (8, 1024, 2), (256, 1024, 2), (64, 1000, 1)):
        st = L.hs2_topk_select_blocks_workspace_size(c.ref(), bs, topk, 128,
                                                     ctypes.byref(ctypes.c_size_t()))
        assert st == expect, (bs, topk, L.hs2_last_error())
    scores = torch.zeros((2, 5000))
    idx = torch.zeros((2, 1152), dtype=torch.int32)
    cnt = torch.zeros(2, dtype=torch.int32)
    # too small a workspace, then too short an idx row: refused before any launch
    st = L.hs2_topk_select_blocks(c.ref(), scores.data_ptr(), 5000, 64, 1024, 128,
                                  idx.data_ptr(), 1152, cnt.data_ptr(), ctypes.c_void_p(256),
                                  256, None)
    assert st == 3 and b"workspace" in L.hs2_last_error()
    st = L.hs2_topk_select_blocks(c.ref(), scores.data_ptr(), 5000, 64, 1024, 128,
                                  idx.data_ptr(), 1000, cnt.data_ptr(), ctypes.c_void_p(256),
                                  1 << 20, None)
    assert st == 1 and b"idx_stride" in L.hs2_last_error()


def test_context_parallel_argument_checks(L):
    c = cpu_cache(batch=1, lens=(5000,))
    P = ctypes.c_void_p
    ws = P(256)
    # NULL outputs, a bad scale, a short score stride, bad merge shapes: refused before any launch
    assert L.hs2_full_attn(c.ref(), P(256), ctypes.c_float(0.088), None, 1, P(256), ws,
                           1 << 20, None) == 1
    assert L.hs2_full_attn(c.ref(), P(256), ctypes.c_float(-1.0), P(256), 1, P(256), ws,
                           1 << 20, None) == 1
    assert L.hs2_score_pass(c.ref(), P(256), ctypes.c_float(0.088), P(256), P(256), 100, ws,
                            1 << 20, None) == 1
    assert b"score_stride" in L.hs2_last_error()
    assert L.hs2_lse_merge(0, 1, 32, P(256), P(256), P(256), 1, None, None) == 1
    assert L.hs2_cp_merge_select(32, 1, (ctypes.c_int32 * 1)(5000), P(256), 1024, 128, P(256),
                                 1152, P(256), None) == 2          # 32 x 1024 keys: too many
    assert L.hs2_cp_localize(1, (ctypes.c_int64 * 1)(4000), (ctypes.c_int32 * 1)(1000), P(256),
                             1152, P(256), P(256), 100, P(256), None) == 1


def declared_signatures():
    """name -> (return type, [parameter types]) of every function include/*.h declares."""
    sigs = {}
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if not fn.endswith(".h"):
            continue
        src = open(os.path.join(ROOT, "include", fn)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"#[^\n]*", "", src)
        for m in re.finditer(r"([A-Za-z_][A-Za-z0-9_ ]*?[\s\*]+)(hs2_[a-z0-9_]+)\s*\(([^)]*)\)\s*;", src):
            ret, name, params = m.group(1).strip(), m.group(2), m.group(3).strip()
            if params in ("", "void"):
                sigs[name] = (ret, [])
                continue
            types = []
            for p in params.split(","):
                p = " ".join(p.split())
                # drop the parameter name (the last identifier) unless the parameter is unnamed
                t = re.sub(r"\s*\b[A-Za-z_][A-Za-z0-9_]*$", "", p) if not p.endswith("*") else p
                types.append(t if t else p)
            sigs[name] = (ret, types)
    return sigs


def ctype_class(t: str) -> str:
    t = t.replace("const", "").strip()
    if "*" in t:
        return "pointer"
    return {"int32_t": "i32", "int64_t": "i64", "uint32_t": "u32", "uint64_t": "u64",
            "size_t": "size", "float": "f32", "int": "i32", "hs2_status": "i32"}.get(t, t)


def argtype_class(a) -> str:
    if a in (ctypes.c_void_p, ctypes.c_char_p) or hasattr(a, "_type_") and \
            isinstance(getattr(a, "_type_", None), type):
        return "pointer"
    return {ctypes.c_int32: "i32", ctypes.c_int64: "i64", ctypes.c_uint32: "u32",
            ctypes.c_uint64: "u64", ctypes.c_size_t: "size", ctypes.c_float: "f32"}.get(a, repr(a))


def test_binding_argtypes_match_the_header(L):
    """Every argument list the binding declares has the header's length and, argument by
    argument, the same class (pointer, 32/64-bit integer, size_t, float)."""
    sigs = declared_signatures()
    assert "hs2_block_decode" in sigs and len(sigs["hs2_block_decode"][1]) == 19
    checked = 0
    for name, (ret, params) in sorted(sigs.items()):
        fn = getattr(L, name)
        if fn.argtypes is None:
            assert not params, f"{name}: the binding sets no argument types"
            continue
        got = [argtype_class(a) for a in fn.argtypes]
        want = [ctype_class(p) for p in params]
        assert got == want, (name, got, want)
        checked += 1
    assert checked >= 20


def test_view_struct_matches_the_header():
    """The binding's hs2_kv_view has the header's fields in the header's order, with the same
    widths, so every offset agrees (the library reads the struct by those offsets)."""
    src = open(os.path.join(ROOT, "include", "hs2.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    body = re.search(r"typedef struct hs2_kv_view \{(.*?)\} hs2_kv_view;", src, flags=re.S).group(1)
    fields = []
    for decl in body.split(";"):
        decl = " ".join(decl.split())
        if not decl:
            continue
        name = re.search(r"([A-Za-z_][A-Za-z0-9_]*)$", decl).group(1)
        fields.append((name, ctype_class(decl[: -len(name)].strip())))
    got = [(n, argtype_class(t)) for n, t in hs2._KvView._fields_]
    assert got == fields
    offsets, off = [], 0
    for _, cls in fields:   # natural alignment on a 64-bit host
        size = {"i32": 4, "u32": 4, "f32": 4}.get(cls, 8)
        off = (off + size - 1) // size * size
        offsets.append(off)
        off += size
    assert [getattr(hs2._KvView, n).offset for n, _ in hs2._KvView._fields_] == offsets
    assert ctypes.sizeof(hs2._KvView) == (off + 7) // 8 * 8


def test_view_layout_agrees_with_the_c_compiler(tmp_path):
    """The header compiles as plain C (C99, no CUDA headers), and gcc lays hs2_kv_view out at
    the offsets the binding uses."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("gcc is not installed")
    names = [n for n, _ in hs2._KvView._fields_]
    prints = "".join(f'printf("%zu\\n", offsetof(hs2_kv_view, {n}));' for n in names)
    (tmp_path / "lay.c").write_text(
        "#include <stdio.h>\n#include <stddef.h>\n#include \"hs2.h\"\n"
        f"int main(void){{{prints} printf(\"%zu\\n\", sizeof(hs2_kv_view)); return 0;}}\n")
    exe = tmp_path / "lay"
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-I" + os.path.join(ROOT, "include"),
                           str(tmp_path / "lay.c"), "-o", str(exe)])
    out = [int(x) for x in subprocess.check_output([str(exe)]).split()]
    assert out[:-1] == [getattr(hs2._KvView, n).offset for n in names]
    assert out[-1] == ctypes.sizeof(hs2._KvView)
