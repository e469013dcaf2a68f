"""The C-ABI library loads without a GPU, exports every entry point the
header declares, and rejects bad arguments on the host (no kernel runs)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from paged_int8_kv_b200 import build
    build.build()
    return ctypes.CDLL(build.LIB)


def _declared():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"\b(kv8_[a-z0-9_]+)\s*\(", src)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert "kv8_paged_decode_attention" in names and len(names) >= 7
    for n in names:
        assert hasattr(lib, n), n


def test_binding_names_match_header():
    import paged_int8_kv_b200 as pk
    assert sorted(pk.EXPORTED) == _declared()
    for n in pk.EXPORTED:
        assert callable(getattr(pk, n))


def test_status_strings():
    import paged_int8_kv_b200 as pk
    assert pk.kv8_status_string(0) == "KV8_OK"
    assert pk.kv8_status_string(3) == "KV8_ERR_WORKSPACE"
    assert pk.kv8_status_string(99) == "KV8_ERR_UNKNOWN"


def test_workspace_bytes_closed_form():
    import paged_int8_kv_b200 as pk
    # batch 64, 32 q heads, 32K context, chunks of 512 -> 64 chunks
    ws = pk.kv8_decode_workspace_bytes(64, 32, 128, 32768, 512)
    ml = 64 * 32 * 64 * 2 * 4          # (m, l) per (sequence, head, chunk)
    o = 64 * 32 * 64 * 128 * 4         # unnormalised output per chunk
    tickets = 64 * 32 * 4              # one merge ticket per (sequence, head)
    counter = 16                       # the work counter, padded
    assert ws == ((ml + 255) // 256) * 256 + o + tickets + counter
    assert pk.kv8_decode_workspace_bytes(64, 32, 128, 512, 512) == 0
    assert pk.kv8_decode_workspace_bytes(64, 32, 128, 32768, 0) == 0
    assert pk.kv8_decode_workspace_bytes(64, 32, 64, 32768, 512) == 0


def _decode(lib, **kw):
    a = dict(q=16, kc=16, vc=16, ks=16, vs=16, bt=16, cl=16, batch=1, hq=8,
             hkv=2, d=128, bs=16, mbs=4, nb=8, maxlen=64, scale=0.0, chunk=0,
             ws=0, wsb=0, out=16, odt=0, stream=0)
    a.update(kw)
    f = lib.kv8_paged_decode_attention
    P, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    f.restype = i32
    f.argtypes = [P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, i64, i32,
                  ctypes.c_float, i32, P, ctypes.c_size_t, P, i32, P]
    return f(a["q"], a["kc"], a["vc"], a["ks"], a["vs"], a["bt"], a["cl"],
             a["batch"], a["hq"], a["hkv"], a["d"], a["bs"], a["mbs"], a["nb"],
             a["maxlen"], a["scale"], a["chunk"], a["ws"], a["wsb"], a["out"],
             a["odt"], a["stream"])


def test_host_validation_rejects_before_launch(lib):
    # Every call below fails its host checks, so no pointer is dereferenced.
    assert _decode(lib, d=64) == 2                 # head_dim unsupported
    assert _decode(lib, bs=32) == 2                # block size unsupported
    assert _decode(lib, hq=12, hkv=4) == 2         # group of 3 not built
    assert _decode(lib, hq=8, hkv=3) == 1          # not a multiple
    assert _decode(lib, maxlen=65) == 1            # > mbs * block_size
    assert _decode(lib, chunk=24) == 1             # not a block multiple
    assert _decode(lib, odt=7) == 1                # bad output dtype
    assert _decode(lib, q=0) == 1                  # null pointer
    assert _decode(lib, kc=8) == 1                 # misaligned cache
    assert _decode(lib, chunk=16, maxlen=64) == 3  # split needs a workspace
    assert _decode(lib, batch=0) == 0              # nothing to do
    f = lib.kv8_quantize_append
    P, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    f.restype = i32
    f.argtypes = [P, P, P, i64, i32, i32, i32, i64, P, P, P, P, P]
    assert f(16, 16, 16, 4, 2, 64, 16, 8, 16, 16, 16, 16, 0) == 2
    assert f(16, 16, 16, -1, 2, 128, 16, 8, 16, 16, 16, 16, 0) == 1
    assert f(16, 16, 16, 0, 2, 128, 16, 8, 16, 16, 16, 16, 0) == 0
    assert f(0, 16, 16, 4, 2, 128, 16, 8, 16, 16, 16, 16, 0) == 1
    # the decode form is an argument of each call; unknown forms are refused
    # before anything else is looked at
    g = lib.kv8_paged_decode_attention_form
    g.restype = i32
    g.argtypes = [P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, i64, i32,
                  ctypes.c_float, i32, P, ctypes.c_size_t, P, i32, i32, P]
    for form in (-1, 99):
        assert g(16, 16, 16, 16, 16, 16, 16, 1, 8, 2, 128, 16, 4, 8, 64, 0.0, 0,
                 0, 0, 16, 0, form, 0) == 1
    assert g(16, 16, 16, 16, 16, 16, 16, 1, 8, 2, 64, 16, 4, 8, 64, 0.0, 0,
             0, 0, 16, 0, 2, 0) == 2                # head_dim unsupported


def test_kivi_host_validation(lib):
    # Every call below fails (or finishes) in its host checks: no pointer is
    # dereferenced and no kernel is launched.
    P, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    a = lib.kv8_kivi_append
    a.restype = i32
    a.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, i64, i32, P, P, P]

    def app(k=16, batch=2, hkv=2, d=128, bs=16, mbs=4, nb=8, max_new=4, cache=16):
        return a(k, 16, 16, 16, 16, batch, hkv, d, bs, mbs, nb, max_new, cache, 16, 0)
    assert app(d=64) == 2            # head_dim unsupported
    assert app(bs=32) == 2           # block size unsupported
    assert app(max_new=-1) == 1      # negative bound
    assert app(batch=-1) == 1
    assert app(k=0) == 1             # null rows
    assert app(cache=8) == 1         # misaligned cache
    assert app(max_new=0) == 0       # nothing to append
    assert app(batch=0) == 0
    f = lib.kv8_kivi_paged_decode_attention
    f.restype = i32
    f.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, i32, i64, i32,
                  ctypes.c_float, i32, P, ctypes.c_size_t, P, i32, P]

    def dec(q=16, batch=1, hq=8, hkv=2, d=128, bs=16, mbs=4, maxlen=64,
            chunk=0, ws=0, odt=1):
        return f(q, 16, 16, 16, 16, batch, hq, hkv, d, bs, mbs, 8, maxlen, 0.0,
                 chunk, ws, 0, 16, odt, 0)
    assert dec(d=64) == 2            # head_dim unsupported
    assert dec(hq=6, hkv=2) == 2     # group of 3 not built
    assert dec(hq=8, hkv=3) == 1     # not a multiple
    assert dec(maxlen=65) == 1       # > mbs * block_size
    assert dec(chunk=24) == 1        # not a block multiple
    assert dec(odt=7) == 1           # bad output dtype
    assert dec(q=0) == 1             # null pointer
    assert dec(q=8) == 1             # misaligned q
    assert dec(chunk=16) == 3        # a split needs a workspace
    assert dec(batch=0) == 0         # nothing to do


def test_check_indices_host_validation(lib):
    P, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    f = lib.kv8_check_indices
    f.restype = i32
    f.argtypes = [P, P, i32, i32, i64, i32, P, i64, P, P]
    assert f(16, 16, 2, 4, 8, 64, 0, 0, 0, 0) == 1      # no counts buffer
    assert f(16, 16, 2, 4, 8, 64, 0, 0, 18, 0) == 1     # misaligned counts
    assert f(16, 16, -1, 4, 8, 64, 0, 0, 16, 0) == 1    # negative batch
    assert f(0, 16, 2, 4, 8, 64, 0, 0, 16, 0) == 1      # tables missing
    assert f(16, 16, 2, 0, 8, 64, 0, 0, 16, 0) == 1     # empty rows
    assert f(16, 16, 0, 4, 8, 64, 0, 3, 16, 0) == 1     # slots missing
    assert f(16, 16, 0, 4, 8, 64, 12, 3, 16, 0) == 1    # misaligned slots
    assert f(16, 16, 2, 4, 0, 64, 0, 0, 16, 0) == 1     # no blocks


def test_chunk_suggestion(lib):
    # no GPU here: the suggestion assumes 148 SMs x 12 resident warps and
    # cuts the longest context into equal block-aligned chunks of 64..512
    # tokens so that sequences x KV heads x chunks >= 1776 warps
    f = lib.kv8_decode_chunk_tokens
    f.restype = ctypes.c_int32
    f.argtypes = [ctypes.c_int32] * 3
    assert f(64, 8, 32768) == 512          # 64 chunks: already 9x the warps
    assert f(32, 8, 4017) == 512           # 7 splits wanted: 8 chunks of <= 512
    assert f(256, 8, 544) == 272           # enough items unsplit; 2 of <= 512
    assert f(2, 2, 256) == 64              # floor of 4 pages per chunk
    assert f(1, 1, 64) == 0 and f(1, 1, 65) == 64
    assert f(0, 8, 100) == 0 and f(4, 0, 100) == 0 and f(4, 8, 0) == 0
    for b, h, t in ((1, 1, 10**6), (7, 3, 12345), (512, 8, 128)):
        c = f(b, h, t)
        assert c % 16 == 0 and 64 <= c <= 512


def test_product_path_is_independent_of_the_oracle():
    # the library and its binding neither import, link nor load anything
    # under oracle/ (the oracle is test infrastructure only), and the oracle
    # shares no source with the CUDA path
    import glob
    import os
    import re
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    pkg = os.path.join(root, "paged_int8_kv_b200")
    for path in glob.glob(os.path.join(pkg, "**", "*"), recursive=True):
        if not path.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
            continue
        text = open(path, encoding="utf-8").read()
        assert not re.search(r"^\s*(import|from)\s+oracle\b", text, re.M), path
        assert "kv8_oracle" not in text and "oracle/" not in text, path
    for path in glob.glob(os.path.join(root, "oracle", "*")):
        if path.endswith((".c", ".h", ".py")):
            text = open(path, encoding="utf-8").read()
            assert not re.search(r"^\s*(import|from)\s+paged_int8_kv_b200\b", text, re.M), path
            assert not re.search(r"#\s*include\s*[<\"].*(csrc|kv8_|kv8\.h)", text), path
            assert not re.search(r"libkv8(?!_oracle)", text), path
