"""The C-ABI library loads and exports every entry point ``include/iskv.h``
declares, and its host-side argument checks work without a GPU."""

import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "iskv.h")


def _lib():
    so = os.path.join(ROOT, "online_rank_kv_b200", "libiskv.so")
    if not os.path.exists(so):
        import importlib.util
        spec = importlib.util.spec_from_file_location(
            "_iskv_build", os.path.join(ROOT, "online_rank_kv_b200", "build.py"))
        mod = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(mod)
        mod.build()
    import online_rank_kv_b200 as ik
    return ik


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"ISKV_API\s+[\w\s\*]+?\b(iskv_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("iskv_create", "iskv_append", "iskv_compress_block", "iskv_decode_attention",
              "iskv_reconstruct", "iskv_destroy", "iskv_status", "iskv_sync"):
        assert n in names


def test_every_declared_symbol_is_exported():
    ik = _lib()
    out = subprocess.run(["nm", "-D", "--defined-only", ik.lib_path()], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r" T (iskv_\w+)", out))
    for n in _declared():
        assert n in exported, n
        assert hasattr(ik.LIB, n)
    assert set(ik.EXPORTED) == set(_declared())


def test_config_struct_layout_matches_header(tmp_path):
    ik = _lib()
    src = tmp_path / "sz.c"
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "iskv.h"\n'
                   'int main(){printf("%zu %zu %zu %zu",sizeof(iskv_config),'
                   'offsetof(iskv_config,rope_theta),offsetof(iskv_config,sync),'
                   'offsetof(iskv_config,ring_extra));return 0;}\n')
    exe = tmp_path / "sz"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)],
                   check=True)
    got = [int(x) for x in subprocess.run([str(exe)], capture_output=True, text=True,
                                          check=True).stdout.split()]
    C = ik._Cfg
    assert got == [ctypes.sizeof(C), C.rope_theta.offset, C.sync.offset, C.ring_extra.offset]


def test_defaults_and_strings():
    ik = _lib()
    c = ik._Cfg()
    assert ik.LIB.iskv_config_default(ctypes.byref(c)) == 0
    assert (c.kv_heads, c.q_heads, c.head_dim, c.rank_k, c.rank_v, c.window, c.block) == \
        (8, 32, 128, 32, 64, 1024, 64)
    assert ik.LIB.iskv_config_default(None) == -1
    for code in (0, -1, -2, -3, -4, -5, -6, -7, -8, -9):
        assert ik.LIB.iskv_strerror(code) != b"unknown status"
    assert set(ik._ERRORS) == {-1, -2, -3, -4, -5, -6, -7, -8, -9}
    assert ik.LIB.iskv_strerror(42) == b"unknown status"


@pytest.mark.parametrize("field,value,code", [
    ("head_dim", 64, -7), ("block", 32, -7), ("rank_k", 24, -7), ("rank_v", 144, -7),
    ("q_heads", 12, -1), ("window", 100, -1), ("layers", 0, -1), ("layers", 129, -1),
    ("kv_dtype", 3, -1), ("coef_dtype", 7, -1), ("max_deferred", 65, -1),
    ("ring_extra", 10, -1), ("max_tokens", 0, -1), ("q_heads", 8 * 9, -7),
    ("rope_theta", 0.5, -1), ("sync", 2, -1),
])
def test_create_rejects_bad_configs_before_touching_the_gpu(field, value, code):
    ik = _lib()
    c = ik._Cfg()
    ik.LIB.iskv_config_default(ctypes.byref(c))
    setattr(c, field, value)
    h = ctypes.c_void_p(123)
    assert ik.LIB.iskv_create(ctypes.byref(c), None, ctypes.byref(h)) == code
    assert h.value is None


def test_null_handles():
    ik = _lib()
    assert ik.LIB.iskv_destroy(None) == 0
    assert ik.LIB.iskv_create(None, None, None) == -1
    T = ctypes.c_int64()
    assert ik.LIB.iskv_get_counts(None, 0, ctypes.byref(T), None) == -1
    assert ik.LIB.iskv_status(None) == -1
    assert ik.LIB.iskv_compress_block(None, 0, 0, None) == -1


def test_every_handle_call_refuses_a_null_handle_on_the_host():
    """Each entry point that takes a cache returns INVALID_ARG for a NULL
    handle (or NULL operands) before any CUDA call, so these run without a GPU."""
    ik = _lib()
    L = ik.LIB
    n = ctypes.c_int(7)
    a, b = ctypes.c_int64(), ctypes.c_int64()
    calls = {
        "iskv_append": lambda: L.iskv_append(None, 0, None, None, 1, None, ctypes.byref(n)),
        "iskv_compress_block_async": lambda: L.iskv_compress_block_async(None, 0, 0, None, None),
        "iskv_sync": lambda: L.iskv_sync(None, 0, None),
        "iskv_decode_attention": lambda: L.iskv_decode_attention(None, 0, None, None, None),
        "iskv_decode_kernel": lambda: L.iskv_decode_kernel(None, 0, ctypes.byref(n)),
        "iskv_reconstruct": lambda: L.iskv_reconstruct(None, 0, 0, None, None),
        "iskv_get_factors": lambda: L.iskv_get_factors(None, 0, 0, None, None, None, None),
        "iskv_kv_bytes": lambda: L.iskv_kv_bytes(None, ctypes.byref(a), ctypes.byref(b)),
        "iskv_decode_attention_noalloc": lambda: L.iskv_decode_attention_noalloc(None, None, None, None),
        "iskv_quantize_rows": lambda: L.iskv_quantize_rows(None, 32, None, 0, None, None, None),
    }
    for name, call in calls.items():
        assert call() == -1, name
    assert n.value == 7                       # outputs untouched on refusal


def test_binding_structs_match_the_header_layout(tmp_path):
    """The ctypes mirrors of iskv_config and iskv_decode_operands have the C
    structs' size and field offsets (compiled here with the host compiler)."""
    import shutil
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    ik = _lib()
    structs = {"iskv_config": ik._Cfg, "iskv_decode_operands": ik.DecodeOperands}
    lines = ['#include <cstddef>', '#include <cstdio>', '#include "iskv.h"', "int main() {"]
    for cname, py in structs.items():
        lines.append(f'    std::printf("{cname} size %zu\\n", sizeof({cname}));')
        for fname, _ in py._fields_:
            lines.append(f'    std::printf("{cname} {fname} %zu\\n", offsetof({cname}, {fname}));')
    lines.append("}")
    src = tmp_path / "layout.cpp"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run([cxx, "-std=c++17", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)],
                   check=True)
    got = {}
    for line in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.splitlines():
        cname, field, value = line.split()
        got[(cname, field)] = int(value)
    for cname, py in structs.items():
        assert got[(cname, "size")] == ctypes.sizeof(py), cname
        for fname, _ in py._fields_:
            assert got[(cname, fname)] == getattr(py, fname).offset, (cname, fname)


def test_code_format_checks_on_the_host():
    """Latent-channel code formats: words per row, and create refuses a format
    whose groups do not cover the rank or use an unsupported width."""
    ik = _lib()
    q = ik.QuantFormat.of([(8 * 2, 8), (16, 2)])
    assert ik.LIB.iskv_quant_words(ctypes.byref(q)) == 16 * 8 // 32 + 16 * 2 // 32
    assert ik.LIB.iskv_quant_words(ctypes.byref(ik.QuantFormat.of([(16, 3)]))) == -1
    assert ik.LIB.iskv_quant_words(ctypes.byref(ik.QuantFormat.of([(24, 8)]))) == -1
    assert ik.LIB.iskv_quant_words(None) == -1
    for qk, qv in (([(16, 8)], [(32, 8), (32, 4)]),          # K groups cover 16 of 32
                   ([(32, 8)], [(32, 8), (32, 5)]),          # 5-bit codes
                   ([(32, 0)], [(64, 8)])):                  # no coded group
        cfg = ik.Config(rank_k=32, rank_v=64, coef_quant=1, quant_k=qk, quant_v=qv)
        h = ctypes.c_void_p(1)
        assert ik.LIB.iskv_create(ctypes.byref(cfg._c()), None, ctypes.byref(h)) == -1
        assert h.value is None
