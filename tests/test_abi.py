"""CPU-side checks of the C ABI: the library loads without a GPU, exports
every symbol include/mla.h declares, and rejects bad arguments before it
touches the device.  No compute call is made here."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mla.h")
PKG = os.path.join(ROOT, "latent_compressed_attention_absorbed_b200")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mla_[a-z_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def built():
    from latent_compressed_attention_absorbed_b200 import build
    return build.build()


def test_header_declares_the_entry_points():
    from latent_compressed_attention_absorbed_b200 import binding
    assert _declared() == sorted(binding.EXPORTS)


def test_library_exports_every_declared_symbol(built):
    out = subprocess.run(["nm", "-D", "--defined-only", built], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (mla_[a-z_]+)$", out, flags=re.M))
    missing = set(_declared()) - exported
    assert not missing, missing


def test_library_loads_and_reports_version(built):
    from latent_compressed_attention_absorbed_b200 import binding
    lib = binding.Library(built)
    assert lib.version() == 101
    assert lib.lib.mla_last_error() == b""


def test_argument_errors_need_no_device(built):
    from latent_compressed_attention_absorbed_b200 import binding as bd
    lib = bd.Library(built)
    L = lib.lib
    # NULL dims
    assert L.mla_decode(None, None, None, None, None, None, None, 1, 1, None, None, 0, None) == -1
    assert b"dims" in L.mla_last_error()
    # odd RoPE width
    d = bd.Dims(128, 512, 63, 128, 128, bd.MLA_DTYPE_BF16, 10000.0, 0.0)
    assert L.mla_decode(ctypes.byref(d), None, None, None, None, None, None, 1, 1, None, None, 0, None) == -2
    # unknown dtype
    d = bd.Dims(128, 512, 64, 128, 128, 7, 10000.0, 0.0)
    assert L.mla_append_cache(ctypes.byref(d), None, None, None, 1, 1, None, None) == -1
    # negative batch
    d = bd.Dims(4, 32, 8, 16, 16, bd.MLA_DTYPE_F32, 10000.0, 0.0)
    assert L.mla_decode(ctypes.byref(d), None, None, None, None, None, None, -1, 1, None, None, 0, None) == -1
    # q_len out of range
    assert L.mla_decode(ctypes.byref(d), None, None, None, None, None, None, 1, 0, None, None, 0, None) == -1
    # empty batch is a successful no-op
    assert L.mla_decode(ctypes.byref(d), None, None, None, None, None, None, 0, 1, None, None, 0, None) == 0
    # NULL tensors
    assert L.mla_decode(ctypes.byref(d), None, None, None, None, None, None, 2, 1, None, None, 0, None) == -1
    # misaligned pointer
    buf = ctypes.create_string_buffer(256)
    a = ctypes.addressof(buf)
    a16 = (a + 15) & ~15
    p_ok, p_bad = ctypes.c_void_p(a16), ctypes.c_void_p(a16 + 2)
    seq = ctypes.c_void_p(a16)
    cache = bd.Cache(a16, 2, 4, 4 * 40, 40)
    assert L.mla_decode(ctypes.byref(d), p_bad, p_ok, p_ok, p_ok, ctypes.byref(cache), seq, 2, 1, p_ok, p_ok,
                        1 << 20, None) == -3
    # cache stride narrower than a row (d_c + d_r = 40)
    cache = bd.Cache(a16, 2, 4, 4 * 32, 32)
    assert L.mla_decode(ctypes.byref(d), p_ok, p_ok, p_ok, p_ok, ctypes.byref(cache), seq, 2, 1, p_ok, p_ok,
                        1 << 20, None) == -2
    # cache with too few sequences
    cache = bd.Cache(a16, 1, 4, 4 * 40, 40)
    assert L.mla_decode(ctypes.byref(d), p_ok, p_ok, p_ok, p_ok, ctypes.byref(cache), seq, 2, 1, p_ok, p_ok,
                        1 << 20, None) == -2


def test_binding_refuses_to_run_without_the_library(tmp_path):
    from latent_compressed_attention_absorbed_b200 import binding
    with pytest.raises(FileNotFoundError):
        binding.Library(str(tmp_path / "libmla.so"))


def test_product_code_never_touches_the_oracle():
    # Only tests, smoke() and the CPU-baseline leg of bench.py may use oracle/.
    for dirpath, _, files in os.walk(PKG):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert not re.search(r"^\s*(from|import)\s+oracle\b", text, flags=re.M), f
                assert "mla_oracle" not in text, f


def test_oracle_never_touches_the_product():
    odir = os.path.join(ROOT, "oracle")
    for f in os.listdir(odir):
        if f.endswith(".py"):
            text = open(os.path.join(odir, f), encoding="utf-8").read()
            assert "latent_compressed_attention_absorbed_b200" not in text, f
            assert "libmla" not in text, f
