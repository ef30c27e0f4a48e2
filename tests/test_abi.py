"""CPU checks of the C ABI: the library builds for sm_100a, loads, and exports every function
include/llvq.h declares; calls that need a device fail with a status code, not a crash."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "llvq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(llvq_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from codebook_free_lattice_b200 import build
    build.build()
    import codebook_free_lattice_b200 as L
    return L.lib()


def test_header_declares_the_boundary():
    fns = declared_functions()
    for f in ("llvq_codec_create", "llvq_codec_destroy", "llvq_codec_info", "llvq_decode", "llvq_gemv",
              "llvq_gemm_smallbatch", "llvq_get_error", "llvq_status_string"):
        assert f in fns


def test_library_exports_every_declared_symbol(lib):
    for f in declared_functions():
        assert hasattr(lib, f), f


def test_binding_lists_the_same_names():
    import codebook_free_lattice_b200 as L
    assert sorted(L.EXPORTED) == [f for f in declared_functions() if f in L.EXPORTED]
    assert set(declared_functions()) <= set(L.EXPORTED)


def test_status_strings(lib):
    import codebook_free_lattice_b200 as L
    assert L.llvq_status_string(0) == "ok"
    assert L.llvq_status_string(1) == "invalid argument"
    assert L.llvq_status_string(99) == "unknown status"


def test_host_argument_checks_without_device(lib):
    """Null handles and pointers are rejected before any device work."""
    import codebook_free_lattice_b200 as L
    assert lib.llvq_codec_create(48, None) == L.LLVQ_ERR_ARG
    h = C.c_void_p()
    assert lib.llvq_codec_create(40, C.byref(h)) == L.LLVQ_ERR_UNSUPPORTED
    assert lib.llvq_decode(None, None, 8, 1, None, None) == L.LLVQ_ERR_ARG
    assert lib.llvq_gemv(None, None, None, None, None) == L.LLVQ_ERR_ARG
    flags = C.c_uint32()
    assert lib.llvq_get_error(None, None, C.byref(flags)) == L.LLVQ_ERR_ARG
    assert lib.llvq_encode(None, None, 1, None, 8, None) == L.LLVQ_ERR_ARG
    assert lib.llvq_gemm_smallbatch(None, None, None, 1, None, None) == L.LLVQ_ERR_ARG
    assert lib.llvq_decode_noalloc(72, None, 16, 1, None, None) == L.LLVQ_ERR_UNSUPPORTED
    assert "48-bit" in L.lib().llvq_last_error_message().decode()
    assert lib.llvq_search(None, 13, 0, 1.0, None, 1, None, None, None, 0, None, None) == L.LLVQ_ERR_ARG
    assert lib.llvq_spherical_gptq(None, 13, 1, 24, None, None, None, None, None, 0, None) == L.LLVQ_ERR_ARG
    # workspace: the block matrices (cols^2 doubles) plus per-row scratch, each part 256-aligned
    assert lib.llvq_spherical_gptq_workspace(4096, 4104) == 4104 * 4104 * 8 + 4096 * 24 * (4 + 1 + 8)
    assert lib.llvq_spherical_gptq_workspace(3, 48) == 48 * 48 * 8 + 512 + 256 + 768   # 288, 72, 576 B rounded up
    for bad in ((-1, 48), (8, 40), (8, 0), (70000, 48)):
        assert lib.llvq_spherical_gptq_workspace(*bad) == 0


def test_flag_values_match_the_header():
    import codebook_free_lattice_b200 as L
    src = open(os.path.join(ROOT, "include", "llvq.h")).read()
    for name in ("LLVQ_FLAG_INDEX_RANGE", "LLVQ_FLAG_WAIT_TIMEOUT", "LLVQ_FLAG_NOT_CODED", "LLVQ_FLAG_SEARCH_INPUT"):
        val = int(re.search(r"#define\s+" + name + r"\s+(0x[0-9a-fA-F]+)u", src).group(1), 16)
        assert getattr(L, name) == val


def test_ncu_record_hash_ignores_comments(tmp_path, monkeypatch):
    """The bench ties its committed ncu record to the kernel code, not to comments or spacing."""
    import shutil

    import bench
    src = os.path.join(ROOT, "codebook_free_lattice_b200", "csrc")
    dst = tmp_path / "codebook_free_lattice_b200" / "csrc"
    shutil.copytree(src, dst)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_sources_hash()
    f = dst / "kernels.cuh"
    f.write_text("// a new comment line\n" + f.read_text().replace("#pragma once", "#pragma once   /* note */"))
    assert bench.kernel_sources_hash() == h0
    f.write_text(f.read_text() + "\nconstexpr int kExtra = 1;\n")
    assert bench.kernel_sources_hash() != h0


def test_no_device_is_a_status_not_a_crash(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    import codebook_free_lattice_b200 as L
    h = C.c_void_p()
    assert lib.llvq_codec_create(48, C.byref(h)) == L.LLVQ_ERR_CUDA
    assert not h.value


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    import codebook_free_lattice_b200 as L
    monkeypatch.setattr(L, "_lib", None)
    monkeypatch.setattr(L, "LIB_PATH", str(tmp_path / "absent.so"))
    with pytest.raises(ImportError):
        L.lib()
