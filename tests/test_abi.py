"""C ABI of libjssa.so on the CPU: the library builds, loads and exports every entry
point that include/jssa.h declares; host-side validation rejects bad arguments
before any CUDA call (so these run without a GPU)."""
import ctypes as C
import os
import re
import subprocess

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "jssa.h")


@pytest.fixture(scope="module")
def lib():
    from token_level_sparse_jssa_b200 import build
    build.build()
    from token_level_sparse_jssa_b200 import _binding
    return _binding.load()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"JSSA_API\s+[\w\s\*]+?\b(jssa_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("jssa_project_keys", "jssa_score", "jssa_topk", "jssa_indexed_attn", "jssa_decode_step",
                     "jssa_dense_decode", "jssa_workspace_size"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    from token_level_sparse_jssa_b200 import _binding
    out = subprocess.run(["nm", "-D", "--defined-only", _binding.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\sT\s(jssa_\w+)$", out, flags=re.M))
    assert set(declared_functions()) <= exported
    for name in declared_functions():
        assert hasattr(lib, name)
    assert set(_binding.EXPORTS) == set(declared_functions())


def test_header_compiles_as_plain_c(tmp_path):
    src = tmp_path / "t.c"
    src.write_text('#include "jssa.h"\nint main(void){ jssa_layout L; (void)L; return (int)JSSA_OK; }\n')
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.dirname(HEADER), "-c", str(src),
                    "-o", str(tmp_path / "t.o")], check=True)


def test_layout_struct_matches_header_size(tmp_path):
    from token_level_sparse_jssa_b200 import Layout
    src = tmp_path / "s.c"
    src.write_text('#include <stdio.h>\n#include "jssa.h"\nint main(void){ printf("%zu", sizeof(jssa_layout)); return 0; }\n')
    exe = tmp_path / "s"
    subprocess.run(["gcc", "-I", os.path.dirname(HEADER), str(src), "-o", str(exe)], check=True)
    assert int(subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout) == C.sizeof(Layout)


def test_status_strings_and_version(lib):
    from token_level_sparse_jssa_b200 import status_string, version
    assert status_string(0) == "ok"
    assert "workspace" in status_string(3)
    assert status_string(99) == "unknown status"
    assert version() >= 10000


def _layout(**kw):
    from token_level_sparse_jssa_b200 import Layout
    L = Layout()
    B, Hq, Hkv, d, r, T = kw.get("B", 2), kw.get("Hq", 8), kw.get("Hkv", 2), kw.get("d", 128), kw.get("r", 32), \
        kw.get("T", 1024)
    L.mode, L.B, L.Hq, L.Hkv, L.d_k, L.d_v, L.r, L.out_dtype = kw.get("mode", 0), B, Hq, Hkv, d, kw.get("dv", d), r, \
        kw.get("out", 0)
    L.T_cap = T
    L.kp_dtype = kw.get("kp", 0)
    for i, v in enumerate((Hkv * T * d, T * d, d)):
        L.k_stride[i] = v
        L.v_stride[i] = v
    for i, v in enumerate((Hkv * T * r, T * r, r)):
        L.kp_stride[i] = v
    for key in ("k_stride", "v_stride", "kp_stride"):
        if key in kw:
            for i, v in enumerate(kw[key]):
                getattr(L, key)[i] = v
    return L


FAKE = 0x10000  # a 16-byte aligned non-null value; validation rejects the call before it is used


@pytest.mark.parametrize("kw,code", [
    (dict(Hq=7), 1),                 # Hq not a multiple of Hkv
    (dict(r=0), 1),
    (dict(r=256), 1),                # r > d
    (dict(r=24), 2),                 # r not a supported power of two
    (dict(d=96), 2),                 # unsupported head dim
    (dict(Hq=64, Hkv=2), 2),         # G = 32
    (dict(dv=64), 1),                # d_v != d_k in GQA -> invalid? d_v < d_k is unsupported
    (dict(mode=1), 2),               # MLA needs Hkv=1, 576/512, 128 heads
    (dict(mode=5), 1),
    (dict(out=3), 1),
    (dict(T=0), 1),
    (dict(k_stride=(8, 8, 100)), 1),  # stride not a multiple of 16 bytes
    (dict(kp_stride=(0, 0, 64)), 2),  # Kp rows must be contiguous
    (dict(kp=2), 1),                  # unknown Kp storage type
    (dict(kp=1, r=8, d=64), 2),       # E4M3 rows of 8 bytes
    (dict(kp=1, r=16, kp_stride=(24, 24, 16)), 1),  # E4M3 strides must be multiples of 16 bytes
])
def test_bad_layouts_are_rejected_on_the_host(lib, kw, code):
    L = _layout(**kw)
    got = lib.jssa_project_keys(C.byref(L), FAKE, FAKE, FAKE, FAKE, None, 1, None)
    if kw == dict(dv=64):
        assert got in (1, 2)
    else:
        assert got == code


def test_mla_dense_decode_validates_on_the_host(lib):
    # the latent layout has a dense (full-cache comparator) path: its arguments are checked
    # before anything is launched
    L = _layout(mode=1, B=1, Hq=128, Hkv=1, d=576, dv=512, r=64)
    assert lib.jssa_dense_decode(C.byref(L), None, FAKE, FAKE, FAKE, 0, 1.0, FAKE, None, C.c_void_p(FAKE), 1 << 30,
                                 None) == 1
    assert lib.jssa_dense_decode(C.byref(L), FAKE, FAKE, FAKE, FAKE, -1, 1.0, FAKE, None, C.c_void_p(FAKE), 1 << 30,
                                 None) == 1
    bad = _layout(mode=1, B=1, Hq=64, Hkv=1, d=576, dv=512, r=64)   # the latent kernel takes 128 heads
    assert lib.jssa_dense_decode(C.byref(bad), FAKE, FAKE, FAKE, FAKE, 0, 1.0, FAKE, None, C.c_void_p(FAKE), 1 << 30,
                                 None) == 2


def test_bad_arguments_are_rejected_before_launch(lib):
    L = _layout()
    ws = C.c_void_p(FAKE)
    # null pointers
    assert lib.jssa_project_keys(C.byref(L), None, FAKE, FAKE, FAKE, None, 4, None) == 1
    assert lib.jssa_project_keys(C.byref(L), FAKE, FAKE, FAKE, None, None, 4, None) == 1
    # misaligned cache pointer
    assert lib.jssa_project_keys(C.byref(L), FAKE + 2, FAKE, FAKE, FAKE, None, 4, None) == 1
    # n_tokens out of range
    assert lib.jssa_project_keys(C.byref(L), FAKE, FAKE, FAKE, FAKE, None, -1, None) == 1
    assert lib.jssa_project_keys(C.byref(L), FAKE, FAKE, FAKE, FAKE, None, 5000, None) == 1
    # n_tokens = 0 is a no-op that touches nothing
    assert lib.jssa_project_keys(C.byref(L), None, None, None, None, None, 0, None) == 0
    # k < 1, negative window
    assert lib.jssa_topk(C.byref(L), FAKE, FAKE, 0, 0, FAKE, FAKE, None, 0, None) == 1
    assert lib.jssa_topk(C.byref(L), FAKE, FAKE, 4, -1, FAKE, FAKE, None, 0, None) == 1
    assert lib.jssa_indexed_attn(C.byref(L), FAKE, FAKE, FAKE, None, 4, FAKE, FAKE, 0, 1.0, FAKE, None, ws, 1 << 30,
                                 None) == 1
    assert lib.jssa_decode_step(C.byref(L), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, -1, 4, 0, 1.0, FAKE, None, None,
                                None, ws, 1 << 30, None) == 1
    assert lib.jssa_dense_decode(C.byref(L), FAKE, FAKE, FAKE, FAKE, -3, 1.0, FAKE, None, ws, 1 << 30, None) == 1
    assert lib.jssa_dense_decode(None, FAKE, FAKE, FAKE, FAKE, 0, 1.0, FAKE, None, ws, 1 << 30, None) == 1
    # workspace status helpers check their arguments
    assert lib.jssa_workspace_init(None, 0, None) == 3
    assert lib.jssa_workspace_init(C.c_void_p(FAKE + 16), 1024, None) == 3  # not 256-byte aligned
    flags = C.c_int32(0)
    assert lib.jssa_read_device_status(None, 0, C.byref(flags), None) == 3


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU error path")
def test_workspace_size_without_a_device_reports_a_cuda_error(lib):
    n = C.c_size_t(0)
    assert lib.jssa_workspace_size(C.byref(_layout()), 16, 0, C.byref(n)) == 4


def test_package_import_does_not_load_the_library_and_fails_loudly_when_missing(tmp_path):
    code = ("import token_level_sparse_jssa_b200 as j, token_level_sparse_jssa_b200._binding as b;"
            "assert b._lib is None\n"
            "try:\n    b.load(r'%s')\nexcept RuntimeError as e:\n    print('LOUD', e)\n" % (tmp_path / "missing.so"))
    out = subprocess.run(["python", "-c", code], capture_output=True, text=True, cwd=ROOT, check=True).stdout
    assert "LOUD" in out and "no fallback" in out


def test_calibration_entry_points_validate_on_the_host(lib):
    L = _layout(B=2, Hq=8, Hkv=2, d=128, r=32, T=1024)
    n = C.c_size_t(0)
    assert lib.jssa_calibrate_workspace_size(C.byref(L), C.byref(n)) == 0
    # status word (256 B) + [Hkv][2 moments + 3 Jacobi matrices][d][d] doubles + [Hkv][2][8] doubles
    assert n.value == 256 + ((2 * 5 * 128 * 128 + 2 * 2 * 8) * 8 + 255) // 256 * 256
    assert lib.jssa_calibrate_workspace_size(C.byref(L), None) == 1
    ws = C.c_void_p(FAKE)
    big = n.value
    assert lib.jssa_calibrate(C.byref(L), None, FAKE, 100, FAKE, None, ws, big, None) == 1       # no queries
    assert lib.jssa_calibrate(C.byref(L), FAKE, FAKE, 0, FAKE, None, ws, big, None) == 1         # no tokens
    assert lib.jssa_calibrate(C.byref(L), FAKE, FAKE, 1025, FAKE, None, ws, big, None) == 1      # beyond T_cap
    assert lib.jssa_calibrate(C.byref(L), FAKE + 8, FAKE, 100, FAKE, None, ws, big, None) == 1   # misaligned
    assert lib.jssa_calibrate(C.byref(L), FAKE, FAKE, 100, FAKE, None, ws, big - 256, None) == 3  # small workspace
    assert lib.jssa_calibrate(C.byref(L), FAKE, FAKE, 100, FAKE, None, C.c_void_p(FAKE + 64), big, None) == 3


def test_voting_and_gather_entry_points_validate_on_the_host(lib):
    L = _layout()
    ws = C.c_void_p(FAKE)
    args = [FAKE, FAKE, FAKE, FAKE, FAKE, 0, 16, 0]
    assert lib.jssa_vote_select(C.byref(L), *args, C.c_float(0.0), FAKE, FAKE, ws, 1 << 30, None) == 1   # sm_scale
    assert lib.jssa_vote_select(C.byref(L), *args, C.c_float(-1.0), FAKE, FAKE, ws, 1 << 30, None) == 1
    bad_k = [FAKE, FAKE, FAKE, FAKE, FAKE, 0, 0, 0]
    assert lib.jssa_vote_select(C.byref(L), *bad_k, C.c_float(0.1), FAKE, FAKE, ws, 1 << 30, None) == 1   # k = 0
    assert lib.jssa_vote_select(C.byref(L), None, *args[1:], C.c_float(0.1), FAKE, FAKE, ws, 1 << 30, None) == 1
    n = C.c_size_t(0)
    assert lib.jssa_gather_size(C.byref(L), 0, 0, C.byref(n)) == 1


def test_staging_copy_validates_on_the_host(lib):
    # null pointers, sizes that are not whole 16-byte words and misaligned pointers are
    # rejected before any CUDA call; an empty copy is a no-op
    assert lib.jssa_copy_mapped(None, FAKE, 16, None) == 1
    assert lib.jssa_copy_mapped(FAKE, None, 16, None) == 1
    assert lib.jssa_copy_mapped(FAKE, FAKE, 24, None) == 1
    assert lib.jssa_copy_mapped(FAKE + 8, FAKE, 16, None) == 1
    assert lib.jssa_copy_mapped(FAKE, FAKE + 4, 16, None) == 1
    assert lib.jssa_copy_mapped(None, None, 0, None) == 0
