"""Host-side checks that need no GPU: the C ABI library builds, loads and exports every entry
point that include/mcs.h declares; the binding declares the same set."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mcs.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mcs_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from free_sparse_attention_reuse_b200 import build
    path = build.build()
    return ctypes.CDLL(path)


def test_header_declares_the_documented_entry_points():
    names = declared_functions()
    for n in ("mcs_dense_attn", "mcs_group", "mcs_select", "mcs_sparse_attn", "mcs_residual", "mcs_anchor",
              "mcs_workspace_size", "mcs_status_string", "mcs_sync_status", "mcs_abi_version"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in declared_functions():
        assert hasattr(lib, n), f"{n} not exported"


def test_binding_covers_every_declared_symbol():
    from free_sparse_attention_reuse_b200 import EXPORTS
    assert sorted(EXPORTS) == declared_functions()


def test_status_strings_without_gpu(lib):
    lib.mcs_status_string.restype = ctypes.c_char_p
    lib.mcs_abi_version.restype = ctypes.c_int
    assert lib.mcs_abi_version() == 1
    assert lib.mcs_status_string(0) == b"MCS_OK"
    assert b"BAD_INDEX" in lib.mcs_status_string(6)
    assert b"unknown" in lib.mcs_status_string(99)


def test_library_is_built_for_sm100a(lib):
    # the fatbin's ELF note names the architecture; check via the build flags instead of
    # reading compiled code: the build must pass exactly this gencode
    from free_sparse_attention_reuse_b200 import build
    assert "arch=compute_100a,code=sm_100a" in build.flags()


def test_product_path_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "free_sparse_attention_reuse_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".cpp", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", text, re.M), f
                assert "mcs_oracle" not in text, f


def test_missing_library_fails_loudly(tmp_path):
    from free_sparse_attention_reuse_b200 import _lib
    saved = _lib._lib
    _lib._lib = None
    try:
        with pytest.raises(RuntimeError, match="libmcs.so not found"):
            _lib.load(str(tmp_path / "absent" / "libmcs.so"))
    finally:
        _lib._lib = saved


def test_binding_refuses_host_tensors():
    # the product path has no CPU fallback: host tensors are rejected before any call
    import torch
    from free_sparse_attention_reuse_b200 import api
    q = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        api.dense_attn(q, q, q)
    with pytest.raises(ValueError, match="CUDA"):
        api.sparse_attn(q, q, q, torch.zeros(1, 1, 128, dtype=torch.int32), 64,
                        torch.zeros(1, 1, 2, 8, dtype=torch.int32))
    with pytest.raises(ValueError, match="CUDA"):
        api.perquery_attn(q, q, q, 8)


def test_shape_limits_rejected_before_any_device_call():
    # shape checks come first in every entry point, so these return without a GPU
    from free_sparse_attention_reuse_b200 import _lib
    lib = _lib.load()
    for B, H, N, d in ((1, 1, (1 << 24) + 128, 128),   # N > 2^24
                       (1, 300, 1 << 24, 64),          # B*H*N > 2^32 - 1
                       (256, 256, 128, 64),            # B*H > 65535
                       (1, 1, 1024, 96)):              # d not in {64, 128}
        s = _lib.Shape(B, H, N, d, 0.0)
        assert lib.mcs_dense_attn(s, None, None, None, None, None, None) == 2
        assert lib.mcs_workspace_size(s, 128, 16) == 0
    assert lib.mcs_dense_attn(_lib.Shape(1, 1, 0, 64, 0.0), None, None, None, None, None, None) == 1


def test_host_staging_size_without_gpu():
    from free_sparse_attention_reuse_b200 import _lib
    lib = _lib.load()
    s = _lib.Shape(1, 24, 32256, 128, 0.0)
    assert lib.mcs_host_staging_size(s, 2) == 2 * 4 * 2 * 32256 * 128 * 2
    assert lib.mcs_host_staging_size(s, 100) == lib.mcs_host_staging_size(s, 24)  # at most B*H heads
    assert lib.mcs_host_staging_size(s, 0) == 0
    assert lib.mcs_host_staging_size(_lib.Shape(1, 1, 1024, 96, 0.0), 1) == 0
    # argument errors return before any device call
    assert lib.mcs_sparse_attn_host(s, None, None, None, None, 128, None, 16, None, None, 2, None, 0, None) == 1


def test_host_binding_checks_where_tensors_live():
    import torch
    from free_sparse_attention_reuse_b200 import api
    q = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16)
    perm = torch.zeros(1, 1, 128, dtype=torch.int32)
    idx = torch.zeros(1, 1, 2, 8, dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA"):  # the metadata must be on the device
        api.sparse_attn_host(q, q, q, perm, 64, idx)
    with pytest.raises(ValueError, match="bfloat16"):
        api.sparse_attn_host(q.float(), q, q, perm, 64, idx)


def test_binding_rejects_mismatched_shapes_before_any_call():
    # a tensor of the wrong shape or dtype would send the kernels past the end of a buffer: the
    # binding refuses it (on any device) before the library is called
    import torch
    from free_sparse_attention_reuse_b200 import api
    B, H, N, d, C = 1, 2, 256, 64, 64
    q = torch.zeros(B, H, N, d, dtype=torch.bfloat16)
    perm = torch.zeros(B, H, N, dtype=torch.int32)
    idx = torch.zeros(B, H, N // C, 16, dtype=torch.int32)
    bad = [
        (lambda: api.dense_attn(q, q[:, :1], q), "K must have shape"),
        (lambda: api.dense_attn(q, q, q, O=torch.zeros(B, H, N, 32, dtype=torch.bfloat16)), "O must have shape"),
        (lambda: api.dense_attn(q, q, q, lse=torch.zeros(B, H, N, dtype=torch.float64)), "lse must be torch.float32"),
        (lambda: api.sparse_attn(q, q, q, perm[:, :, :128], C, idx), "perm must have shape"),
        (lambda: api.sparse_attn(q, q, q, perm, C, idx[:, :, :2]), "idx must have shape"),
        (lambda: api.sparse_attn(q, q, q, perm, C, idx, R=q.float()), "R must be"),
        (lambda: api.sparse_attn(q, q, q, perm.long(), C, idx), "perm must be torch.int32"),
        (lambda: api.sparse_attn(q, q, q, perm, C, idx, out=q[:, :, :128]), "out must have shape"),
        (lambda: api.residual(q, q, q, perm, C, idx, q[:, :1]), "O_full must have shape"),
        (lambda: api.select(q, q, perm, C, 16, idx=idx[..., :8].contiguous()), "idx must hold k = 16"),
        (lambda: api.select(q, q, perm, C, 16, lse=torch.zeros(B, H, N - 1)), "lse must have shape"),
        (lambda: api.anchor(q, q, q, C, 16, out=(q, perm, idx[..., :4].contiguous(), q)), "idx must hold k = 16"),
        (lambda: api.select_blocks(q, q, perm, C, 64, 2, method="mean"), "method must be"),
        (lambda: api.perquery_attn(q, q, q, 8, out=q[:1, :1]), "out must have shape"),
        (lambda: api.group(q[0], C), "4-d"),
        (lambda: api.sparse_attn_host(q, q, q.float(), perm, C, idx), "hV must be torch.bfloat16"),
        (lambda: api.sparse_attn_host(q, q, q, perm, C, idx, out=q[:, :1]), "out must have shape"),
    ]
    for call, msg in bad:
        with pytest.raises((ValueError, TypeError), match=msg):
            call()


def test_c_program_uses_the_abi_without_python(tmp_path):
    # the ABI is plain C: a C program includes include/mcs.h, links libmcs.so and gets the
    # documented statuses back (argument paths only, no device needed)
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    from free_sparse_attention_reuse_b200 import _lib
    libdir = os.path.dirname(_lib.LIB_PATH)
    exe = tmp_path / "c_abi_check"
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                        os.path.join(ROOT, "tests", "c_abi_check.c"), "-o", str(exe), "-L", libdir, "-lmcs",
                        f"-Wl,-rpath,{libdir}"], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and "c abi ok" in r.stdout, r.stdout + r.stderr
