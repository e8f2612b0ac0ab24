"""Host-only checks of the C-ABI boundary: the library builds and loads,
exports every entry point include/moe_sparse.h declares, and rejects bad
descriptors and arguments synchronously without touching a GPU."""

import ctypes
import os
import re

import pytest

from intra_expert_activation_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_sparse.h")
CHECK_HEADER = os.path.join(ROOT, "include", "moe_sparse_check.h")


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(_lib.LIB_PATH):
        from intra_expert_activation_b200 import build
        build.build()
    return _lib.load()


def declared_functions(header=HEADER):
    src = open(header).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_sparse_\w+)\s*\(", src)))


def good_desc(**kw):
    d = dict(d_model=512, d_ff=384, n_experts=4, top_k_max=2, max_tokens=64, renormalize=1,
             n_shared=0, d_ff_shared=0, dtype=_lib.MOE_BF16, path=0, debug=0, device=0,
             gemv_max_tokens=0, gather_max_density=0.0)
    d.update(kw)
    return _lib.moe_sparse_desc(**d)


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), f"{n} declared in moe_sparse.h but not exported"
    assert set(names) == set(_lib.SIGNATURES), "binding and header disagree"


def test_only_the_abi_is_exported():
    out = os.popen(f"nm -D --defined-only {_lib.LIB_PATH}").read()
    syms = {l.split()[-1] for l in out.splitlines() if " T " in l}
    ours = {s for s in syms if s.startswith("moe_")}
    assert ours == set(declared_functions())


def test_struct_sizes_match_header():
    assert ctypes.sizeof(_lib.moe_sparse_desc) == 16 * 4
    assert ctypes.sizeof(_lib.moe_stats) == 15 * 8


def test_valid_desc_accepted(lib):
    assert lib.moe_sparse_validate_desc(ctypes.byref(good_desc())) == _lib.MOE_OK
    f32 = good_desc(dtype=_lib.MOE_F32, d_model=256, d_ff=512)
    assert lib.moe_sparse_validate_desc(ctypes.byref(f32)) == _lib.MOE_OK
    shared = good_desc(n_shared=2, d_ff_shared=256)
    assert lib.moe_sparse_validate_desc(ctypes.byref(shared)) == _lib.MOE_OK
    gate = good_desc(score=_lib.MOE_SCORE_GATE)
    assert lib.moe_sparse_validate_desc(ctypes.byref(gate)) == _lib.MOE_OK


@pytest.mark.parametrize("kw,code", [
    (dict(d_model=0), _lib.MOE_ERR_INVALID),
    (dict(d_model=320), _lib.MOE_ERR_UNSUPPORTED),           # bf16 needs d % 256
    (dict(d_ff=100), _lib.MOE_ERR_UNSUPPORTED),              # bf16 needs d_ff % 128
    (dict(n_experts=300), _lib.MOE_ERR_UNSUPPORTED),
    (dict(top_k_max=5), _lib.MOE_ERR_INVALID),               # > n_experts
    (dict(max_tokens=-1), _lib.MOE_ERR_INVALID),
    (dict(max_tokens=70000), _lib.MOE_ERR_UNSUPPORTED),
    (dict(dtype=7), _lib.MOE_ERR_INVALID),
    (dict(path=9), _lib.MOE_ERR_INVALID),
    (dict(score=2), _lib.MOE_ERR_INVALID),
    (dict(n_shared=1, d_ff_shared=0), _lib.MOE_ERR_UNSUPPORTED),
    (dict(n_shared=9, d_ff_shared=128), _lib.MOE_ERR_INVALID),
    (dict(dtype=_lib.MOE_F32, d_model=256, d_ff=512, path=3), _lib.MOE_ERR_UNSUPPORTED),
    (dict(gather_max_density=1.5), _lib.MOE_ERR_INVALID),
    (dict(gemv_max_tokens=-2), _lib.MOE_ERR_INVALID),
    (dict(out_f32=3), _lib.MOE_ERR_INVALID),
])
def test_bad_desc_rejected(lib, kw, code):
    d = good_desc(**kw)
    assert lib.moe_sparse_validate_desc(ctypes.byref(d)) == code
    assert lib.moe_sparse_last_error(None)
    ctx = ctypes.c_void_p()
    assert lib.moe_sparse_init(ctypes.byref(d), ctypes.byref(ctx)) == code
    assert not ctx.value


def test_null_desc_and_ctx(lib):
    assert lib.moe_sparse_validate_desc(None) == _lib.MOE_ERR_INVALID
    ctx = ctypes.c_void_p()
    assert lib.moe_sparse_init(None, ctypes.byref(ctx)) == _lib.MOE_ERR_INVALID
    assert lib.moe_sparse_forward(None, None, 1, None, None, None, None, None, 0.0, 1, None,
                                  None) == _lib.MOE_ERR_INVALID
    assert lib.moe_sparse_get_stats(None, None, None) == _lib.MOE_ERR_INVALID
    assert lib.moe_sparse_destroy(None) == _lib.MOE_OK


def test_workspace_bytes_scale_with_tokens(lib):
    small = ctypes.c_size_t()
    big = ctypes.c_size_t()
    assert lib.moe_sparse_workspace_bytes(ctypes.byref(good_desc(max_tokens=16)),
                                          ctypes.byref(small)) == _lib.MOE_OK
    assert lib.moe_sparse_workspace_bytes(ctypes.byref(good_desc(max_tokens=4096)),
                                          ctypes.byref(big)) == _lib.MOE_OK
    assert 0 < small.value < big.value
    # h^T, X_perm and Y dominate: at least P * (2*d + 4*d) bytes
    assert big.value >= 4096 * 2 * (2 * 512 + 4 * 512)


def test_stage_names(lib):
    names = [lib.moe_sparse_stage_name(i).decode() for i in range(len(_lib.STAGES))]
    assert tuple(names) == _lib.STAGES
    assert lib.moe_sparse_stage_name(len(_lib.STAGES)) is None


def test_init_without_gpu_fails_cleanly(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    ctx = ctypes.c_void_p()
    st = lib.moe_sparse_init(ctypes.byref(good_desc()), ctypes.byref(ctx))
    assert st == _lib.MOE_ERR_CUDA
    assert not ctx.value
    assert lib.moe_sparse_last_error(None)


def test_binding_refuses_missing_library(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "nope.so"))
    monkeypatch.setattr(_lib, "_LIB", None)
    with pytest.raises(RuntimeError, match="missing"):
        _lib.load()


def test_header_is_plain_c_and_links(lib, tmp_path):
    """A C11 program compiled against include/moe_sparse.h with warnings as
    errors links against the library and gets the host-only answers
    (descriptor checks, workspace size, stage names, clean init failure)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if not cc:
        pytest.skip("no C compiler")
    exe = str(tmp_path / "c_abi_check")
    pkg = os.path.dirname(_lib.LIB_PATH)
    r = subprocess.run([cc, "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic",
                        "-I", os.path.join(ROOT, "include"),
                        os.path.join(ROOT, "tests", "c_abi_check.c"), "-o", exe,
                        "-L", pkg, "-lmoe_sparse", f"-Wl,-rpath,{pkg}"],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip().endswith("OK"), r.stdout + r.stderr


@pytest.mark.timeout(600)
def test_checked_build_exports_the_same_abi():
    """build.py --check compiles the kernels' bounds checks in (MOE_CHECK=1)
    into a separate library with the same exported entry points, which the
    binding loads under MOE_SPARSE_LIB=check."""
    import subprocess
    import sys
    from intra_expert_activation_b200 import build
    path = build.build(check=True)
    assert path.endswith("libmoe_sparse_check.so") and os.path.exists(path)
    out = os.popen(f"nm -D --defined-only {path}").read()
    syms = {l.split()[-1] for l in out.splitlines() if " T " in l}
    # the ABI plus the checked build's test hook (include/moe_sparse_check.h)
    check_only = set(declared_functions(CHECK_HEADER))
    assert check_only == set(_lib.CHECK_SIGNATURES)
    assert {s for s in syms if s.startswith("moe_")} == set(declared_functions()) | check_only
    r = subprocess.run([sys.executable, "-c",
                        "from intra_expert_activation_b200 import _lib; print(_lib.LIB_PATH)"],
                       capture_output=True, text=True, cwd=ROOT,
                       env={**os.environ, "MOE_SPARSE_LIB": "check"})
    assert r.returncode == 0 and r.stdout.strip() == path, r.stdout + r.stderr
