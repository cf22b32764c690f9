"""Host-side checks of the C-ABI library (no GPU needed): it loads, exports every declared symbol,
and rejects bad arguments on the host before touching a device."""
import ctypes
import os
import re

import pytest

import gated_delta_rule_120_b200 as kda
from gated_delta_rule_120_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    _build.build()
    return kda.lib()


def declared_symbols():
    src = ""
    for name in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if name.endswith(".h"):
            with open(os.path.join(ROOT, "include", name)) as f:
                src += f.read()
    return sorted(set(re.findall(r"KDA_API\s+[\w\s\*]+?\b(kda_\w+)\s*\(", src)))


def test_every_declared_symbol_is_exported(L):
    syms = declared_symbols()
    assert len(syms) >= 6
    assert set(syms) == set(kda.ABI_SYMBOLS)
    for s in syms:
        assert hasattr(L, s), s


def test_status_strings(L):
    for code in range(6):
        assert kda.status_string(code).startswith("KDA_")
    assert kda.status_string(99) == "KDA_ERR_UNKNOWN"
    assert L.kda_version().decode().count(".") == 2


def _ws(B, T, H, Dk, Dv, C, N, dt):
    out = ctypes.c_size_t(0)
    rc = kda.lib().kda_chunk_fwd_workspace_size(B, T, H, Dk, Dv, C, N, dt, ctypes.byref(out))
    return rc, out.value


def test_workspace_size_queries(L):
    rc, n = _ws(2, 4096, 32, 128, 128, 64, 2, kda.KDA_DTYPE_BF16)
    assert rc == kda.KDA_OK and n > 0 and n % 256 == 0
    rc, n1 = _ws(1, 1000, 4, 32, 32, 64, 3, kda.KDA_DTYPE_F32)
    assert rc == kda.KDA_OK
    rc, n2 = _ws(1, 1000, 4, 32, 32, 64, 30, kda.KDA_DTYPE_F32)
    assert rc == kda.KDA_OK and n2 >= n1  # more sequences => more partial chunks
    assert _ws(1, 256, 1, 96, 128, 64, 1, kda.KDA_DTYPE_BF16)[0] == kda.KDA_ERR_UNSUPPORTED
    assert _ws(1, 256, 1, 32, 32, 48, 1, kda.KDA_DTYPE_F32)[0] == kda.KDA_ERR_UNSUPPORTED
    assert _ws(1, 256, 1, 256, 32, 64, 1, kda.KDA_DTYPE_F32)[0] == kda.KDA_ERR_UNSUPPORTED
    assert _ws(1, -1, 1, 32, 32, 64, 1, kda.KDA_DTYPE_F32)[0] == kda.KDA_ERR_INVALID_ARG
    assert _ws(1, 256, 0, 32, 32, 64, 1, kda.KDA_DTYPE_F32)[0] == kda.KDA_ERR_INVALID_ARG
    assert _ws(1, 256, 1, 32, 32, 64, 1, 7)[0] == kda.KDA_ERR_INVALID_ARG
    out = ctypes.c_size_t(0)
    assert L.kda_chunk_fwd_workspace_size(1, 1, 1, 1, 1, 64, 1, 0, None) == kda.KDA_ERR_INVALID_ARG
    del out


def test_grid_limits_are_refused_on_host(L):
    """Shapes beyond the kernels' launch grids are UNSUPPORTED before any size is computed: more
    than 65535 heads, or more chunk x head items (here 2^30 empty sequences x 4 heads) or sequence
    x head chains than an int counts; the largest fitting head count still sizes."""
    F32, BF16 = kda.KDA_DTYPE_F32, kda.KDA_DTYPE_BF16
    assert _ws(1, 64, 65536, 32, 32, 64, 1, F32)[0] == kda.KDA_ERR_UNSUPPORTED
    assert _ws(1, 0, 4, 32, 32, 64, 1 << 30, F32)[0] == kda.KDA_ERR_UNSUPPORTED
    assert _ws(1, 0, 2, 32, 32, 64, 1 << 29, F32)[0] == kda.KDA_ERR_UNSUPPORTED  # 2 N H = 2^31
    rc, n = _ws(1, 64, 65535, 32, 32, 64, 1, F32)
    assert rc == kda.KDA_OK and n > 65535 * 64 * 32 * 4
    assert _fwd(H=65536) == kda.KDA_ERR_UNSUPPORTED
    assert _fwd(dt=F32, Dk=32, Dv=32, cu=FAKE, B=1, T=0, N=1 << 30, H=4) == kda.KDA_ERR_UNSUPPORTED
    sz = ctypes.c_size_t(0)
    assert L.kda_chunk_bwd_workspace_size(1, 64, 65536, 32, 32, 1, F32, ctypes.byref(sz)) == \
        kda.KDA_ERR_UNSUPPORTED
    assert L.kda_chunk_bwd_workspace_size(1, 0, 4, 32, 32, 1 << 30, BF16, ctypes.byref(sz)) == \
        kda.KDA_ERR_UNSUPPORTED


FAKE = 1 << 20  # a 256-aligned non-null address: never dereferenced, the host rejects first


def _fwd(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, dt=kda.KDA_DTYPE_BF16, la=FAKE, beta=FAKE, s0=None, cu=None,
             N=1, B=1, T=64, H=1, Dk=128, Dv=128, C=64, o=FAKE, sT=None, ws=FAKE, wsb=1 << 40,
             stream=None)
    a.update(kw)
    return kda.lib().kda_chunk_fwd(a["q"], a["k"], a["v"], a["dt"], a["la"], a["beta"], a["s0"],
                                   a["cu"], a["N"], a["B"], a["T"], a["H"], a["Dk"], a["Dv"],
                                   a["C"], a["o"], a["sT"], a["ws"], a["wsb"], a["stream"])


def test_prefill_argument_errors_are_caught_on_host(L):
    E = kda
    assert _fwd(q=None) == E.KDA_ERR_INVALID_ARG
    assert _fwd(o=None) == E.KDA_ERR_INVALID_ARG
    assert _fwd(beta=None) == E.KDA_ERR_INVALID_ARG
    assert _fwd(q=FAKE + 8) == E.KDA_ERR_INVALID_ARG  # misaligned
    assert _fwd(la=FAKE + 4) == E.KDA_ERR_INVALID_ARG
    assert _fwd(s0=FAKE + 4) == E.KDA_ERR_INVALID_ARG
    assert _fwd(Dk=64) == E.KDA_ERR_UNSUPPORTED  # bf16 path is 128 x 128, C = 64
    assert _fwd(C=32) == E.KDA_ERR_UNSUPPORTED
    assert _fwd(dt=kda.KDA_DTYPE_F32, C=48, Dk=32, Dv=32) == E.KDA_ERR_UNSUPPORTED
    assert _fwd(N=2) == E.KDA_ERR_INVALID_ARG  # N must equal B without cu_seqlens
    assert _fwd(cu=FAKE, B=2, N=2) == E.KDA_ERR_INVALID_ARG  # packed input needs B == 1
    assert _fwd(T=-5) == E.KDA_ERR_INVALID_ARG
    assert _fwd(H=0) == E.KDA_ERR_INVALID_ARG
    assert _fwd(ws=None) == E.KDA_ERR_WORKSPACE
    assert _fwd(ws=FAKE + 16) == E.KDA_ERR_WORKSPACE
    assert _fwd(wsb=1024) == E.KDA_ERR_WORKSPACE
    assert _fwd(dt=3) == E.KDA_ERR_INVALID_ARG
    assert _fwd(N=0, B=0, T=0) == E.KDA_OK  # nothing to do, nothing launched


def _step(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, dt=kda.KDA_DTYPE_BF16, la=FAKE, beta=FAKE, S=FAKE, o=FAKE,
             N=4, H=2, Dk=128, Dv=128, stream=None)
    a.update(kw)
    return kda.lib().kda_recurrent_step(a["q"], a["k"], a["v"], a["dt"], a["la"], a["beta"],
                                        a["S"], a["o"], a["N"], a["H"], a["Dk"], a["Dv"],
                                        a["stream"])


def test_decode_argument_errors_are_caught_on_host(L):
    E = kda
    assert _step(S=None) == E.KDA_ERR_INVALID_ARG
    assert _step(S=FAKE + 4) == E.KDA_ERR_INVALID_ARG
    assert _step(q=None) == E.KDA_ERR_INVALID_ARG
    assert _step(Dv=130) == E.KDA_ERR_UNSUPPORTED
    assert _step(Dv=6) == E.KDA_ERR_UNSUPPORTED
    assert _step(Dk=129) == E.KDA_ERR_UNSUPPORTED
    assert _step(N=-1) == E.KDA_ERR_INVALID_ARG
    assert _step(dt=9) == E.KDA_ERR_INVALID_ARG
    assert _step(N=0) == E.KDA_OK


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    monkeypatch.setattr(kda, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(kda, "_lib", None)
    with pytest.raises(ImportError):
        kda.lib()


def test_fusion_struct_layout_matches_the_header(tmp_path):
    """The binding's ctypes mirror of kda_fusion_t has the C compiler's size and offsets."""
    import ctypes
    import subprocess

    import gated_delta_rule_120_b200 as kda

    src = tmp_path / "layout.c"
    fields = [f[0] for f in kda.Fusion._fields_]
    body = "".join(f'  printf("%zu\\n", offsetof(kda_fusion_t, {f}));\n' for f in fields)
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "kda.h"\nint main(void) {\n'
                   '  printf("%zu\\n", sizeof(kda_fusion_t));\n' + body + "  return 0;\n}\n")
    exe = tmp_path / "layout"
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    subprocess.run(["gcc", "-std=c11", "-I", os.path.join(root, "include"), "-o", str(exe),
                    str(src)], check=True)
    got = [int(x) for x in subprocess.run([str(exe)], check=True, capture_output=True,
                                          text=True).stdout.split()]
    want = [ctypes.sizeof(kda.Fusion)] + [getattr(kda.Fusion, f).offset for f in fields]
    assert got == want


def test_backward_workspace_and_argument_errors_on_host(L):
    """The backward's size query and its host-side argument checks (no device work)."""
    import ctypes

    sz = ctypes.c_size_t(0)
    assert L.kda_chunk_bwd_workspace_size(2, 4096, 32, 128, 128, 2, 1, ctypes.byref(sz)) == 0
    # records (T and B included) + two state arrays + dV' for 256 chunks x 32 heads
    assert sz.value > 2 * 256 * 32 * 128 * 128 * 4
    assert L.kda_chunk_bwd_workspace_size(2, 64, 4, 256, 128, 2, 0, ctypes.byref(sz)) == \
        kda.KDA_ERR_UNSUPPORTED
    assert L.kda_chunk_bwd_workspace_size(2, 64, 0, 64, 64, 2, 0, ctypes.byref(sz)) == \
        kda.KDA_ERR_INVALID_ARG
    # null tensors with tokens present -> INVALID_ARG before any launch
    args = [None] * 3 + [0] + [None] * 4 + [1, 1, 16, 1, 32, 32] + [None] * 9 + [0, None]
    assert L.kda_chunk_bwd(*args) == kda.KDA_ERR_INVALID_ARG
    # N != B without cu_seqlens
    args = [None] * 3 + [0] + [None] * 4 + [3, 2, 0, 1, 32, 32] + [None] * 9 + [0, None]
    assert L.kda_chunk_bwd(*args) == kda.KDA_ERR_INVALID_ARG


def test_binding_refuses_host_tensors():
    """No CPU fallback: host tensors are refused by every entry point before anything reaches the
    library, and the size queries refuse dtypes the library has no kernel for."""
    import torch

    q = torch.zeros((1, 64, 2, 32))
    beta = torch.zeros((1, 64, 2))
    with pytest.raises(ValueError, match="CUDA tensor"):
        kda.kda_chunk_fwd(q, q, q, q, beta, chunk=32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        kda.kda_chunk_fwd_noalloc(q, q, q, q, beta, chunk=32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        kda.kda_chunk_bwd(q, q, q, q, beta, q)
    with pytest.raises(ValueError, match="CUDA tensor"):
        kda.kda_recurrent_fwd(q, q, q, q, beta, torch.zeros((1, 2, 32, 32)))
    with pytest.raises(ValueError, match="CUDA tensor"):
        kda.kda_recurrent_step(q[0], q[0], q[0], q[0], beta[0], torch.zeros((64, 2, 32, 32)))
    with pytest.raises(TypeError):
        kda.kda_chunk_fwd_workspace_size(1, 64, 2, 128, 128, 64, 1, torch.float16)
    with pytest.raises(TypeError):
        kda.kda_chunk_bwd_workspace_size(1, 64, 2, 128, 128, 1, torch.float16)


def test_selftest_limit_is_checked_on_host(L):
    """The failure-detection self-test refuses limits outside [1 ns, 1 s] before launching."""
    assert L.kda_selftest_wait_timeout(0, None) == kda.KDA_ERR_INVALID_ARG
    assert L.kda_selftest_wait_timeout(1_000_000_001, None) == kda.KDA_ERR_INVALID_ARG


def test_headers_compile_as_c_and_the_library_links(L, tmp_path):
    """A C99 program (tests/c_abi/kda_abi_check.c) includes the headers with no CUDA or C++ header,
    links libkda.so and gets the host-side answers of the ABI."""
    import shutil
    import subprocess

    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no gcc")
    exe = tmp_path / "kda_abi_check"
    pkg = os.path.dirname(_build.LIB)
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_abi", "kda_abi_check.c"),
                    "-L", pkg, "-lkda", f"-Wl,-rpath,{pkg}", "-o", str(exe)], check=True)
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stdout + run.stderr
    assert run.stdout.startswith("ok ")


def test_product_path_never_reaches_the_oracle(L):
    """The oracle is test infrastructure: the package's Python files, the CUDA sources and the
    headers never name it, and libkda.so links no library besides the C/C++ runtime (the CUDA
    runtime is linked statically)."""
    import shutil
    import subprocess

    pkg = os.path.dirname(_build.LIB)
    roots = [pkg, os.path.join(pkg, "csrc"), os.path.join(ROOT, "include")]
    for d in roots:
        for name in os.listdir(d):
            if name.endswith((".py", ".cu", ".cuh", ".h")):
                with open(os.path.join(d, name)) as f:
                    assert "oracle" not in f.read().lower(), os.path.join(d, name)
    readelf = shutil.which("readelf")
    if readelf is None:
        pytest.skip("no readelf")
    dyn = subprocess.run([readelf, "-d", _build.LIB], capture_output=True, text=True,
                         check=True).stdout
    needed = re.findall(r"\(NEEDED\)\s+Shared library: \[([^\]]+)\]", dyn)
    assert needed and all(re.match(r"(libstdc\+\+|libgcc_s|libc|libm|ld-linux|libdl|librt|"
                                   r"libpthread)", n) for n in needed), needed


def test_oracle_shares_nothing_with_the_library():
    """The other direction: the oracle's C source includes only system headers and its Python
    module imports nothing from the package, the CUDA sources or the synthetic-input module."""
    odir = os.path.join(ROOT, "oracle")
    with open(os.path.join(odir, "kda_oracle.c")) as f:
        src = f.read()
    assert re.findall(r'#include\s+"', src) == []  # no local header at all
    with open(os.path.join(odir, "__init__.py")) as f:
        py = f.read()
    for name in ("gated_delta_rule_120_b200", "kda_synth", "csrc", "libkda.so"):
        assert name not in py, name


def test_noalloc_limit_matches_the_header():
    """The binding's copy of the no-allocation scratch limit is the value include/kda.h declares."""
    with open(os.path.join(ROOT, "include", "kda.h")) as f:
        m = re.search(r"#define\s+KDA_NOALLOC_SCRATCH_BYTES\s+\(\(size_t\)(\d+)\s*<<\s*(\d+)\)",
                      f.read())
    assert m, "KDA_NOALLOC_SCRATCH_BYTES not found"
    assert kda.NOALLOC_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))
