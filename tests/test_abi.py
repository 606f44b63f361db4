"""CPU-only checks of the C-ABI boundary: the library loads, exports every
symbol include/clusterattn.h declares, and rejects invalid arguments on the
host before touching CUDA.  No compute call is made here."""

import ctypes
import os
import re
import subprocess
import sys

import pytest

import means_cluster_attention_b200 as ca
from means_cluster_attention_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "clusterattn.h")


def header_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ca_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def test_header_declares_expected_entry_points():
    syms = header_symbols()
    for s in ("ca_forward", "ca_forward_bf16", "ca_sync_status", "ca_status_string", "ca_last_error"):
        assert s in syms


def test_library_exports_every_header_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (ca_[a-z0-9_]+)\b", out))
    missing = [s for s in header_symbols() if s not in exported]
    assert not missing, f"declared but not exported: {missing}"
    for s in header_symbols():
        getattr(lib, s)


def test_binding_covers_header():
    assert sorted(_lib.SIGNATURES) == header_symbols()


def test_library_has_no_dynamic_cudart_dependency(lib):
    out = subprocess.run(["ldd", _lib.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcudart" not in out


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(OSError):
        _lib.load(str(tmp_path / "nope.so"))


def test_status_strings(lib):
    for code in range(6):
        assert lib.ca_status_string(code)
    assert b"sm_100a" in lib.ca_version()


# Dummy device-pointer values: never dereferenced, because validation fails
# before any CUDA call.
P = 1 << 20
GOOD = dict(B=2, H=3, L=128, d=64, K=16, iters=3, W=32, alpha=0.5)


def _call(lib, fn="ca_forward", q=P, k=P, v=P, out=P, assign=None, cent=None, **kw):
    a = dict(GOOD)
    a.update(kw)
    f = getattr(lib, fn)
    return f(q, k, v, a["B"], a["H"], a["L"], a["d"], a["K"], a["iters"], a["W"], a["alpha"], out,
             assign, cent, None)


@pytest.mark.parametrize("kw,status", [
    (dict(K=129, L=128), 1),            # K > L
    (dict(K=0), 1),
    (dict(K=129, L=4096), 2),           # K above the supported maximum
    (dict(d=32), 2),                    # unsupported head dim
    (dict(d=0), 1),
    (dict(B=0), 1),
    (dict(H=-1), 1),
    (dict(L=0), 1),
    (dict(iters=-1), 1),
    (dict(W=-2), 1),
    (dict(alpha=1.5), 1),
    (dict(alpha=-0.1), 1),
    (dict(alpha=float("nan")), 1),
    (dict(alpha=float("inf")), 1),
    (dict(B=255, H=256, L=1 << 11), 1),        # B*H*L*d >= 2^31
    (dict(B=1 << 10, H=1 << 7, L=16), 2),      # B*H above 65535
])
@pytest.mark.parametrize("fn", ["ca_forward", "ca_forward_bf16"])
def test_invalid_arguments_rejected_on_host(lib, fn, kw, status):
    assert _call(lib, fn, **kw) == status
    assert lib.ca_last_error()


@pytest.mark.parametrize("ptrs", [dict(q=None), dict(k=None), dict(v=None), dict(out=None),
                                  dict(q=P + 2), dict(out=P + 8), dict(cent=P + 4)])
def test_bad_pointers_rejected_on_host(lib, ptrs):
    assert _call(lib, **ptrs) == 1
    assert lib.ca_last_error()


def test_trace_rejects_bad_dtype(lib):
    st = lib.ca_forward_trace(P, P, P, 7, 1, 1, 64, 64, 4, 1, 8, 0.5, P, None, None, None, None)
    assert st == 1


def test_product_package_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "means_cluster_attention_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", text, re.M), f
                assert "liboracle" not in text, f


def test_source_hash_ignores_comments_but_not_code():
    # The bench reports a kernel's DRAM traffic only while the code the
    # counters were taken on is unchanged; comment edits must not count.
    base = b"__global__ void f(int *p) {\n    p[0] = 1;  // store\n}\n"
    commented = b"// header note\n/* block\n   comment */\n__global__ void f(int *p) {\n\n    p[0] = 1;\n}\n"
    changed = b"__global__ void f(int *p) {\n    p[0] = 2;\n}\n"
    assert build._code_only(base) == build._code_only(commented)
    assert build._code_only(base) != build._code_only(changed)
    assert re.fullmatch(r"[0-9a-f]{16}", build.source_hash("fused_forward"))


def test_debug_error_hook_validates_code_on_host(lib):
    # only CA_ERR_TIMEOUT (4) and CA_ERR_DEVICE (5) may be recorded; anything
    # else is rejected before a launch, so this needs no GPU
    for bad in (0, 1, 2, 3, 6, -1):
        assert lib.ca_debug_record_error(bad, None) == 1


def test_checked_build_exports_every_header_symbol_and_is_selected_by_env():
    path = build.build(checked=True)
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (ca_[a-z0-9_]+)\b", out))
    assert not [s for s in header_symbols() if s not in exported]
    code = ("import os, sys; sys.path.insert(0, %r); from means_cluster_attention_b200 import _lib; "
            "lib = _lib.load(); print(lib._name)") % ROOT
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                       env=dict(os.environ, CA_CHECKED="1"), check=True)
    assert r.stdout.strip().endswith("libclusterattn_checked.so")
