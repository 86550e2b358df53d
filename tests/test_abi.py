"""The C-ABI library loads on a machine without a GPU and exports every entry
point that include/adacluster.h declares; the product package never imports
the oracle."""
import ctypes
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "adacluster.h")


def declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ac_[a-z_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from clustered_sparse_attention_head_b200 import build
    path = build()
    return ctypes.CDLL(path)


def test_header_declares_the_boundary():
    names = declared()
    for n in ["ac_cluster_q", "ac_cluster_k", "ac_select", "ac_sparse_attn", "ac_forward"]:
        assert n in names


def test_binding_constants_match_the_header():
    import re
    from clustered_sparse_attention_head_b200 import _abi
    hdr = open(os.path.join(ROOT, "include", "adacluster.h")).read()
    flags = dict(re.findall(r"#define (AC_FLAG_\w+) (\d+)u", hdr))
    assert set(flags) == {n for n in dir(_abi) if n.startswith("AC_FLAG_")}
    for name, val in flags.items():
        assert getattr(_abi, name) == int(val), name


def test_every_declared_symbol_is_exported(lib):
    from clustered_sparse_attention_head_b200 import _abi
    names = declared()
    assert sorted(_abi.EXPORTS) == names
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    lib.ac_status_string.restype = ctypes.c_char_p
    for code in range(8):
        s = lib.ac_status_string(code).decode()
        assert s and s != "unknown status"


def test_nothing_but_declared_symbols_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", lib._name], capture_output=True, text=True).stdout
    syms = {l.split()[-1] for l in out.splitlines() if " T " in l}
    assert {s for s in syms if s.startswith("ac_")} == set(declared())


def test_create_rejects_bad_config_without_launching(lib):
    from clustered_sparse_attention_head_b200 import _abi
    L = _abi.load()
    ctx = ctypes.c_void_p()
    bad = _abi.ac_config(1, 100, 96, 1, 4, 4, 1, 0, 0, 0, 0.0, 0, 0, 0.9, 0)   # d = 96
    assert L.ac_create(ctypes.byref(bad), ctypes.byref(ctx)) == _abi.AC_ERR_UNSUPPORTED
    bad = _abi.ac_config(1, 100, 64, 1, 0, 4, 1, 0, 0, 0, 0.0, 0, 0, 0.9, 0)   # kq = 0
    assert L.ac_create(ctypes.byref(bad), ctypes.byref(ctx)) == _abi.AC_ERR_INVALID_ARG
    bad = _abi.ac_config(1, 100, 64, 1, 4, 4, 1, 0, 0, 0, 0.0, 0, 0, 0.0, 0)   # top_p = 0
    assert L.ac_create(ctypes.byref(bad), ctypes.byref(ctx)) == _abi.AC_ERR_INVALID_ARG
    bad = _abi.ac_config(1, 100, 64, 1, 4, 4, 1, 0, 1, 0, 0.0, 0, 0, 0.9, 0)   # adaptive, nmax 0
    assert L.ac_create(ctypes.byref(bad), ctypes.byref(ctx)) == _abi.AC_ERR_INVALID_ARG
    assert not ctx.value


def test_product_does_not_import_oracle():
    code = ("import sys; import clustered_sparse_attention_head_b200 as p; "
            "from clustered_sparse_attention_head_b200 import api, _abi; "
            "assert 'oracle' not in sys.modules, 'oracle imported'")
    subprocess.check_call([sys.executable, "-c", code], cwd=ROOT)


def test_no_unresolved_internal_symbols(lib):
    """Every internal launcher the entry points call is defined in the library."""
    out = subprocess.run(["nm", "-D", "--undefined-only", lib._name], capture_output=True, text=True).stdout
    assert not [l for l in out.splitlines() if "_ZN2ac" in l], out


def _cfg(**over):
    from clustered_sparse_attention_head_b200 import _abi
    base = dict(heads=2, n=1000, d=128, dtype=_abi.AC_BF16, kq=10, kk=20, iters=3, adaptive_q=0, adaptive_k=0,
                tau_rule=_abi.AC_TAU_ABS, tau_value=0.0, nmax_q=0, nmax_k=0, top_p=0.9, flags=0,
                score_mode=_abi.AC_SCORE_CENTROID, top_k=0, text_keys=0)
    base.update(over)
    return _abi.ac_config(**base)


@pytest.mark.parametrize("over, code", [
    (dict(heads=0), "AC_ERR_INVALID_ARG"),
    (dict(n=0), "AC_ERR_INVALID_ARG"),
    (dict(iters=-1), "AC_ERR_INVALID_ARG"),
    (dict(d=32), "AC_ERR_UNSUPPORTED"),
    (dict(dtype=7), "AC_ERR_INVALID_ARG"),
    (dict(kq=1001), "AC_ERR_INVALID_ARG"),
    (dict(kk=1001), "AC_ERR_INVALID_ARG"),
    (dict(kk=0), "AC_ERR_INVALID_ARG"),
    (dict(top_p=-0.5), "AC_ERR_INVALID_ARG"),
    (dict(top_p=float("nan")), "AC_ERR_INVALID_ARG"),
    (dict(score_mode=9), "AC_ERR_INVALID_ARG"),
    (dict(top_k=-1), "AC_ERR_INVALID_ARG"),
    (dict(text_keys=-1), "AC_ERR_INVALID_ARG"),
    (dict(text_keys=1000), "AC_ERR_INVALID_ARG"),
    (dict(text_keys=990), "AC_ERR_INVALID_ARG"),          # 10 video keys left for kk = 20 clusters
    (dict(heads=2 ** 20, n=2 ** 11), "AC_ERR_UNSUPPORTED"),  # H * N beyond the int32 index range
    (dict(adaptive_q=1, nmax_q=0), "AC_ERR_INVALID_ARG"),
    (dict(adaptive_k=1, nmax_k=40, tau_rule=5), "AC_ERR_INVALID_ARG"),
    (dict(adaptive_k=1, nmax_k=40, tau_value=-1.0), "AC_ERR_INVALID_ARG"),
    (dict(adaptive_k=1, nmax_k=40, tau_value=float("nan")), "AC_ERR_INVALID_ARG"),
])
def test_every_config_check(lib, over, code):
    """Each argument check of ac_create rejects its case on the host, before
    any device call, and leaves the output handle empty."""
    from clustered_sparse_attention_head_b200 import _abi
    L = _abi.load()
    ctx = ctypes.c_void_p()
    cfg = _cfg(**over)
    assert L.ac_create(ctypes.byref(cfg), ctypes.byref(ctx)) == getattr(_abi, code)
    assert not ctx.value
