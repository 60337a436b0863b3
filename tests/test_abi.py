"""The C-ABI library loads, exports every symbol include/fk.h declares, and rejects bad
arguments on the host before any device work (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def fk():
    import __graft_entry__
    __graft_entry__.build()
    from exact_lloyd_means_b200 import fk as m
    return m


def _declared():
    src = open(os.path.join(ROOT, "include", "fk.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fk_[a-z_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(fk):
    lib = ctypes.CDLL(fk.LIB_PATH)
    names = _declared()
    assert "fk_lloyd" in names and "fk_assign" in names and "fk_update" in names
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(fk.EXPORTED) == names


def test_only_declared_symbols_are_exported(fk):
    out = os.popen(f"nm -D --defined-only {fk.LIB_PATH}").read()
    exported = sorted(set(re.findall(r"\bT (fk_[a-z_]+)\b", out)))
    assert exported == _declared()


def test_status_strings(fk):
    for code, name in [(0, "FK_OK"), (1, "FK_ERR_INVALID_ARG"), (2, "FK_ERR_UNSUPPORTED"),
                       (3, "FK_ERR_WORKSPACE"), (4, "FK_ERR_CUDA"), (5, "FK_ERR_TIMEOUT"),
                       (6, "FK_ERR_DEVICE")]:
        assert fk.status_string(code) == name
    assert fk.version() >= 1


def test_workspace_size_validation(fk):
    import torch
    n = fk.fk_workspace_size(65536, 128, 256, torch.float32, "l2")
    assert n > 65536 * 128 * 4  # holds the two bf16 planes of X
    assert fk.fk_workspace_size(65536, 128, 256, torch.bfloat16, "l2") < n
    assert fk.fk_workspace_size(65536, 128, 256, torch.float32, "cosine") > n
    for args, code in [((10, 128, 11), fk.FK_ERR_INVALID_ARG),
                       ((10, 0, 2), fk.FK_ERR_INVALID_ARG),
                       ((0, 8, 1), fk.FK_ERR_INVALID_ARG),
                       ((10, 6, 2), fk.FK_ERR_UNSUPPORTED),
                       ((2 ** 31, 8, 2), fk.FK_ERR_INVALID_ARG)]:
        with pytest.raises(fk.FkError) as e:
            fk.fk_workspace_size(*args, torch.float32, "l2")
        assert e.value.status == code
    with pytest.raises(fk.FkError) as e:
        fk.fk_workspace_size(100, 12, 4, torch.bfloat16, "l2")
    assert e.value.status == fk.FK_ERR_UNSUPPORTED
    with pytest.raises(fk.FkError) as e:
        fk.fk_workspace_size(100, 16, 4, torch.bfloat16, "cosine")
    assert e.value.status == fk.FK_ERR_UNSUPPORTED


def test_host_side_checks_need_no_device(fk):
    lib = fk._lib
    # null workspace / null inputs are rejected before any CUDA call
    assert lib.fk_assign(None, 0, 100, 8, None, 4, None, None, None, 0, None) == \
        fk.FK_ERR_INVALID_ARG
    assert lib.fk_assign(16, 0, 100, 8, 16, 4, 16, None, None, 0, None) == fk.FK_ERR_WORKSPACE
    assert lib.fk_assign(16, 0, 100, 8, 16, 4, 16, None, 256, 10, None) == fk.FK_ERR_WORKSPACE
    assert lib.fk_assign(8, 0, 100, 8, 16, 4, 16, None, 256, 1 << 30, None) == \
        fk.FK_ERR_UNSUPPORTED  # X not 16-byte aligned
    assert lib.fk_lloyd(16, 0, 100, 8, 4, 0, -1, 16, 16, None, None, None, None, 256, 1 << 30,
                        None) == fk.FK_ERR_INVALID_ARG
    # C_new overlapping C_old
    assert lib.fk_update(16, 0, 100, 8, 4, 16, 4096, 4100, 16, 16, None, None, 256, 1 << 30,
                         None) == fk.FK_ERR_INVALID_ARG
    assert lib.fk_get_device_error(None, 0, None, None) == fk.FK_ERR_INVALID_ARG


def test_binding_rejects_cpu_tensors(fk):
    import torch
    X = torch.zeros(10, 8)
    with pytest.raises(ValueError):
        fk.fk_assign(X, torch.zeros(2, 8), torch.zeros(10, dtype=torch.int32),
                     torch.zeros(256, dtype=torch.uint8))


def test_pre_split_dtype_is_assign_only(fk):
    lib = fk._lib
    n32 = fk.fk_workspace_size(4096, 100, 64, fk.FK_F32, "l2")
    nx2 = fk.fk_workspace_size(4096, 100, 64, fk.FK_BF16X2, "l2")
    assert nx2 < n32  # no room for the planes of X: the caller holds them
    with pytest.raises(fk.FkError) as e:
        fk.fk_workspace_size(4096, 100, 64, fk.FK_BF16X2, "cosine")
    assert e.value.status == fk.FK_ERR_UNSUPPORTED
    big = 1 << 30
    assert lib.fk_lloyd(256, fk.FK_BF16X2, 100, 8, 4, 0, 1, 256, 256, None, None, None, None,
                        256, big, None) == fk.FK_ERR_UNSUPPORTED
    assert lib.fk_update(256, fk.FK_BF16X2, 100, 8, 4, 256, 4096, 8192, 256, 256, None, None,
                         256, big, None) == fk.FK_ERR_UNSUPPORTED
    assert lib.fk_update_partial(256, fk.FK_BF16X2, 100, 8, 4, 256, 256, 256, 256, 256, None,
                                 256, big, None) == fk.FK_ERR_UNSUPPORTED
    assert lib.fk_split_points(None, 100, 8, 256, None) == fk.FK_ERR_INVALID_ARG
    assert lib.fk_split_points(256, 100, 6, 256, None) == fk.FK_ERR_UNSUPPORTED
    assert lib.fk_split_points(8, 100, 8, 256, None) == fk.FK_ERR_UNSUPPORTED


def test_ivf_lists_host_checks(fk):
    lib = fk._lib
    big = 1 << 30
    assert lib.fk_ivf_lists(None, 0, 100, 8, 4, 256, 256, 256, None, 256, big, None) == \
        fk.FK_ERR_INVALID_ARG
    # X_lists overlapping X
    assert lib.fk_ivf_lists(4096, 0, 100, 8, 4, 256, 256, 256, 4096 + 64, 256, big, None) == \
        fk.FK_ERR_INVALID_ARG
    assert lib.fk_ivf_lists(4096, 0, 100, 8, 4, 256, 256, 256, None, 256, 10, None) == \
        fk.FK_ERR_WORKSPACE


def test_ivf_search_host_checks(fk):
    lib = fk._lib
    big = 1 << 30
    ok = dict(Q=256, nq=10, d=8, C=256, nlist=4, Xl=256, Xn=256, Xp=None, rad=None, off=256,
              rid=256, N=100,
              nprobe=2, k=3, flags=0, dist=256, ids=256, probes=None, ws=256, wsb=big)

    def call(**kw):
        a = dict(ok, **kw)
        return lib.fk_ivf_search(a["Q"], a["nq"], a["d"], a["C"], a["nlist"], a["Xl"], a["Xn"],
                                 a["Xp"], a["rad"], a["off"], a["rid"], a["N"], a["nprobe"], a["k"], a["flags"],
                                 a["dist"],
                                 a["ids"], a["probes"], a["ws"], a["wsb"], None, None)

    for bad in (dict(nprobe=5), dict(nprobe=0), dict(k=0), dict(k=33), dict(nq=0),
                dict(N=0), dict(Q=None), dict(Xn=None), dict(ids=None),
                dict(nq=1 << 30, nprobe=4)):
        assert call(**bad) == fk.FK_ERR_INVALID_ARG, bad
    for bad in (dict(d=6), dict(Q=8), dict(Xl=264), dict(probes=258), dict(Xp=264),
                dict(rad=258)):
        assert call(**bad) == fk.FK_ERR_UNSUPPORTED, bad
    assert call(wsb=10) == fk.FK_ERR_WORKSPACE
    assert call(ws=None) == fk.FK_ERR_WORKSPACE
    assert lib.fk_ivf_norms(None, 10, 8, 256, None) == fk.FK_ERR_INVALID_ARG
    assert lib.fk_ivf_radii(None, 4, 256, 256, 8, 256, None) == fk.FK_ERR_INVALID_ARG
    assert lib.fk_ivf_radii(256, 4, 256, 256, 6, 256, None) == fk.FK_ERR_UNSUPPORTED
    assert lib.fk_ivf_norms(256, 10, 6, 256, None) == fk.FK_ERR_UNSUPPORTED
    with pytest.raises(fk.FkError) as e:
        fk.ivf_search_workspace(10, 8, 4, 100, 5, 3, device="cpu")
    assert e.value.status == fk.FK_ERR_INVALID_ARG
    # the workspace grows with the queries' pairs and the coarse batch
    s1 = fk.ivf_search_workspace(1000, 8, 64, 100, 8, 10, device="meta").numel()
    s2 = fk.ivf_search_workspace(2000, 8, 64, 100, 8, 10, device="meta").numel()
    assert s2 > s1 > 1000 * 8 * 10 * 12


def test_fault_injection_workspace_needs_no_device(fk):
    """FK_FAULT=workspace (read when the library is first used, so in a child process):
    every workspace check fails with FK_ERR_WORKSPACE, before any device work."""
    import subprocess
    import sys
    code = (
        "import ctypes, sys\n"
        f"sys.path.insert(0, {ROOT!r})\n"
        "from exact_lloyd_means_b200 import fk\n"
        "lib = fk._lib\n"
        "r1 = lib.fk_assign(16, 0, 100, 8, 16, 4, 16, None, 256, 1 << 30, None)\n"
        "r2 = lib.fk_lloyd(16, 0, 100, 8, 4, 0, 1, 16, 16, None, None, None, None, 256, 1 << 30, None)\n"
        "print(r1, r2)\n")
    env = dict(os.environ, FK_FAULT="workspace")
    out = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                         timeout=300)
    assert out.returncode == 0, out.stderr
    r1, r2 = (int(x) for x in out.stdout.split())
    assert r1 == fk.FK_ERR_WORKSPACE and r2 == fk.FK_ERR_WORKSPACE


def test_binding_without_the_library_fails_loudly(tmp_path):
    """The product path has no CPU fallback: the binding, copied where no libfk.so sits
    beside it, refuses to import and says how to build the library."""
    import shutil
    import subprocess
    import sys
    pkg = tmp_path / "exact_lloyd_means_b200"
    pkg.mkdir()
    shutil.copy(os.path.join(ROOT, "exact_lloyd_means_b200", "fk.py"), pkg / "fk.py")
    (pkg / "__init__.py").write_text("")
    r = subprocess.run([sys.executable, "-c", "import exact_lloyd_means_b200.fk"],
                       cwd=tmp_path, capture_output=True, text=True, timeout=120)
    assert r.returncode != 0
    assert "ImportError" in r.stderr and "build the CUDA library first" in r.stderr


def test_product_package_never_imports_the_oracle():
    """Only tests/, the smoke check and the bench's baseline legs may use oracle/: no module
    of the product package imports it."""
    import re
    pat = re.compile(r"^\s*(import\s+oracle\b|from\s+oracle\b)", re.M)
    pkg = os.path.join(ROOT, "exact_lloyd_means_b200")
    for dirpath, _, files in os.walk(pkg):
        for name in files:
            if name.endswith(".py"):
                with open(os.path.join(dirpath, name)) as f:
                    assert not pat.search(f.read()), os.path.join(dirpath, name)
