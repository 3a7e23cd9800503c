"""The C-ABI library on a machine without a GPU: it loads, exports every
symbol include/gsq.h declares, and rejects bad arguments on the host before
any device work (no compute call is made here)."""
import ctypes as C
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def gsq():
    from post_weight_quantization_philox_b200 import build
    build.build()
    from post_weight_quantization_philox_b200 import gsq as g
    return g


def declared_symbols():
    hdr = open(os.path.join(ROOT, "include", "gsq.h")).read()
    return sorted(set(re.findall(r"^GSQ_API\s+[\w\s\*]*?\b(gsq_\w+)\s*\(", hdr, re.M)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for name in ["gsq_init", "gsq_step", "gsq_harden_pack", "gsq_recon_error",
                 "gsq_last_loss", "gsq_destroy"]:
        assert name in syms


def test_library_exports_every_declared_symbol(gsq):
    out = subprocess.run(["nm", "-D", "--defined-only", gsq.LIB_PATH],
                         capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r" T (gsq_\w+)$", out, re.M))
    assert set(declared_symbols()) <= exported
    assert sorted(gsq.EXPORTS) == declared_symbols()
    lib = C.CDLL(gsq.LIB_PATH)
    for s in declared_symbols():
        assert getattr(lib, s) is not None


def test_packed_bytes_and_error_strings(gsq):
    assert gsq.gsq_packed_bytes(gsq.GSQ_GRID_2BIT, 4096, 4096) == 4096 * 4096 // 4
    assert gsq.gsq_packed_bytes(gsq.GSQ_GRID_TERNARY, 14336, 4096) == 14336 * 4096 // 4
    assert gsq.gsq_packed_bytes(gsq.GSQ_GRID_3BIT_LOCAL, 4096, 14336) == 4096 * 14336 * 3 // 8
    for bad in [(7, 8, 128), (0, 0, 128), (0, 8, 100), (0, 8, 0)]:
        with pytest.raises(gsq.GSQError) as e:
            gsq.gsq_packed_bytes(*bad)
        assert e.value.status == gsq.GSQ_ERR_INVALID_ARG
    for st in range(-7, 1):
        assert gsq.error_string(st) and gsq.error_string(st) != "unknown status"
    assert gsq.error_string(-99) == "unknown status"


def test_init_rejects_bad_arguments_before_device_work(gsq):
    import numpy as np
    W = np.zeros((8, 256), np.float32)
    X = np.zeros((4, 256), np.float32)
    cases = [
        (dict(W=W[:, :200], X=X[:, :200]), gsq.GSQ_ERR_INVALID_ARG),   # K % 128
        (dict(W=W, X=X, grid_mode=5), gsq.GSQ_ERR_INVALID_ARG),        # mode
        (dict(W=np.zeros((0, 256), np.float32), X=X), gsq.GSQ_ERR_INVALID_ARG),
        (dict(W=W, X=np.zeros((0, 256), np.float32)), gsq.GSQ_ERR_INVALID_ARG),
        (dict(W=W, X=X, group=64), gsq.GSQ_ERR_UNSUPPORTED),           # group
    ]
    for kw, status in cases:
        with pytest.raises(gsq.GSQError) as e:
            gsq.gsq_init(**kw)
        assert e.value.status == status


def test_null_context_handling(gsq):
    lib = gsq.lib()
    assert lib.gsq_destroy(None) == gsq.GSQ_OK
    assert lib.gsq_step(None, 1.0, 1e-3, 0.9, 0.99) == gsq.GSQ_ERR_INVALID_ARG
    d = C.c_double()
    assert lib.gsq_last_loss(None, C.byref(d)) == gsq.GSQ_ERR_INVALID_ARG
    assert lib.gsq_harden_pack(None, None, None, None) == gsq.GSQ_ERR_INVALID_ARG
    out = C.c_void_p()
    assert lib.gsq_init(C.byref(out), None, 0, None, 0, 8, 128, 8, 128, 0, None, 0,
                        None) == gsq.GSQ_ERR_INVALID_ARG
    assert lib.gsq_init(None, None, 0, None, 0, 8, 128, 8, 128, 0, None, 0,
                        None) == gsq.GSQ_ERR_INVALID_ARG


def test_release_without_pools(gsq):
    """With no device allocation made there is no pool to trim: a no-op that succeeds
    without touching a device."""
    assert gsq.lib().gsq_release_cached_memory() == gsq.GSQ_OK
    assert gsq.lib().gsq_set_cached_memory_limit(1 << 30) == gsq.GSQ_OK
    assert gsq.lib().gsq_set_cached_memory_limit(2 ** 64 - 1) == gsq.GSQ_OK


def test_binding_has_no_fallback(monkeypatch, tmp_path):
    """Importing the binding without the shared library raises."""
    import importlib.util
    src = os.path.join(ROOT, "post_weight_quantization_philox_b200", "gsq.py")
    dst = tmp_path / "gsq_copy.py"
    dst.write_text(open(src).read())
    spec = importlib.util.spec_from_file_location("gsq_copy", dst)
    mod = importlib.util.module_from_spec(spec)
    with pytest.raises(ImportError):
        spec.loader.exec_module(mod)


def test_failure_hooks_are_host_only(gsq):
    """The allocation-failure hook and the pool query need no device until
    the library has allocated on one."""
    lib = gsq.lib()
    assert lib.gsq_debug_fail_alloc(3) == gsq.GSQ_OK
    assert lib.gsq_debug_fail_alloc(-1) == gsq.GSQ_OK
    b = C.c_uint64(7)
    assert lib.gsq_debug_pool_used(0, C.byref(b)) == gsq.GSQ_OK and b.value == 0
    assert lib.gsq_debug_pool_used(-1, C.byref(b)) == gsq.GSQ_ERR_INVALID_ARG
    assert lib.gsq_debug_pool_used(0, None) == gsq.GSQ_ERR_INVALID_ARG
    assert lib.gsq_debug_stall_probe(None) == gsq.GSQ_ERR_INVALID_ARG


def test_row_shard_init_rejects_bad_offsets_on_host(gsq):
    import numpy as np
    W = np.zeros((8, 256), np.float32)
    X = np.zeros((4, 256), np.float32)
    for row0, st16 in [(-1, 0), (0, 2), (1 << 60, 0)]:
        out = C.c_void_p()
        rc = gsq.lib().gsq_init_rows(C.byref(out), W.ctypes.data, gsq.GSQ_F32, X.ctypes.data,
                                     gsq.GSQ_F32, 8, 256, 4, 128, 0, None, 0, row0, st16, None)
        assert rc == gsq.GSQ_ERR_INVALID_ARG and not out.value
