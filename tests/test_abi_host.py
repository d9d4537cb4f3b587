"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point include/eta.h declares, and rejects bad arguments before
launching anything."""
import ctypes
import os
import re

import pytest

import learned_threshold_sparse_b200 as eta

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    src = open(os.path.join(ROOT, "include", "eta.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(eta_[a-z_0-9]+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    names = _declared_symbols()
    assert "eta_decode" in names and "eta_block_summary_update" in names
    lib = eta.library()
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) <= set(eta.SYMBOLS) | {n for n in names if hasattr(eta, n)}
    for n in names:
        assert hasattr(eta, n), f"binding lacks {n}"


def test_status_strings():
    for code in range(8):
        assert eta.eta_status_string(code)
    assert "sm_100a" in eta.eta_build_info()


def _params(**over):
    fake = 1 << 20  # aligned, never dereferenced on the host
    p = eta.eta_decode_params()
    p.cache = eta.eta_cache_desc(1, 16, 4, 128, 64, 4096, eta.ETA_BF16, fake, fake, fake)
    p.summary = eta.eta_summary_desc(fake, fake, fake)
    p.q = fake
    p.tau_mode = eta.ETA_TAU_CALIBRATED
    p.c_tau = fake
    p.scale = 0.088
    p.beta = 5.0
    p.z = 2.0
    p.n_local_blocks = 2
    p.screen_enabled = 1
    p.out = fake
    for k, v in over.items():
        if "." in k:
            a, b = k.split(".")
            setattr(getattr(p, a), b, v)
        else:
            setattr(p, k, v)
    return p


@pytest.mark.parametrize("over,code", [
    ({"cache.head_dim": 96}, eta.ETA_ERR_UNSUPPORTED),
    ({"cache.block_size": 48}, eta.ETA_ERR_UNSUPPORTED),
    ({"cache.n_q_heads": 12, "cache.n_kv_heads": 8}, eta.ETA_ERR_INVALID_ARG),
    ({"cache.n_q_heads": 48, "cache.n_kv_heads": 4}, eta.ETA_ERR_UNSUPPORTED),
    ({"cache.batch": 0}, eta.ETA_ERR_INVALID_ARG),
    ({"cache.max_ctx": 0}, eta.ETA_ERR_INVALID_ARG),
    ({"cache.kv_dtype": 7}, eta.ETA_ERR_INVALID_ARG),
    ({"cache.k_cache": None}, eta.ETA_ERR_INVALID_ARG),
    ({"cache.v_cache": (1 << 20) + 8}, eta.ETA_ERR_INVALID_ARG),
    ({"q": None}, eta.ETA_ERR_INVALID_ARG),
    ({"out": (1 << 20) + 4}, eta.ETA_ERR_INVALID_ARG),
    ({"summary.mu": None}, eta.ETA_ERR_INVALID_ARG),
    ({"tau_mode": eta.ETA_TAU_LEARNED}, eta.ETA_ERR_INVALID_ARG),
    ({"c_tau": None}, eta.ETA_ERR_INVALID_ARG),
    ({"scale": 0.0}, eta.ETA_ERR_INVALID_ARG),
    ({"scale": float("nan")}, eta.ETA_ERR_INVALID_ARG),
    ({"beta": -1.0}, eta.ETA_ERR_INVALID_ARG),
    ({"z": 0.0}, eta.ETA_ERR_INVALID_ARG),
    ({"z": float("nan")}, eta.ETA_ERR_INVALID_ARG),
    ({"offset_a": float("inf")}, eta.ETA_ERR_INVALID_ARG),
    ({"n_local_blocks": -2}, eta.ETA_ERR_INVALID_ARG),
    ({"attend_impl": 9}, eta.ETA_ERR_INVALID_ARG),
    ({"lse": (1 << 20) + 2}, eta.ETA_ERR_INVALID_ARG),
])
def test_invalid_arguments_rejected_before_launch(over, code):
    p = _params(**over)
    assert eta.library().eta_decode(ctypes.byref(p), None) == code
    n = ctypes.c_size_t(0)
    assert eta.library().eta_decode_workspace_size(ctypes.byref(p), ctypes.byref(n)) == code


@pytest.mark.parametrize("over", [{"cache.head_dim": 96}, {"cache.batch": 0}, {"q": None}, {"scale": 0.0},
                                  {"attend_impl": 9}])
def test_graph_create_validates_like_decode(over):
    p = _params(**over)
    h = ctypes.c_void_p(123)
    code = eta.library().eta_decode(ctypes.byref(p), None)
    assert code != eta.ETA_OK
    assert eta.library().eta_decode_graph_create(ctypes.byref(p), ctypes.byref(h)) == code
    assert h.value is None  # no handle on failure


def test_graph_create_rejects_timing_events_and_null():
    p = _params()
    p.timing_events[1] = 1 << 12
    h = ctypes.c_void_p()
    assert eta.library().eta_decode_graph_create(ctypes.byref(p), ctypes.byref(h)) == eta.ETA_ERR_INVALID_ARG
    assert eta.library().eta_decode_graph_create(None, ctypes.byref(h)) == eta.ETA_ERR_INVALID_ARG
    assert eta.library().eta_decode_graph_create(ctypes.byref(_params()), None) == eta.ETA_ERR_INVALID_ARG
    assert eta.library().eta_decode_graph_launch(None, None) == eta.ETA_ERR_INVALID_ARG
    assert eta.library().eta_decode_graph_destroy(None) == eta.ETA_ERR_INVALID_ARG


def test_step_graph_validation():
    lib = eta.library()
    h = ctypes.c_void_p()
    fake = 1 << 20
    d = eta.eta_step_desc()
    assert lib.eta_step_graph_create(None, ctypes.byref(h)) == eta.ETA_ERR_INVALID_ARG
    assert lib.eta_step_graph_create(ctypes.byref(d), ctypes.byref(h)) == eta.ETA_ERR_INVALID_ARG  # no decode
    bad = _params(**{"cache.head_dim": 96})
    d.decode = ctypes.pointer(bad)
    assert lib.eta_step_graph_create(ctypes.byref(d), ctypes.byref(h)) == eta.ETA_ERR_UNSUPPORTED
    p = _params()
    p.timing_events[0] = 1 << 12
    d.decode = ctypes.pointer(p)
    assert lib.eta_step_graph_create(ctypes.byref(d), ctypes.byref(h)) == eta.ETA_ERR_INVALID_ARG
    assert h.value is None
    assert lib.eta_step_graph_create(ctypes.byref(d), None) == eta.ETA_ERR_INVALID_ARG
    good = _params()
    d.decode = ctypes.pointer(good)
    d.k_new = fake  # an append needs all three of k_new, v_new, positions
    assert lib.eta_step_graph_create(ctypes.byref(d), ctypes.byref(h)) == eta.ETA_ERR_INVALID_ARG
    d.k_new = None
    d.h2d_bytes = 64  # a copy needs both ends
    d.h2d_dst = fake
    assert lib.eta_step_graph_create(ctypes.byref(d), ctypes.byref(h)) == eta.ETA_ERR_INVALID_ARG
    d.h2d_bytes = 0
    d.d2h_bytes = 64
    d.d2h_src = fake
    assert lib.eta_step_graph_create(ctypes.byref(d), ctypes.byref(h)) == eta.ETA_ERR_INVALID_ARG


def test_diag_wait_timeout_validation():
    assert eta.library().eta_diag_wait_timeout(None, None) == eta.ETA_ERR_INVALID_ARG
    assert eta.library().eta_diag_wait_timeout((1 << 20) + 64, None) == eta.ETA_ERR_INVALID_ARG


def test_null_params():
    assert eta.library().eta_decode(None, None) == eta.ETA_ERR_INVALID_ARG
    assert eta.library().eta_decode_workspace_size(None, None) == eta.ETA_ERR_INVALID_ARG
    assert eta.library().eta_read_device_status(None, None) == eta.ETA_ERR_INVALID_ARG


def test_summary_update_validation():
    fake = 1 << 20
    c = eta.eta_cache_desc(1, 4, 4, 64, 64, 4096, eta.ETA_F32, fake, fake, fake)
    s = eta.eta_summary_desc(fake, fake, fake)
    lib = eta.library()
    assert lib.eta_block_summary_update(ctypes.byref(c), ctypes.byref(s), None, 1, None) == eta.ETA_ERR_INVALID_ARG
    assert lib.eta_block_summary_update(ctypes.byref(c), ctypes.byref(s), fake, 0, None) == eta.ETA_ERR_INVALID_ARG
    assert lib.eta_block_summary_update(ctypes.byref(c), ctypes.byref(s), fake, 65, None) == eta.ETA_ERR_INVALID_ARG
    s2 = eta.eta_summary_desc(fake + 2, fake, fake)
    assert lib.eta_block_summary_update(ctypes.byref(c), ctypes.byref(s2), fake, 1, None) == eta.ETA_ERR_INVALID_ARG
    c2 = eta.eta_cache_desc(1, 4, 4, 80, 64, 4096, eta.ETA_F32, fake, fake, fake)
    assert lib.eta_block_summary_update(ctypes.byref(c2), ctypes.byref(s), fake, 1, None) == eta.ETA_ERR_UNSUPPORTED


def test_struct_layout_matches_header(tmp_path):
    # Compile a C probe of include/eta.h and compare every field offset and
    # struct size with the ctypes mirror used by the binding.
    fields = {
        "eta_cache_desc": eta.eta_cache_desc,
        "eta_summary_desc": eta.eta_summary_desc,
        "eta_decode_params": eta.eta_decode_params,
        "eta_prefill_params": eta.eta_prefill_params,
        "eta_calib_params": eta.eta_calib_params,
        "eta_step_desc": eta.eta_step_desc,
    }
    lines = ["#include <stdio.h>", "#include <stddef.h>", '#include "eta.h"', "int main(void) {"]
    for sname, cls in fields.items():
        lines.append(f'printf("{sname} size %zu\\n", sizeof({sname}));')
        for fname, _ in cls._fields_:
            lines.append(f'printf("{sname} {fname} %zu\\n", offsetof({sname}, {fname}));')
    lines.append("return 0; }")
    src = tmp_path / "probe.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "probe"
    import subprocess
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    got = {}
    for ln in out:
        if ln.strip():
            a, b, c = ln.split()
            got[(a, b)] = int(c)
    for sname, cls in fields.items():
        assert got[(sname, "size")] == ctypes.sizeof(cls), sname
        for fname, _ in cls._fields_:
            assert got[(sname, fname)] == getattr(cls, fname).offset, (sname, fname)


def test_append_kv_validation():
    fake = 1 << 20
    c = eta.eta_cache_desc(1, 4, 4, 64, 64, 4096, eta.ETA_BF16, fake, fake, fake)
    s = eta.eta_summary_desc(fake, fake, fake)
    lib = eta.library()
    assert lib.eta_append_kv(ctypes.byref(c), ctypes.byref(s), None, fake, fake, None) == eta.ETA_ERR_INVALID_ARG
    assert lib.eta_append_kv(ctypes.byref(c), ctypes.byref(s), fake, fake + 8, fake, None) == eta.ETA_ERR_INVALID_ARG
    assert lib.eta_append_kv(ctypes.byref(c), ctypes.byref(s), fake, fake, fake + 2, None) == eta.ETA_ERR_INVALID_ARG
    c2 = eta.eta_cache_desc(1, 4, 4, 96, 64, 4096, eta.ETA_BF16, fake, fake, fake)
    assert lib.eta_append_kv(ctypes.byref(c2), ctypes.byref(s), fake, fake, fake, None) == eta.ETA_ERR_UNSUPPORTED


def _prefill_ok():
    fake = 1 << 20  # never dereferenced: every case below fails validation before a launch
    p = eta.eta_prefill_params()
    p.batch, p.n_q_heads, p.n_kv_heads, p.head_dim, p.seq_len, p.kv_stride = 1, 8, 2, 128, 1000, 1024
    p.dtype = eta.ETA_BF16
    p.q = p.k = p.v = p.out = fake
    p.tau_mode = eta.ETA_TAU_LEARNED
    p.w_tau = p.b_tau = fake
    p.scale, p.beta, p.offset_a = 0.088, 5.0, 0.0
    p.workspace, p.workspace_bytes = fake, eta.PREFILL_WORKSPACE_BYTES
    return p


@pytest.mark.parametrize("field,value,code", [
    ("seq_len", 0, 1), ("kv_stride", 999, 1), ("n_kv_heads", 3, 1), ("head_dim", 64, 2), ("dtype", 0, 2),
    ("q", 0, 1), ("k", (1 << 20) + 8, 1), ("w_tau", (1 << 20) + 4, 1), ("scale", 0.0, 1),
    ("beta", -1.0, 1), ("beta", float("nan"), 1), ("tau_mode", 7, 1), ("workspace_bytes", 16, 3),
    ("workspace", 0, 3), ("lse", (1 << 20) + 2, 1),
])
def test_prefill_validation(field, value, code):
    p = _prefill_ok()
    setattr(p, field, value)
    assert eta.library().eta_prefill(ctypes.byref(p), None) == code


def test_prefill_size_limits():
    p = _prefill_ok()
    p.batch, p.n_q_heads, p.n_kv_heads, p.seq_len, p.kv_stride = 64, 64, 64, 1 << 20, 1 << 20
    assert eta.library().eta_prefill(ctypes.byref(p), None) == eta.ETA_ERR_UNSUPPORTED
    # one grid row per 128-query tile: at most 65535 tiles
    p = _prefill_ok()
    p.n_q_heads = p.n_kv_heads = 1
    p.seq_len = p.kv_stride = 65535 * 128 + 1
    assert eta.library().eta_prefill(ctypes.byref(p), None) == eta.ETA_ERR_UNSUPPORTED
    p = _prefill_ok()
    p.tau_mode = eta.ETA_TAU_CALIBRATED
    p.c_tau = None
    assert eta.library().eta_prefill(ctypes.byref(p), None) == eta.ETA_ERR_INVALID_ARG


def test_calibration_host_solver_matches_the_oracle_solver():
    # host-only entry point: no device involved
    import numpy as np
    from oracle import eta_calib_oracle as co

    rng = np.random.default_rng(9)
    S = rng.standard_normal(20000) * 1.5
    w = rng.uniform(0.05, 1.0, 20000)
    lo, hi, nb = -6.0, 6.0, 600
    hist = np.stack([co.histogram(S, w, lo, hi, nb), co.histogram(S * 0.5, w, lo, hi, nb)])
    targets = np.array([0.38, 0.1], np.float32)
    c = np.zeros(2, np.float32)
    rc = eta.library().eta_calibrate_constants(hist.ctypes.data, 2, nb, lo, hi, targets.ctypes.data, c.ctypes.data)
    assert rc == eta.ETA_OK
    for h in range(2):
        ref = co.histogram_constant(hist[h], lo, hi, float(targets[h]))
        assert abs(float(c[h]) - ref) <= 1e-5 * max(1.0, abs(ref))


def test_calibration_validation():
    fake = 1 << 20
    p = eta.eta_calib_params(1, 4, 2, 128, 100, 100, eta.ETA_BF16, fake, fake, 0.088, -8.0, 8.0, 512, fake)
    lib = eta.library()
    for field, value, code in [("nbins", 0, 1), ("hi", -9.0, 1), ("head_dim", 96, 2), ("hist", fake + 4, 1),
                               ("kv_stride", 50, 1), ("n_kv_heads", 3, 1)]:
        q = eta.eta_calib_params.from_buffer_copy(p)
        setattr(q, field, value)
        assert lib.eta_calibration_histogram(ctypes.byref(q), None) == code, field


def test_c_example_compiles_and_links(tmp_path):
    # tests/c/decode_example.c drives one decode step through the C ABI from
    # plain C99 (no Python); here it must compile warning-free and link
    # against libeta.so (running it needs a GPU)
    import subprocess
    cuda = "/usr/local/cuda"
    exe = tmp_path / "decode_example"
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                        "-I", os.path.join(cuda, "include"), os.path.join(ROOT, "tests", "c", "decode_example.c"),
                        "-L", os.path.join(ROOT, "learned_threshold_sparse_b200"), "-leta",
                        "-L", os.path.join(cuda, "lib64"), "-lcudart", "-lm", "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
