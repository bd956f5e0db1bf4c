"""The C-ABI library loads, exports every entry point include/eta.h declares,
and rejects bad arguments on the host before launching anything (no GPU needed)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "eta.h")


def declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"ETA_API\s+[\w\s\*]+?\b(eta_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared()
    for n in ("eta_build_block_meta", "eta_predict_tau", "eta_decode_sparse", "eta_decode_dense", "eta_screen",
              "eta_decode_workspace_bytes", "eta_read_device_status", "eta_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol():
    from learned_block_sparse_b200 import binding
    out = subprocess.run(["nm", "-D", "--defined-only", binding.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (eta_\w+)", out))
    for n in declared():
        assert n in exported, n
        assert hasattr(binding.lib, n)
    assert set(binding.EXPORTED) == set(declared())
    # nothing else leaks out of the library's C++ internals as eta_ symbols
    assert exported == set(declared())


def test_abi_version_and_status_strings():
    from learned_block_sparse_b200 import binding
    assert binding.lib.eta_abi_version() == 3
    assert binding.status_string(0) == "ok"
    assert "workspace" in binding.status_string(3)
    assert binding.status_string(99) == "unknown status"


def _shape(**kw):
    from learned_block_sparse_b200 import binding
    d = dict(batch=1, n_q_heads=4, n_kv_heads=2, head_dim=128, block_size=32, capacity=1024, kv_dtype=1, q_dtype=1)
    d.update(kw)
    return binding.Shape(**d)


@pytest.mark.parametrize("kw,expect", [
    (dict(head_dim=96), 2), (dict(block_size=48, capacity=960), 2), (dict(n_q_heads=6, n_kv_heads=4), 1),
    (dict(n_q_heads=32, n_kv_heads=2), 2), (dict(capacity=1000), 1), (dict(batch=0), 1), (dict(kv_dtype=7), 1),
])
def test_shape_validation(kw, expect):
    from learned_block_sparse_b200 import binding
    s = _shape(**kw)
    p = binding.make_params()
    k = ctypes.c_void_p(4096)
    st = binding.lib.eta_decode_dense(ctypes.byref(s), ctypes.byref(p), k, k, k, 100, None, 0, k, k, 1 << 20, None)
    assert st == expect
    assert binding.lib.eta_decode_workspace_bytes(ctypes.byref(s), ctypes.byref(p)) == 0


def test_argument_validation_before_launch():
    from learned_block_sparse_b200 import binding
    s = _shape()
    p = binding.make_params()
    L = binding.lib
    a16 = ctypes.c_void_p(1 << 20)
    bad = ctypes.c_void_p((1 << 20) + 2)
    meta = binding.Meta(1 << 20, 1 << 20, 1 << 20)
    # n_tokens out of range, null and misaligned pointers
    assert L.eta_decode_sparse(ctypes.byref(s), ctypes.byref(p), a16, a16, a16, meta, 0, a16, 0, a16, None, a16,
                               1 << 30, None) == 1
    assert L.eta_decode_sparse(ctypes.byref(s), ctypes.byref(p), a16, a16, a16, meta, 2000, a16, 0, a16, None,
                               a16, 1 << 30, None) == 1
    assert L.eta_decode_sparse(ctypes.byref(s), ctypes.byref(p), a16, bad, a16, meta, 100, a16, 0, a16, None, a16,
                               1 << 30, None) == 1
    assert L.eta_decode_sparse(ctypes.byref(s), ctypes.byref(p), a16, a16, a16, meta, 100, None, 0, a16, None,
                               a16, 1 << 30, None) == 1
    # workspace: null, misaligned, too small
    assert L.eta_decode_sparse(ctypes.byref(s), ctypes.byref(p), a16, a16, a16, meta, 100, a16, 0, a16, None,
                               None, 1 << 30, None) == 3
    assert L.eta_decode_sparse(ctypes.byref(s), ctypes.byref(p), a16, a16, a16, meta, 100, a16, 0, a16, None,
                               ctypes.c_void_p((1 << 20) + 16), 1 << 30, None) == 3
    assert L.eta_decode_sparse(ctypes.byref(s), ctypes.byref(p), a16, a16, a16, meta, 100, a16, 0, a16, None,
                               a16, 64, None) == 3
    # params
    for bad_p in (binding.make_params(beta=0.0), binding.make_params(n_local=0), binding.make_params(n_splits=-1),
                  binding.make_params(z=float("nan")), binding.make_params(gate=2),
                  binding.make_params(sub_blocks=3), binding.make_params(sub_blocks=-1)):
        assert L.eta_decode_dense(ctypes.byref(s), ctypes.byref(bad_p), a16, a16, a16, 100, None, 0, a16, a16,
                                  1 << 30, None) == 1
    # per-row lengths: the length array is required; max_tokens bounded by the capacity
    assert L.eta_decode_dense_ragged(ctypes.byref(s), ctypes.byref(p), a16, a16, a16, None, 100, None, 0, a16,
                                     a16, 1 << 30, None) == 1
    assert L.eta_decode_dense_ragged(ctypes.byref(s), ctypes.byref(p), a16, a16, a16, a16, s.capacity + 1, None, 0,
                                     a16, a16, 1 << 30, None) == 1
    assert L.eta_decode_sparse_ragged(ctypes.byref(s), ctypes.byref(p), a16, a16, a16, meta, a16, 100, None, 0,
                                      None, None, None, a16, None, a16, 1 << 30, None) == 1   # no thresholds
    # sub-block envelope: sub-blocks of fewer than 16 tokens, and paged stores, are not supported
    for bs, r in ((32, 4), (16, 2)):
        s2 = _shape(block_size=bs)
        p2 = binding.make_params(sub_blocks=r)
        assert L.eta_screen(ctypes.byref(s2), ctypes.byref(p2), a16, meta, 100, a16, 0, None, a16, 1 << 30,
                            None) == 2, (bs, r)
    assert L.eta_decode_workspace_bytes(ctypes.byref(s), ctypes.byref(binding.make_params(sub_blocks=2))) > 0
    pages = binding.Pages(1 << 20, 64)
    p2 = binding.make_params(sub_blocks=2)
    assert L.eta_decode_sparse_paged(ctypes.byref(s), ctypes.byref(p2), a16, a16, a16, pages, meta, a16, 100, a16,
                                     0, None, None, None, a16, None, a16, 1 << 30, None) == 2
    # metadata block range
    assert L.eta_build_block_meta(ctypes.byref(s), a16, -1, 3, meta, None) == 1
    assert L.eta_build_block_meta(ctypes.byref(s), a16, 0, 33, meta, None) == 1
    assert L.eta_build_block_meta(ctypes.byref(s), a16, 5, 5, meta, None) == 0      # empty range: no-op
    # more cache (or pool) rows than a 32-bit row index reaches: unsupported, for the builders too
    big = _shape(batch=128, n_q_heads=16, n_kv_heads=16, block_size=16, capacity=1 << 20)
    assert L.eta_build_block_meta(ctypes.byref(big), a16, 0, 1, meta, None) == 2
    assert L.eta_build_block_meta_paged(ctypes.byref(s), a16, binding.Pages(1 << 20, 1 << 26), 0, 1, meta,
                                        None) == 2
    assert L.eta_build_block_meta_paged(ctypes.byref(s), a16, binding.Pages(1 << 20, 64), 0, 0, meta, None) == 0
    assert L.eta_predict_tau(ctypes.byref(s), None, a16, a16, a16, None) == 1
    # screen diagnostics: every buffer required, the fp64 output 8-byte aligned
    assert L.eta_screen_diagnostics(ctypes.byref(s), ctypes.byref(p), 100, a16, 0, a16, a16, a16, None, a16, a16,
                                    None) == 1
    assert L.eta_screen_diagnostics(ctypes.byref(s), ctypes.byref(p), 100, a16, 0, a16, a16, a16, a16, a16,
                                    ctypes.c_void_p((1 << 20) + 4), None) == 1
    assert L.eta_screen_diagnostics(ctypes.byref(s), ctypes.byref(p), 0, a16, 0, a16, a16, a16, a16, a16, a16,
                                    None) == 1
    st = ctypes.c_int(0)
    assert L.eta_read_device_status(None, None, ctypes.byref(st)) == 1
    assert L.eta_workspace_init(bad, 1 << 20, None) == 3


def test_workspace_size_grows_with_splits_and_capacity():
    from learned_block_sparse_b200 import binding
    s = _shape()
    a = binding.workspace_bytes(s, binding.make_params(n_splits=4))
    b = binding.workspace_bytes(s, binding.make_params(n_splits=8))
    c = binding.workspace_bytes(_shape(capacity=4096), binding.make_params(n_splits=8))
    assert a < b < c and a % 256 == 0


def test_binding_structs_match_the_header(tmp_path):
    """The ctypes mirrors of eta_shape_t, eta_params_t, eta_meta_t, eta_pages_t and
    eta_screen_out_t have the header's sizes and field offsets (a C probe compiled
    against include/eta.h)."""
    from learned_block_sparse_b200 import binding
    structs = {"eta_shape_t": binding.Shape, "eta_params_t": binding.Params, "eta_meta_t": binding.Meta,
               "eta_pages_t": binding.Pages, "eta_screen_out_t": binding.ScreenOut}
    lines = ['#include <stddef.h>', '#include <stdio.h>', '#include "eta.h"', 'int main(void) {']
    for cname, py in structs.items():
        lines.append(f'  printf("{cname} size %zu\\n", sizeof({cname}));')
        for fname, _ in py._fields_:
            lines.append(f'  printf("{cname} {fname} %zu\\n", offsetof({cname}, {fname}));')
    lines += ['  return 0;', '}']
    src = tmp_path / "probe.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "probe"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), "-I", "/usr/local/cuda/include", str(src), "-o",
                    str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    got = {}
    for line in out:
        if line:
            c, f, v = line.split()
            got[(c, f)] = int(v)
    for cname, py in structs.items():
        assert got[(cname, "size")] == ctypes.sizeof(py), cname
        for fname, _ in py._fields_:
            assert got[(cname, fname)] == getattr(py, fname).offset, (cname, fname)
