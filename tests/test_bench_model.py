"""The benchmark's byte model (the numerator of the roofline fraction): K+V
bytes of the admitted union blocks with the partial last block counted by its
valid rows, metadata of the screened blocks (r columns per block with the
sub-block envelope), and the split partials only for segments that cross
thread-block ranges. The dense K+V bytes are pinned to the cache sizes printed
in the pages' Table 5 (thelatestinai.com)."""
import json
import os

import numpy as np
import pytest

import bench
from learned_block_sparse_b200 import synth


def _w(**kw):
    d = dict(name="m", dtype="bf16", B=2, Hq=8, Hkv=2, d=128, n=32 * 100 + 5, bs=32, z=1.0, tau_mode="const",
             densities=(0.4,), seed=1)
    d.update(kw)
    return synth.Workload(**d)


def test_kv_bytes_count_the_valid_rows_of_the_last_block():
    w = _w()
    ucnt = np.full((w.B, w.Hkv), 40, np.int64)          # every list ends with the partial block
    hcnt = np.full((w.B, w.Hq), 20, np.int64)
    m = bench.byte_model(w, ucnt, hcnt, S=148)
    row = w.d * 2
    last = w.n - (w.nb - 1) * w.bs                       # 5 valid rows
    assert m["kv"] == 2 * row * (int(ucnt.sum()) * w.bs - w.B * w.Hkv * (w.bs - last))
    assert m["union_blocks"] == int(ucnt.sum())
    assert m["d_union"] == pytest.approx(ucnt.sum() / (w.B * w.Hkv * w.nb))
    assert m["d_head"] == pytest.approx(hcnt.sum() / (w.B * w.Hq * w.nb))


@pytest.mark.parametrize("r", [1, 2, 4])
def test_metadata_bytes_scale_with_sub_blocks(r):
    w = _w(bs=64, n=64 * 50 + 1)
    ucnt = np.full((w.B, w.Hkv), 10, np.int64)
    hcnt = np.full((w.B, w.Hq), 5, np.int64)
    m = bench.byte_model(w, ucnt, hcnt, S=148, r=r)
    assert m["meta"] == w.B * w.Hkv * w.n_screened * r * (2 * w.d + 1) * 4


def test_partials_only_for_segments_crossing_ranges():
    w = _w(B=1, Hkv=2, Hq=2)
    hcnt = np.ones((1, 2), np.int64)
    # T = 300 entries over S = 3 ranges of 100: segment 0 = [0, 150) crosses one boundary (2 parts),
    # segment 1 = [150, 300) crosses one (2 parts)
    ucnt = np.array([[150, 150]], np.int64)
    m = bench.byte_model(w, ucnt, hcnt, S=3)
    partial = (w.d + 2) * 4 * w.G
    base = bench.byte_model(w, ucnt, hcnt, S=1)           # one range: no partials
    assert m["decode_kernel"] - base["decode_kernel"] == 4 * partial
    # fewer entries than ranges: every entry is its own range
    small = np.array([[1, 2]], np.int64)
    m2 = bench.byte_model(w, small, hcnt, S=148)
    b2 = bench.byte_model(w, small, hcnt, S=1)
    assert m2["decode_kernel"] - b2["decode_kernel"] == 2 * partial   # segment 1 has 2 entries -> 2 parts


def test_dense_kv_bytes_match_table5_cache_sizes():
    """Table 5's KV column (H_Q 32, H_KV 4, d_h 64, fp16): 2 GB at B 32 and 64K
    tokens, doubling with L and with B. The byte model's dense K+V bytes of the
    same shapes in a 2-byte dtype must be exactly those sizes (GiB)."""
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "table5_kv_bytes.json")
    g = json.load(open(path))
    for row in g["rows"]:
        w = _w(B=row["B"], Hq=32, Hkv=g["h_kv"], d=g["head_dim"], n=row["L"], bs=64)
        ucnt = np.full((w.B, w.Hkv), w.nb, np.int64)
        hcnt = np.full((w.B, w.Hq), w.nb, np.int64)
        m = bench.byte_model(w, ucnt, hcnt, S=148)
        assert m["dense_kv"] == row["gib"] << 30, row
        assert m["kv"] == m["dense_kv"]           # every block admitted: the dense bytes
