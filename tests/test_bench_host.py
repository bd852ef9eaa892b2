"""CPU checks of the host logic of bench.py: which kernel family a workload
runs on, the rule that a recorded DRAM-traffic figure is used only for the
device sources it was captured on, and the work counts behind the metric."""
import dataclasses
import os

import numpy as np
import pytest

import bench
from workloads import WORKLOADS


@pytest.mark.parametrize("name,family", [
    ("long", "tile"), ("vit", "short"), ("unet_cross", "short"), ("tiny", "short"), ("unet_self", "tile"),
    ("long_fp8", "tile"), ("vit3136_neighborhood", "tile"),
    ("decode_gqa", "decode"), ("decode_gqa_small", "decode"),
    ("long_bwd", "bwd"), ("prefill_gqa_bwd", "bwd"),
])
def test_kernel_family(name, family):
    assert bench.kernel_family(WORKLOADS[name]) == family


def test_split_kv_with_many_rows_per_kv_head_uses_the_tile_kernel():
    w = dataclasses.replace(WORKLOADS["decode_gqa"], Nq=64)  # 4 x 64 rows per K/V head
    assert bench.kernel_family(w) == "tile"


def write_traffic(root, name, traffic, sha):
    import json
    os.makedirs(os.path.join(root, "profiles"), exist_ok=True)
    with open(os.path.join(root, "profiles", "traffic.json"), "w") as f:
        json.dump({f"attn_fwd_{name}": {"traffic_bytes_per_launch": traffic, "kernel_source_sha": sha}}, f)


def test_recorded_traffic_only_for_the_sources_it_was_taken_on(tmp_path, monkeypatch):
    w = WORKLOADS["long"]
    sha = bench.kernel_source_hash("tile")  # computed on the real sources
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    # the current sources' hash (the temporary root holds no sources)
    monkeypatch.setattr(bench, "kernel_source_hash", lambda family="tile": sha)
    assert bench.recorded_traffic(w) is None  # no record
    write_traffic(str(tmp_path), "long", 123456, "0" * 16)
    assert bench.recorded_traffic(w) is None  # record of other sources
    write_traffic(str(tmp_path), "long", 123456, sha)
    assert bench.recorded_traffic(w) == 123456.0
    write_traffic(str(tmp_path), "vit", 1, sha)
    assert bench.recorded_traffic(w) is None  # another workload's record


def test_committed_traffic_records_are_well_formed():
    import json
    recs = json.load(open(os.path.join(os.path.dirname(bench.__file__), "profiles", "traffic.json")))
    for key, rec in recs.items():
        assert key.startswith(("attn_fwd_", "attn_bwd_"))
        assert rec["traffic_bytes_per_launch"] > 0 and len(rec["kernel_source_sha"]) == 16
        assert os.path.exists(os.path.join(os.path.dirname(bench.__file__), "profiles", rec["summary"]))


def test_kernel_source_hash_depends_on_family_sources():
    hashes = {f: bench.kernel_source_hash(f) for f in ("tile", "short", "decode", "bwd")}
    assert len(set(hashes.values())) == 4 and all(len(h) == 16 for h in hashes.values())


def test_flops_dense_causal_backward_and_fp8():
    long = WORKLOADS["long"]
    assert long.flops() == 4.0 * 8 * 32 * 4096 * 4096 * 128
    assert WORKLOADS["long_causal"].flops() == long.flops() / 2
    assert WORKLOADS["long_bwd"].flops() == 2.5 * long.flops()
    assert WORKLOADS["long_fp8"].flops() == long.flops()  # same count whatever the input format
    assert bench.workload_flops(long) == long.flops()


def brute_keys_per_row(kind, W, size, shift, n, causal):
    out = []
    for i in range(n):
        ri, ci = divmod(i, W)
        c = 0
        for j in range(n):
            rj, cj = divmod(j, W)
            if kind == "neighborhood":
                ok = abs(ri - rj) < size and abs(ci - cj) < size
            else:
                ok = (ri + shift) // size == (rj + shift) // size and (ci + shift) // size == (cj + shift) // size
            if causal and j > i:
                ok = False
            c += ok
        out.append(c)
    return np.array(out)


@pytest.mark.parametrize("mask2d,causal", [(("neighborhood", 7, 2), False), (("neighborhood", 7, 3), True),
                                           (("window", 6, 3), False), (("window", 6, 4, 2), True)])
def test_mask2d_work_count_matches_brute_force(mask2d, causal):
    w = dataclasses.replace(WORKLOADS["vit3136_neighborhood"], B=1, Hq=1, Hkv=1, Nq=50, Nk=50,
                            mask2d=mask2d, is_causal=causal)
    shift = mask2d[3] if len(mask2d) > 3 else 0
    ref = brute_keys_per_row(mask2d[0], mask2d[1], mask2d[2], shift, 50, causal)
    np.testing.assert_array_equal(bench.mask2d_keys_per_row(w), ref)
    assert bench.workload_flops(w) == 4.0 * w.d * ref.sum()


def test_vit3136_neighborhood_counts_the_visible_pairs():
    """5.76 GFLOP of visible pairs: a 9 x 9 neighbourhood on the 56 x 56 grid."""
    w = WORKLOADS["vit3136_neighborhood"]
    per_row = bench.mask2d_keys_per_row(w)
    assert per_row.max() == 81 and per_row.min() == 25  # interior and corner tokens
    assert abs(bench.workload_flops(w) - 5.76e9) < 0.01e9
