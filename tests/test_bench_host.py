"""Host-side logic of the benchmark, on the CPU: the compulsory-byte formula
behind `roofline.achieved` and the source-hash guard on the committed DRAM
traffic figures behind `roofline.traffic`."""
import hashlib
import json
import os

import numpy as np
import pytest

import bench
import workloads as W


# Compulsory HBM bytes per call: E (s_u + s_y + gated (s_w + s_v)) + H bins 8,
# bins = N + 1 (L + 1 for a partial filter, the kept bins when masked).  The
# values are that formula evaluated by hand for each workload's shape.
@pytest.mark.parametrize("name,expected", [
    ("fp32_n1k", 8 * 1024 * 8 + 8 * 1025 * 8),                        # 131,136
    ("gated_bf16_n4k", 64 * 768 * 4096 * 8 + 768 * 4097 * 8),         # 1,635,784,704
    ("fp16_n32k", 8 * 256 * 32768 * 4 + 256 * 32769 * 8),             # 335,546,368
    ("dna_bf16_n1m", (1 << 27) * 4 + 128 * ((1 << 20) + 1) * 8),      # 1,610,613,760
    ("partial_bf16_n8k", 16 * 768 * 8192 * 8 + 768 * 2049 * 8),       # 817,895,424
    ("sparse_bf16_n8k", 16 * 768 * 8192 * 8 + 768 * 2048 * 8),        # 817,889,280: round(0.25 * 8193) bins
    ("dna_bf16_n4m_l1m", (1 << 27) * 4 + 32 * ((1 << 20) + 1) * 8),   # 805,306,624
])
def test_algorithmic_bytes(name, expected):
    assert bench.algorithmic_bytes(W.WORKLOADS[name]) == expected


# The tensor-core paths store each spectrum bin as complex fp16 (4 bytes).
@pytest.mark.parametrize("name,path,expected", [
    ("gated_bf16_n4k", "tc_fused", 64 * 768 * 4096 * 8 + 768 * 4097 * 4),       # 1,623,198,720
    ("fp16_n32k", "tc_staged", 8 * 256 * 32768 * 4 + 256 * 32769 * 4),         # 301,990,912
    ("gated_bf16_n4k", "simt_fused", 64 * 768 * 4096 * 8 + 768 * 4097 * 8),
])
def test_algorithmic_bytes_at_the_stored_filter_width(name, path, expected):
    assert bench.algorithmic_bytes(W.WORKLOADS[name], path) == expected


# Issued MMA flops per output element, from the instruction shapes of the
# 32 x 32 x 8 engine: 8*32 + 16*(32 + 8) = 896 for a zero-padded transform
# with half its outputs kept; 16*(32 + 32 + 8) = 1152 for a full one; three
# two blocks of 4096 per 8192 outputs (unmasked N = 8192) and four packed 1K
# sequences per 8192-point row keep 4096 outputs per transform like N = 4096.
@pytest.mark.parametrize("name,path,expected", [
    ("gated_bf16_n4k", "tc_fused", 896.0),
    ("gated_bf16_n1k", "tc_fused", 896.0),
    ("sparse_bf16_n8k", "tc_fused", 1152.0),
    ("partial_bf16_n8k", "tc_fused", 896.0),
    ("fp16_n16k", "tc_fused", 896.0),
    ("fp16_n32k", "tc_staged", 1152.0),
    ("fp32_n1k", "simt_fused", 0.0),
])
def test_mma_flops_per_element(name, path, expected):
    assert bench.mma_flops_per_elem(W.WORKLOADS[name], path)[1] == expected


def test_roofline_takes_the_slower_of_bytes_and_flops():
    w = W.WORKLOADS["gated_bf16_n4k"]
    r = bench.roofline_entry(w, "tc_fused", 0.5, 6531.9, 1607.7)
    t_hbm = 1623198720 / 6531.9e9
    t_mma = 896.0 * w.elems / 1607.7e12
    assert abs(r["hbm_frac"] - t_hbm / 0.5e-3) < 1e-12
    assert abs(r["frac"] - max(t_hbm, t_mma) / 0.5e-3) < 1e-12
    assert r["bound"] == "hbm"


def _fake_root(tmp_path, src_text, recorded_hash):
    (tmp_path / "profiles").mkdir()
    (tmp_path / "k.cu").write_text(src_text)
    entry = {"bytes_per_launch": 123, "source": "k.cu", "source_sha256": recorded_hash}
    (tmp_path / "profiles" / "dram_traffic.json").write_text(json.dumps({"w:path": entry}))
    return str(tmp_path)


def test_traffic_is_read_while_the_source_is_unchanged(tmp_path, monkeypatch):
    src = "kernel source\n"
    root = _fake_root(tmp_path, src, hashlib.sha256(src.encode()).hexdigest())
    monkeypatch.setattr(bench, "ROOT", root)
    assert bench.read_traffic("w:path")["bytes_per_launch"] == 123
    assert bench.read_traffic("other:path") is None


def test_traffic_is_dropped_once_the_source_changes(tmp_path, monkeypatch):
    root = _fake_root(tmp_path, "kernel source, edited\n", hashlib.sha256(b"kernel source\n").hexdigest())
    monkeypatch.setattr(bench, "ROOT", root)
    assert bench.read_traffic("w:path") is None


def test_committed_traffic_entries_name_existing_sources():
    with open(os.path.join(bench.ROOT, "profiles", "dram_traffic.json")) as f:
        d = json.load(f)
    assert d
    for key, ent in d.items():
        assert os.path.isfile(os.path.join(bench.ROOT, ent["source"])), key
        assert ent["bytes_per_launch"] == ent["dram_bytes_read"] + ent["dram_bytes_write"], key
        assert "--clock-control none" in ent["command"], key


def test_monarch_flop_count_and_kept_bins():
    """Monarch-aligned mask of the flagship shape: all c2 kept issues the dense
    896 flops per output; keeping c2 in {0..3, 28..31} skips 24 of the 32
    per-c2 products of S3 and S3' and two of the four K steps of S2'
    (2 * 24 * 8 * 128*16*16 + 16 * 128*64*16*2 fewer flops per 32768-output
    tile: 672 per output)."""
    assert bench.monarch_mma_flops_per_elem(0xFFFFFFFF) == 896.0
    assert bench.monarch_mma_flops_per_elem(0xF000000F) == 672.0
    w = W.WORKLOADS["monarch_bf16_n4k"]
    m = W.monarch_binmask(w.monarch_keep, w.N)
    M = 2 * w.N
    assert np.array_equal(m, m[(M - np.arange(M)) % M])          # Hermitian
    assert abs(W.monarch_kept_fraction(w) - 0.25) < 0.01
    assert W.make_mask(w) is None                                  # no block mask besides it
    assert np.all(W.monarch_binmask(0xFFFFFFFF, 1024) == 1)


def test_backward_bytes_and_grad_output_stream():
    # gated bf16 flagship shape: u, dy, w, v read and du, dw, dv written
    # (7 x 2 B per element), K_f read once at 4 B per bin, dk written in fp32
    w = W.WORKLOADS["gated_bf16_n4k"]
    assert bench.backward_bytes(w, "tc_fused") == w.elems * 14 + w.H * (w.N + 1) * 4 + w.H * w.L * 4
    p = W.WORKLOADS["partial_bf16_n8k"]
    assert bench.backward_bytes(p, "tc_fused") == p.elems * 14 + p.H * (p.L + 1) * 4 + p.H * p.L * 4
    small = W.Workload("t", index=99, B=2, H=3, N=64, L=64, dtype="bf16", gated=True, k_kind="scaled")
    dy = W.make_grad_output(small)
    assert dy.shape == (2, 3, 64) and np.array_equal(dy, W.make_grad_output(small))
    assert not np.array_equal(dy, W.make_input(small))                     # its own stream
    assert np.array_equal(dy, W.round_to(dy, "bf16"))
    assert set(bench.BACKWARD_WORKLOADS) <= set(W.WORKLOADS)
