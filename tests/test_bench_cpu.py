"""Host-side accounting of bench.py (no GPU): the algorithmic bytes and
FLOPs behind the roofline fractions, counted here a second way, and the
rule that an ncu traffic figure is reported only for the exact kernel source
it was taken on."""
import json
import os

import pytest

import bench
from selective_state_space_29_b200 import workloads as wl


def test_scan_bytes_of_the_mid_workload():
    w = wl.SCAN_WORKLOADS["mid_bf16"]
    tc = w.batch * w.length * w.channels
    # u, delta read and y written (bf16); B, C per (batch, token, state); A, D; final state
    want = tc * 2 * 3 + 2 * w.batch * w.length * w.nstate * 2 + w.channels * (w.nstate + 1) * 4 \
        + w.batch * w.channels * w.nstate * 4
    assert abs(bench.scan_bytes(w) - want) <= 0.01 * want
    assert 300e6 < bench.scan_bytes(w) < 310e6       # ~6.06 bytes per token-channel


def test_scan_bytes_of_the_long_workload():
    w = wl.SCAN_WORKLOADS["long_bf16"]
    tc = w.batch * w.length * w.channels
    assert tc == 2_147_483_648
    # 3 x 2 bytes per token-channel, B and C 64 bytes per token, A, D, final state
    want = 6 * tc + 64 * w.length + w.channels * 17 * 4 + w.channels * 16 * 4
    assert bench.scan_bytes(w) == want
    assert 12.95e9 < bench.scan_bytes(w) < 12.96e9


def test_bench_defaults_to_the_largest_single_gpu_config(monkeypatch):
    monkeypatch.setattr("sys.argv", ["bench.py"])
    args = bench.parse_args()
    assert args.workload == "long_bf16"
    big = max(wl.SCAN_WORKLOADS.values(), key=bench.scan_bytes)
    assert big.name == args.workload


def test_ssd_bytes_of_the_mid_workload():
    w = wl.SSD_WORKLOADS["ssd_mid_bf16"]
    x_and_y = 2 * w.batch * w.length * w.channels * 2
    dt = w.batch * w.length * w.heads * 2
    bc = 2 * w.batch * w.length * w.nstate * 2
    state = w.batch * w.channels * w.nstate * 4
    assert bench.ssd_bytes(w) == x_and_y + dt + bc + state + w.heads * 4 + w.channels * 4


def test_ssd_mma_flops_by_enumerating_causal_blocks():
    w = wl.SSD_WORKLOADS["ssd_mid_bf16"].with_(length=1000)   # ragged last chunk counts as a whole chunk
    q, p, n = bench.SSD_CHUNK, 64, w.nstate
    k = q // 16
    blocks = sum(1 for row in range(k) for col in range(k) if col <= row)
    per_chunk = 2 * q * n * p                       # C S_in
    per_chunk += blocks * 2 * 16 * n * 16           # causal blocks of C B^T
    per_chunk += blocks * 2 * 16 * 16 * p           # causal blocks of M X
    per_chunk += 2 * n * q * p                      # B_w^T X
    chunks = (w.length + q - 1) // q
    assert bench.ssd_mma_flops(w) == w.batch * w.heads * chunks * per_chunk


def test_backward_bytes_of_the_mid_workload():
    w = wl.SCAN_WORKLOADS["mid_bf16"]
    tc = w.batch * w.length * w.channels
    bc = w.batch * w.length * w.nstate
    # u, delta, dy read; du, ddelta written; B, C read (bf16) and dB, dC written (fp32); A, D and gradients
    want = 5 * 2 * tc + bc * (2 * 2 + 2 * 4) + 2 * w.channels * (w.nstate + 1) * 4
    assert bench.backward_bytes(w) == want


def test_traffic_is_reported_only_for_the_profiled_source(tmp_path, monkeypatch):
    rec = json.load(open(os.path.join(bench.ROOT, "profiles", "traffic.json")))
    kernels = {e["kernel"] for e in rec["entries"]}
    assert {"scan_chunks_kernel", "state_update_kernel", "ssd_chunk_kernel", "scan_backward_kernel"} <= kernels
    for e in rec["entries"]:
        got = bench.profiled_traffic(e["kernel"], e["workload"])
        if e["source_hash"] == bench.source_hash(e["kernel"]):
            assert got == e["dram_bytes_per_launch"]
        else:
            assert got is None
    assert bench.profiled_traffic("scan_chunks_kernel", "no_such_workload") is None
    # a different source hash (an edited kernel) hides the figure
    monkeypatch.setattr(bench, "source_hash", lambda kernel="": "0" * 16)
    assert bench.profiled_traffic("scan_chunks_kernel", "mid_bf16") is None


@pytest.mark.parametrize("kernel", sorted(bench.KERNEL_SOURCES))
def test_kernel_sources_exist(kernel):
    for name in bench.KERNEL_SOURCES[kernel]:
        assert os.path.exists(os.path.join(bench.ROOT, "selective_state_space_29_b200", "csrc", name))
