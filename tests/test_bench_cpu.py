"""bench.py's host-side arithmetic, on CPU: the roofline numerator of a step
(indexer FP8 key bytes, read once per sequence and index group, plus the bf16
latent rows the attention gathers), the whole-job throughput over ranks, and
the DRAM traffic recorded from an ncu capture, which is used only while the
kernel source it was captured on is unchanged."""
import hashlib
import types

import torch

import bench

KEY_B = 128          # e4m3 indexer key
ROW_B = 576 * 2      # bf16 latent row


def _inp(T, vis, n_layers=1, index_share=1, mtp_index_share=False, topk=2048):
    B = len(vis) // T
    return types.SimpleNamespace(
        B=B, T=T, q_vis=torch.tensor(vis, dtype=torch.int32),
        q_offsets=torch.arange(B + 1, dtype=torch.int32) * T, n_layers=n_layers,
        index_share=index_share, mtp_index_share=mtp_index_share, topk=topk)


def test_batch32_128k_step_bytes():
    keys, gathered = bench.algorithmic_bytes(_inp(1, [131072] * 32))
    assert keys == 536_870_912                 # 32 x 131072 keys x 128 B
    assert gathered == 75_497_472              # 32 x 2048 rows x 1152 B


def test_short_rows_gather_only_what_is_visible():
    keys, gathered = bench.algorithmic_bytes(_inp(1, [1000, 3000]))
    assert keys == (1000 + 3000) * KEY_B
    assert gathered == (1000 + 2048) * ROW_B


def test_mtp_verify_reads_keys_once_per_sequence():
    vis = [100, 101, 102, 5000, 5001, 5002]    # 2 sequences x 3 positions
    keys, gathered = bench.algorithmic_bytes(_inp(3, vis))
    assert keys == (102 + 5002) * KEY_B        # the longest position of each sequence
    assert gathered == (100 + 101 + 102 + 3 * 2048) * ROW_B
    # position 0's selection reused: one key scan and one gather per sequence
    keys, gathered = bench.algorithmic_bytes(_inp(3, vis, mtp_index_share=True))
    assert keys == (100 + 5000) * KEY_B
    assert gathered == (100 + 2048) * ROW_B


def test_index_share_scans_keys_once_per_group_and_gathers_per_layer():
    vis = [4000, 9000]
    for n_layers, share, groups in [(4, 4, 1), (6, 4, 2), (9, 8, 2), (3, 1, 3)]:
        keys, gathered = bench.algorithmic_bytes(_inp(1, vis, n_layers=n_layers, index_share=share))
        assert keys == groups * (4000 + 9000) * KEY_B
        assert gathered == n_layers * (2048 + 2048) * ROW_B


def test_job_throughput_counts_every_rank_over_the_slowest_time():
    assert bench.job_throughput(32, 1, 20, 4.0) == 32 * 20 / 4e-3
    assert bench.job_throughput(32, 4, 20, 4.0) == 4 * bench.job_throughput(32, 1, 20, 4.0)
    assert bench.reduce_over_ranks(3.5, 1) == 3.5


def test_recorded_traffic_is_dropped_once_the_kernel_source_changes(tmp_path, monkeypatch):
    csrc = tmp_path / "sparse_attention_decode_lightning_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    src = csrc / "k.cu"
    src.write_bytes(b"__global__ void k() {}\n")
    sha = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    (tmp_path / "profiles" / "k.md").write_text(
        f"# capture\n\ntraffic_bytes_per_launch: 123456\nsource_sha256_16: {sha}\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("k.cu", "k.md") == 123456
    src.write_bytes(b"__global__ void k() { }\n")        # the kernel changed since the capture
    assert bench.measured_traffic("k.cu", "k.md") is None
    assert bench.measured_traffic("k.cu", "absent.md") is None
