"""The bench's host-side arithmetic (no GPU): the algorithmic bytes and FLOPs the roofline divides by,
and the traffic record it reports."""
import hashlib
import json
import os

import bench
from denoiser_attention_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_algorithmic_bytes_and_flops_of_the_batch_workload():
    # K + V of (16384 context + 16 block) tokens x 2 kv heads x 64 sequences at 2 x 128 x 2 bytes
    a = synth.workload("batch_bf16").attn
    assert bench.kv_bytes_of(a) == 64 * (16384 + 16) * 2 * 2 * 128 * 2 == 1074790400
    # 4 G S d per key and kv head (QK^T and PV), G S = 256 query rows per kv head
    assert bench.attn_flops_of(a) == 64 * (16384 + 16) * 2 * 4 * 16 * 16 * 128
    assert abs(bench.attn_flops_of(a) / 1e9 - 275.1) < 0.1


def test_algorithmic_bytes_of_the_ragged_workload_follow_its_lengths():
    a = synth.workload("ragged_paged").attn
    assert bench.kv_bytes_of(a) == sum(int(L) + 16 for L in a.ctx_lens) * 2 * 2 * 128 * 2


def test_traffic_record_is_tied_to_the_kernel_source():
    rec = json.load(open(os.path.join(ROOT, "profiles", "attn_tc_kernel_traffic.json")))["batch_bf16"]
    assert rec["dram_bytes_per_launch"] == rec["dram_bytes_read"] + rec["dram_bytes_write"]
    src = os.path.join(ROOT, "denoiser_attention_b200", "csrc", "attn_tc.cu")
    matches = hashlib.sha256(open(src, "rb").read()).hexdigest() == rec["source_sha256"]
    # reported only while the capture was taken on this version of the kernel source
    assert bench.measured_traffic("batch_bf16") == (rec["dram_bytes_per_launch"] if matches else None)
    assert bench.measured_traffic("decode_bf16") is None


def test_shard_ranges_cover_the_batch():
    for world in (1, 2, 3, 8):
        spans = [bench.shard_range(64 * world, world, r) for r in range(world)]
        assert spans[0][0] == 0 and spans[-1][1] == 64 * world
        assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
