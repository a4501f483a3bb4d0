"""Multi-rank plumbing of bench.py on CPU (gloo, world size 2): the timing
reduction takes the maximum over ranks, and the reference arm runs on rank 0
only (other ranks exit 0 without work)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks(torch, dist, 10.0 + 5.0 * rank, torch.device("cpu"))
        out[rank] = got
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
        assert dict(out) == {0: 15.0, 1: 15.0}


def test_max_over_ranks_single_process():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(torch, None, 3.5, torch.device("cpu")) == 3.5


def test_reference_arm_nonzero_rank_does_nothing(capsys):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    args = bench.parse_args(["--impl", "reference", "--steps", "3", "--warmup", "1"])
    assert bench.run_reference(args, rank=1, world=2) == 0
    assert capsys.readouterr().out == ""


def test_reference_arm_rank0_prints_one_line(capsys):
    import json
    import sys
    sys.path.insert(0, ROOT)
    import bench
    args = bench.parse_args(["--impl", "reference", "--steps", "3", "--warmup", "1",
                             "--workload", "tiny_decode_bf16"])
    assert bench.run_reference(args, rank=0, world=1) == 0
    lines = capsys.readouterr().out.strip().splitlines()
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["value"] > 0 and rec["unit"] == "tokens/s"
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["cpu_baseline"]["kind"] == "oracle"


def test_describe_plan_names_the_schedule_and_variants():
    """The bench's `kernel` field is the launch fqr_append_plan_query reports,
    in words (checked here on plans shaped like the library's)."""
    import sys
    sys.path.insert(0, ROOT)
    import bench
    lat = dict(schedule=1, grid=139, block_threads=384, tasks=1664, warp_check=1, bulk_tails=0,
               request_tails=0)
    d = bench.describe_plan(lat)
    assert "latency schedule" in d and "139 blocks of 384 threads" in d
    assert "1664 warp tasks" in d and "warp-level batch check" in d and "bulk" not in d
    d = bench.describe_plan(dict(lat, warp_check=0, bulk_tails=1, request_tails=1))
    assert "block batch prologue" in d and "bulk-copy tails" in d and "own the tails" in d
    d = bench.describe_plan(dict(schedule=2, grid=296, block_threads=256, tasks=9212,
                                 warp_check=0, bulk_tails=0, request_tails=0))
    assert "streaming schedule" in d and "296 blocks of 256 threads" in d and "9212 units" in d


def test_prefill_replicas_keep_the_batch_shape():
    """Every replica of the headline workload has the same tokens per request
    (so every timed step does the same work) but its own positions, pages and
    data; bytes per launch stay within a fraction of a percent."""
    import sys
    sys.path.insert(0, ROOT)
    import numpy as np
    import bench
    import workloads
    ws = bench.replica_workloads("ragged_prefill_fp8", min_bytes=1, max_replicas=2)
    assert len(ws) == 2
    a, b = ws
    assert a.T == b.T and np.array_equal(a.q_indptr, b.q_indptr)
    assert not np.array_equal(a.seq_lens, b.seq_lens)
    assert not np.array_equal(a.page_table, b.page_table)
    assert not np.array_equal(a.qkv[:4], b.qkv[:4])
    ba, bb = (workloads.append_bytes(w)["total"] for w in ws)
    assert abs(ba - bb) / ba < 1e-3
    # decode workloads keep one token per request in every replica
    ds = bench.replica_workloads("qwen3_decode_bf16", min_bytes=1, max_replicas=3)
    assert len(ds) == 2 and {w.T for w in ds} == {128}


def test_traffic_record_needs_the_current_kernel_sources(tmp_path, monkeypatch):
    """The traffic figure is used only when the ncu record was taken on the
    sources the library is built from now."""
    import json
    import sys
    sys.path.insert(0, ROOT)
    import bench
    rec = {"kernel_sources": bench.kernel_source_hash(),
           "workloads": {"ragged_prefill_fp8": {"dram_read_bytes": 100, "gpc_write_bytes": 50,
                                                "dram_write_bytes": 40}}}
    path = tmp_path / "traffic.json"
    path.write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "TRAFFIC_RECORD", str(path))
    t, parts = bench.profiled_traffic("ragged_prefill_fp8")
    assert t == 150 and parts["dram_write"] == 40
    assert bench.profiled_traffic("qwen3_decode_bf16")[0] is None
    rec["kernel_sources"] = "0" * 16
    path.write_text(json.dumps(rec))
    assert bench.profiled_traffic("ragged_prefill_fp8")[0] is None


def test_both_arms_name_the_same_config():
    """The GPU arm's line and the reference arm's line carry the same config
    block, derived from the workload alone."""
    import sys
    sys.path.insert(0, ROOT)
    import bench
    import workloads
    w = workloads.ragged_prefill_fp8()
    c = bench.config_block(w)
    assert c == bench.config_block(workloads.ragged_prefill_fp8())
    assert c["replicas"] == len(bench.replica_workloads("ragged_prefill_fp8"))
    assert c["workload"] == w.name and c["tokens_per_step"] == 9212 and "L2" in c["l2"]


def test_kernel_source_hash_ignores_comments_and_layout():
    """The hash that keys the traffic record follows the kernels' code only."""
    import sys
    sys.path.insert(0, ROOT)
    import bench
    a = "int f(int x) {  // the identity\n  return x; /* no\n change */ }\n"
    b = "int f(int x) {\n/* a different\n comment */ return x;\n}"
    assert bench._code_tokens(a) == bench._code_tokens(b) == "int f(int x) { return x; }"
    assert bench._code_tokens("return x + 1;") != bench._code_tokens("return x;")
    assert bench.kernel_source_hash() == bench.kernel_source_hash()


def test_cpu_leg_checks_the_e2e_outputs_byte_for_byte():
    """The cpu_baseline leg compares the e2e leg's host outputs of one step
    with the oracle's outputs of the same call: identical when they are the
    oracle's own, not identical once one byte of out_q differs."""
    import sys
    sys.path.insert(0, ROOT)
    import bench
    import numpy as np
    import oracle
    import workloads
    w = workloads.APPEND_CONFIGS["tiny_decode_bf16"]()
    es = w.kv_esize
    dt = np.uint16 if es == 2 else np.uint8
    kc = np.zeros((w.num_pages, w.page_size, w.Hkv, 128), dt)
    vc = np.zeros_like(kc)
    oq, qs, fl = oracle.new_outputs(w)
    assert oracle.append_paged(w, kc, vc, oq, None, fl) == 0
    sample = {"out_q": torch.from_numpy(oq.view(np.int16).copy()),
              "flags": torch.from_numpy(fl.copy())}
    res = bench.cpu_baseline(w, 0.05, sample)
    assert res["e2e_check"]["identical"] == {"out_q": True, "flags": True}
    sample["out_q"].view(-1)[7] ^= 1
    res = bench.cpu_baseline(w, 0.05, sample)
    assert res["e2e_check"]["identical"] == {"out_q": False, "flags": True}
