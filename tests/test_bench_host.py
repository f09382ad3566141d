"""Host-side logic of bench.py on CPU: the multi-rank timing reduction over
gloo (world size 2), the JSON line of the reference arm, and the stored
traffic lookup."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    bench.dist_init("gloo")
    # each rank reports its own step times; the job time is the max over ranks
    mine = [1.0 + rank, 2.0 - rank, 5.0 * (rank + 1)]
    mx = bench.dist_max(mine)
    sm = bench.dist_sum([1.0])
    bench.dist_barrier()
    bench.dist_finish()
    q.put((rank, mx, sm))


def test_dist_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, sm in res:
        assert mx == [2.0, 2.0, 10.0]
        assert sm == [2.0]


def test_single_rank_reduction_is_identity():
    assert bench.dist_max([3.0, 4.0]) == [3.0, 4.0]


def test_reference_arm_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "0"], capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
    # every input buffer's SHA-256, reproducible from the seeded generator
    from block_scaled_precision_requant_b200 import synth

    hashes = line["config"]["inputs_sha256"]
    assert hashes == bench.input_hashes(synth.make_workload("decode"))
    assert sorted(hashes) == ["a_bf16", "scale2", "w_e4m3", "w_packed"]
    assert all(len(v) == 64 and int(v, 16) >= 0 for v in hashes.values())


def test_reference_arm_non_zero_rank_exits_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1"],
                         capture_output=True, text=True, timeout=120, cwd=ROOT, env=env)
    assert out.returncode == 0 and out.stdout.strip() == ""


def test_units_and_bytes():
    from block_scaled_precision_requant_b200 import synth

    assert bench.decode_bytes(1, 4096, 4096) == 18890752
    u, unit, _ = bench.units_per_step(synth.WORKLOADS["ffn_up"])
    assert unit == "TOPS" and abs(u - 2 * 2048 * 14336 * 4096 / 1e12) < 1e-9


def test_stored_traffic_requires_matching_source(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    src = bench.kernel_source_hash("decode_kernel")
    (prof / "dram_traffic.txt").write_text(f"decode_kernel decode {src} 123\ndecode_kernel decode deadbeef 7\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda kernel: src)
    assert bench.stored_traffic("decode_kernel", "decode") == 123.0
    assert bench.stored_traffic("gemm_kernel", "decode") is None
    assert bench.stored_traffic("no_such_kernel", "decode") is None


def _csrc_copy(tmp_path, monkeypatch):
    import shutil

    src = os.path.join(bench.ROOT, "block_scaled_precision_requant_b200", "csrc")
    root = tmp_path / "r"
    csrc = root / "block_scaled_precision_requant_b200" / "csrc"
    shutil.copytree(src, csrc)
    monkeypatch.setattr(bench, "ROOT", str(root))
    return csrc


def test_source_hash_ignores_comments_not_code(tmp_path, monkeypatch):
    csrc = _csrc_copy(tmp_path, monkeypatch)
    h0 = bench.kernel_source_hash("decode_kernel")
    f = csrc / "decode.cu"
    text = f.read_text()
    f.write_text("// a new comment line\n/* and a block\n   comment */\n" + text.replace("\n\n", "\n\n\n", 3))
    assert bench.kernel_source_hash("decode_kernel") == h0
    f.write_text(text.replace("return MR <= 2 ? 32 : 8;", "return MR <= 2 ? 32 : 16;"))
    assert bench.kernel_source_hash("decode_kernel") != h0


def test_source_hash_follows_the_kernels_own_sources(tmp_path, monkeypatch):
    csrc = _csrc_copy(tmp_path, monkeypatch)
    assert bench.kernel_sources("decode_kernel") == ["api.cu", "common.cuh", "decode.cu", "kernels.h", "quant.cuh"]
    assert bench.kernel_sources("gemm_kernel") == ["api.cu", "common.cuh", "gemm_tc.cu", "kernels.h"]
    # a kernel launched from two layers depends on both
    assert bench.kernel_sources("nvfp4_gemv_kernel") == ["api.cu", "common.cuh", "fp_cvt.cuh", "kernels.h",
                                                         "nvfp4_enc.cuh", "nvfp4_gemv.cu", "w4a4.cu"]
    h = {k: bench.kernel_source_hash(k) for k in bench.KERNEL_UNITS}
    # a new, unrelated translation unit changes neither
    (csrc / "other.cu").write_text("__global__ void other_kernel() {}\n")
    assert {k: bench.kernel_source_hash(k) for k in bench.KERNEL_UNITS} == h
    # a shared header changes both; a kernel's own unit changes only it
    (csrc / "common.cuh").write_text((csrc / "common.cuh").read_text() + "\nconstexpr int kProbe = 1;\n")
    h2 = {k: bench.kernel_source_hash(k) for k in bench.KERNEL_UNITS}
    assert all(h2[k] != h[k] for k in h)
    (csrc / "gemm_tc.cu").write_text((csrc / "gemm_tc.cu").read_text() + "\nstatic int probe_value = 2;\n")
    assert bench.kernel_source_hash("gemm_kernel") != h2["gemm_kernel"]
    assert bench.kernel_source_hash("decode_kernel") == h2["decode_kernel"]

