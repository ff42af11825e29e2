"""Host logic of the multi-GPU benchmark path on CPU: two gloo ranks on 127.0.0.1.

The fused linear has no exchange step (every token row is independent), so N GPUs
run N replicas; the only collectives are the timing barrier and the max-over-ranks
reduction of the elapsed time."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    r, w, local = bench.dist_init(world)
    try:
        bench.barrier(w)
        t = bench.max_over_ranks(10.0 + 5.0 * r, w)   # rank-dependent elapsed times
        q.put((r, w, local, t))
    finally:
        bench.dist_done(w)


@pytest.mark.timeout(120)
def test_two_gloo_ranks_take_the_max_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(90)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(world))
    assert [g[0] for g in got] == [0, 1]
    assert all(g[1] == 2 for g in got)
    assert all(g[3] == 15.0 for g in got)   # every rank sees the slowest rank's time


def test_single_process_needs_no_process_group():
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        os.environ.pop(k, None)
    assert bench.dist_init(1) == (0, 1, 0)
    assert bench.max_over_ranks(3.5, 1) == 3.5


def test_gemm_traffic_tracks_the_kernel_source(tmp_path, monkeypatch):
    """roofline.traffic comes from the committed ncu capture only while the GEMM sources
    hash to the value recorded beside it."""
    import hashlib
    src = tmp_path / "k.cuh"
    src.write_bytes(b"kernel v1")
    prof = tmp_path / "gemm_traffic_block2048_w4a8.md"
    digest = hashlib.sha256(b"kernel v1").hexdigest()
    prof.write_text(f"# t\n\n    traffic_bytes_per_launch: 1234\n    source_sha256: {digest}\n")
    monkeypatch.setattr(bench, "traffic_file", lambda w: str(tmp_path / f"gemm_traffic_{w}.md"))
    monkeypatch.setattr(bench, "GEMM_SOURCES", [str(src)])
    assert bench.gemm_traffic("block2048_w4a8") == 1234
    assert bench.gemm_traffic("block4096_w4a8_t10") is None   # no capture for that workload
    src.write_bytes(b"kernel v2")                              # the kernel changed since
    assert bench.gemm_traffic("block2048_w4a8") is None


def test_gemm_traffic_ignores_host_side_edits(tmp_path, monkeypatch):
    """Only the device code before the host-side marker identifies the kernel."""
    marker = bench.HOST_SIDE_MARKER.decode()
    src = tmp_path / "g.cuh"
    src.write_text(f"__global__ void k() {{}}\n{marker}\nint host_a();\n")
    digest = bench.gemm_device_source_hash([str(src)])
    prof = tmp_path / "gemm_traffic_block2048_w4a8.md"
    prof.write_text(f"    traffic_bytes_per_launch: 77\n    source_sha256: {digest}\n")
    monkeypatch.setattr(bench, "traffic_file", lambda w: str(tmp_path / f"gemm_traffic_{w}.md"))
    monkeypatch.setattr(bench, "GEMM_SOURCES", [str(src)])
    assert bench.gemm_traffic("block2048_w4a8") == 77
    src.write_text(f"__global__ void k() {{}}\n{marker}\nint host_b();\n")   # host side only
    assert bench.gemm_traffic("block2048_w4a8") == 77
    src.write_text(f"__global__ void k() {{ int x; }}\n{marker}\nint host_b();\n")  # device
    assert bench.gemm_traffic("block2048_w4a8") is None


def test_bench_names_the_gemm_instance_of_each_linear():
    """The bench line's per-linear entries name the GEMM instance from the library's
    plan: 224-token pairs with the weights in TMEM on the hidden-4096 block, 256-token
    pairs for its attention output projection at 4288 tokens, one CTA with 256-deep
    stages at 16 tokens."""
    import activation_quantized_gemm_wq_b200 as wq
    assert bench.gemm_instance(wq, 8512, 4096, 16384) == (
        "256 channels x 224 tokens on a CTA pair, 128-deep stages, int8 weights in TMEM")
    assert bench.gemm_instance(wq, 4288, 2048, 2048) == (
        "256 channels x 256 tokens on a CTA pair, 128-deep stages")
    assert bench.gemm_instance(wq, 16, 16384, 4096) == (
        "128 channels x 16 tokens on one CTA, 256-deep stages, int8 weights in TMEM, "
        "K split 4 ways")


def test_cpu_baseline_reports_each_linear():
    """The oracle's timing on the host: the aggregate over the sample, the same sample
    on one thread, and each linear's time extrapolated to the full token batch."""
    from activation_quantized_gemm_wq_b200 import synth as S
    r = bench.cpu_baseline(S.TINY, rows=4)
    assert r["kind"] == "oracle" and r["unit"] == "TOPS" and r["value"] > 0
    assert r["cores"] >= 1 and r["single_thread"]["cores"] == 1
    assert [p["linear"] for p in r["per_linear"]] == [
        f"{lin.name} {lin.K}->{lin.N}" for lin in S.TINY.linears]
    assert all(p["seconds_full_batch"] >= 0 and p["tops"] > 0 for p in r["per_linear"])


def test_peaks_file_is_read_only_when_it_holds_numbers(tmp_path):
    f = tmp_path / "peaks.json"
    f.write_text('{"hbm_gbs": 6550.5, "bf16_tflops": 1630, "bf16_tflops_sustained": 1410}')
    assert bench.peaks(str(f)) == (1630.0, 1410.0, 6550.5, "measured")
    f.write_text('{"hbm_gbs": 6550.5, "bf16_tflops": 1630}')   # no sustained figure
    assert bench.peaks(str(f)) == (1630.0, 1630.0, 6550.5, "measured")
    fallback = (bench.FALLBACK_BF16_TFLOPS, bench.FALLBACK_BF16_TFLOPS_SUSTAINED,
                bench.FALLBACK_HBM_GBS, "fallback")
    for bad in ('{"hbm_gbs": {"value": 6550}, "bf16_tflops": 1630}', '[1, 2, 3]', 'not json',
                '{"hbm_gbs": 0, "bf16_tflops": 1630}', '{"bf16_tflops": 1630}',
                '{"hbm_gbs": "6550", "bf16_tflops": 1630}'):
        f.write_text(bad)
        assert bench.peaks(str(f)) == fallback, bad
    assert bench.peaks(str(tmp_path / "absent.json")) == fallback
