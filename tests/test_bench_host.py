"""Host-side logic of bench.py that needs no GPU: the DRAM traffic recorded in the ncu
summaries under profiles/ and how it is scaled to a launch."""
import os

import bench


def _write_summary(root, kernel, workload, sha, traffic, units):
    os.makedirs(os.path.join(root, "profiles"), exist_ok=True)
    with open(os.path.join(root, "profiles", f"{kernel}_{workload}.md"), "w") as fh:
        fh.write(f"# `{kernel}` on the `{workload}` workload\n\n")
        fh.write(f"- dram_bytes_per_launch: `{traffic}`\n")
        fh.write(f"- units_per_launch: `{units}` (algorithmic bytes of this launch, from the same command)\n")
        fh.write(f"- sources_sha256: `{sha}`\n")


def test_recorded_traffic_scales_by_units(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "sources_sha256", lambda: "abc")
    _write_summary(str(tmp_path), "k_x", "w", "abc", 1000, 500)
    assert bench.recorded_traffic("k_x", "w", 500) == 1000.0
    assert bench.recorded_traffic("k_x", "w", 250) == 500.0      # a launch with half the units


def test_recorded_traffic_stale_or_missing(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "sources_sha256", lambda: "new")
    _write_summary(str(tmp_path), "k_x", "w", "old", 1000, 500)
    assert bench.recorded_traffic("k_x", "w", 500) is None      # sources changed since the capture
    assert bench.recorded_traffic("k_y", "w", 500) is None      # no summary at all


def _rank_main(rank, ws, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    try:
        # rank r timed (10 + r) ms for the steps and (20 - r) ms end to end
        got = bench.max_over_ranks([10.0 + rank, 20.0 - rank], "cpu")
        q.put((rank, got, bench.job_throughput(ws, 8, 100, got[0])))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    """The N > 1 reduction on two CPU ranks (gloo): every rank gets the element-wise maximum,
    and the whole-job throughput counts every rank's tokens over the slowest rank's time."""
    import socket
    import torch.multiprocessing as tmp
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    ctx = tmp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, thr in res:
        assert got == [11.0, 20.0]
        assert abs(thr - 2 * 8 * 100 / 0.011) < 1e-6 * thr


def test_max_over_ranks_single_process():
    assert bench.max_over_ranks([3.0, 4.5], "cpu") == [3.0, 4.5]
    assert bench.job_throughput(1, 8, 200, 11.0) == 8 * 200 / 0.011


def test_code_hash_ignores_comments_only():
    """The profile summaries stay valid across comment edits, not across code edits."""
    a = 'int f(int x) {  // twice\n  return 2 * x;  /* doubled */\n}\nconst char *s = "//not a comment";\n'
    b = '/* a new header */\nint f(int x) {\n\n  return 2 * x;\n}\nconst char *s = "//not a comment";\n'
    c = 'int f(int x) {\n  return 3 * x;\n}\nconst char *s = "//not a comment";\n'
    assert bench.strip_c_comments(a) == bench.strip_c_comments(b)
    assert bench.strip_c_comments(a) != bench.strip_c_comments(c)
    assert '"//not a comment"' in bench.strip_c_comments(a)


def test_clock_summary_keeps_only_samples_under_load():
    """Clock samples outside the loaded window (nvidia-smi start-up, idle tail) do not count."""
    ln = "{sm}, 1965, 700.5, 0x0000000000000000, Not Active, Not Active, Not Active, {cap}"
    lines = [(0.0, ln.format(sm=345, cap="Not Active")), (1.0, ln.format(sm=1965, cap="Not Active")),
             (1.2, ln.format(sm=1800, cap="Active")), (1.4, ln.format(sm=1965, cap="Not Active")),
             (9.0, ln.format(sm=400, cap="Not Active"))]
    got = bench.summarize_clock_lines(lines, 0.5, 2.0)
    assert got["samples"] == 3 and got["sm_mhz"] == 1965.0 and got["sm_max_mhz"] == 1965.0
    assert got["reasons"] == ["sw_power_cap"]
    assert bench.summarize_clock_lines(lines)["samples"] == 5
    assert bench.summarize_clock_lines([(0.0, "garbage")]) is None


def test_extra_workloads_default_and_none():
    a = bench.parse([])
    assert a.workload == "decode_T8"
    assert bench.extra_workloads(a) == ["layer_T1", "prefill_T4096", "stack30_T1", "prefill_T10000",
                                        "prefill_T40000", "block_T8"]
    assert bench.extra_workloads(bench.parse(["--extra", "none"])) == []
    assert bench.extra_workloads(bench.parse(["--workload", "prefill_T4096", "--extra", "layer_T1,prefill_T4096"])) \
        == ["layer_T1"]
    assert set(bench.WORKLOAD_T) == set(bench.mi.WORKLOADS)
