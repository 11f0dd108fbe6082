"""bench.py host logic without a GPU: the max-over-ranks timing with 2 gloo ranks, the
weak-scaling aggregate, the oracle reference arm and the stale-profile check."""
import io
import json
import os
import socket
import contextlib

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        t = bench.max_over_ranks(10.0 + 5.0 * rank)
        seed = bench.rank_seed(rank)
        q.put((rank, t, seed))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [r[1] for r in res] == [15.0, 15.0]      # every rank sees the slowest time
    assert res[0][2] != res[1][2]                    # each rank draws its own batch


def test_whole_job_value_is_weak_scaling_aggregate():
    f = 1e12
    assert bench.whole_job_tflops(f, 1, 10, 1000.0) == pytest.approx(10.0)
    assert bench.whole_job_tflops(f, 4, 10, 1000.0) == pytest.approx(40.0)


def test_reference_arm_prints_one_json_line():
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        rc = bench.main(["--impl", "reference", "--steps", "2", "--warmup", "3",
                         "--workload", "tiny"])
    assert rc == 0
    lines = [l for l in buf.getvalue().splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_do_nothing(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"]) == 0
    assert buf.getvalue() == ""


def test_warmup_minimum():
    with pytest.raises(SystemExit):
        bench.main(["--warmup", "2"])


def test_profile_traffic_only_for_current_sources(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    csrc = tmp_path / "exact_io_aware_60_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "fa_bwd.cuh").write_text("kernel v1")
    (csrc / "fa_fwd.cuh").write_text("forward v1")
    (csrc / "fa_api.cu").write_text("int launch_bwd(int a) {\n  return a;\n}\nint launch_fwd(int b) {\n  return b;\n}\n")
    (tmp_path / "profiles").mkdir()
    sha = bench.kernel_source_sha("fa_bwd_kernel")
    (tmp_path / "profiles" / "fa_bwd_kernel_gpt2.txt").write_text(
        f"source_sha: {sha}\ndram_bytes_per_launch: 12345\n")
    assert bench.profile_traffic("fa_bwd_kernel", "gpt2") == 12345.0
    # another kernel's code, or another launch function, does not touch this profile
    (csrc / "fa_fwd.cuh").write_text("forward v2")
    (csrc / "fa_api.cu").write_text("int launch_bwd(int a) {\n  return a;\n}\nint launch_fwd(int b) {\n  return b + 1;\n}\n")
    assert bench.profile_traffic("fa_bwd_kernel", "gpt2") == 12345.0
    # its own launch function or header does
    (csrc / "fa_api.cu").write_text("int launch_bwd(int a) {\n  return a + 1;\n}\nint launch_fwd(int b) {\n  return b + 1;\n}\n")
    assert bench.profile_traffic("fa_bwd_kernel", "gpt2") is None
    (csrc / "fa_api.cu").write_text("int launch_bwd(int a) {\n  return a;\n}\nint launch_fwd(int b) {\n  return b + 1;\n}\n")
    assert bench.profile_traffic("fa_bwd_kernel", "gpt2") == 12345.0
    (csrc / "fa_bwd.cuh").write_text("kernel v2")
    assert bench.profile_traffic("fa_bwd_kernel", "gpt2") is None


def test_source_hash_ignores_comments_and_layout_only(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    csrc = tmp_path / "exact_io_aware_60_b200" / "csrc"
    csrc.mkdir(parents=True)
    f = csrc / "k.cuh"
    f.write_text("int a = 1;  // one\nint b = 2;\n")
    h0 = bench.kernel_source_sha()
    f.write_text("/* header\n   text */\nint a = 1;   // first value, reworded\n\n\nint b = 2;\n")
    assert bench.kernel_source_sha() == h0
    f.write_text("int a = 1;\nint b = 3;\n")
    assert bench.kernel_source_sha() != h0
    (csrc / "note.txt").write_text("not a CUDA source")
    f.write_text("int a = 1;  // one\nint b = 2;\n")
    assert bench.kernel_source_sha() == h0


def test_visible_pairs_counts():
    import numpy as np
    T, N = 8, 1024
    ones = np.ones((T, T), np.uint8)
    assert bench.visible_pairs(N, ones, True) == N * (N + 1) // 2
    assert bench.visible_pairs(N, ones, False) == N * N
    assert bench.visible_pairs(300, np.ones((3, 3), np.uint8), False) == 300 * 300
    eye = np.eye(T, dtype=np.uint8)
    assert bench.visible_pairs(N, eye, False) == T * 128 * 128
    assert bench.visible_pairs(N, eye, True) == T * 128 * 129 // 2


@pytest.mark.parametrize("flags,suffix", [(["--dropout", "0.1"], "dropout p=0.1"),
                                          (["--block-sparse"], "block-sparse")])
def test_reference_arm_follows_the_measured_path(flags, suffix):
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        rc = bench.main(["--impl", "reference", "--steps", "2", "--warmup", "3",
                         "--workload", "tiny"] + flags)
    assert rc == 0
    d = json.loads(buf.getvalue().strip().splitlines()[-1])
    assert suffix in d["config"]["workload"] and d["value"] > 0


def test_dropout_and_block_sparse_are_exclusive():
    with pytest.raises(SystemExit):
        bench.main(["--impl", "reference", "--dropout", "0.1", "--block-sparse"])
    with pytest.raises(SystemExit):
        bench.main(["--impl", "reference", "--dropout", "1.0"])


def test_profiled_kernels_have_their_sources_and_launchers():
    """Every kernel whose profile bench.py reads names real files and a launch function
    that exists in fa_api.cu (a rename must not silently drop it from the hash)."""
    import os
    csrc = os.path.join(bench.ROOT, "exact_io_aware_60_b200", "csrc")
    api = open(os.path.join(csrc, "fa_api.cu"), encoding="utf-8").read()
    for kernel, (files, functions) in bench.KERNEL_SOURCES.items():
        for n in files:
            assert os.path.exists(os.path.join(csrc, n)), (kernel, n)
        launcher = functions[0]
        text = bench._function_text(api, launcher)
        assert text.startswith(f"int {launcher}(") and "return FA_OK;" in text, kernel
        # the helpers the launcher calls (tensor maps, workspace layout, schedule, launch)
        # are hashed too: each must be found as a definition and be called by the launcher
        # or by another of the listed helpers
        texts = {fn: bench._function_text(api, fn) for fn in functions[1:]}
        for fn, t in texts.items():
            assert t and f"{fn}(" in t.splitlines()[0] and t.rstrip().endswith("}"), (kernel, fn)
            callers = [text] + [u for g, u in texts.items() if g != fn]
            assert any(f"{fn}(" in c for c in callers), (kernel, fn, "not called")


def test_function_text_skips_declarations_and_calls():
    src = ("int helper(int a);\n"
           "static int user(int b) {\n    return helper(b) + 1;\n}\n"
           "int helper(int a) {\n    return a * 2;\n}\n")
    t = bench._function_text(src, "helper")
    assert t.startswith("int helper(int a) {") and "a * 2" in t
    assert bench._function_text(src, "missing") == ""


def test_reference_arm_config_matches_ours():
    """Both arms print the same config dict for the same flags (so the two lines are
    recognisably the same workload)."""
    import argparse
    from exact_io_aware_60_b200 import workloads as W
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3",
                           "--workload", "tiny"]) == 0
    d = json.loads(buf.getvalue().strip().splitlines()[-1])
    args = argparse.Namespace(block_sparse=False, fp8=False, dropout=0.0)
    assert d["config"] == bench.config_dict(W.WORKLOADS["tiny"], args, 1)
    for key in ("flops_per_step", "parallelism", "l2", "workload"):
        assert key in d["config"]


def test_effective_flops_of_key_padding():
    from exact_io_aware_60_b200 import workloads as W
    w = W.WORKLOADS["bert"]
    assert bench.effective_flops(w, [w.N] * w.B) == w.nominal_flops()
    f, b = bench.effective_flops(w, [w.N // 2] * w.B)
    assert f == w.nominal_flops()[0] / 2 and b == 2.5 * f
    g = W.WORKLOADS["gpt2"]
    assert bench.effective_flops(g, [g.N] * g.B)[0] == 4.0 * g.d * g.B * g.H * g.N * (g.N + 1) / 2
