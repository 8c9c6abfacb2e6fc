"""The N > 1 plumbing of bench.py (replicas, barrier, max-over-ranks timing) on two
gloo ranks on the CPU."""

import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench

    r, w, _ = bench.dist_setup(world)
    try:
        bench.barrier(w)
        # each rank times a different amount of work: the job's time is the slowest rank's
        t = bench.max_over_ranks(10.0 * (r + 1), w)
        out.put((r, w, t))
    finally:
        bench.dist_teardown(w)


@pytest.mark.timeout(120)
def test_two_gloo_ranks_take_the_max_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(90)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert got == [(0, 2, 20.0), (1, 2, 20.0)]


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.5, 1) == 3.5
    bench.barrier(1)


def test_kernel_source_digest_follows_only_its_kernel():
    sys.path.insert(0, ROOT)
    import bench

    # a recorded ncu figure is keyed to the code a kernel can depend on: its file without the
    # other kernels' bodies, plus the shared headers
    text = ("#include <x>\nconstexpr int k = 1;\n"
            "template <int D>\n__global__ void __launch_bounds__(384, 1)\n    ka(int a) {\n  if (a) { a = 2; }\n}\n"
            "__global__ void __launch_bounds__(256) kb(int b) { b = 3; }\n")
    base_a = bench.kernel_source_digest("bwd_sm100.cu", "ka", text)
    base_b = bench.kernel_source_digest("bwd_sm100.cu", "kb", text)
    t_a = text.replace("a = 2", "a = 5")    # change inside ka
    t_b = text.replace("b = 3", "b = 7")    # change inside kb
    t_top = text.replace("k = 1", "k = 2")  # change outside both kernels
    assert bench.kernel_source_digest("bwd_sm100.cu", "ka", t_a) != base_a
    assert bench.kernel_source_digest("bwd_sm100.cu", "kb", t_a) == base_b
    assert bench.kernel_source_digest("bwd_sm100.cu", "ka", t_b) == base_a
    assert bench.kernel_source_digest("bwd_sm100.cu", "kb", t_b) != base_b
    assert bench.kernel_source_digest("bwd_sm100.cu", "ka", t_top) != base_a
    assert bench.kernel_source_digest("bwd_sm100.cu", "kb", t_top) != base_b
    t_comment = text.replace("constexpr int k = 1;", "// a comment\nconstexpr int k = 1;  /* another */")
    assert bench.kernel_source_digest("bwd_sm100.cu", "ka", t_comment) == base_a  # comments do not count


def test_roofline_peak_follows_the_sampled_clock():
    sys.path.insert(0, ROOT)
    import bench

    peaks = {"bf16_tflops": 1617.9, "bf16_tflops_sustained": 1374.1, "source": "measured"}
    full = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}  # flag, clock not lowered
    low = {"sm_mhz": 1500.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    none = {"sm_mhz": None, "sm_max_mhz": None, "reasons": []}
    assert bench.tensor_peak(peaks, full)[0] == 1617.9
    assert bench.tensor_peak(peaks, low)[0] == 1374.1
    assert bench.tensor_peak(peaks, none)[0] == 1617.9


def test_wait_event_polls_until_done_and_gives_up():
    sys.path.insert(0, ROOT)
    import bench

    class Ev:  # stands in for a CUDA event: completes on the third query
        n = 0

        def query(self):
            self.n += 1
            return self.n >= 3

    ev = Ev()
    bench.wait_event(ev)
    assert ev.n == 3

    class Never:
        def query(self):
            return False

    with pytest.raises(RuntimeError):
        bench.wait_event(Never(), limit_s=0.01)
