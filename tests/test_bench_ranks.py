"""The multi-rank host logic of bench.py on CPU: two gloo ranks (one process
each, 127.0.0.1) agree on the job time as the max over ranks, the whole-job
value counts every replica, and a single rank needs no process group."""
import datetime
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, times, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=30))
    try:
        torch.distributed.barrier()
        q.put((rank, bench.max_over_ranks(times[rank], world, torch.device("cpu"))))
    finally:
        torch.distributed.destroy_process_group()


@pytest.mark.parametrize("times", [(12.5, 17.25), (9.0, 3.0)])
def test_max_over_ranks_two_gloo_ranks(times):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, times, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = {}
    try:
        for _ in procs:
            r, v = q.get(timeout=60)
            got[r] = v
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    assert got == {0: max(times), 1: max(times)}


def test_single_rank_needs_no_group():
    assert not torch.distributed.is_initialized()
    assert bench.max_over_ranks(4.5, 1, torch.device("cpu")) == 4.5


def test_whole_job_value_counts_every_replica():
    f = 106.17e9                                      # flop of one replica's step
    one = bench.whole_job_value(1, f, 0.36)
    assert one == pytest.approx(f / 0.36e-3 / 1e12)
    # weak scaling: N replicas in the same time are N times the work
    assert bench.whole_job_value(8, f, 0.36) == pytest.approx(8 * one)
    # the max-over-ranks time decides: a slower rank lowers the job's value
    assert bench.whole_job_value(2, f, 0.40) < bench.whole_job_value(2, f, 0.36)


@pytest.mark.parametrize("name", ["tiny", "opensora_low"])
def test_oracle_arm_samples_fit_the_workload(name):
    """The timed oracle samples (cpu_baseline and the reference arm) stay
    inside the workload: the temporal sample takes at most a frame's tokens,
    so a frame smaller than the default sample (tiny: 64 tokens) still runs."""
    import argparse
    import synth
    w = synth.BY_NAME[name]
    cb = bench.cpu_baseline(w, budget_s=0.2)
    assert cb["kind"] == "oracle" and cb["value"] > 0 and cb["single_thread"]["value"] > 0
    line = bench.run_reference(argparse.Namespace(cpu_budget=0.2, steps=1, warmup=3), w)
    assert line["impl"] == "reference" and line["value"] > 0


def test_step_kind_per_workload():
    """Each workload takes the step its layout calls for: the image-DiT block
    (T = 1 with the Q/K RMSNorm), the V-Major step (T = 1 with change
    fractions) or the ST-DiT block."""
    import synth
    kinds = {w.name: bench.step_kind(w) for w in synth.WORKLOADS}
    assert kinds == {"tiny": "st", "opensora_low": "st", "video_1080p": "st", "image_4096px": "image",
                     "vmajor_2304px": "vmajor"}


@pytest.mark.parametrize("workload,launch", [("image_4096px", "ring"), ("opensora_low", "ring"),
                                             ("video_1080p", "ring"), ("vmajor_2304px", "cached_kv")])
def test_traffic_record_matches_the_attention_source(workload, launch):
    """The committed DRAM counters of each workload's roofline launch belong to
    the attention source as it stands (the bench reports them as
    roofline.traffic only then), and lie between what the launch must read (Q,
    K and V once; part of O may still be in L2 when the launch ends) and its
    algorithmic bytes plus the K/V re-reads of the ring walk."""
    import synth
    got = bench.kernel_traffic(workload, launch)
    assert got is not None, "profiles/traffic.json was captured on another attention source"
    w = synth.BY_NAME[workload]
    t = w.B * w.T * w.S * w.C * w.elem_bytes
    assert 0.98 * 3 * t <= got <= 1.6 * 4 * t
