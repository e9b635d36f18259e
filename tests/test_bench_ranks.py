"""The multi-rank plumbing of bench.py, on the CPU: the max-over-ranks timing
reduction over a 2-rank gloo group, and the reference arm's rule that only
rank 0 works (the other ranks exit 0 at once)."""
import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 10.0 * (rank + 1)             # rank r took 10*(r+1) ms
        out = bench.aggregate_over_ranks(ms, tokens_per_step=85, steps=4, world=world,
                                         dist=dist)
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


def test_aggregate_takes_max_over_ranks_gloo():
    world, port = 2, 29517
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        ms, value = res[r]
        assert ms == 20.0                         # the slowest rank's time
        assert value == pytest.approx(85 * 4 * world / 0.020)


def test_aggregate_single_rank():
    sys.path.insert(0, ROOT)
    import bench
    ms, value = bench.aggregate_over_ranks(5.0, 10, 2, 1)
    assert ms == 5.0 and value == pytest.approx(10 * 2 / 0.005)


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--gpus", "2"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_bench_mirrors_library_dispatch_constants():
    """bench.py counts the kernels a forward launches from the library's
    dispatch limits; its copies of those limits must match kernels.h."""
    import re
    sys.path.insert(0, ROOT)
    import bench
    src = open(os.path.join(ROOT, "mixture_experts_expert_route_b200", "csrc",
                            "kernels.h")).read()
    def const(name):
        return int(re.search(rf"constexpr\s+\w+\s+{name}\s*=\s*(\d+)", src).group(1))
    assert bench.SMALL_T == const("kSmallT")
    assert bench.CHUNK == const("kChunk")
    assert bench.SMALL_AMAX == const("kSmallAmaxElems")
    # decode T=1 (small path, bf16): route+permute, gate/up (gathers), down, combine
    assert bench.kernels_per_forward(1, 2, 8, False, 4096) == 4
    # FP8 T=1, x of 5.6 KB: amax and x codes in the route kernel, plus h quantisation
    assert bench.kernels_per_forward(1, 4, 32, True, 2880) == 5
    # FP8 T=2048: route, count, scan + scatter, amax, x codes, gather, 2 GEMMs,
    # quant, combine
    assert bench.kernels_per_forward(2048, 4, 32, True, 2880) == 10
    # prefill bf16 T=4096: route, count, scan + scatter, gather, 2 GEMMs, combine
    assert bench.kernels_per_forward(4096, 8, 128, False, 2048) == 7
    # token cap 64 (no gather kernel): route, count, scan + scatter, 2 GEMMs, combine
    assert bench.kernels_per_forward(1000, 3, 96, False, 128) == 6
    # with adapters: the gather kernel and two shrink GEMMs more
    assert bench.kernels_per_forward(4096, 8, 128, False, 2048, lora=True) == 9
    assert bench.kernels_per_forward(1, 2, 8, False, 4096, lora=True) == 7
    # the token-tile cap (pair tiles above 64): twice the mean per expert
    assert bench.gemm_token_cap(64, 2, 8) == 32
    assert bench.gemm_token_cap(40, 2, 2) == 96
    assert bench.gemm_token_cap(4096, 8, 128) == 256


def test_gemm_code_hash_ignores_comments_only():
    """The traffic provenance key follows the code: comments and blank lines do
    not change it, code does, and literals holding comment markers survive."""
    import bench
    src = 'int a = 1; // one\n/* block\n comment */ const char* s = "x // y /* z */";\n\nchar c = \'"\';\n'
    same = 'int a = 1;   \n const char* s = "x // y /* z */"; // trailing\nchar c = \'"\'; /* c */\n'
    assert bench.strip_comments(src) == bench.strip_comments(same)
    assert '"x // y /* z */"' in bench.strip_comments(src)
    assert bench.strip_comments(src) != bench.strip_comments(src.replace("a = 1", "a = 2"))
    assert len(bench.gemm_source_hash()) == 12
