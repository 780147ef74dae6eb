"""Host-side logic of bench.py that needs no GPU: the multi-rank reduction (two gloo ranks on
the CPU) and the reference arm (the CPU oracle) with its JSON line."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # each rank: its own token count and device times
        out = bench.combine_ranks(torch, dist, tokens=100 + rank, dev_ms=2.0 + rank,
                                  e2e_ms=10.0 - rank, device=torch.device("cpu"))
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


def test_combine_ranks_sums_tokens_and_takes_max_time_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(2):
        assert results[r] == (201.0, 3.0, 10.0)


def test_combine_ranks_single_process():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.combine_ranks(torch, None, 7, 1.5, 2.5, torch.device("cpu")) == (7.0, 1.5, 2.5)


def test_reference_arm_prints_one_json_line():
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "2", "--warmup", "1"], capture_output=True, text=True,
                       timeout=600, cwd=ROOT)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["unit"] == "tokens/s" and j["value"] > 0
    assert j["cpu_baseline"]["kind"] == "oracle"
    assert 1 <= j["cpu_baseline"]["cores"] <= len(os.sched_getaffinity(0))
    assert j["e2e"]["h2d_bytes_per_step"] == 0 and j["higher_is_better"] is True
    assert j["steps"] == 2 and j["warmup"] >= 3


@pytest.mark.parametrize("n", [1, 3, 7])
def test_oracle_token_shares_write_what_the_whole_batch_writes(n):
    # the all-cores CPU baseline splits the batch into token ranges; run one after another
    # and on threads, the ranges must leave the cache and Q output exactly as one call does
    from concurrent.futures import ThreadPoolExecutor

    import numpy as np
    sys.path.insert(0, ROOT)
    import bench
    import workloads as W
    from oracle import runners as R
    w = W.ragged_store(31, lengths=[40, 3, 70], cache_lengths=[5, 60, 0], n_q_heads=4,
                       n_kv_heads=2, head_dim=64, page_size=16, rope_dim=64, theta=1e4,
                       interleaved=False, max_seq_len=256)
    want = R.oracle_ragged_store(w)
    assert want.err == 0
    for threaded in (False, True):
        calls, store, q_out = bench.oracle_token_shares(w, n)
        if threaded:
            with ThreadPoolExecutor(n) as ex:
                errs = list(ex.map(lambda f: f(), calls))
        else:
            errs = [f() for f in calls]
        assert errs == [0] * n
        assert np.array_equal(store, want.storage)
        assert np.array_equal(q_out, want.q_out)


def test_algorithmic_bytes_of_the_named_workloads():
    # the per-unit figures the roofline uses, as the design states them: bytes the method
    # must move per token (QKV read, Q written, K / V written; cache rows read where the op
    # reads them), plus the distinct freqs_cis rows for the rotating ops
    sys.path.insert(0, ROOT)
    import bench
    import workloads as W

    def per_token_without_freqs(w, total, freqs_rows_bytes):
        return (total - freqs_rows_bytes) / w.total_tokens

    w = W.llama3_8b_prefill()
    fr = len(set(bench.positions_ragged(w.lengths, [0] * 8))) * 128 * 4
    assert bench.bytes_ragged(w) == 10433 * 24576 + fr
    assert bench.bytes_ragged(w) == 257437184
    w8 = W.llama3_8b_prefill_fp8_cache()
    assert bench.bytes_ragged(w8) == 10433 * (6144 * 2 + 4096 * 2 + 2048 * 1) + fr
    n = W.per_head_norm()
    frn = len(set(bench.positions_ragged(n.lengths, n.cache.cache_lengths.tolist()))) * 128 * 4
    assert per_token_without_freqs(n, bench.bytes_ragged(n), frn) == 40960
    d = W.dual_band_minimax()
    frd = len(set(bench.positions_ragged(d.lengths,
                                         d.main_cache.cache_lengths.tolist()))) * 64 * 4
    assert per_token_without_freqs(d, bench.bytes_dual(d), frd) == 45568
    di = W.dual_band_minimax_in_place()
    assert per_token_without_freqs(di, bench.bytes_dual(di), frd) == 41472
    r = W.radd_minimax()
    assert bench.bytes_radd(r) == 32768 * 12288
    b = W.decode_bshd()
    frb = len(set(int(c) for c in b.cache.cache_lengths.tolist())) * 128 * 2
    assert bench.bytes_bshd(b) == 256 * (20736 - 256) + frb
    g = W.mla_kv_a_proj()
    assert bench.bytes_gemv(g) == (576 * 7168 + 7168 + 512 + 576) * 2


@pytest.mark.parametrize("n", [1, 4])
def test_oracle_token_shares_of_the_dual_band_write_what_the_whole_batch_writes(n):
    # the same for the two-band launch, whose bands keep caches and page sizes of their own
    from concurrent.futures import ThreadPoolExecutor

    import numpy as np
    sys.path.insert(0, ROOT)
    import bench
    import workloads as W
    from oracle import runners as R
    w = W.dual_band(33, lengths=[30, 1, 45], cache_lengths=[3, 70, 0], main_q_heads=4,
                    main_kv_heads=2, index_q_heads=2, index_kv_heads=1, head_dim=64,
                    main_page_size=16, index_page_size=8, rope_dim=32, theta=1e4,
                    interleaved=True, max_seq_len=256)
    want = R.oracle_dual(w)
    assert want.err == 0
    calls, (ms, ist), (qm, qi) = bench.oracle_token_shares(w, n)
    with ThreadPoolExecutor(n) as ex:
        assert list(ex.map(lambda f: f(), calls)) == [0] * n
    assert np.array_equal(ms, want.main_storage) and np.array_equal(ist, want.index_storage)
    assert np.array_equal(qm, want.q_main_out) and np.array_equal(qi, want.q_index_out)


def test_batch_prefix_takes_the_first_sequences_of_the_batch():
    sys.path.insert(0, ROOT)
    import bench
    full = bench.make_workload("dual_band_minimax", 0)
    w, k = bench.batch_prefix("dual_band_minimax", 5000)
    assert w.total_tokens == 5000 and w.lengths[:-1] == full.lengths[:k - 1]
    assert w.lengths[-1] <= full.lengths[k - 1]
    assert w.cache_lengths_of(w.main_cache) == full.cache_lengths_of(full.main_cache)[:k]


def test_source_hash_of_each_workload_covers_its_kernel_files():
    """A summary's hash covers the host code, the shared device headers and its kernel's
    files: workloads of one kernel share it, and editing one kernel's file leaves the other
    kernels' hashes as they were (checked on a copy of the sources)."""
    import shutil
    import tempfile
    import bench
    by_kernel = {}
    for w in bench.WORKLOADS:
        h = bench.kernel_source_hash(w)
        assert len(h) == 16 and int(h, 16) >= 0
        by_kernel.setdefault(bench.KERNEL_FILES[bench.WORKLOADS[w]], set()).add(h)
    assert all(len(v) == 1 for v in by_kernel.values())
    assert len({next(iter(v)) for v in by_kernel.values()}) == len(by_kernel)
    with tempfile.TemporaryDirectory() as d:
        shutil.copytree(os.path.join(bench.ROOT, "rope_paged_kv_b200", "csrc"),
                        os.path.join(d, "rope_paged_kv_b200", "csrc"))
        root = bench.ROOT
        try:
            bench.ROOT = d
            before = {w: bench.kernel_source_hash(w) for w in bench.WORKLOADS}
            with open(os.path.join(d, "rope_paged_kv_b200", "csrc", "gemv_norm.cuh"), "a") as f:
                f.write("\n")
            after = {w: bench.kernel_source_hash(w) for w in bench.WORKLOADS}
        finally:
            bench.ROOT = root
    changed = {w for w in before if before[w] != after[w]}
    assert changed == {w for w in bench.WORKLOADS
                       if bench.WORKLOADS[w] == "matmul_fused_partial_rmsnorm"}
