"""Host-side logic on CPU: the seeded generator, the workload table, and the
multi-process (replica) plumbing of bench.py with gloo ranks (world size 2)."""
import json
import multiprocessing as mp
import os
import socket
import subprocess
import sys
import types

import numpy as np
import pytest

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_generator_is_seeded_and_counter_based():
    a = synth.normal_bf16((1000,), 7, 3)
    b = synth.normal_bf16((1000,), 7, 3)
    c = synth.normal_bf16((1000,), 8, 3)
    assert np.array_equal(a, b) and not np.array_equal(a, c)
    # any sub-range of a stream can be drawn on its own
    tail = synth.normal_bf16((400,), 7, 3, start=600)
    assert np.array_equal(tail, a[600:])
    x = synth.bf16_to_f32(synth.normal_bf16((200000,), 1, 1))
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1) < 0.01


def test_bf16_rounding_is_nearest_even():
    v = np.array([1.0, 1.00390625, 1.01171875, -2.5, 3.0e-3], dtype=np.float32)  # halfway cases at 1+2^-8
    bits = synth.f32_to_bf16(v)
    back = synth.bf16_to_f32(bits)
    assert back[0] == 1.0 and back[1] == 1.0 and back[2] == 1.015625 and back[3] == -2.5


def test_workload_table():
    s = synth.SHAPES
    assert (s[0].H, s[0].d, s[0].Lq, s[0].P_tok, s[0].NP, s[0].Kp, s[0].r) == (2, 64, 256, 256, 8, 2, 64)
    assert (s[1].H, s[1].Lq, s[1].P_tok, s[1].Lc, s[1].L, s[1].r) == (12, 4680, 12480, 49920, 54600, 256)
    assert (s[2].H, s[2].Lq, s[2].Lc) == (40, 4680, 49920)
    assert (s[3].H, s[3].Lq, s[3].P_tok, s[3].Lc, s[3].r, s[3].NP) == (40, 10800, 28800, 115200, 512, 12)
    assert s[4].host_pages and s[4].NP == 48 and s[4].n_segments == 9
    for sh in s:
        assert sh.L % 8 == 0 and sh.r % 64 == 0
    assert synth.segment_bounds(48, 9).tolist() == [0, 5, 10, 16, 21, 26, 32, 37, 42, 48]
    t = synth.tau_schedule(12)
    assert t[0] == 1.0 and abs(t[-1] - 0.35) < 1e-7 and np.all(np.diff(t) < 0)


def test_biased_pages_and_segment_choice():
    x = synth.make_inputs(synth.SHAPES[4].replace(F_tok=32, page_tok=0), 1004)
    lo, hi = x.seg_begin[x.s_star], x.seg_begin[x.s_star + 1]
    assert len(set(x.biased)) == 3 and all(lo <= c < hi for c in x.biased)
    cos = x.e_seg @ x.e_cur / (np.linalg.norm(x.e_seg, axis=1) * np.linalg.norm(x.e_cur))
    assert int(np.argmax(cos)) == x.s_star


def _rank_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank), HSA_BENCH_BACKEND="gloo")
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    r, w, _ = bench.dist_setup(world)
    m = bench.max_over_ranks(10.0 * (r + 1), w)
    bench.barrier(w)
    q.put((r, w, m))
    dist.destroy_process_group()


def test_replica_timing_is_max_over_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_rank_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert out == [(0, 2, 20.0), (1, 2, 20.0)]


def test_reference_arm_two_ranks_prints_one_line():
    """torchrun with 2 gloo ranks: rank 0 alone runs the oracle arm and prints one JSON line."""
    port = free_port()
    env = dict(os.environ, HSA_BENCH_BACKEND="gloo", OMP_NUM_THREADS="2")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--workload", "0", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    res = json.loads(lines[0])
    assert res["impl"] == "reference" and res["unit"] == "query-tokens/s" and res["value"] > 0
    assert res["cpu_baseline"]["kind"] == "oracle" and res["e2e"]["h2d_bytes_per_step"] == 0


def _sharded_worker(rank, world, port, q):
    """A head-sharded retrieval over gloo: each rank's partial page scores are the
    oracle's scores of its heads; the plumbing sums them over the ranks and ranks."""
    import numpy as np
    import torch
    import torch.distributed as dist

    import oracle
    import synth
    from hybrid_sparse_attention_hkv_b200.sharded import head_range, sharded_retrieval
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    H, d, Lq, NP, Kp = 5, 16, 96, 12, 3
    kbar = synth.normal_f32((NP, H, d), 5, 1, sigma=0.5).astype(np.float64)
    Q = synth.normal_bf16((Lq, H, d), 5, 2, offset=synth.normal_f32((H, d), 5, 3))
    h0, h1 = head_range(H, rank, world)
    qbar = oracle.pooled_query(Q[:, h0:h1])

    def partial():
        return torch.from_numpy(oracle.page_scores(kbar[:, h0:h1], qbar).copy())

    def select(s):
        s = s.numpy()
        return sorted(sorted(range(NP), key=lambda p: (-s[p], p))[:Kp])

    sel = sharded_retrieval(partial, lambda t: dist.all_reduce(t, op=dist.ReduceOp.SUM), select)
    full, _ = oracle.select_pages(kbar, Q, Kp, dtype=np.float64)
    q.put((rank, (h0, h1), sel, full.tolist()))
    dist.destroy_process_group()


def test_head_sharded_retrieval_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_sharded_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, hr0, s0, full0), (r1, hr1, s1, full1) = out
    assert hr0 == (0, 3) and hr1 == (3, 5)  # 5 heads over 2 ranks
    assert s0 == s1 == full0 == full1  # every rank selects the unsharded pages


def test_head_ranges_cover_every_head_once():
    from hybrid_sparse_attention_hkv_b200.sharded import head_range
    for H in (1, 2, 5, 12, 40):
        for world in (1, 2, 3, 4, 8):
            if world > H:
                continue
            r = [head_range(H, k, world) for k in range(world)]
            assert r[0][0] == 0 and r[-1][1] == H
            assert all(a[1] == b[0] for a, b in zip(r, r[1:]))
            assert max(b - a for a, b in r) - min(b - a for a, b in r) <= 1


def test_kernel_count_of_a_step():
    """The bench's launch count: the traced calls of one step and the kernels each
    launches add up to the per-step launches of the ncu launch list (14B 720p: 12
    kernels a step, the block selection's scores kernel twice)."""
    sys.path.insert(0, ROOT)
    import bench
    c3 = synth.SHAPES[3]
    step = ["page_scores_partial", "select_pages_final", "kc128_from_pages", "gather", "pool", "block_select",
            "linformer_proj", "linformer_reduce", "attn_plan", "attention_merge"]
    assert bench.kernels_in_scope("block_select", c3) == 3
    assert sum(bench.kernels_in_scope(n, c3) for n in step) == 12
    assert bench.kernels_in_scope("block_select", c3, joint=True) == 2
    no_history = types.SimpleNamespace(Lc=0)  # no cached KV: the intra map alone
    assert bench.kernels_in_scope("block_select", no_history) == 2
    assert bench.kernels_in_scope("store_fetch", synth.SHAPES[4]) == 2


def test_bench_pair_count_and_kept_fractions():
    """The FLOP count behind the attention roofline: selected query-key pairs from
    the selection lists, partial query and key blocks at their real sizes.  A
    hand-worked selection (H = 2, Lq = 200, Lc = 300: query blocks of 128 + 72 and
    4 x 64 - 56, cached blocks 128 + 128 + 44) gives 103072 pairs, and a token-level
    mask built from the same lists counts the same."""
    import torch
    sys.path.insert(0, ROOT)
    import bench
    H, Lq, Lc = 2, 200, 300
    shape = types.SimpleNamespace(H=H, Lq=Lq, Lc=Lc)
    inter = [[[0, 2], [1]], [[0, 1, 2], [2]]]            # [h][128-row query block] -> cached blocks
    intra = [[[0], [3], [0, 1, 2, 3], [2]], [[0], [1], [2], [3]]]  # [h][64-row query block] -> chunk blocks

    def buffers(lists, n_blocks):
        idx = torch.full((H, len(lists[0]), n_blocks), -1, dtype=torch.int32)
        cnt = torch.zeros(H, len(lists[0]), dtype=torch.int32)
        for h, rows in enumerate(lists):
            for i, kept in enumerate(rows):
                idx[h, i, :len(kept)] = torch.tensor(kept, dtype=torch.int32)
                cnt[h, i] = len(kept)
        return idx, cnt

    ii, ic = buffers(inter, 3)
    qi, qc = buffers(intra, 4)
    sel = types.SimpleNamespace(inter_idx=ii, inter_cnt=ic, intra_idx=qi, intra_cnt=qc)
    pairs, f_inter, f_intra = bench.exact_pairs(shape, sel)
    assert pairs == 103072
    mask = np.zeros((H, Lq, Lc + Lq), dtype=bool)
    for h in range(H):
        for t in range(Lq):
            for j in inter[h][t // 128]:
                mask[h, t, 128 * j:min(Lc, 128 * j + 128)] = True
            for j in intra[h][t // 64]:
                mask[h, t, Lc + 64 * j:Lc + min(Lq, 64 * j + 64)] = True
    assert int(mask.sum()) == pairs
    assert f_inter == 7 / 12 and f_intra == 11 / 32
    per_inter, per_intra = bench.kept_fraction_per_head(shape, sel)
    assert per_inter == [0.5, 0.6667] and per_intra == [0.4375, 0.25]


def test_bench_work_model_closed_forms():
    """The algorithmic work the bench divides by: Linformer FLOPs
    H (4 r L d + 4 Lq r d) (93.2 GFLOP at the 1.3B 480p workload) and gather bytes
    4 Lc H d x 2 (613 MB at 1.3B 480p, 2.04 GB at 14B 480p, 4.72 GB at 14B 720p)."""
    sys.path.insert(0, ROOT)
    import bench
    c1, c2, c3 = synth.SHAPES[1], synth.SHAPES[2], synth.SHAPES[3]
    w1 = bench.step_work(c1)
    assert abs(w1["proj_flops"] + w1["lin_attn_flops"] - 93.2e9) < 0.05e9
    assert w1["proj_flops"] == w1["proj_hist_flops"] + w1["proj_chunk_flops"]
    assert round(w1["gather_bytes"] / 1e6) == 613
    assert round(bench.step_work(c2)["gather_bytes"] / 1e7) == 204
    assert round(bench.step_work(c3)["gather_bytes"] / 1e7) == 472
