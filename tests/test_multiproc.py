"""N > 1 host paths on the CPU: world size 2 over gloo.

The benchmark runs one independent replica per GPU (the decode path has no
exchange step); what the ranks share is the barrier and the max-over-ranks
timing. Both, and the reference arm's rank-0-only output under torchrun, are
checked here without a GPU."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    import bench
    got = bench.max_over_ranks(10.0 + 5.0 * rank, dist, "cpu")
    dist.barrier()
    q.put((rank, got))
    dist.destroy_process_group()


def test_max_over_ranks_gloo_world_2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res == {0: 15.0, 1: 15.0}


def test_max_over_ranks_without_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, None, "cpu") == 3.5


def test_reference_arm_under_torchrun_prints_once():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--workload", "tiny", "--gpus", "2", "--steps", "1", "--warmup", "0"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"


def _shard_worker(rank, world, port, q):
    """Rank-local oracle decode and rectify of this rank's KV heads; the
    outputs are gathered on every rank and compared with one process."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    import numpy as np

    import oracle as orc
    from block_sparse_attention_quest_b200.sharding import kv_head_range, q_head_range
    from workload import Spec, decode_inputs, make_cache, rectify_inputs
    spec = Spec(batch=2, n_q_heads=12, n_kv_heads=3, head_dim=64, len0=700, steps=2,
                dtype="bf16", r=0.1, n_min=4, f=16)
    K, V = make_cache(spec)
    h0, h1 = kv_head_range(spec.n_kv_heads, rank, world)
    a0, a1 = q_head_range(spec.n_q_heads, spec.n_kv_heads, rank, world)
    st = orc.State(K[:, h0:h1], V[:, h0:h1], spec.len0, spec.group)
    outs = []
    for step in range(spec.steps):
        qq, kn, vn = decode_inputs(spec, step)
        res = st.decode(qq[:, a0:a1], kn[:, h0:h1], vn[:, h0:h1], spec.r, spec.n_min, 1.0)
        outs.append(res["out"])
    q_f, k_f, v_f = rectify_inputs(spec, 0, st.length, spec.f)
    outs.append(st.rectify(q_f[:, :, a0:a1], k_f[:, :, h0:h1], v_f[:, :, h0:h1], spec.f, 1.0))
    local = torch.from_numpy(np.concatenate([o.reshape(-1) for o in outs]))
    sizes = [torch.zeros(1, dtype=torch.int64) for _ in range(world)]
    dist.all_gather(sizes, torch.tensor([local.numel()]))
    # gloo gathers equal sizes: pad to the largest share, trim afterwards
    big = max(int(s.item()) for s in sizes)
    parts = [torch.zeros(big, dtype=local.dtype) for _ in sizes]
    dist.all_gather(parts, torch.cat([local, torch.zeros(big - local.numel(), dtype=local.dtype)]))
    parts = [p[:int(s.item())] for p, s in zip(parts, sizes)]
    ranges = [torch.zeros(2, dtype=torch.int64) for _ in range(world)]
    dist.all_gather(ranges, torch.tensor([h0, h1]))
    q.put((rank, [tuple(r.tolist()) for r in ranges], [p.numpy() for p in parts]
           if rank == 0 else None))
    dist.destroy_process_group()


def test_kv_head_shards_partition_and_match_one_process():
    import numpy as np

    sys.path.insert(0, ROOT)
    import oracle as orc
    from block_sparse_attention_quest_b200.sharding import kv_head_range
    from workload import Spec, decode_inputs, make_cache, rectify_inputs
    # ranges: contiguous, disjoint, covering, balanced
    for H in (1, 3, 8):
        for world in range(1, H + 1):
            rs = [kv_head_range(H, r, world) for r in range(world)]
            assert rs[0][0] == 0 and rs[-1][1] == H
            assert all(a[1] == b[0] for a, b in zip(rs, rs[1:]))
            sizes = [b - a for a, b in rs]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1
    with pytest.raises(ValueError):
        kv_head_range(2, 0, 3)

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    world = 2
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict((r, (rng, parts)) for r, rng, parts in (q.get(timeout=120) for _ in procs))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    ranges, parts = got[0]
    assert ranges == [(0, 2), (2, 3)]
    # one process over every head
    spec = Spec(batch=2, n_q_heads=12, n_kv_heads=3, head_dim=64, len0=700, steps=2,
                dtype="bf16", r=0.1, n_min=4, f=16)
    K, V = make_cache(spec)
    st = orc.State(K, V, spec.len0, spec.group)
    full = []
    for step in range(spec.steps):
        qq, kn, vn = decode_inputs(spec, step)
        full.append(st.decode(qq, kn, vn, spec.r, spec.n_min, 1.0)["out"])
    q_f, k_f, v_f = rectify_inputs(spec, 0, st.length, spec.f)
    full.append(st.rectify(q_f, k_f, v_f, spec.f, 1.0))
    # reassemble: each rank's flat buffer holds its heads of every output in order
    G = spec.group
    for rank, (h0, h1) in enumerate(ranges):
        flat, off = parts[rank], 0
        for ref in full:
            shape = list(ref.shape)
            axis = 1 if ref.ndim == 3 else 2            # decode [B,Hq,d]; rectify [B,f,Hq,d]
            shape[axis] = (h1 - h0) * G
            n = int(np.prod(shape))
            mine = flat[off:off + n].reshape(shape)
            off += n
            sl = [slice(None)] * ref.ndim
            sl[axis] = slice(h0 * G, h1 * G)
            assert np.array_equal(mine, ref[tuple(sl)])
        assert off == flat.size
