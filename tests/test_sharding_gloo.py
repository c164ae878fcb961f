"""Multi-rank path on the CPU: two gloo ranks each run the recurrence (the fp64
oracle stands in for the GPU kernel here) on the sequences the sharding helper
assigns them; gathering the shards reproduces a single full run exactly, with
no exchange between ranks before the final check."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from linear_recurrent_lm_wkv7_b200 import sharding


def test_assign_sequences_balances_and_covers():
    lengths = [7231, 3968, 5229, 5520, 5868, 5253, 769, 895, 3887, 1619, 2620, 2046, 1786, 4109, 6339, 945]
    for ws in (1, 2, 3, 4, 8):
        owned = sharding.assign_sequences(lengths, ws)
        flat = sorted(i for o in owned for i in o)
        assert flat == list(range(len(lengths)))
        loads = [sum(lengths[i] for i in o) for o in owned]
        assert max(loads) - min(loads) <= max(lengths)
    assert sharding.assign_sequences([5, 5, 5], 2) == sharding.assign_sequences([5, 5, 5], 2)


def test_dense_shard_partitions():
    for B in (1, 4, 7):
        for ws in (1, 2, 3, 4):
            got = [i for r in range(ws) for i in sharding.dense_shard(B, ws, r)]
            assert got == list(range(B))


def test_packed_shard_offsets():
    offs = [0, 5, 5, 12, 20]
    ranges, new = sharding.packed_shard(offs, [3, 1])
    assert ranges == [(12, 20), (5, 5)]
    assert new == [0, 8, 8]


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import oracle
    import wkv7_inputs as W

    inp = W.make_packed([40, 3, 70, 0, 25, 64], [2, 0, 5, 1, 0, 3], 2, io="bf16", wdt="f32", s0_std=0.1, seed=31)
    offs = inp.seq_offsets.tolist()
    lengths = [offs[i + 1] - offs[i] for i in range(len(offs) - 1)]
    owned = sharding.assign_sequences(lengths, world)[rank]
    ranges, new = sharding.packed_shard(offs, owned)
    t = {k: v.double().numpy() for k, v in inp.tensors().items()}
    take = lambda x: np.concatenate([x[s:e] for s, e in ranges], axis=0) if ranges else x[:0]
    s0 = inp.s0.double().numpy()[owned]
    y, sT = oracle.forward(*(take(t[n]) for n in ("r", "w_log", "k", "v", "a", "b")), s0,
                           seq_offsets=np.array(new, dtype=np.int32))
    np.save(os.path.join(out_dir, f"y{rank}.npy"), y)
    np.save(os.path.join(out_dir, f"s{rank}.npy"), sT)
    np.save(os.path.join(out_dir, f"owned{rank}.npy"), np.array(owned, dtype=np.int64))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_reproduce_full_run(tmp_path, oracle_mod):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    import wkv7_inputs as W

    inp = W.make_packed([40, 3, 70, 0, 25, 64], [2, 0, 5, 1, 0, 3], 2, io="bf16", wdt="f32", s0_std=0.1, seed=31)
    t = {k: v.double().numpy() for k, v in inp.tensors().items()}
    offs = inp.seq_offsets.numpy()
    y_full, s_full = oracle_mod.forward(*(t[n] for n in ("r", "w_log", "k", "v", "a", "b")),
                                        inp.s0.double().numpy(), seq_offsets=offs)
    seen = set()
    for rank in range(world):
        owned = np.load(tmp_path / f"owned{rank}.npy").tolist()
        y = np.load(tmp_path / f"y{rank}.npy")
        s = np.load(tmp_path / f"s{rank}.npy")
        pos = 0
        for j, i in enumerate(owned):
            n = offs[i + 1] - offs[i]
            np.testing.assert_array_equal(y[pos:pos + n], y_full[offs[i]:offs[i + 1]])
            np.testing.assert_array_equal(s[j], s_full[i])
            pos += n
            seen.add(i)
    assert seen == set(range(len(offs) - 1))


# ------------------------------------------------------------------ one sequence cut across ranks
def test_token_ranges_cover_in_chunk_steps():
    for T in (0, 1, 63, 64, 100, 16384, 16385):
        for n in (1, 2, 3, 4, 8):
            rg = sharding.token_ranges(T, n)
            assert len(rg) == n and rg[0][0] == 0 and rg[-1][1] == T
            assert all(rg[j][1] == rg[j + 1][0] for j in range(n - 1))
            assert all(t0 % 64 == 0 for t0, _ in rg[1:] if t0 < T)
            sizes = [(t1 - t0 + 63) // 64 for t0, t1 in rg]
            assert max(sizes) - min(sizes) <= 1


def test_start_states_fold_the_maps_in_order():
    rng = np.random.default_rng(3)
    maps = [(rng.standard_normal((4, 4)), rng.standard_normal((4, 4))) for _ in range(4)]
    s0 = rng.standard_normal((4, 4))
    apply = lambda S, M, Q: (S @ M if S is not None else 0.0) + Q
    st = sharding.start_states(maps + [None], s0, apply)
    assert len(st) == 5 and st[0] is s0
    S = s0
    for j, (M, Q) in enumerate(maps):
        S = S @ M + Q
        np.testing.assert_allclose(st[j + 1], S)
    assert sharding.start_states([None], None, apply) == [None]


def _seq_worker(rank, world, port, out_dir):
    """Rank j holds token range j of one batch; its map (the oracle stands in for
    wkv7_state_map), the all-gather of the maps over gloo, the scan, and the
    range's forward from its start state."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import oracle
    import wkv7_inputs as W

    inp = W.make_prefill(2, 300, 2, io="bf16", wdt="f32", s0_std=0.1, seed=33)
    t = {k: v.double().numpy() for k, v in inp.tensors().items()}
    t0, t1 = sharding.token_ranges(inp.T, world)[rank]
    part = {n: x[:, t0:t1] for n, x in t.items()}
    if rank < world - 1:
        M, Q = oracle.state_map(*(part[n] for n in ("w_log", "k", "v", "a", "b")))
    else:
        M = Q = np.zeros((inp.B, inp.H, 64, 64))
    stacks = sharding.gather_maps(torch.from_numpy(np.stack([M, Q])), None)
    maps = [(m[0].numpy(), m[1].numpy()) for m in stacks[:rank]] + [None]
    apply = lambda S, M_, Q_: (S @ M_ if S is not None else 0.0) + Q_
    S = sharding.start_states(maps, inp.s0.double().numpy(), apply)[-1]
    y, sT = oracle.forward(*(part[n] for n in ("r", "w_log", "k", "v", "a", "b")), S)
    np.save(os.path.join(out_dir, f"seq_y{rank}.npy"), y)
    np.save(os.path.join(out_dir, f"seq_s{rank}.npy"), sT)
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_split_one_sequence(tmp_path, oracle_mod, world):
    mp.start_processes(_seq_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    import wkv7_inputs as W

    inp = W.make_prefill(2, 300, 2, io="bf16", wdt="f32", s0_std=0.1, seed=33)
    t = {k: v.double().numpy() for k, v in inp.tensors().items()}
    y_full, s_full = oracle_mod.forward(*(t[n] for n in ("r", "w_log", "k", "v", "a", "b")), inp.s0.double().numpy())
    ys = [np.load(tmp_path / f"seq_y{j}.npy") for j in range(world)]
    np.testing.assert_allclose(np.concatenate(ys, axis=1), y_full, rtol=0, atol=1e-10)
    np.testing.assert_allclose(np.load(tmp_path / f"seq_s{world - 1}.npy"), s_full, rtol=0, atol=1e-10)
