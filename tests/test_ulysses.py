"""The head-sharded multi-GPU layout (int8_kv_cache_action_b200.ulysses) as two gloo ranks on CPU.

The per-rank attention here is the CPU oracle (test infrastructure) on the rank's heads: the test pins
the exchanges and the sharding, i.e. that sequence-sharded inputs, exchanged to head shards, attended
per head and exchanged back, give exactly the single-process result for every token and head (each
head's attention and INT8 cache are independent of the others)."""
import math
import os
import socket

import numpy as np
import pytest
import torch

WORLD = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _cfg():
    from int8_kv_cache_action_b200.workloads import small_config
    # 4 heads (2 per rank), 300 queries (150 per rank), ring of 4 frames, prior heads and text tails
    return small_config(heads=4, head_dim=64, tokens_per_frame=100, n_frames=3, window=4, prior_frames=(3, 2))


def _rank_main(rank, port, out_dir):
    import torch.distributed as dist
    from int8_kv_cache_action_b200 import ulysses as U
    from int8_kv_cache_action_b200.workloads import make_inputs
    from oracle import attention as att
    from oracle.ring import OracleCache
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    try:
        cfg = _cfg()
        inp = make_inputs(cfg)
        hg = cfg.heads // WORLD

        def shard(x):                      # this rank's token shard of a full [S, H, D] tensor
            n = x.shape[0] // WORLD
            return x[rank * n:(rank + 1) * n].float()

        # exchange layout: the head shard of every token, in global token order
        q_h = U.seq_to_heads(shard(inp.q))
        assert torch.equal(q_h, inp.q.float()[:, rank * hg:(rank + 1) * hg])
        assert torch.equal(U.heads_to_seq(q_h), shard(inp.q))
        # the path per rank: append the prior segments' exchanged K/V into a cache of the rank's heads,
        # then attention of the exchanged current segment on those heads, output exchanged back
        oc = OracleCache(hg, cfg.head_dim, cfg.tokens_per_frame, cfg.window_frames, cfg.capacity_frames,
                         cfg.head_store_tokens)
        for seg, kv in zip(cfg.prior, inp.prior):
            oc.append(U.seq_to_heads(shard(kv.k)).numpy(), U.seq_to_heads(shard(kv.v)).numpy(), seg.n_frames,
                      U.head_slice(kv.head_k.float(), rank, hg).numpy(), U.head_slice(kv.head_v.float(), rank, hg).numpy())
        out_h, _ = att.attention(oc, U.seq_to_heads(shard(inp.q)).numpy(), U.seq_to_heads(shard(inp.k_cur)).numpy(),
                                 U.seq_to_heads(shard(inp.v_cur)).numpy(),
                                 U.head_slice(inp.k_txt.float(), rank, hg).numpy(),
                                 U.head_slice(inp.v_txt.float(), rank, hg).numpy(), cfg.current,
                                 1.0 / math.sqrt(cfg.head_dim))
        out = U.heads_to_seq(torch.from_numpy(out_h))
        np.save(os.path.join(out_dir, f"out{rank}.npy"), out.numpy())
    finally:
        dist.destroy_process_group()


def test_head_sharded_attention_equals_single_process(tmp_path):
    import torch.multiprocessing as mp
    from int8_kv_cache_action_b200.workloads import make_inputs
    from oracle import attention as att
    from oracle.ring import OracleCache
    mp.start_processes(_rank_main, args=(_free_port(), str(tmp_path)), nprocs=WORLD, start_method="spawn")
    cfg = _cfg()
    inp = make_inputs(cfg)
    f = lambda t: t.float().numpy()
    oc = OracleCache(cfg.heads, cfg.head_dim, cfg.tokens_per_frame, cfg.window_frames, cfg.capacity_frames,
                     cfg.head_store_tokens)
    for seg, kv in zip(cfg.prior, inp.prior):
        oc.append(f(kv.k), f(kv.v), seg.n_frames, f(kv.head_k), f(kv.head_v))
    ref, _ = att.attention(oc, f(inp.q), f(inp.k_cur), f(inp.v_cur), f(inp.k_txt), f(inp.v_txt), cfg.current,
                           1.0 / math.sqrt(cfg.head_dim))
    got = np.concatenate([np.load(tmp_path / f"out{r}.npy") for r in range(WORLD)])
    assert got.shape == ref.shape
    assert np.array_equal(got, ref)


def _uneven_main(rank, port, out_dir):
    import torch.distributed as dist
    from int8_kv_cache_action_b200 import ulysses as U
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    try:
        errors = 0
        for fn, x in ((U.seq_to_heads, torch.zeros(4, 3, 8)), (U.heads_to_seq, torch.zeros(5, 2, 8))):
            try:
                fn(x)
            except ValueError:
                errors += 1
        np.save(os.path.join(out_dir, f"err{rank}.npy"), np.array([errors]))
    finally:
        dist.destroy_process_group()


def test_exchange_rejects_uneven_splits(tmp_path):
    # 3 heads or 5 tokens do not split over 2 ranks: refused on the host before any collective runs
    import torch.multiprocessing as mp
    mp.start_processes(_uneven_main, args=(_free_port(), str(tmp_path)), nprocs=WORLD, start_method="spawn")
    assert [int(np.load(tmp_path / f"err{r}.npy")[0]) for r in range(WORLD)] == [2, 2]
