"""Tensor-parallel head sharding (Glm5NextLayer `mixer_all_reduce`) on CPU ranks: two gloo
processes each run the oracle block on their half of the heads (kda_gated_delta_gate_b200.tp
shards the weights), multiply by their o_proj slice, and all-reduce the partial outputs; the
FP64 sum equals the unsharded block's output, and the BF16 reduction (the default of TPBlock)
stays within its rounding bound of it. This covers the sharding and the collective on the
host (world sizes 2 and 4); the GPU kernels on the shards are tested in test_gpu_tp.py."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out_dir: str):
    import oracle
    from kda_gated_delta_gate_b200.tp import shard_block_weights
    from synth import block_hidden, block_weights
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        W = block_weights(hidden=64, H=4, D=16, rank=8, seed=9, std=0.2)
        h = block_hidden(11, 64, seed=9)
        sh = shard_block_weights(W, rank, world)
        h0 = rank * (W.H // world)
        r = np.random.default_rng(9)
        hs_full = r.standard_normal((W.H, 16, 16)) * 0.1
        cs_full = oracle.bf16_round(r.standard_normal((3 * W.H * 16, 3)))
        qkv, c0, c1 = W.H * 16, h0 * 16, (h0 + sh.H) * 16
        cs = np.concatenate([cs_full[c0:c1], cs_full[qkv + c0:qkv + c1], cs_full[2 * qkv + c0:2 * qkv + c1]])
        mine = oracle.block_prefill(sh, h, hs_full[h0:h0 + sh.H], cs)
        part = torch.from_numpy(oracle.linear(mine["o_norm_out"], sh.o_proj))
        dist.all_reduce(part, op=dist.ReduceOp.SUM)
        # every rank's heads and conv channels, gathered for the check on rank 0
        st = torch.from_numpy(mine["h_state"]).contiguous()
        states = [torch.empty_like(st) for _ in range(world)]
        dist.all_gather(states, st)
        if rank == 0:
            full = oracle.block_prefill(W, h, hs_full, cs_full)
            ref = oracle.linear(full["o_norm_out"], W.o_proj)
            np.testing.assert_allclose(part.numpy(), ref, rtol=1e-12, atol=1e-12)
            got = oracle.bf16_round(part.numpy())
            assert np.all(np.abs(got - full["final_out"]) <= 2.0 ** -8 * np.abs(full["final_out"]) + 1e-30)
            np.testing.assert_allclose(torch.cat(states).numpy(), full["h_state"], rtol=1e-12, atol=1e-14)
        # the default reduction of the block output in BF16: each rank's partial rounded to BF16,
        # summed by the collective in BF16; within a few BF16 steps of the unsharded output
        p64 = torch.from_numpy(oracle.linear(mine["o_norm_out"], sh.o_proj))
        part16 = p64.to(torch.bfloat16)
        mag = p64.abs()  # sum over ranks of |partial|: each BF16 rounding is relative to its operands
        dist.all_reduce(part16, op=dist.ReduceOp.SUM)
        dist.all_reduce(mag, op=dist.ReduceOp.SUM)
        if rank == 0:
            full = oracle.block_prefill(W, h, hs_full, cs_full)
            ref = oracle.linear(full["o_norm_out"], W.o_proj)
            got16 = part16.double().numpy()
            # one rounding of each partial and one per addition, each at most half a BF16 step
            bound = world * 2.0 ** -8 * (mag.numpy() + np.abs(ref)) + 1e-30
            assert np.all(np.abs(got16 - ref) <= bound)
            open(os.path.join(out_dir, "ok"), "w").write("ok")
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_head_sharded_block_all_reduce_matches_unsharded(tmp_path, world):
    """world = 4 leaves one head per rank."""
    port = _free_port()
    mp.spawn(_rank_main, args=(world, port, str(tmp_path)), nprocs=world, join=True)
    assert (tmp_path / "ok").exists()


def test_shard_rejects_uneven_split():
    from kda_gated_delta_gate_b200.tp import head_range
    with pytest.raises(ValueError):
        head_range(6, 0, 4)
    assert head_range(8, 3, 4) == (6, 8)
