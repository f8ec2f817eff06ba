"""Tensor-parallel head sharding on the GPU kernels: the two halves of the heads run one after
the other on one device (no inter-rank waiting; the sum of their partials stands in for the
all-reduce, which test_tp_gloo.py checks across processes). Each shard's recurrent state is
bit-identical to the unsharded block's state for those heads; the summed output matches the
unsharded block and the oracle, with the partials in FP32 and in BF16 (the default: the block
output is reduced in BF16)."""
import numpy as np
import pytest
import torch

import kda_gated_delta_gate_b200 as kda
import oracle
from kda_gated_delta_gate_b200.tp import TPBlock, shard_block_weights
from synth import block_hidden, block_weights
from tests.gpu_harness import np64, rel_l2
from tests.test_gpu_block import _device_weights

pytestmark = pytest.mark.gpu
TOL_BF16 = 2e-2


@pytest.fixture(autouse=True)
def _status(cuda_ok):
    kda.device_status(clear=True)
    yield
    assert kda.device_status(clear=True) == 0


def _to_device(W):
    import dataclasses
    return dataclasses.replace(W, **{f.name: getattr(W, f.name).cuda() for f in dataclasses.fields(W)
                                     if isinstance(getattr(W, f.name), torch.Tensor)})


@pytest.mark.parametrize("hidden,H,D,rank,T,world,rd", [(256, 4, 64, 64, 130, 2, "fp32"),
                                                        (4096, 32, 128, 128, 256, 2, "fp32"),
                                                        (4096, 32, 128, 128, 256, 2, "bf16")])
def test_tp_prefill_shards_sum_to_unsharded_block(hidden, H, D, rank, T, world, rd):
    Wt = block_weights(hidden, H, D, rank, seed=21, std=0.05 if hidden < 4096 else 0.02)
    h = block_hidden(T, hidden, seed=21).cuda()
    # unsharded block
    ws = kda.Workspace(kda.dims(H, D), hidden, rank, max_tokens=T)
    hs = torch.zeros((H, D, D), device="cuda")
    cs = torch.zeros((3 * H * D, 3), dtype=torch.bfloat16, device="cuda")
    dw = _device_weights(Wt)  # held: the struct keeps only raw pointers
    kda.kda_block_prefill(kda.block_weights_struct(dw), h, T, hs, cs, 0.0, ws)
    torch.cuda.synchronize()
    full = ws.view("final_out", (T, hidden), torch.bfloat16).clone()
    ws.close()
    # the shards, one after the other
    Wd = _to_device(Wt)
    total = torch.zeros((T, hidden), device="cuda")
    for r in range(world):
        sh = shard_block_weights(Wd, r, world)
        blk = TPBlock(sh, max_tokens=T, reduce_dtype=rd)
        hs_r = torch.zeros((sh.H, D, D), device="cuda")
        cs_r = torch.zeros((3 * sh.H * D, 3), dtype=torch.bfloat16, device="cuda")
        total += blk.prefill(h, T, hs_r, cs_r).float()
        torch.cuda.synchronize()
        h0 = r * sh.H
        assert torch.equal(hs_r, hs[h0:h0 + sh.H]), r
        blk.close()
    out = total.to(torch.bfloat16)
    assert rel_l2(np64(out), np64(full)) <= 1e-2
    ref = oracle.block_prefill(Wt, h.cpu(), np.zeros((H, D, D)), np.zeros((3 * H * D, 3)))
    assert rel_l2(np64(out), ref["final_out"]) <= TOL_BF16


def test_tp_decode_shards_sum_to_unsharded_block():
    hidden, H, D, rank, N, world = 256, 4, 64, 64, 3, 2
    Wt = block_weights(hidden, H, D, rank, seed=23, std=0.05)
    h = block_hidden(N, hidden, seed=23).cuda()
    g = torch.Generator().manual_seed(23)
    hs0 = torch.randn((N, H, D, D), generator=g) * 0.1
    cs0 = torch.randn((N, 3 * H * D, 3), generator=g).to(torch.bfloat16)
    ws = kda.Workspace(kda.dims(H, D), hidden, rank, max_tokens=8)
    hs = [hs0[n].cuda().clone() for n in range(N)]
    cs = [cs0[n].cuda().clone() for n in range(N)]
    dw = _device_weights(Wt)  # held: the struct keeps only raw pointers
    hp, cp = kda.ptr_array(hs), kda.ptr_array(cs)
    kda.kda_block_decode(kda.block_weights_struct(dw), h, N, hp, cp, ws)
    torch.cuda.synchronize()
    full = ws.view("final_out", (N, hidden), torch.bfloat16).clone()
    ws.close()
    Wd = _to_device(Wt)
    total = torch.zeros((N, hidden), device="cuda")
    qkv = H * D
    for r in range(world):
        sh = shard_block_weights(Wd, r, world)
        h0, c0, c1 = r * sh.H, r * sh.H * D, (r + 1) * sh.H * D
        blk = TPBlock(sh, max_tokens=8, reduce_dtype="fp32")
        hs_r = [hs0[n, h0:h0 + sh.H].cuda().contiguous() for n in range(N)]
        cs_r = [torch.cat([cs0[n, c0:c1], cs0[n, qkv + c0:qkv + c1], cs0[n, 2 * qkv + c0:2 * qkv + c1]]).cuda()
                for n in range(N)]
        hp_r, cp_r = kda.ptr_array(hs_r), kda.ptr_array(cs_r)
        total += blk.decode(h, N, hp_r, cp_r)
        torch.cuda.synchronize()
        for n in range(N):
            assert torch.equal(hs_r[n], hs[n][h0:h0 + sh.H]), (r, n)
        blk.close()
    assert rel_l2(np64(total.to(torch.bfloat16)), np64(full)) <= 1e-2
