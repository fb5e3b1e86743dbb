"""Data-parallel host logic at world size 2 over gloo (CPU, no GPU): splitting
the tokens across ranks and all-reducing the adapter gradients reproduces the
full-batch dA and dB of the oracle."""
import os
import socket

import numpy as np
import torch
import torch.multiprocessing as mp

from bit_nf4_quantized_24_b200 import dp
from bit_nf4_quantized_24_b200 import workloads as wl


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_dir):
    import oracle
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        p = wl.draw_small(5, 37, 48, 128, 8, 16.0)
        codes, aq, dq, _ = oracle.nf4_quantize(p["W"].numpy())
        _, Wp = oracle.nf4_dequantize(codes, aq, dq, p["N"], p["K"])
        a, b = dp.token_shard(p["M"], rank, world)
        bits = wl.bf16_bits
        _, dA, dB, _ = oracle.linear_bwd(bits(p["X"][a:b]), bits(p["dY"][a:b]), Wp, bits(p["A"]), bits(p["B"]),
                                         p["scale"], want_dx=False)
        tA, tB = torch.from_numpy(dA), torch.from_numpy(dB)
        dp.allreduce_adapter_grads(tA, tB)
        np.save(os.path.join(out_dir, f"dA{rank}.npy"), tA.numpy())
        np.save(os.path.join(out_dir, f"dB{rank}.npy"), tB.numpy())
    finally:
        dist.destroy_process_group()


def test_token_shard_covers_everything():
    for M in (0, 1, 7, 4096):
        for world in (1, 2, 3, 8):
            spans = [dp.token_shard(M, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == M
            assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
            assert max(e - s for s, e in spans) - min(e - s for s, e in spans) <= 1


def test_allreduce_of_sharded_adapter_grads_equals_full_batch(tmp_path, oracle):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    p = wl.draw_small(5, 37, 48, 128, 8, 16.0)
    codes, aq, dq, _ = oracle.nf4_quantize(p["W"].numpy())
    _, Wp = oracle.nf4_dequantize(codes, aq, dq, p["N"], p["K"])
    bits = wl.bf16_bits
    _, dA, dB, _ = oracle.linear_bwd(bits(p["X"]), bits(p["dY"]), Wp, bits(p["A"]), bits(p["B"]), p["scale"],
                                     want_dx=False)
    for r in range(world):
        gA = np.load(tmp_path / f"dA{r}.npy")
        gB = np.load(tmp_path / f"dB{r}.npy")
        assert np.allclose(gA, dA, rtol=1e-12, atol=1e-12)
        assert np.allclose(gB, dB, rtol=1e-12, atol=1e-12)
