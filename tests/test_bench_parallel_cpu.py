"""Host logic of ``bench.py --parallel`` on the CPU: two and three gloo ranks.

The --parallel modes split one matrix over the ranks (FC1 by rows, FC2 by
inputs, or the FC1 -> FC2 block) and exchange the partial results with a
collective.  Here the shapes are small, each rank's product is the FP64 oracle
on its own shard (standing in for the GPU library), and the step the bench
times must return the whole matrix's product on every rank.  The byte
accounting the bench reports is checked against the whole matrices.
"""
from __future__ import annotations

import json
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SMALL = {"fc1": (256, 512), "fc2": (128, 256)}


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, outdir):
    import datetime
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bcq_synth as S
    import bench
    from oracle import bcq_oracle as O
    from weight_only_quantized_bcq_b200 import sharded as T

    class OracleShard(T.ShardedLinear):
        """A shard whose product is the oracle (host tensors)."""

        def __init__(self, plan, signs, alpha):
            self.plan, self.group = plan, None
            self.m, self.n = plan.local_m, plan.local_n
            self.signs, self.alpha = signs, alpha

        def local_product(self, x_local):
            return torch.from_numpy(O.bcq_matmul(x_local.numpy(), self.signs.numpy(), self.alpha.numpy(),
                                                 self.plan.g)).float()

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        q, g, batch = 3, 64, 2
        gen = S.generator(11)
        whole = {}
        for name, (m, n) in SMALL.items():
            whole[name] = (S.draw_signs(gen, q, m, n), S.draw_alpha(gen, q, m, n, g, 0.02))
        x = S.draw_x(S.generator(77), batch, SMALL["fc1"][1])
        x2 = S.draw_x(S.generator(78), batch, SMALL["fc2"][1])
        res = {}
        for mode in ("rows", "inputs", "paired"):
            plans = bench.parallel_plans(mode, q, g, world, rank, shapes=SMALL)
            mats = {"rows": ["fc1"], "inputs": ["fc2"], "paired": ["fc1", "fc2"]}[mode]
            lins = [OracleShard(p, *T.take_shard(p, *whole[nm])) for p, nm in zip(plans, mats)]
            xin = x2 if mode == "inputs" else x
            xin = T.take_input_slice(plans[0], xin) if mode == "inputs" else xin
            y = bench.parallel_step(mode, lins, xin)
            s1, a1 = whole["fc1"]
            s2, a2 = whole["fc2"]
            if mode == "rows":
                ref = O.bcq_matmul(x.numpy(), s1.numpy(), a1.numpy(), g)
            elif mode == "inputs":
                ref = O.bcq_matmul(x2.numpy(), s2.numpy(), a2.numpy(), g)
            else:
                h = torch.from_numpy(O.bcq_matmul(x.numpy(), s1.numpy(), a1.numpy(), g)).float().to(torch.float16)
                ref = O.bcq_matmul(h.numpy(), s2.numpy(), a2.numpy(), g)
            ref = torch.from_numpy(ref)
            wb, mb = bench.parallel_bytes(plans, batch)
            res[mode] = {"err": float((y.double() - ref).abs().max() / ref.abs().max()),
                         "whole": wb, "mine": mb, "shape": list(y.shape)}
        with open(os.path.join(outdir, f"rank{rank}.json"), "w") as f:
            json.dump(res, f)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_parallel_steps_return_the_whole_product(tmp_path, world):
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    sys.path.insert(0, ROOT)
    from weight_only_quantized_bcq_b200.roofline import algorithmic_bytes
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    q, g, b = 3, 64, 2
    want_whole = {"rows": algorithmic_bytes(256, 512, q, g, b), "inputs": algorithmic_bytes(128, 256, q, g, b)}
    want_whole["paired"] = want_whole["rows"] + want_whole["inputs"]
    for mode in ("rows", "inputs", "paired"):
        for r in res:
            assert r[mode]["err"] < 1e-6, (mode, r[mode])          # fp32 exchange of FP64 partials
            assert r[mode]["whole"] == want_whole[mode]
            assert r[mode]["shape"] == [b, 256 if mode == "rows" else 128]
        # Each rank's shard is a part of the whole: the shards' weight bytes add up.
        assert sum(r[mode]["mine"] for r in res) >= want_whole[mode]
