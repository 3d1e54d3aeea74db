"""Expert parallelism on the GPU kernels (needs a B200): two or three ranks simulated in
one process on one GPU (each rank with its own packed buffers of its expert block and
its own workspaces), the all-to-all exchanges done in between by slicing device
tensors, which is what NCCL would move.  The combined output of every rank is checked
against the oracle at the parity tolerances (routing bit-exact)."""
import numpy as np
import pytest

import synth
from tests import harness as H

pytestmark = pytest.mark.gpu


def _exchange(sends, counts):
    """sends[r]: rank r's rows in destination order, counts[r][d]: rows r -> d.
    Returns what every rank receives, sources in rank order."""
    import torch
    world = len(sends)
    out = []
    for d in range(world):
        parts = []
        for r in range(world):
            o = int(np.sum(counts[r][:d]))
            parts.append(sends[r][o:o + int(counts[r][d])])
        out.append(torch.cat(parts))
    return out


@pytest.mark.parametrize("world,T,balanced", [(2, 4, False), (3, 12, True), (2, 96, True)])
def test_expert_parallel_ranks_on_one_gpu(world, T, balanced):
    import torch

    import bit_routed_expert_fp32_b200 as moe
    import oracle
    from bit_routed_expert_fp32_b200.ep import (ExpertParallelLayer, GpuBackend, pack_rank,
                                                partition_experts)
    cfg = synth.micro(T=T, H=256, E=16, k=4, I=128, S=1, formats="mixed", zipf=1.1, seed=90 + T)
    layer = synth.Layer(cfg, 0)
    pop = None
    if balanced:
        Lc = oracle.logits(synth.calibration_tokens(cfg, 256), layer.router_w)
        pop = np.bincount(oracle.select(Lc, layer.router_b, cfg.k)[0].ravel(), minlength=cfg.E)
    owner = partition_experts(cfg.E, world, pop)
    ranks, cases = [], []
    for r in range(world):
        local, shared, e_local = pack_rank(cfg, layer.fmt, layer.expert, owner, r)
        be = GpuBackend(cfg, layer.router_w, layer.router_b, local, e_local, shared, T, max_rows=world * T * cfg.k)
        ranks.append(ExpertParallelLayer(cfg.E, cfg.k, r, world, owner, be, comm=None))
        cases.append(H.make_case(cfg, step=700 + 10 * r))
    xs = [moe.bf16_to_device(c.x) for c in cases]
    # 1. dispatch on every rank
    disp = [ep.dispatch(x) for ep, x in zip(ranks, xs)]
    counts = [d[2] for d in disp]
    recv_rows = _exchange([d[0] for d in disp], counts)
    recv_ids = _exchange([d[1] for d in disp], counts)
    # 3. local experts
    outs = [ep.compute(rr, ri) for ep, rr, ri in zip(ranks, recv_rows, recv_ids)]
    # 4. back to the sources: rank d returns, per source r, the rows it received from r
    recv_counts = [[counts[r][d] for r in range(world)] for d in range(world)]
    back = _exchange(outs, recv_counts)
    for r in range(world):
        y = ranks[r].combine(back[r])
        torch.cuda.synchronize()
        for st, det in ranks[r].backend.errors():
            assert st == 0, (moe.STATUS[st], hex(det))
        # routing of this rank's tokens is the oracle's
        rt = ranks[r].backend.rt
        np.testing.assert_array_equal(rt["topk_ids"][:T].cpu().numpy(), cases[r].ids)
        np.testing.assert_array_equal(rt["perm"][:T * cfg.k].cpu().numpy(), cases[r].perm)
        H.check_outputs(moe.bf16_to_host(y), H.oracle_outputs(cases[r], list(range(T))))
