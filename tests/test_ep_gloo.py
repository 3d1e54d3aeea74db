"""Expert parallelism (bit_routed_expert_fp32_b200/ep.py) on CPU ranks over gloo.

The partition of the experts into contiguous blocks, the split sizes, the two
all-to-all exchanges and the bookkeeping that brings every expert output back to its
(token, slot) are the product's host logic; here they run on world_size 2 and 3 gloo
ranks with an oracle-backed stand-in for the kernels (fp64 rows, so the exchanged
result must equal the single-process oracle to rounding), and each rank's output is
compared with the oracle's layer output for its own tokens.
"""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from bit_routed_expert_fp32_b200.ep import ExpertParallelLayer, block_starts, partition_experts  # noqa: E402


class OracleBackend:
    """Stand-in for ep.GpuBackend on CPU: the oracle's routing and expert FFNs in fp64,
    rows as float64 torch tensors (bf16 values of the tokens)."""

    def __init__(self, layer, cfg, owner, rank):
        import oracle
        self.oracle, self.layer, self.cfg = oracle, layer, cfg
        self.owner = np.asarray(owner)
        self.start = block_starts(self.owner, int(self.owner.max()) + 1)[rank]
        self.rank = rank

    @staticmethod
    def _bits(rows):
        import synth
        return synth.f32_to_bf16_bits(rows.numpy().astype(np.float32))

    def new_rows(self, n, f32=False):
        import torch
        return torch.empty((n, self.cfg.H), dtype=torch.float64)

    def new_int(self, n):
        import torch
        return torch.empty(n, dtype=torch.int32)

    def to_dev(self, a):
        import torch
        return torch.from_numpy(np.ascontiguousarray(a))

    def route(self, x):
        o, c = self.oracle, self.cfg
        L = o.logits(self._bits(x), self.layer.router_w)
        ids, gates = o.select(L, self.layer.router_b, c.k)
        counts, offsets, perm, inv = o.permute(ids, c.E)
        return ids, gates, perm, inv, counts

    def gather(self, x, perm, k):
        import torch
        return x[torch.from_numpy(np.asarray(perm, dtype=np.int64) // k)].clone()

    def experts(self, rows, local_ids):
        import torch
        c = self.cfg
        out = torch.zeros_like(rows)
        ids = local_ids.numpy()
        for le in np.unique(ids):
            e = int(self.start + le)
            assert self.owner[e] == self.rank, "a row reached a rank that does not own its expert"
            sel = np.nonzero(ids == le)[0]
            y = self.oracle.expert_ffn(c.H, c.I, int(self.layer.fmt[e]), self.layer.expert(e),
                                       self._bits(rows[torch.from_numpy(sel)]))
            out[torch.from_numpy(sel)] = torch.from_numpy(y)
        return out

    def shared(self, x):
        import torch
        c = self.cfg
        if not c.S:
            return None
        return torch.from_numpy(self.oracle.expert_ffn(c.H, c.I, int(self.layer.fmt[c.E]), self.layer.expert(c.E),
                                                       self._bits(x)))

    def combine(self, T, k, rows_back, inv_perm, gates, y_shared):
        y = np.zeros((T, self.cfg.H))
        rb = rows_back.numpy()
        for t in range(T):
            for j in range(k):
                y[t] += gates[t][j] * rb[inv_perm[t * k + j]]
        if y_shared is not None:
            y += y_shared.numpy()
        return y


def _cfg():
    import synth
    return synth.micro(T=12, H=128, E=16, k=4, I=64, S=1, formats="mixed", zipf=1.1, seed=71)


def _rank_main(rank, world, port, popularity_balanced, out_dir):
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist

    import oracle
    import synth
    from datetime import timedelta
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        cfg = _cfg()
        layer = synth.Layer(cfg, 0)
        pop = None
        if popularity_balanced:
            Lc = oracle.logits(synth.calibration_tokens(cfg, 256), layer.router_w)
            ids_c, _ = oracle.select(Lc, layer.router_b, cfg.k)
            pop = np.bincount(ids_c.ravel(), minlength=cfg.E)
        owner = partition_experts(cfg.E, world, pop)
        xb = synth.tokens(cfg, 0, 500 + rank)                     # this rank's tokens
        x = torch.from_numpy(synth.bf16_bits_to_f32(xb).astype(np.float64))
        ep = ExpertParallelLayer(cfg.E, cfg.k, rank, world, owner, OracleBackend(layer, cfg, owner, rank))
        y = ep.forward(x)
        # the single-process oracle on the same tokens
        L = oracle.logits(xb, layer.router_w)
        ids, gates = oracle.select(L, layer.router_b, cfg.k)
        ref = oracle.forward_tokens(layer, xb, ids, gates, range(cfg.T))
        np.save(os.path.join(out_dir, f"y{rank}.npy"), np.asarray(y))
        np.save(os.path.join(out_dir, f"ref{rank}.npy"), ref)
        np.save(os.path.join(out_dir, f"owner{rank}.npy"), owner)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,balanced", [(2, False), (2, True), (3, True)])
def test_expert_parallel_matches_the_oracle_on_gloo_ranks(world, balanced, tmp_path):
    import torch.multiprocessing as mp
    port = 29600 + 10 * world + int(balanced)
    mp.spawn(_rank_main, args=(world, port, balanced, str(tmp_path)), nprocs=world, join=True)
    for r in range(world):
        y = np.load(tmp_path / f"y{r}.npy")
        ref = np.load(tmp_path / f"ref{r}.npy")
        np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    owners = [np.load(tmp_path / f"owner{r}.npy") for r in range(world)]
    assert all((o == owners[0]).all() for o in owners)


def test_partition_blocks():
    # equal blocks without popularity
    o = partition_experts(16, 3)
    assert list(np.bincount(o)) == [6, 5, 5] or list(np.bincount(o)) == [5, 5, 6] or sorted(np.bincount(o)) == [5, 5, 6]
    assert (np.diff(o) >= 0).all() and o[0] == 0 and o[-1] == 2
    # popularity: the hot experts get a rank of their own, every rank keeps one expert
    pop = np.array([100, 1, 1, 1, 1, 1, 1, 1], float)
    o = partition_experts(8, 2, pop)
    assert list(o) == [0, 1, 1, 1, 1, 1, 1, 1]
    o = partition_experts(4, 4, np.array([0, 0, 0, 10.0]))
    assert list(o) == [0, 1, 2, 3]
    # balanced loads: the max load over ranks is within one expert of the ideal
    rng = np.random.default_rng(0)
    pop = rng.zipf(1.5, size=256).astype(float)
    o = partition_experts(256, 8, pop)
    loads = np.bincount(o, weights=pop, minlength=8)
    assert loads.max() <= pop.sum() / 8 + pop.max()
    with pytest.raises(ValueError):
        partition_experts(4, 5)
