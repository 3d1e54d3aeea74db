"""Expert parallelism: the routed experts of one layer split over several GPUs.

The pages run their engine on more than one consumer GPU (molayo1419.me, "Delta
Inference Engine", the multi-GPU paragraph); on B200 a whole layer fits one GPU, so
this is for layers (or models) larger than one GPU's HBM, or for spreading one layer's
expert bytes over several GPUs' HBM bandwidth.  Every rank holds the router, the shared
expert and its own block of routed experts.  One step on rank r with its tokens x_r:

  1. route x_r with the full router (moe_route): ids, gates, and the rows of x_r in
     expert-major order (perm); experts are owned in contiguous id blocks, so that
     order is also destination-rank order;
  2. gather the rows (moe_gather_rows) and send each rank its rows, with the local id of
     each row's expert (all-to-all; the split sizes come from the per-expert counts);
  3. every rank runs its own experts on the rows it received, each row with one expert
     and gate 1 (moe_route_fixed + moe_forward on the local packed buffer);
  4. the output rows go back to their sources (all-to-all, the reverse splits), in the
     order they were sent;
  5. the source adds the shared expert (run locally) and combines: y[t] = sum_j g[t][j]
     row[inv_perm[t k + j]] + y_shared[t] (moe_combine_pairs).

The exchanges are torch.distributed all_to_all_single calls (NCCL on GPUs; the CUDA
kernels never read another GPU's memory, and nothing uses cluster multicast).  The
steps are also available one by one (dispatch, compute, combine), so that a test can
drive several ranks in one process with the exchange done in between.

The arithmetic of every step runs in the library's kernels through `GpuBackend`;
another backend (same five methods) can stand in for it, which is how the partition
and the exchanges are tested on CPU ranks.
"""
from __future__ import annotations

import numpy as np


def partition_experts(E: int, world: int, popularity=None) -> np.ndarray:
    """Owner rank of each expert: contiguous id blocks.  Without popularity the blocks
    are as equal in size as possible; with it (expected tokens per expert, e.g. counts
    measured on a calibration batch) the block boundaries are placed where the running
    sum of popularity crosses r/world of the total, so that every rank gets about the
    same number of rows; every rank keeps at least one expert."""
    if world < 1 or E < world:
        raise ValueError("need 1 <= world <= E")
    if popularity is None:
        return (np.arange(E) * world // E).astype(np.int32)
    pop = np.asarray(popularity, dtype=np.float64)
    if pop.shape != (E,) or np.any(pop < 0):
        raise ValueError("popularity must be E non-negative values")
    cum = np.cumsum(pop + 1e-9)
    owner = np.minimum((cum / cum[-1] * world - 1e-12).astype(np.int64), world - 1)
    # every rank at least one expert: fix up ends of blocks that came out empty
    bounds = [0]
    for r in range(1, world):
        b = int(np.searchsorted(owner, r, side="left"))
        b = max(b, bounds[-1] + 1)
        b = min(b, E - (world - r))
        bounds.append(b)
    bounds.append(E)
    out = np.empty(E, dtype=np.int32)
    for r in range(world):
        out[bounds[r]:bounds[r + 1]] = r
    return out


def block_starts(owner: np.ndarray, world: int) -> np.ndarray:
    """First expert id of every rank's block (owner must be contiguous and ascending)."""
    if np.any(np.diff(owner) < 0) or owner[0] != 0 or owner[-1] != world - 1:
        raise ValueError("owner must assign contiguous ascending id blocks")
    return np.searchsorted(owner, np.arange(world), side="left").astype(np.int64)


class ExpertParallelLayer:
    """One rank of an expert-parallel routed-MoE layer.

    backend: route(x) -> (ids [T][k], gates [T][k], perm, inv_perm, counts [E] (host));
             gather(x, perm, k) -> rows in perm order;
             experts(rows, local_ids) -> the local experts' outputs, one row per row;
             shared(x) -> the shared expert's output rows (or None);
             combine(T, k, rows_back, inv_perm, gates, shared) -> y;
             and the tensor helpers new_int(n), new_rows(n), to_host(t), to_dev(a).
    comm:    all_to_all(out, inp, out_splits, in_splits) (torch.distributed by default)."""

    def __init__(self, E, k, rank, world, owner, backend, comm=None):
        self.E, self.k, self.rank, self.world = E, k, rank, world
        self.owner = np.asarray(owner, dtype=np.int32)
        self.starts = block_starts(self.owner, world)
        self.backend = backend
        self.comm = comm if comm is not None else TorchComm()
        self._st = None

    # ---- step 1: route, gather, split sizes ------------------------------------------
    def dispatch(self, x):
        """Returns (rows to send, their local expert ids, rows per destination rank)."""
        b = self.backend
        T = int(x.shape[0])
        ids, gates, perm, inv_perm, counts = b.route(x)
        counts = np.asarray(counts, dtype=np.int64)
        send_counts = np.bincount(self.owner, weights=counts, minlength=self.world).astype(np.int64)
        rows = b.gather(x, perm, self.k)
        expert_of_row = np.repeat(np.arange(self.E, dtype=np.int64), counts)
        local = (expert_of_row - self.starts[self.owner[expert_of_row]]).astype(np.int32)
        self._st = dict(T=T, gates=gates, inv_perm=inv_perm, send_counts=send_counts, x=x)
        return rows, b.to_dev(local), send_counts

    # ---- step 3: the local experts on the received rows ------------------------------
    def compute(self, recv_rows, recv_ids):
        return self.backend.experts(recv_rows, recv_ids)

    # ---- step 5: shared expert and combine --------------------------------------------
    def combine(self, back_rows):
        st, b = self._st, self.backend
        y_shared = b.shared(st["x"])
        return b.combine(st["T"], self.k, back_rows, st["inv_perm"], st["gates"], y_shared)

    # ---- the whole step over the process group ----------------------------------------
    def forward(self, x):
        rows, local_ids, send_counts = self.dispatch(x)
        b, c = self.backend, self.comm
        recv_counts = c.exchange_counts(send_counts)
        n_recv = int(recv_counts.sum())
        recv_rows = b.new_rows(n_recv)
        recv_ids = b.new_int(n_recv)
        c.all_to_all(recv_rows, rows, recv_counts, send_counts)
        c.all_to_all(recv_ids, local_ids, recv_counts, send_counts)
        out_rows = self.compute(recv_rows, recv_ids)
        back = b.new_rows(int(send_counts.sum()), f32=True)
        c.all_to_all(back, out_rows, send_counts, recv_counts)
        return self.combine(back)


class TorchComm:
    """The exchanges over torch.distributed (NCCL for CUDA tensors, gloo for CPU ones)."""

    def __init__(self, group=None):
        self.group = group

    def exchange_counts(self, send_counts: np.ndarray) -> np.ndarray:
        import torch
        import torch.distributed as dist
        dev = "cuda" if dist.get_backend(self.group) == "nccl" else "cpu"
        s = torch.as_tensor(send_counts, dtype=torch.int64, device=dev)
        r = torch.empty_like(s)
        dist.all_to_all_single(r, s, group=self.group)
        return r.cpu().numpy()

    def all_to_all(self, out, inp, out_splits, in_splits):
        import torch.distributed as dist
        dist.all_to_all_single(out, inp, [int(v) for v in out_splits], [int(v) for v in in_splits],
                               group=self.group)


class GpuBackend:
    """The library's kernels for one rank: the full router, this rank's experts and the
    shared expert, each with its own workspace.

    packed_local:  packed buffer (host) of this rank's experts as a layer of E_local
                   routed experts, top-1, no shared expert (moe_pack_experts);
    packed_shared: packed buffer of the shared expert as a one-expert layer, or None."""

    def __init__(self, cfg, router_w, router_b, packed_local, e_local, packed_shared, max_tokens,
                 max_rows=None, device="cuda"):
        import dataclasses

        import torch

        import bit_routed_expert_fp32_b200 as moe
        self.moe, self.torch, self.dev = moe, torch, device
        self.cfg = cfg
        self.H, self.k = cfg.H, cfg.k
        self.router_w = torch.from_numpy(np.ascontiguousarray(router_w, np.float32)).to(device)
        self.router_b = None if router_b is None else torch.from_numpy(
            np.ascontiguousarray(router_b, np.float32)).to(device)
        route_cfg = dataclasses.replace(cfg, S=0)
        self.route_cfg = route_cfg
        self.ws_route = torch.empty(moe.moe_workspace_size(route_cfg, max_tokens), dtype=torch.uint8, device=device)
        moe.moe_workspace_init(self.ws_route)
        self.rt = moe.alloc_routing(route_cfg, max_tokens, device)
        max_rows = max_rows or max_tokens * cfg.k
        self.local_cfg = dataclasses.replace(cfg, E=e_local, k=1, S=0)
        self.local = self._expert_set(self.local_cfg, packed_local, max_rows)
        self.shared_cfg = None if packed_shared is None else dataclasses.replace(cfg, E=1, k=1, S=0)
        self.shared_set = None if packed_shared is None else self._expert_set(self.shared_cfg, packed_shared,
                                                                              max_tokens)

    def _expert_set(self, cfg, packed, max_rows):
        torch, moe = self.torch, self.moe
        ws = torch.empty(moe.moe_workspace_size(cfg, max_rows), dtype=torch.uint8, device=self.dev)
        moe.moe_workspace_init(ws)
        return dict(cfg=cfg, packed=torch.from_numpy(packed).to(self.dev), ws=ws,
                    rt=moe.alloc_routing(cfg, max_rows, self.dev),
                    ones=torch.ones(max(max_rows, 1), dtype=torch.float32, device=self.dev),
                    zeros=torch.zeros(max(max_rows, 1), dtype=torch.int32, device=self.dev))

    # tensors: token rows travel as bf16, expert output rows come back as fp32 (the
    # combine then rounds once, as the single-GPU layer does)
    def new_rows(self, n, f32=False):
        return self.torch.empty((n, self.H), dtype=self.torch.float32 if f32 else self.torch.bfloat16,
                                device=self.dev)

    def new_int(self, n):
        return self.torch.empty(n, dtype=self.torch.int32, device=self.dev)

    def to_dev(self, a):
        return self.torch.from_numpy(np.ascontiguousarray(a)).to(self.dev)

    def to_host(self, t):
        return t.cpu().numpy()

    # steps
    def route(self, x):
        T = int(x.shape[0])
        self.moe.moe_route(self.route_cfg, T, x, self.router_w, self.router_b, self.rt, self.ws_route)
        counts = self.rt["counts"].cpu().numpy()          # the split sizes (one small copy)
        return (self.rt["topk_ids"][:T], self.rt["topk_w"][:T], self.rt["perm"][:T * self.k],
                self.rt["inv_perm"][:T * self.k], counts)

    def gather(self, x, perm, k):
        rows = self.new_rows(int(perm.numel()))
        if rows.shape[0]:
            self.moe.moe_gather_rows(x, perm, k, rows, self.ws_route)
        return rows

    def _run(self, S, x, ids):
        moe = self.moe
        n = int(x.shape[0])
        y = self.new_rows(n, f32=True)
        if n == 0:
            return y
        moe.moe_route_fixed(S["cfg"], n, x, ids, S["ones"], S["rt"], S["ws"])
        moe.moe_forward(S["cfg"], n, S["packed"], x, S["rt"], y, moe.PATH_AUTO | moe.OUT_F32, S["ws"])
        return y

    def experts(self, rows, local_ids):
        return self._run(self.local, rows, local_ids)

    def shared(self, x):
        if self.shared_set is None:
            return None
        return self._run(self.shared_set, x, self.shared_set["zeros"])

    def combine(self, T, k, rows_back, inv_perm, gates, y_shared):
        y = self.new_rows(T)
        self.moe.moe_combine_pairs(T, k, rows_back, inv_perm, gates, y_shared, y, self.ws_route)
        return y

    def errors(self):
        """(status, detail) of every workspace this backend used (synchronises)."""
        out = [self.moe.moe_get_error(self.ws_route), self.moe.moe_get_error(self.local["ws"])]
        if self.shared_set is not None:
            out.append(self.moe.moe_get_error(self.shared_set["ws"]))
        return out


def pack_rank(cfg, fmt, expert_fn, owner, rank):
    """Host packed buffers of one rank: (its routed experts as an E_local-expert top-1
    layer without shared expert, the shared expert as a one-expert layer or None,
    E_local)."""
    import dataclasses

    import bit_routed_expert_fp32_b200 as moe
    ids = np.nonzero(np.asarray(owner) == rank)[0]
    lcfg = dataclasses.replace(cfg, E=len(ids), k=1, S=0)
    lfmt = np.asarray(fmt, dtype=np.uint8)[ids]
    local = moe.pack_layer(lcfg, lfmt, lambda e: expert_fn(int(ids[e])))
    shared = None
    if cfg.S:
        scfg = dataclasses.replace(cfg, E=1, k=1, S=0)
        shared = moe.pack_layer(scfg, np.asarray(fmt, dtype=np.uint8)[cfg.E:cfg.E + 1], lambda e: expert_fn(cfg.E))
    return local, shared, len(ids)
