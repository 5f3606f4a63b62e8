"""Expert parallelism (EP) of the MoE layer over G GPUs, one process per GPU.

The pages' servers split the model over several GPUs: the official deployment uses tensor and
expert parallelism over eight GPUs (page "Beam 1.0 501B", the model-information page's
introduction: TP8/EP8) and the workstation recipe tensor parallelism over four (page "Running
Beam-1.0 (501B) on workstation GPUs", its serving command).  EP changes
where each expert runs, not what the layer computes: rank d holds global experts d*El ..
d*El+El-1 (El = E / G) and routes its own tokens over all E experts; every routed row travels
to its expert's owner, is run there, and its result travels back to be combined.

One step of rank ``rank`` (every rank takes the same collective steps in the same order):
  1. route its tokens (router kernel: ids, w, counts, offsets, perm, inv);
  2. all-gather the per-expert counts into C [G, E] and copy C to the host;
  3. plan: the rows it sends to / receives from every rank (``plan`` below, and the device
     plan kernel for the receive-side expert ids);
  4. move the rows to their owners -- ``transport="peer"``: the dispatch kernel stores each
     row straight into the owner's receive buffer over NVLink (CUDA IPC mappings), then a
     barrier; ``transport="collective"``: the gather kernel lines the rows up in expert order
     and one all-to-all (NCCL) delivers them;
  5. run the owner's experts on the rows it received (the experts-only entry point);
  6. bring the results back and combine -- ``peer``: a barrier, then the combine kernel reads
     every result from its owner's output buffer over NVLink; ``collective``: an all-to-all back,
     then the combine kernel.
The combine keeps the single-GPU layer's f32 accumulation order, so for the same expert
kernels the output equals the single-GPU layer's bit for bit.

The orchestration below is host logic only; every step on the data runs in the library's
kernels (or the collective library).  ``ops`` is the set of device steps; it defaults to the
CUDA library, and the only other implementation lives in the CPU tests of this host logic.
"""
from __future__ import annotations

import numpy as np

from . import _abi


def plan(counts_all, rank: int) -> dict:
    """Host plan of one EP step from C [G, E] (row s: rows rank s routes to each global expert).

    send[d]      rows this rank sends to rank d (its rows of d's experts, contiguous in its
                 expert-ordered perm);
    recv[s]      rows this rank receives from rank s;
    recv_total   sum of recv; recv_totals[d] the same for every rank d (capacity checks);
    dst_off_expert_major[g], dst_off_source_major[g]: where this rank's first row of global
                 expert g lands in its owner's receive buffer, for the two buffer layouts
                 (expert-major: for each local expert, the rows of rank 0, 1, ...; source-major:
                 the rows of rank 0 expert by expert, then rank 1, ... -- an all-to-all's order);
    recv_ids_expert_major, recv_ids_source_major: local expert id of every received row.
    """
    C = np.asarray(counts_all, dtype=np.int64)
    if C.ndim != 2:
        raise ValueError("counts_all must be [G, E]")
    G, E = C.shape
    if E % G:
        raise ValueError(f"{E} experts do not split evenly over {G} ranks")
    if not 0 <= rank < G:
        raise ValueError(f"rank {rank} outside 0 .. {G - 1}")
    El = E // G
    by_owner = C.reshape(G, G, El)                   # [source, owner, local expert]
    send = by_owner[rank].sum(axis=1)
    recv = by_owner[:, rank].sum(axis=1)
    recv_totals = by_owner.sum(axis=(0, 2))
    tot = C.sum(axis=0).reshape(G, El)               # [owner, local expert] over all sources
    em = np.zeros(E, dtype=np.int64)
    sm = np.zeros(E, dtype=np.int64)
    for g in range(E):
        d, e = divmod(g, El)
        em[g] = tot[d, :e].sum() + C[:rank, g].sum()
        sm[g] = by_owner[:rank, d].sum() + by_owner[rank, d, :e].sum()
    mine = by_owner[:, rank]                         # [source, local expert]
    ids_em = np.repeat(np.arange(El), mine.sum(axis=0))
    ids_sm = np.concatenate([np.repeat(np.arange(El), mine[s]) for s in range(G)]) if G else np.zeros(0, np.int64)
    return dict(G=G, E=E, El=El, send=send.tolist(), recv=recv.tolist(), recv_total=int(recv.sum()),
                recv_totals=recv_totals.tolist(), dst_off_expert_major=em, dst_off_source_major=sm,
                recv_ids_expert_major=ids_em.astype(np.int32), recv_ids_source_major=ids_sm.astype(np.int32))


def check_capacity(pl: dict, capacity: int) -> None:
    """Raises ValueError if the plan sends any rank more rows than its receive buffers hold.
    Every rank plans from the same gathered counts, so every rank raises together, before any
    row moves."""
    over = [d for d, n in enumerate(pl["recv_totals"]) if n > capacity]
    if over:
        raise ValueError(f"ranks {over} would receive {[pl['recv_totals'][d] for d in over]} rows; "
                         f"the receive buffers hold {capacity}")


def shard_bank(bank, rank: int, ranks: int):
    """The bank of rank's experts (records rank*El .. rank*El+El-1 of the full bank layout)."""
    from . import make_bank
    E = int(bank.num_experts)
    if E % ranks:
        raise ValueError(f"{E} experts do not split evenly over {ranks} ranks")
    El = E // ranks
    base = int(bank.base_dev or 0) + rank * El * int(bank.record_stride)
    return make_bank(base, El, bank.hidden, bank.intermediate, bank.record_stride, list(bank.codes_off),
                     list(bank.scales_off), list(bank.global_off), bank.global_mode)


class CudaOps:
    """The device steps of an EP step, on the library's kernels (current CUDA device)."""

    def __init__(self):
        from . import lib
        lib()                                        # fails loudly without the built library

    def route(self, logits, k):
        from . import moe_nvfp4_route
        return moe_nvfp4_route(logits, k)

    def gather_rows(self, x, perm, k):
        from . import moe_nvfp4_gather_rows
        return moe_nvfp4_gather_rows(x, perm, k)

    def recv_plan(self, counts_all, rank, recv_rows, layout):
        from . import moe_nvfp4_ep_plan
        return moe_nvfp4_ep_plan(counts_all, rank, recv_rows, layout)

    def experts(self, rows, ids, shard, y=None, path=_abi.PATH_AUTO, sorted_ids=False):
        from . import moe_nvfp4_experts
        return moe_nvfp4_experts(rows, ids, shard, y_rows=y, path=path, sorted_ids=sorted_ids)

    def combine(self, y, w, inv, k, x=None, x_next=None):
        from . import moe_nvfp4_combine
        return moe_nvfp4_combine(y, w, inv, k, x=x, x_next=x_next)

    def dispatch(self, x, route, dst_off, recv_ptrs, capacity):
        from . import moe_nvfp4_ep_dispatch
        moe_nvfp4_ep_dispatch(x, route, dst_off, recv_ptrs, capacity)

    def peer_combine(self, route, dst_off, y_ptrs, hidden, capacity, x=None, x_next=None):
        from . import moe_nvfp4_ep_combine
        return moe_nvfp4_ep_combine(route, dst_off, y_ptrs, hidden, capacity, x=x, x_next=x_next)


def _view(ptr: int, shape, dtype, device):
    """A torch tensor over device memory at ptr (no copy), for the IPC buffers."""
    import torch
    itemsize = torch.empty((), dtype=dtype).element_size()
    typestr = {1: "|u1", 2: "<i2", 4: "<f4"}[itemsize]

    class _Iface:
        __cuda_array_interface__ = {"shape": tuple(int(s) for s in shape), "typestr": typestr,
                                    "data": (int(ptr), False), "version": 3}
    t = torch.as_tensor(_Iface(), device=device)
    return t.view(dtype) if t.dtype != dtype else t


class ExpertParallel:
    """One rank's share of an expert-parallel MoE layer.

    bank: the FULL bank layout (every rank passes the same descriptor shape; only this rank's
    records need to be resident: base_dev + rank*El*record_stride onward for El records).
    group: a torch.distributed process group (default: the world); transport "peer" (NVLink
    kernels over CUDA IPC buffers, NCCL only for the counts and the barriers) or "collective"
    (all-to-all).  capacity_rows: rows each rank's receive buffers hold (peer transport); a step
    that would send any rank more raises ValueError on every rank before anything moves.
    """

    def __init__(self, bank, k: int, group=None, transport: str = "peer", capacity_rows: int = 0,
                 ops=None, path: int = _abi.PATH_AUTO):
        import torch
        import torch.distributed as dist
        if transport not in ("peer", "collective"):
            raise ValueError(f"unknown transport {transport!r}")
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.E, self.H, self.k = int(bank.num_experts), int(bank.hidden), int(k)
        if self.E % self.world:
            raise ValueError(f"{self.E} experts do not split evenly over {self.world} ranks")
        self.El = self.E // self.world
        self.transport = transport
        self.ops = ops if ops is not None else CudaOps()
        self.path = path
        self.shard = shard_bank(bank, self.rank, self.world)
        self.capacity = int(capacity_rows)
        self._own = []
        self._opened = []
        self.recv_x_ptrs = self.recv_y_ptrs = None
        self.device = torch.device("cuda", torch.cuda.current_device()) if torch.cuda.is_available() else None
        if transport == "peer":
            if self.capacity < 1:
                raise ValueError("the peer transport needs capacity_rows >= 1")
            self._make_buffers()

    # -- peer buffers ------------------------------------------------------------------------
    def _make_buffers(self) -> None:
        """Creates this rank's receive buffers and maps every peer's.  Every rank learns whether all
        of them succeeded (an all-gather of the outcome) and all raise together if one failed, so
        that no rank is left waiting in a later collective."""
        import torch.distributed as dist
        from . import (moe_nvfp4_ep_buffer_close, moe_nvfp4_ep_buffer_create, moe_nvfp4_ep_buffer_destroy,
                       moe_nvfp4_ep_buffer_open)
        cap, H = self.capacity, self.H
        err = None
        mine = None
        try:
            px, hx = moe_nvfp4_ep_buffer_create(cap * H * 2)
            self._own.append(px)
            py, hy = moe_nvfp4_ep_buffer_create(cap * H * 4)
            self._own.append(py)
            mine = (hx, hy)
        except Exception as exc:            # reported to every rank below
            err = repr(exc)
        handles = [None] * self.world
        dist.all_gather_object(handles, mine, group=self.group)
        xs, ys = [], []
        if all(h is not None for h in handles):
            try:
                for d, (hxd, hyd) in enumerate(handles):
                    if d == self.rank:
                        xs.append(px)
                        ys.append(py)
                        continue
                    a = moe_nvfp4_ep_buffer_open(hxd)
                    self._opened.append(a)
                    b = moe_nvfp4_ep_buffer_open(hyd)
                    self._opened.append(b)
                    xs.append(a)
                    ys.append(b)
            except Exception as exc:
                err = repr(exc)
        outcome = [None] * self.world
        dist.all_gather_object(outcome, err, group=self.group)
        failed = {d: e for d, e in enumerate(outcome) if e is not None}
        if failed or any(h is None for h in handles):
            for p in self._opened:
                moe_nvfp4_ep_buffer_close(p)
            self._opened = []
            dist.barrier(group=self.group)          # no peer still maps this rank's buffers
            for p in self._own:
                moe_nvfp4_ep_buffer_destroy(p)
            self._own = []
            raise RuntimeError(f"expert-parallel buffers could not be set up: {failed}")
        self.recv_x_ptrs, self.recv_y_ptrs = xs, ys
        self._recv_x = _view(px, (cap, H), _bf16(), self.device)
        self._recv_y = _view(py, (cap, H), _f32(), self.device)

    def close(self) -> None:
        """Unmaps the peers' buffers and frees this rank's (collective: every rank calls it)."""
        import torch.distributed as dist
        from . import moe_nvfp4_ep_buffer_close, moe_nvfp4_ep_buffer_destroy
        if not self._own:
            return
        import torch
        torch.cuda.synchronize()
        dist.barrier(group=self.group)
        for p in self._opened:
            moe_nvfp4_ep_buffer_close(p)
        self._opened = []
        dist.barrier(group=self.group)
        for p in self._own:
            moe_nvfp4_ep_buffer_destroy(p)
        self._own = []

    # -- one step -----------------------------------------------------------------------------
    def _barrier(self) -> None:
        """Stream-ordered barrier: an all-reduce of one element on the group's collective stream,
        which the current stream waits for."""
        import torch
        import torch.distributed as dist
        t = torch.ones(1, dtype=torch.int32, device=self.device)
        dist.all_reduce(t, group=self.group)

    def _counts(self, counts):
        import torch
        import torch.distributed as dist
        flat = counts.new_empty(self.world * self.E)
        dist.all_gather_into_tensor(flat, counts.contiguous(), group=self.group)
        C = flat.view(self.world, self.E)
        return C, C.cpu().numpy()

    def forward(self, x, logits, x_next=None):
        """out [T, H] of this rank's tokens (x [T, H] bf16, logits [T, E] f32); with x_next, also
        x_next = bf16(x + out)."""
        k = self.k
        r = self.ops.route(logits, k)
        C, C_host = self._counts(r["counts"])
        pl = plan(C_host, self.rank)
        if self.transport == "collective":
            return self._collective(x, r, C, pl, x_next)
        return self._peer(x, r, C, pl, x_next)

    def _collective(self, x, r, C, pl, x_next):
        import torch.distributed as dist
        k, H = self.k, self.H
        rows = self.ops.gather_rows(x, r["perm"], k)
        recv = rows.new_empty((pl["recv_total"], H))
        dist.all_to_all_single(recv, rows, pl["recv"], pl["send"], group=self.group)
        _, ids = self.ops.recv_plan(C, self.rank, pl["recv_total"], _abi.EP_SOURCE_MAJOR)
        y = self.ops.experts(recv, ids, self.shard, path=self.path)
        back = y.new_empty((rows.shape[0], H))
        dist.all_to_all_single(back, y, pl["send"], pl["recv"], group=self.group)
        return self.ops.combine(back, r["w"], r["inv"], k, x=x, x_next=x_next)

    def _peer(self, x, r, C, pl, x_next):
        check_capacity(pl, self.capacity)
        Rr = pl["recv_total"]
        dst_off, ids = self.ops.recv_plan(C, self.rank, Rr, _abi.EP_EXPERT_MAJOR)
        self.ops.dispatch(x, r, dst_off, self.recv_x_ptrs, self.capacity)
        self._barrier()                  # every row has reached its owner
        self.ops.experts(self._recv_x[:Rr], ids, self.shard, y=self._recv_y[:Rr], path=self.path, sorted_ids=True)
        self._barrier()                  # every owner's results are ready
        return self.ops.peer_combine(r, dst_off, self.recv_y_ptrs, self.H, self.capacity, x=x, x_next=x_next)


def _bf16():
    import torch
    return torch.bfloat16


def _f32():
    import torch
    return torch.float32
