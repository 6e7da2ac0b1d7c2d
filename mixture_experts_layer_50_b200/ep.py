"""Expert-parallel MoE layer: the routed experts spread over the ranks of a process group.

"Mixture-of-Experts : routage et capacité" slides, "Le problème — Communication", "L'idée —
Communication" and "Support visuel — Communication": each device holds some experts; a token's
row goes to the device of every expert it picked (dispatch all-to-all) and the expert outputs
come back to the token's device (combine all-to-all).

One process per GPU.  Rank ``r`` routes its own tokens with the full router (replicated), owns
the experts ``[first(r), first(r+1))`` and a copy of the shared expert.  A forward pass:

1. ``moe_route`` on the rank's tokens: ids, gates and the per-expert demand;
2. all-gather of the demands (E + 1 int32 per rank, the last entry the rank's token count);
3. ``moe_ep_plan`` (host, C): the capacity share of this rank per expert, every rank's kept
   counts, the row runs to send and where received runs land;
4. ``moe_permute_ep``: this rank's kept rows in the send layout (expert-major);
5. dispatch: one grouped point-to-point exchange of the row runs (NCCL on GPUs), or with
   ``transport="p2p"`` the dispatch passes of step 4 write the kept rows straight into the
   owners' receive buffers over peer memory (CUDA IPC mappings; NVLink on a multi-GPU node);
6. ``moe_ep_expert_ffn``: the owned experts on the received rows (tcgen05 grouped GEMMs), and
   the shared expert on the rank's own tokens, written straight into y;
7. combine trip: the same runs back to their source ranks (NCCL), or with ``"p2p"`` nothing:
   step 8 reads the outputs where the owners wrote them (``moe_ep_combine_p2p``);
8. ``moe_ep_combine``: the gate-weighted sum onto y.

The result on every rank equals the single-device layer over the concatenation of all ranks'
tokens (rank 0's first), capacity included: an expert serves that concatenated batch in token
order.  Every step of the layer runs in the library's kernels; torch.distributed only moves
the demands and the rows.
"""
from __future__ import annotations

from typing import Optional, Sequence

import torch

from . import _native as nat


def shard_experts(W_gu: torch.Tensor, W_down: torch.Tensor, E: int, n_shared: int, world: int,
                  rank: int):
    """This rank's slices of the full expert weights ``[E + S][..]``: its owned experts, then
    the shared expert (copies, contiguous)."""
    e0, e1 = nat.moe_ep_first_expert(world, rank, E), nat.moe_ep_first_expert(world, rank + 1, E)
    idx = list(range(e0, e1)) + list(range(E, E + n_shared))
    sel = torch.tensor(idx, dtype=torch.long, device=W_gu.device)
    return W_gu.index_select(0, sel).contiguous(), W_down.index_select(0, sel).contiguous()


def exchange_rows(send_buf: torch.Tensor, recv_buf: torch.Tensor, sends: Sequence, recvs: Sequence,
                  rank: int, group=None):
    """Point-to-point exchange of row runs: every run ``(peer, expert, row, rows)`` of ``sends``
    goes from ``send_buf[row:row+rows]`` to ``peer``; every run of ``recvs`` arrives from
    ``peer`` into ``recv_buf[row:row+rows]``.  Runs with ``peer == rank`` are copied locally.
    The messages of one call form one group (``batch_isend_irecv``: one NCCL group on GPUs,
    gloo on CPU tensors); runs with the same peer are posted in the same order on both sides
    and tagged with their expert id."""
    import torch.distributed as dist
    local_in = {(e, rows): row for peer, e, row, rows in recvs if peer == rank}
    ops = []
    for peer, e, row, rows in sends:
        src = send_buf[row:row + rows]
        if peer == rank:
            dst_row = local_in.pop((e, rows))
            recv_buf[dst_row:dst_row + rows].copy_(src)
        else:
            ops.append(dist.P2POp(dist.isend, src, peer, group, tag=e))
    for peer, e, row, rows in recvs:
        if peer != rank:
            ops.append(dist.P2POp(dist.irecv, recv_buf[row:row + rows], peer, group, tag=e))
    if local_in:
        raise RuntimeError(f"rank {rank}: local runs without a matching send: {local_in}")
    if ops:
        for req in dist.batch_isend_irecv(ops):
            req.wait()


def loopback_exchange(send_bufs: Sequence[torch.Tensor], recv_bufs: Sequence[torch.Tensor],
                      sends: Sequence[Sequence], recvs: Sequence[Sequence]):
    """The same exchange for ranks emulated in one process (``send_bufs[r]`` is rank r's send
    buffer ...): each run is copied straight from its sender's buffer to its receiver's.
    Checks that every run has exactly one counterpart of the same size."""
    pending = {}
    for r, lst in enumerate(recvs):
        for peer, e, row, rows in lst:
            key = (peer, r, e)
            if key in pending:
                raise RuntimeError(f"two receive runs for {key}")
            pending[key] = (row, rows)
    for r, lst in enumerate(sends):
        for peer, e, row, rows in lst:
            dst_row, n = pending.pop((r, peer, e))
            if n != rows:
                raise RuntimeError(f"run {r}->{peer} expert {e}: {rows} rows sent, {n} expected")
            recv_bufs[peer][dst_row:dst_row + rows].copy_(send_bufs[r][row:row + rows])
    if pending:
        raise RuntimeError(f"receive runs without a sender: {sorted(pending)}")


def all_plans(world: int, E: int, capacity: int, demand_all) -> list:
    """Every rank's plan from the all-gathered demands (each rank can compute the others')."""
    return [nat.moe_ep_plan(world, r, E, capacity, demand_all) for r in range(world)]


def peer_runs(rank: int, plans: Sequence[dict], direction: str) -> list:
    """This rank's runs for ``moe_ep_copy_runs`` as (src_row, dst_rank, dst_row, rows):
    ``"dispatch"``: each run of its send buffer lands where its owner receives (rank, expert);
    ``"return"``: each run of its receive buffer (expert outputs) goes back to the row of the
    source's send run (rank, expert), i.e. into the source's return buffer."""
    mine, theirs = ("sends", "recvs") if direction == "dispatch" else ("recvs", "sends")
    out = []
    for peer, e, row, rows in plans[rank][mine]:
        dst = {(p, ex): (r, n) for p, ex, r, n in plans[peer][theirs]}
        if (rank, e) not in dst or dst[(rank, e)][1] != rows:
            raise RuntimeError(f"rank {rank} -> {peer} expert {e}: no matching run of {rows} rows")
        out.append((row, peer, dst[(rank, e)][0], rows))
    return out


def expert_tables(rank: int, plans: Sequence[dict], E: int, recv_base: Sequence[int],
                  out_base: Sequence[int], rows: Sequence[int]):
    """Where rank ``rank``'s kept rows of each expert go and come back from: per expert e, the
    receive and output buffer of e's owner (``recv_base``/``out_base`` indexed by rank), the
    row of the owner's buffers where this rank's rows of e start (the owner's receive run for
    (rank, e)), and the owner's buffer size (``rows``).  An expert this rank keeps no row of
    gets this rank's own buffers at row 0 (never read).  Host lists of E entries."""
    recv, out = [recv_base[rank]] * E, [out_base[rank]] * E
    row0, size = [0] * E, [0] * E
    for peer, e, _, n in plans[rank]["sends"]:
        dst = {(p, ex): r for p, ex, r, _ in plans[peer]["recvs"]}
        if (rank, e) not in dst:
            raise RuntimeError(f"rank {rank} -> {peer} expert {e}: no matching receive run")
        recv[e], out[e] = recv_base[peer], out_base[peer]
        row0[e], size[e] = dst[(rank, e)], rows[peer]
    return recv, out, row0, size


class PeerTransport:
    """The rows of an expert-parallel layer moved through peer memory (the peers' allocations
    mapped with CUDA IPC) instead of NCCL messages.  One allocation, made once, holds the
    receive buffer (every rank's rows for this rank's experts: at most world * max_tokens * k
    rows) and, row for row beside it, the output buffer of this rank's experts; its handle is
    exchanged once.  A forward takes two barriers (``barrier``; default: a one-element
    all-reduce on the stream for NCCL groups, else a synchronise and a host barrier):

    1. ``dispatch_fused``: the dispatch passes write each kept row into its owner's receive
       buffer, then the barrier;
    2. the owner's experts write their outputs into its output buffer, then the barrier;
    3. ``combine``: each rank's combine reads its slots' outputs from the owners' output
       buffers (the return trip and the combine in one pass).

    An owner rewrites its receive buffer only after barrier 2 (its experts have read it) and
    its output buffer only after the next forward's barrier 1, which every rank reaches after
    its combine, so no row is overwritten while still in use."""

    def __init__(self, layer: "EPMoELayer", group=None, barrier=None):
        import torch.distributed as dist
        self.layer, self.group = layer, group
        dev = layer.xp.device
        self.rows = max(1, layer.world * layer.max_tokens * layer.k)
        self.buf = torch.empty((2 * self.rows, layer.d), dtype=torch.bfloat16, device=dev)
        self.recv, self.out = self.buf[:self.rows], self.buf[self.rows:]
        handle, offset = nat.ipc_handle(self.buf)
        gathered = [None] * layer.world
        dist.all_gather_object(gathered, (handle, offset, self.rows), group=group)
        self.mapped = []
        row_bytes = layer.d * 2
        self._recv_base, self._out_base, self._rows = [], [], []
        for r, (h, off, n) in enumerate(gathered):
            if r == layer.rank:
                base = self.buf.data_ptr()
            else:
                mapped = nat.ipc_open(h)
                self.mapped.append(mapped)
                base = mapped + off
            self._recv_base.append(base)
            self._out_base.append(base + n * row_bytes)
            self._rows.append(n)
        if barrier is None:
            if dist.get_backend(group) == "nccl":
                flag = torch.zeros(1, dtype=torch.int32, device=dev)
                barrier = lambda: dist.all_reduce(flag, group=group)
            else:
                def barrier():
                    torch.cuda.current_stream(dev).synchronize()
                    dist.barrier(group=group)
        self.barrier = barrier
        self._tables = None

    def expert_tables(self, plans: Sequence[dict]):
        """Per expert e (host lists of E entries): the owner's receive and output buffers, the
        row where this rank's kept rows of e start in them, and their size in rows."""
        L = self.layer
        return expert_tables(L.rank, plans, L.E, self._recv_base, self._out_base, self._rows)

    def _device_tables(self, plans: Sequence[dict]):
        dev = self.buf.device
        recv, out, row0, rows = self.expert_tables(plans)
        i64 = dict(dtype=torch.int64)
        return (torch.tensor(recv, **i64).to(dev), torch.tensor(out, **i64).to(dev),
                torch.tensor(row0, dtype=torch.int32).to(dev), torch.tensor(rows, **i64).to(dev))

    def dispatch_fused(self, x: torch.Tensor, plans: Sequence[dict]) -> torch.Tensor:
        """The dispatch passes with the kept rows written straight into their owners'
        receive buffers (moe_permute_ep_p2p), then the barrier; returns this rank's received
        rows."""
        L = self.layer
        N = L.N
        self._tables = self._device_tables(plans)
        if N > 0:
            recv, _, row0, rows = self._tables
            nat.moe_permute_ep_p2p(
                L.config(N), ids=L.ids[:N], cap=L.cap, x=x, offsets=L.offsets,
                slot_row=L.slot_row[:N], dst_base=recv, dst_row0=row0, dst_rows=rows,
                counts=L.counts, drop_mask=L.drop_mask[:N], ws=L.ws)
        self.barrier()
        return self.recv[:max(1, plans[L.rank]["rows_owned"])]

    def outputs(self, plans: Sequence[dict]) -> torch.Tensor:
        """Where this rank's experts write their outputs (row i: the output of received row i)."""
        return self.out[:max(1, plans[self.layer.rank]["rows_owned"])]

    def combine(self, y: torch.Tensor) -> torch.Tensor:
        """The gate-weighted sum onto y, each slot's output read from its owner's output buffer
        (moe_ep_combine_p2p); follows the barrier after the experts."""
        L = self.layer
        N = L.N
        if self._tables is None:
            raise RuntimeError("PeerTransport.combine before dispatch_fused: no expert tables")
        if N > 0:
            _, out, row0, rows = self._tables
            nat.moe_ep_combine_p2p(L.config(N), ids=L.ids[:N], slot_row=L.slot_row[:N],
                                   gates=L.gates[:N], offsets=L.offsets, src_base=out,
                                   src_row0=row0, src_rows=rows, y=y, ws=L.ws)
        return y

    def close(self):
        torch.cuda.synchronize(self.buf.device)
        for m in self.mapped:
            nat.ipc_close(m)
        self.mapped = []


class EPMoELayer:
    """One rank of an expert-parallel MoE layer (bf16).

    ``W_g [E][d]`` is the full router; ``W_gu``, ``W_down`` hold this rank's experts then the
    shared expert (``shard_experts``).  ``capacity_factor`` applies to the whole concatenated
    batch: C = ceil(T k / E * cf) with T the tokens of all ranks.  ``forward`` runs the whole
    layer with torch.distributed (``group``); the phase methods (``route``, ``set_plan``,
    ``permute``, ``run_experts``, ``combine``) let a caller drive the exchanges itself.
    ``transport``: ``"nccl"`` (grouped point-to-point messages) or ``"p2p"`` (``PeerTransport``:
    the rows written straight into the peers' buffers); a p2p layer is built collectively, by
    every rank of the group, and released with ``close``.
    """

    def __init__(self, *, W_g, W_gu, W_down, k, world: int, rank: int, n_shared=0,
                 score_fn=nat.SOFTMAX, renorm=1, act=nat.SWIGLU, clamp=0.0, bias=None,
                 logit_offset=None, capacity_factor=None, max_tokens: int, group=None,
                 transport: str = "nccl", barrier=None):
        if W_gu.dtype != torch.bfloat16:
            raise ValueError("the expert-parallel layer is bf16")
        self.E, self.d = W_g.shape
        self.F = W_down.shape[2]
        self.k, self.n_shared = k, n_shared
        self.world, self.rank, self.group = world, rank, group
        self.first = nat.moe_ep_first_expert(world, rank, self.E)
        self.n_owned = nat.moe_ep_first_expert(world, rank + 1, self.E) - self.first
        if W_gu.shape[0] != self.n_owned + n_shared or W_down.shape[0] != self.n_owned + n_shared:
            raise ValueError(f"rank {rank} owns {self.n_owned} experts (+{n_shared} shared); "
                             f"got weights for {W_gu.shape[0]}")
        self.W_g, self.W_gu, self.W_down = W_g, W_gu, W_down
        self.score_fn, self.renorm, self.act, self.clamp = score_fn, renorm, act, clamp
        self.bias, self.logit_offset = bias, logit_offset
        self.n_bias_sets = 0 if bias is None else bias.shape[0]
        self.capacity_factor = capacity_factor
        self.max_tokens = max_tokens
        dev = W_gu.device
        self.ws = nat.alloc_ep_workspace(self.config(max_tokens), world, device=dev)
        Nk = max(1, max_tokens * k)
        i32 = dict(dtype=torch.int32, device=dev)
        self.ids = torch.empty((max_tokens, k), **i32)
        self.gates = torch.empty((max_tokens, k), dtype=torch.float32, device=dev)
        self.demand = torch.empty(self.E + 1, **i32)          # + this rank's token count
        self.counts = torch.empty(self.E, **i32)
        self.offsets = torch.empty(self.E + 1, **i32)
        self.slot_row = torch.empty((max_tokens, k), **i32)
        self.drop_mask = torch.empty((max_tokens, k), dtype=torch.uint8, device=dev)
        self.xp = torch.empty((Nk, self.d), dtype=torch.bfloat16, device=dev)
        self.cap = torch.empty(self.E, **i32)
        self.owned_offsets = torch.empty(self.n_owned + 1, **i32)
        self.plan = None
        self.plans = None
        self.N = 0
        if transport not in ("nccl", "p2p"):
            raise ValueError(f"transport must be 'nccl' or 'p2p', not {transport!r}")
        self.transport = PeerTransport(self, group, barrier) if transport == "p2p" else None

    @classmethod
    def from_full_weights(cls, *, W_g, W_gu, W_down, k, E, world, rank, n_shared=0, **kw):
        gu, dn = shard_experts(W_gu, W_down, E, n_shared, world, rank)
        return cls(W_g=W_g, W_gu=gu, W_down=dn, k=k, world=world, rank=rank, n_shared=n_shared,
                   **kw)

    def config(self, N: int, capacity: int = 0) -> "nat.moe_config":
        return nat.make_config(N, self.d, self.E, self.k, self.F, self.n_shared, self.n_bias_sets,
                               self.score_fn, self.renorm, self.act, nat.BF16, self.clamp,
                               capacity)

    # ---- phases ------------------------------------------------------------------------
    def route(self, x: torch.Tensor, modality=None) -> torch.Tensor:
        """Router, scores and top-k on this rank's tokens (no capacity yet).  Returns the
        device int32 [E + 1] vector to all-gather: demand per expert, then the token count."""
        N = x.shape[0]
        if N > self.max_tokens:
            raise ValueError(f"{N} tokens > max_tokens={self.max_tokens}")
        self.N = N
        if N == 0:
            self.demand.zero_()
            return self.demand
        nat.moe_route(self.config(N), x=x, W_g=self.W_g, logit_offset=self.logit_offset,
                      bias=self.bias, modality=modality, ids=self.ids[:N], gates=self.gates[:N],
                      counts=self.counts, demand=self.demand[:self.E], ws=self.ws)
        self.demand[self.E:].fill_(N)
        return self.demand

    def set_plan(self, gathered) -> dict:
        """The plan from the all-gathered [world][E + 1] demands (host array or tensor)."""
        import numpy as np
        g = np.asarray(gathered.cpu() if isinstance(gathered, torch.Tensor) else gathered,
                       dtype=np.int64).reshape(self.world, self.E + 1)
        T = int(g[:, self.E].sum())
        C = nat.moe_capacity(T, self.k, self.E, self.capacity_factor)
        self.plans = all_plans(self.world, self.E, C, g[:, :self.E])
        self.plan = self.plans[self.rank]
        self.plan["capacity"] = C
        self.cap.copy_(torch.from_numpy(self.plan["cap"]), non_blocking=False)
        self.owned_offsets.copy_(torch.from_numpy(self.plan["owned_offsets"]), non_blocking=False)
        return self.plan

    def permute(self, x: torch.Tensor) -> torch.Tensor:
        """This rank's kept rows in the send layout; returns the send buffer."""
        N = self.N
        if N > 0:
            nat.moe_permute_ep(self.config(N), ids=self.ids[:N], cap=self.cap, x=x,
                               offsets=self.offsets, slot_row=self.slot_row[:N], xp=self.xp,
                               counts=self.counts, drop_mask=self.drop_mask[:N], ws=self.ws)
        return self.xp[:max(1, self.plan["rows_kept"])]

    def new_recv_buffer(self) -> torch.Tensor:
        return torch.empty((max(1, self.plan["rows_owned"]), self.d), dtype=torch.bfloat16,
                           device=self.xp.device)

    def new_return_buffer(self) -> torch.Tensor:
        return torch.empty((max(1, self.plan["rows_kept"]), self.d), dtype=torch.bfloat16,
                           device=self.xp.device)

    def run_experts(self, xr: torch.Tensor, x: torch.Tensor, y: torch.Tensor,
                    ye: Optional[torch.Tensor] = None) -> torch.Tensor:
        """The owned experts on the received rows (outputs into ye, a new buffer by default);
        the shared expert's rows go into y."""
        if ye is None:
            ye = torch.empty_like(xr)
        nat.moe_ep_expert_ffn(self.config(self.max_tokens), self.world, self.rank, self.N,
                              self.plan["rows_owned"], xr=xr, owned_offsets=self.owned_offsets,
                              x=x if self.N else None, W_gu=self.W_gu, W_down=self.W_down, ye=ye,
                              y=y if self.n_shared and self.N else None, ws=self.ws)
        return ye

    def combine(self, ye_back: torch.Tensor, y: torch.Tensor) -> torch.Tensor:
        N = self.N
        if N > 0:
            nat.moe_ep_combine(self.config(N), ye=ye_back, slot_row=self.slot_row[:N],
                               gates=self.gates[:N], y=y)
        return y

    # ---- the whole layer over torch.distributed ------------------------------------------
    def forward(self, x: torch.Tensor, modality=None, y: Optional[torch.Tensor] = None):
        import torch.distributed as dist
        if y is None:
            y = torch.empty_like(x)
        demand = self.route(x, modality)
        if dist.get_backend(self.group) == "nccl":
            gathered = torch.empty(self.world * (self.E + 1), dtype=torch.int32,
                                   device=demand.device)
            dist.all_gather_into_tensor(gathered, demand, group=self.group)
        else:  # a CPU backend (gloo) moves host tensors
            gathered = torch.empty(self.world * (self.E + 1), dtype=torch.int32)
            dist.all_gather_into_tensor(gathered, demand.cpu(), group=self.group)
        plan = self.set_plan(gathered)
        if self.transport is not None:
            # the dispatch passes write the kept rows straight into the owners' buffers; the
            # combine reads the outputs back from them
            t = self.transport
            xr = t.dispatch_fused(x, self.plans)
            self.run_experts(xr, x, y, ye=t.outputs(self.plans))
            t.barrier()
            return t.combine(y)
        xp = self.permute(x)
        xr = self.new_recv_buffer()
        exchange_rows(xp, xr, plan["sends"], plan["recvs"], self.rank, self.group)
        ye = self.run_experts(xr, x, y)
        ye_back = self.new_return_buffer()
        exchange_rows(ye, ye_back, plan["recvs"], plan["sends"], self.rank, self.group)
        return self.combine(ye_back, y)

    def close(self):
        """Unmap the peers' buffers (p2p transport)."""
        if self.transport is not None:
            self.transport.close()

    def check_status(self) -> int:
        return nat.moe_check_status(self.ws)


__all__ = ["EPMoELayer", "PeerTransport", "shard_experts", "exchange_rows", "loopback_exchange",
           "all_plans", "peer_runs", "expert_tables"]
