"""MoELayer: a layer's device weights and workspace behind one ``forward`` call."""
from __future__ import annotations

from typing import Optional

import torch

from . import _native as nat


class MoELayer:
    """Forward pass of one MoE FFN layer through ``moe_forward``.

    Weights use the library's storage convention (``W_g [E][d]``, ``W_gu [E+S][2F][d]``
    gate rows then up rows, ``W_down [E+S][d][F]``, shared expert last).  The capacity is
    recomputed per call from ``capacity_factor`` and the call's token count,
    C = ceil(N k / E * cf).  ``overflow`` is what happens to an assignment beyond the
    capacity: ``"drop"`` (it contributes 0) or ``"reroute"`` (the slides' "report" policy: it
    goes to the token's next-best expert if that one has room; ``moe_forward_reroute``).
    The workspace is allocated once for ``max_tokens``.
    """

    def __init__(self, *, W_g, W_gu, W_down, k, n_shared=0, score_fn=nat.SOFTMAX, renorm=1,
                 act=nat.SWIGLU, clamp=0.0, bias=None, logit_offset=None,
                 capacity_factor=None, max_tokens: int, stream=None, overflow: str = "drop"):
        if overflow not in ("drop", "reroute"):
            raise ValueError(f"overflow must be 'drop' or 'reroute', not {overflow!r}")
        self.overflow = overflow
        self.W_g, self.W_gu, self.W_down = W_g, W_gu, W_down
        self.E, self.d = W_g.shape
        self.F = W_down.shape[2]
        self.k, self.n_shared = k, n_shared
        self.score_fn, self.renorm, self.act, self.clamp = score_fn, renorm, act, clamp
        self.bias, self.logit_offset = bias, logit_offset
        self.n_bias_sets = 0 if bias is None else bias.shape[0]
        self.capacity_factor = capacity_factor
        self.dtype = nat.BF16 if W_gu.dtype == torch.bfloat16 else nat.F32
        self.max_tokens = max_tokens
        self.ws = nat.alloc_workspace(self.config(max_tokens), device=W_gu.device)
        self._graphs = {}

    @classmethod
    def from_workload(cls, shape, tensors: dict, max_tokens: Optional[int] = None,
                      overflow: str = "drop"):
        return cls(W_g=tensors["W_g"], W_gu=tensors["W_gu"], W_down=tensors["W_down"],
                   k=shape.k, n_shared=shape.n_shared, score_fn=shape.score_fn,
                   renorm=shape.renorm, act=shape.act, clamp=shape.clamp,
                   bias=tensors.get("bias"), logit_offset=tensors.get("logit_offset"),
                   capacity_factor=shape.capacity_factor,
                   max_tokens=shape.N if max_tokens is None else max_tokens,
                   overflow=overflow)

    def capacity(self, N: int) -> int:
        return nat.moe_capacity(N, self.k, self.E, self.capacity_factor)

    def config(self, N: int) -> "nat.moe_config":
        return nat.make_config(N, self.d, self.E, self.k, self.F, self.n_shared,
                               self.n_bias_sets, self.score_fn, self.renorm, self.act,
                               self.dtype, self.clamp, self.capacity(N))

    def _check_tokens(self, N):
        if N > self.max_tokens:
            raise ValueError(f"{N} tokens > max_tokens={self.max_tokens} of this layer's workspace")

    def forward(self, x: torch.Tensor, modality=None, y=None, route_out: Optional[dict] = None,
                stream=None) -> torch.Tensor:
        N = x.shape[0]
        self._check_tokens(N)
        if y is None:
            y = torch.empty_like(x)
        fwd = nat.moe_forward_reroute if self.overflow == "reroute" else nat.moe_forward
        fwd(self.config(N), x=x, W_g=self.W_g, W_gu=self.W_gu, W_down=self.W_down, y=y,
            logit_offset=self.logit_offset, bias=self.bias, modality=modality,
            route_out=route_out, ws=self.ws, stream=stream)
        return y

    def _forward_host_copies(self, x_host, y_host, modality, stream, sync):
        # host buffers through torch copies on the layer's stream (the C host entry points
        # implement the drop policy only)
        N = x_host.shape[0]
        st = torch.cuda.current_stream() if stream is None else stream
        with torch.cuda.stream(st):
            xd = torch.empty(x_host.shape, dtype=x_host.dtype, device=self.W_gu.device)
            xd.copy_(x_host, non_blocking=True)
            y = self.forward(xd, modality=modality, stream=st)
            y_host[:N].copy_(y, non_blocking=True)
        if sync:
            st.synchronize()
        return y_host

    def forward_graphed(self, x: torch.Tensor, y: torch.Tensor, modality=None) -> torch.Tensor:
        """forward() replayed from a CUDA graph: the first call with a given (x, y, modality)
        captures the layer's launches once (the library's one-time per-device set-up has
        happened in an eager call first); later calls replay them with one graph launch.
        The buffers must stay the same; their contents may change between calls."""
        key = (x.data_ptr(), y.data_ptr(), None if modality is None else modality.data_ptr(),
               x.shape[0])
        g = self._graphs.get(key)
        if g is None:
            self.forward(x, modality=modality, y=y)          # eager run: one-time set-up
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            # thread-local capture: CUDA calls of other threads (a process group's
            # watchdog, pinned-memory workers) do not invalidate the capture
            with torch.cuda.graph(g, capture_error_mode="thread_local"):
                self.forward(x, modality=modality, y=y)
            self._graphs[key] = g
        g.replay()
        return y

    def forward_host(self, x_host: torch.Tensor, y_host: torch.Tensor, modality=None,
                     stream=None) -> torch.Tensor:
        N = x_host.shape[0]
        self._check_tokens(N)
        if self.overflow == "reroute":
            return self._forward_host_copies(x_host, y_host, modality, stream, sync=True)
        nat.moe_forward_host(self.config(N), x_host=x_host, W_g=self.W_g, W_gu=self.W_gu,
                             W_down=self.W_down, y_host=y_host, logit_offset=self.logit_offset,
                             bias=self.bias, modality=modality, ws=self.ws, stream=stream)
        return y_host

    def forward_host_batches(self, x_host: list, y_host: list, modality=None, stream=None):
        """Several host batches with copies overlapped with the layer (pinned buffers)."""
        N = x_host[0].shape[0]
        self._check_tokens(N)
        if self.overflow == "reroute":
            for xb, yb in zip(x_host, y_host):
                self._forward_host_copies(xb, yb, modality, stream, sync=False)
            (torch.cuda.current_stream() if stream is None else stream).synchronize()
            return y_host
        mods = None if modality is None else [modality] * len(x_host)
        nat.moe_forward_host_batches(self.config(N), x_host=x_host, W_g=self.W_g, W_gu=self.W_gu,
                                     W_down=self.W_down, y_host=y_host,
                                     logit_offset=self.logit_offset, bias=self.bias,
                                     modality=mods, ws=self.ws, stream=stream)
        return y_host

    def check_status(self, stream=None) -> int:
        return nat.moe_check_status(self.ws, stream)
