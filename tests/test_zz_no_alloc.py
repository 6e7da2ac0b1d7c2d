"""moe_route_static: routing for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc: a plug-in inside a host process whose memory manager
already owns the whole device, or a latency-critical loop that cannot afford the implicit
synchronisation of an allocation.  moe_route_static gives them moe_route's results with its
scratch in a fixed array inside the library.  This file checks, through the C ABI, that it
returns what moe_route returns, on two calls in a row (the array keeps the previous call's
contents, so the second call must not depend on them), and that a request larger than the
array is refused.  It is collected last so that a failure here leaves every other test run.
"""
import numpy as np
import pytest
import torch

from gpu_util import assert_route_equal
from mixture_experts_layer_50_b200 import _native as nat
from mixture_experts_layer_50_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _outputs(N, E, k):
    return dict(ids=torch.empty((N, k), dtype=torch.int32, device="cuda"),
                gates=torch.empty((N, k), dtype=torch.float32, device="cuda"),
                counts=torch.empty(E, dtype=torch.int32, device="cuda"),
                demand=torch.empty(E, dtype=torch.int32, device="cuda"),
                drop_mask=torch.empty((N, k), dtype=torch.uint8, device="cuda"))


def _case(N, E, k, score_fn, n_sets, cf, seed):
    z = torch.from_numpy(W.random_logits(N, E, seed, scale=1.5)).cuda()
    bias = torch.from_numpy(W.random_bias(n_sets, E, seed + 1)).cuda() if n_sets else None
    mod = torch.from_numpy(W.random_modality(N, seed + 2)).cuda() if n_sets > 1 else None
    C = nat.moe_capacity(N, k, E, cf)
    cfg = nat.make_config(N, 64, E, k, 64, n_bias_sets=n_sets, score_fn=score_fn, capacity=C)
    return cfg, z, bias, mod


def test_route_static_matches_moe_route_on_two_calls(cuda_dev):
    cases = [(16384, 384, 6, W.SIGMOID, 2, None, 31),     # DeepSeek-V4.1-Flash-like routing
             (3001, 64, 2, W.SOFTMAX, 0, 1, 32)]           # ragged N, capacity factor 1
    for cfg, z, bias, mod in (_case(*c) for c in cases):
        N, E, k = cfg.N, cfg.E, cfg.k
        ref = _outputs(N, E, k)
        ws = nat.alloc_workspace(cfg)
        nat.moe_route(cfg, logits=z, bias=bias, modality=mod, ws=ws, **ref)
        assert nat.moe_check_status(ws) == 0
        got = _outputs(N, E, k)
        for t in got.values():
            t.fill_(0x55 if t.dtype == torch.uint8 else -3)
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        nat.moe_route_static(cfg, logits=z, bias=bias, modality=mod, status=status, **got)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        for name in ("ids", "counts", "demand", "drop_mask"):
            assert torch.equal(got[name], ref[name]), name
        g, r = got["gates"].cpu().numpy(), ref["gates"].cpu().numpy()
        assert (np.abs(g - r) / np.maximum(np.abs(r), 1e-30)).max() <= 1e-5
        # and directly against the CPU oracle on the same fp32 logits
        assert_route_equal({n: t.cpu().numpy() for n, t in got.items()}, z.cpu().numpy(), k,
                           cfg.score_fn, cfg.renorm,
                           None if bias is None else bias.cpu().numpy(),
                           None if mod is None else mod.cpu().numpy(), E, cfg.capacity)
        if cfg.capacity > 0:
            assert int(got["drop_mask"].sum()) > 0 or int(got["demand"].max()) <= cfg.capacity


def test_route_static_refuses_requests_beyond_its_array(cuda_dev):
    N, E, k = 65536, 256, 8            # needs about 6 MiB of scratch: more than the 4 MiB
    cfg = nat.make_config(N, 64, E, k, 64)
    out = _outputs(1, E, k)            # never written: the call is refused on the host
    z = torch.zeros(1, E, device="cuda")
    with pytest.raises(nat.MoeError) as err:
        nat.moe_route_static(cfg, logits=z, **out)
    assert err.value.status == nat.MOE_ERR_UNSUPPORTED
    assert "scratch" in str(err.value)
