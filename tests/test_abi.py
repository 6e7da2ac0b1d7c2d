"""The C ABI library: it loads, exports what include/moe.h declares, and rejects bad
arguments on the host before touching the GPU (so these run without one)."""
import ctypes
import os
import re

import pytest

from golden.reader import load

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def nat():
    from conftest import ensure_library
    ensure_library()
    from mixture_experts_layer_50_b200 import _native
    return _native


def _declared_functions():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"^MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text, re.M)
    return names


def test_library_exports_every_declared_function(nat):
    names = _declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(nat.lib, n), n
    assert set(nat.EXPORTED) <= set(names)


def test_config_struct_layout(nat):
    assert ctypes.sizeof(nat.moe_config) == 64
    assert nat.moe_config.capacity.offset == 56
    assert ctypes.sizeof(nat.moe_route_out) == 7 * 8


def test_capacity_against_the_slides(nat):
    g = load("p2_capacity_trace.txt")
    lib = nat.lib
    assert lib.moe_capacity(8, 2, 4, 5, 4) == int(g["C_1.25"])
    assert lib.moe_capacity(8, 2, 4, 1, 1) == int(g["C_1.0"])
    assert lib.moe_capacity(8, 2, 4, 2, 1) == int(g["C_2.0"])
    assert lib.moe_capacity(8, 1, 4, 5, 4) == int(g["C_k1"])
    assert lib.moe_capacity(8, 2, 4, 3, 2) == int(g["C_1.5"])
    assert lib.moe_capacity(8, 2, 4, 0, 1) == 0          # no limit
    assert lib.moe_capacity(100, 2, 64, 1, 1) == 4       # exact ceiling of 3.125
    assert lib.moe_capacity(16384, 2, 64, 5, 4) == 640
    assert lib.moe_capacity(-1, 2, 4, 1, 1) == -1
    assert nat.moe_capacity(16384, 1, 64, 1) == 256


def _cfg(nat, **kw):
    base = dict(N=64, d=256, E=8, k=2, F=512)
    base.update(kw)
    return nat.make_config(**base)


def test_workspace_size(nat):
    small = nat.moe_workspace_size(_cfg(nat, N=16))
    big = nat.moe_workspace_size(_cfg(nat, N=4096))
    assert 0 < small < big
    # xp (N k d bf16) and ye ((N k + N) d bf16) dominate
    c = _cfg(nat, N=4096, n_shared=1)
    assert nat.moe_workspace_size(c) >= 2 * (4096 * 2 * 256 + 4096 * 3 * 256)
    assert nat.moe_workspace_size(_cfg(nat, k=9)) == 0      # k > E
    assert nat.moe_workspace_size(_cfg(nat, E=2000)) == 0   # unsupported E


@pytest.mark.parametrize("bad,code", [
    (dict(k=0), 1), (dict(k=9), 1), (dict(E=0), 1), (dict(N=-1), 1), (dict(d=0), 1),
    (dict(score_fn=7), 1), (dict(act=3), 1), (dict(dtype=5), 1), (dict(renorm=2), 1),
    (dict(E=64, k=33), 2), (dict(E=1500, k=2), 2), (dict(n_shared=2), 2), (dict(d=100), 2),
    (dict(F=12), 2),
])
def test_forward_rejects_bad_config_on_host(nat, bad, code):
    c = _cfg(nat, **bad)
    fake = ctypes.c_void_p(0x100000)
    st = nat.lib.moe_forward(ctypes.byref(c), fake, fake, None, None, None, fake, fake, fake,
                             None, fake, None)
    assert st == code, nat.lib.moe_last_error()
    assert nat.lib.moe_last_error()


def test_forward_rejects_null_and_unaligned_pointers(nat):
    c = _cfg(nat)
    fake = ctypes.c_void_p(0x100000)
    lib = nat.lib
    assert lib.moe_forward(ctypes.byref(c), None, fake, None, None, None, fake, fake, fake,
                           None, fake, None) == nat.MOE_ERR_INVALID_ARG
    assert b"x is NULL" in lib.moe_last_error()
    assert lib.moe_forward(ctypes.byref(c), ctypes.c_void_p(0x100001), fake, None, None, None,
                           fake, fake, fake, None, fake, None) == nat.MOE_ERR_UNSUPPORTED
    assert lib.moe_forward(ctypes.byref(c), fake, fake, None, None, None, fake, fake, fake,
                           None, ctypes.c_void_p(0x100010), None) == nat.MOE_ERR_INVALID_ARG
    assert b"256-byte" in lib.moe_last_error()
    assert lib.moe_forward(None, fake, fake, None, None, None, fake, fake, fake, None, fake,
                           None) == nat.MOE_ERR_INVALID_ARG


def test_bias_and_modality_rules(nat):
    fake = ctypes.c_void_p(0x100000)
    lib = nat.lib
    c = _cfg(nat, n_bias_sets=2)
    # two bias sets need the modality flags
    assert lib.moe_forward(ctypes.byref(c), fake, fake, None, fake, None, fake, fake, fake,
                           None, fake, None) == nat.MOE_ERR_INVALID_ARG
    c = _cfg(nat, n_bias_sets=0)
    assert lib.moe_forward(ctypes.byref(c), fake, fake, None, fake, None, fake, fake, fake,
                           None, fake, None) == nat.MOE_ERR_INVALID_ARG
    c = _cfg(nat, n_bias_sets=1)
    assert lib.moe_route(ctypes.byref(c), fake, None, None, None, None, None, fake, fake, fake,
                         fake, fake, None, fake, None) == nat.MOE_ERR_INVALID_ARG


def test_split_entry_points_validate(nat):
    fake = ctypes.c_void_p(0x100000)
    lib = nat.lib
    c = _cfg(nat)
    assert lib.moe_permute(ctypes.byref(c), None, None, fake, fake, None, fake, fake, fake,
                           None) == nat.MOE_ERR_INVALID_ARG
    assert lib.moe_expert_ffn(ctypes.byref(c), fake, None, None, fake, fake, fake, fake,
                              None) == nat.MOE_ERR_INVALID_ARG
    assert lib.moe_combine(ctypes.byref(c), fake, None, fake, fake, None) == nat.MOE_ERR_INVALID_ARG
    assert lib.moe_route(ctypes.byref(c), None, None, fake, None, None, None, fake, fake, fake,
                         fake, fake, None, fake, None) == nat.MOE_ERR_INVALID_ARG
    assert lib.moe_forward_host(ctypes.byref(c), None, fake, None, None, None, fake, fake,
                                fake, fake, None) == nat.MOE_ERR_INVALID_ARG
    assert lib.moe_check_status(None, None) == nat.MOE_ERR_INVALID_ARG
    assert lib.moe_workspace_init(None, None) == nat.MOE_ERR_INVALID_ARG


def test_binding_refuses_host_tensors(nat):
    import torch
    c = _cfg(nat)
    with pytest.raises(ValueError):
        nat.moe_combine(c, ye=torch.zeros(4), slot_row=torch.zeros(4, dtype=torch.int32),
                        gates=torch.zeros(4), y=torch.zeros(4))


def test_wait_selftest_validates_on_host(nat):
    lib = nat.lib
    assert lib.moe_selftest_wait_timeout(None, 1000, None) == nat.MOE_ERR_INVALID_ARG
    fake = ctypes.c_void_p(256)
    assert lib.moe_selftest_wait_timeout(fake, -1, None) == nat.MOE_ERR_INVALID_ARG
    assert lib.moe_selftest_wait_timeout(fake, 2_000_000_000, None) == nat.MOE_ERR_INVALID_ARG


def _build_c_client(out_dir):
    """Compile and link tests/c_abi_forward.c (plain C99) against the library."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    from conftest import ensure_library
    ensure_library()
    here = os.path.dirname(os.path.abspath(__file__))
    root = os.path.dirname(here)
    pkg = os.path.join(root, "mixture_experts_layer_50_b200")
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    exe = os.path.join(str(out_dir), "c_abi_forward")
    cmd = [gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-O2",
           os.path.join(here, "c_abi_forward.c"), "-I", os.path.join(root, "include"),
           "-I", os.path.join(cuda, "include"), "-L", pkg, "-lmoe_b200",
           "-L", os.path.join(cuda, "lib64"), "-lcudart", f"-Wl,-rpath,{pkg}",
           f"-Wl,-rpath,{os.path.join(cuda, 'lib64')}", "-o", exe]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return exe


def test_header_is_plain_c_and_a_c_client_links(tmp_path):
    """include/moe.h compiles as C99 and a C program links against libmoe_b200.so alone."""
    exe = _build_c_client(tmp_path)
    assert os.path.exists(exe)


def test_ffn_kernel_choice(nat):
    """Which grouped GEMM each preset layer takes, decided on the host from the configuration
    (with no GPU the device attributes fall back to 148 SMs and 126 MB of L2, the B200's)."""
    from mixture_experts_layer_50_b200 import workloads as W
    one_256, one_128 = "1-SM, 128x256 tiles", "1-SM, 128x128 tiles"
    two = "2-SM, 256x256 tiles"
    # decode-sized batches (every group within 64 rows): 64-row tiles
    d64_256, d64_128 = "1-SM, 64x256 tiles", "1-SM, 64x128 tiles"
    want = {
        "mixtral-n16": (d64_128, d64_256), "mixtral-n256": (one_128, one_256),
        # gate/up: 235 MB weight panels per expert stay on the 1-SM kernel
        "mixtral-n4096": (one_256, two), "mixtral-n16384": (one_256, two),
        # ~256 rows per expert: 256-row tiles would pad a third more rows
        "dsv3-n64": (d64_256, d64_256), "dsv3-n8192": (one_256, one_256),
        "v41flash-n64": (d64_256, d64_256), "v41flash-n16384": (one_256, one_256),
        # the shared expert's 16384 rows dominate; 11.5 MB panels
        "capacity-cf1": (two, two), "capacity-cfinf": (two, two),
        "switch-cf1": (two, two), "switch-cfinf": (two, two),
    }
    for name, (gu, dn) in want.items():
        got = nat.moe_ffn_kernels(nat.config_from_shape(W.PRESETS[name]))
        assert gu in got[0] and dn in got[1], (name, got)
    toy = nat.moe_ffn_kernels(nat.config_from_shape(W.PRESETS["toy"]))
    assert "f32" in toy[0] and "f32" in toy[1]
    assert nat.moe_ffn_kernels(_cfg(nat, N=0)) == ("none", "none")
    # truncation keeps the terminating NUL; bad arguments are refused on the host
    buf = ctypes.create_string_buffer(8)
    assert nat.lib.moe_ffn_kernels(ctypes.byref(_cfg(nat)), buf, None, 8) == 0
    assert buf.value == b"grouped"
    assert nat.lib.moe_ffn_kernels(ctypes.byref(_cfg(nat)), buf, None, 0) == nat.MOE_ERR_INVALID_ARG
    assert nat.lib.moe_ffn_kernels(ctypes.byref(_cfg(nat, k=9)), buf, None, 8) == nat.MOE_ERR_INVALID_ARG


@pytest.mark.parametrize("path,kind", [("1sm", "1-SM"), ("1sm128", "x128 tiles"),
                                       ("2sm", "2-SM, 256x256 tiles"), ("swap", "token-in-N"),
                                       ("tall", "1-SM, 256x256 tiles")])
def test_ffn_kernel_override(nat, path, kind, monkeypatch):
    """MOE_B200_GEMM_PATH forces one grouped GEMM for both projections ("1sm" keeps the
    automatic tile width), and moe_ffn_kernels reports the forced choice (the library reads
    the variable at every call)."""
    from mixture_experts_layer_50_b200 import workloads as W
    monkeypatch.setenv("MOE_B200_GEMM_PATH", path)
    for name in ("mixtral-n16", "dsv3-n8192", "capacity-cf1"):
        got = nat.moe_ffn_kernels(nat.config_from_shape(W.PRESETS[name]))
        assert kind in got[0] and kind in got[1], (path, name, got)
    monkeypatch.delenv("MOE_B200_GEMM_PATH")
    got = nat.moe_ffn_kernels(nat.config_from_shape(W.PRESETS["capacity-cf1"]))
    assert "2-SM" in got[0] and "2-SM" in got[1]


def test_expert_parallel_entry_points_validate_on_host(nat):
    """The expert-parallel calls reject bad arguments before touching the GPU."""
    fake = ctypes.c_void_p(0x100000)
    lib = nat.lib
    c = _cfg(nat)
    assert nat.moe_ep_workspace_size(c, 1) >= nat.moe_workspace_size(c)
    assert nat.moe_ep_workspace_size(c, 2) > nat.moe_workspace_size(c)
    assert nat.moe_ep_workspace_size(c, c.E + 1) == 0          # more ranks than experts
    assert nat.moe_ep_workspace_size(c, 0) == 0
    # moe_permute_ep: the per-expert capacity is required
    assert lib.moe_permute_ep(ctypes.byref(c), fake, None, fake, fake, None, fake, fake, None,
                              None, fake, None) == nat.MOE_ERR_INVALID_ARG
    # moe_ep_expert_ffn: rank range, token count, row bound, offsets
    args = lambda world, rank, n, rows, off: (ctypes.byref(c), world, rank, n, rows, fake, off,
                                              fake, fake, fake, fake, fake, fake, None)
    assert lib.moe_ep_expert_ffn(*args(2, 2, 1, 1, fake)) == nat.MOE_ERR_INVALID_ARG
    assert lib.moe_ep_expert_ffn(*args(2, 0, c.N + 1, 1, fake)) == nat.MOE_ERR_INVALID_ARG
    assert lib.moe_ep_expert_ffn(*args(2, 0, 1, 2 * c.N * c.k + 1, fake)) == nat.MOE_ERR_INVALID_ARG
    assert lib.moe_ep_expert_ffn(*args(2, 0, 1, 1, None)) == nat.MOE_ERR_INVALID_ARG
    assert lib.moe_ep_expert_ffn(*args(c.E + 1, 0, 1, 1, fake)) == nat.MOE_ERR_UNSUPPORTED
    f32 = nat.make_config(c.N, 64, c.E, c.k, 64, dtype=nat.F32)
    assert lib.moe_ep_expert_ffn(ctypes.byref(f32), 1, 0, 1, 1, fake, fake, fake, fake, fake,
                                 fake, fake, fake, None) == nat.MOE_ERR_UNSUPPORTED
    assert lib.moe_ep_combine(ctypes.byref(c), fake, None, fake, fake, None) == nat.MOE_ERR_INVALID_ARG
    assert lib.moe_ep_combine(ctypes.byref(f32), fake, fake, fake, fake, None) == nat.MOE_ERR_UNSUPPORTED
    # the peer-memory dispatch and combine: the tables are required, bf16 only
    assert lib.moe_permute_ep_p2p(ctypes.byref(c), fake, fake, fake, fake, fake, None, fake, fake,
                                  None, None, fake, None) == nat.MOE_ERR_INVALID_ARG
    assert lib.moe_permute_ep_p2p(ctypes.byref(f32), fake, fake, fake, fake, fake, fake, fake,
                                  fake, None, None, fake, None) == nat.MOE_ERR_UNSUPPORTED
    p2p = lambda cfg, src_base, ws: lib.moe_ep_combine_p2p(
        ctypes.byref(cfg), fake, fake, fake, fake, src_base, fake, fake, fake, ws, None)
    assert p2p(c, None, fake) == nat.MOE_ERR_INVALID_ARG
    assert p2p(c, fake, None) == nat.MOE_ERR_INVALID_ARG
    assert p2p(f32, fake, fake) == nat.MOE_ERR_UNSUPPORTED
