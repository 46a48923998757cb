"""The C-ABI library without a GPU: it builds, loads, exports every declared entry point,
its structs match the ctypes mirror, and its host-side checks and sizes are right.
No kernel is launched here."""
import ctypes
import os
import re
import subprocess
import tempfile

import numpy as np
import pytest

from oracle import moe_oracle as O
from routing_dispatch_expert_warp_b200 import _abi, build as B
import routing_dispatch_expert_warp_b200 as M

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


@pytest.fixture(scope="module")
def lib():
    B.build()
    return _abi.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 15
    assert set(names) == set(_abi.PROTOTYPES), "ctypes prototypes and header disagree"
    nm = subprocess.run(["nm", "-D", "--defined-only", _abi.LIB_PATH], capture_output=True,
                        text=True, check=True).stdout
    exported = set(re.findall(r"\b(moe_[a-z0-9_]+)$", nm, flags=re.M))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        assert getattr(lib, n) is not None
    assert lib.moe_abi_version() == 5


def test_struct_layout_matches_header(tmp_path):
    prog = tmp_path / "layout.c"
    prog.write_text("""
#include <stdio.h>
#include <stddef.h>
#include "moe.h"
int main(void) {
  printf("%zu %zu %zu %zu\\n", sizeof(moe_config_t), sizeof(moe_load_stats_t),
         sizeof(moe_layer_inputs_t), sizeof(moe_layer_buffers_t));
  printf("%zu %zu %zu\\n", offsetof(moe_config_t, capacity_factor),
         offsetof(moe_load_stats_t, p50), offsetof(moe_load_stats_t, dropped_by_rank));
  printf("%zu %zu\\n", offsetof(moe_layer_inputs_t, bias_row_stride),
         offsetof(moe_layer_buffers_t, stats));
  printf("%zu %zu %zu %zu\\n", sizeof(moe_ep_config_t), sizeof(moe_ep_stats_t),
         offsetof(moe_ep_config_t, recv_rows), offsetof(moe_ep_stats_t, bytes_recv));
  return 0;
}
""")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(prog), "-o",
                    str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()
    got = [int(v) for v in out]
    want = [ctypes.sizeof(_abi.MoeConfig), ctypes.sizeof(_abi.MoeLoadStats),
            ctypes.sizeof(_abi.MoeLayerInputs), ctypes.sizeof(_abi.MoeLayerBuffers),
            _abi.MoeConfig.capacity_factor.offset, _abi.MoeLoadStats.p50.offset,
            _abi.MoeLoadStats.dropped_by_rank.offset, _abi.MoeLayerInputs.bias_row_stride.offset,
            _abi.MoeLayerBuffers.stats.offset,
            ctypes.sizeof(_abi.MoeEpConfig), ctypes.sizeof(_abi.MoeEpStats),
            _abi.MoeEpConfig.recv_rows.offset, _abi.MoeEpStats.bytes_recv.offset]
    assert got == want


@pytest.mark.parametrize("T,E,k,cf", [(64, 8, 2, 1.25), (16384, 256, 8, 1.0), (8192, 8, 2, 1.25),
                                      (10, 3, 1, 1.0), (10, 3, 1, 0.01), (4096, 8, 2, 0.0),
                                      (37, 5, 2, 0.7)])
def test_capacity_matches_oracle(lib, T, E, k, cf):
    cfg = M.make_config(T, 64, 64, E, k, capacity_factor=cf)
    C = O.capacity(float(np.float32(cf)), T, k, E)
    assert M.capacity(cfg) == (-1 if C is None else C)
    A = T * k
    assert M.max_rows(cfg) == (A if C is None else min(A, E * C))
    if C is not None:
        cfg.layout = M.PADDED
        assert M.max_rows(cfg) == E * C


def test_workspace_size_and_bad_configs(lib):
    cfg = M.make_config(4096, 4096, 14336, 8, 2)
    n = M.workspace_size(cfg)
    assert n >= 256 + 16 * 8 * 4 + 4096 * 8 * 4
    bad = [dict(E=0), dict(E=257), dict(k=0), dict(k=9), dict(T=0), dict(T=1 << 40),
           dict(d_model=12), dict(d_model=1 << 26), dict(d_ff=1 << 26), dict(gating=3),
           dict(layout=2), dict(dtype=7)]
    for b in bad:
        kw = dict(T=64, d_model=128, d_ff=256, E=8, k=2)
        kw.update({kk: v for kk, v in b.items() if kk in kw})
        c = M.make_config(**kw)
        for kk, v in b.items():
            if kk not in kw:
                setattr(c, kk, v)
        with pytest.raises(M.MoEError) as ei:
            M.workspace_size(c)
        assert ei.value.status == 1, b
    # k > E
    with pytest.raises(M.MoEError):
        M.workspace_size(M.make_config(64, 128, 256, 4, 5))
    # PADDED without a capacity
    with pytest.raises(M.MoEError):
        M.workspace_size(M.make_config(64, 128, 256, 8, 2, layout=M.PADDED))
    # group limits that cannot hold k experts, or groups that do not divide E
    with pytest.raises(M.MoEError):
        M.workspace_size(M.make_config(64, 128, 256, 8, 4, n_groups=4, topk_groups=1))
    with pytest.raises(M.MoEError):
        M.workspace_size(M.make_config(64, 128, 256, 8, 2, n_groups=3, topk_groups=1))
    for bad in (dict(bias_mode=2), dict(drop_policy=3)):
        with pytest.raises(M.MoEError):
            M.workspace_size(M.make_config(64, 128, 256, 8, 2, **bad))
    # pick-rank drops keep k count planes per block
    a = M.workspace_size(M.make_config(4096, 4096, 4096, 8, 2))
    b = M.workspace_size(M.make_config(4096, 4096, 4096, 8, 2, drop_policy=M.DROP_PICK_RANK))
    assert b - a == 16 * 8 * 4


def test_null_and_misaligned_pointers_rejected_on_host(lib):
    cfg = M.make_config(64, 128, 256, 8, 2, dtype=M.F32)
    ws_bytes = M.workspace_size(cfg)
    L = lib
    # NULL workspace
    st = L.moe_route(ctypes.byref(cfg), 16, 16, None, 0, None, 16, 16, None, ws_bytes, None)
    assert st == 1 and b"workspace" in L.moe_last_error()
    # workspace too small (aligned fake address; nothing is dereferenced on the host)
    st = L.moe_route(ctypes.byref(cfg), 16, 16, None, 0, None, 16, 16, 256, 16, None)
    assert st == 3
    # misaligned x
    st = L.moe_route(ctypes.byref(cfg), 17, 16, None, 0, None, 16, 16, 256, ws_bytes, None)
    assert st == 1 and b"aligned" in L.moe_last_error()
    # NULL outputs
    st = L.moe_dispatch(ctypes.byref(cfg), 16, 16, None, 16, 16, 16, 16, 16, 256, ws_bytes, None)
    assert st == 1
    st = L.moe_combine(ctypes.byref(cfg), 16, None, 16, 16, None)
    assert st == 1
    st = L.moe_load_stats(ctypes.byref(cfg), 16, 16, 16, None, None, None)
    assert st == 1
    # bf16 FFN needs multiples of 64
    cfg2 = M.make_config(64, 96, 256, 8, 2, dtype=M.BF16)
    st = L.moe_expert_ffn(ctypes.byref(cfg2), 16, 16, 16, 16, 16, 16, 16, 16, 256,
                          M.workspace_size(cfg2), None)
    assert st == 2
    assert L.moe_status_string(5) == b"MOE_ERR_TIMEOUT"


def test_score_drop_policy_host_checks(lib):
    """MOE_DROP_SCORE: dispatch needs the scores, the workspace holds the ranking scratch,
    the fixed-scratch dispatch refuses it; the counters check their pointers."""
    L = lib
    cfg = M.make_config(4096, 256, 256, 256, 8, capacity_factor=1.25, drop_policy=M.DROP_SCORE)
    base = M.make_config(4096, 256, 256, 256, 8, capacity_factor=1.25)
    A = 4096 * 8
    r256 = lambda b: -(-b // 256) * 256
    extra = 2 * r256(4 * A) + r256(4 * 256) + r256(4 * 257) + r256(8 * 256) + r256(8 * A)
    assert M.workspace_size(cfg) - M.workspace_size(base) == extra
    ws = M.workspace_size(cfg)
    c = ctypes.byref(cfg)
    st = L.moe_dispatch(c, 16, 16, 16, 16, 16, 16, 16, 16, 256, ws, None)
    assert st == 1 and b"moe_dispatch_scored" in L.moe_last_error()
    st = L.moe_dispatch_scored(c, 16, 16, None, None, 0, 16, 16, 16, 16, 16, 16, 256, ws, None)
    assert st == 1 and b"logits" in L.moe_last_error()
    st = L.moe_dispatch_scored(c, 16, 16, 16, 16, 3, 16, 16, 16, 16, 16, 16, 256, ws, None)
    assert st == 1 and b"bias_row_stride" in L.moe_last_error()
    st = L.moe_dispatch_scored(c, 16, 16, 16, None, 0, 16, 16, 16, 16, 16, 16, 256,
                               M.workspace_size(base), None)
    assert st == 3                       # the base workspace lacks the ranking scratch
    st = L.moe_dispatch_static_scratch(c, 16, 16, 16, 16, 16, 16, 16, 16, None)
    assert st == 2 and b"MOE_DROP_SCORE" in L.moe_last_error()
    for ptrs in ((None, 16, 16, 16, 16), (16, None, 16, 16, 16), (16, 16, None, 16, 16),
                 (16, 16, 16, None, 16), (16, 16, 16, 16, None)):
        idx, ar, r, k, d = ptrs
        st = L.moe_pick_rank_counts(c, idx, ar, None, r, k, d, 256, ws, None)
        assert st == 1 and b"NULL" in L.moe_last_error()


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(_abi, "_lib", None)
    monkeypatch.setattr(_abi, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        _abi.lib()


def test_ep_sizes_and_argument_checks(lib):
    """Expert-parallel host checks (no kernel runs): the receive-buffer bound and rejections."""
    cfg = M.make_config(4096, 256, 128, 256, 8, capacity_factor=1.0)
    C = O.capacity(1.0, 4096, 8, 256)
    ep = _abi.MoeEpConfig(world=8, rank=3, ranks_per_node=4, n_local=32, expert_rank=None,
                          recv_rows=0)
    assert lib.moe_ep_recv_rows_bound(ctypes.byref(cfg), ctypes.byref(ep)) == 8 * min(4096 * 8, 32 * C)
    dropless = M.make_config(100, 256, 128, 8, 2)
    ep1 = _abi.MoeEpConfig(world=4, rank=0, ranks_per_node=1, n_local=2, expert_rank=None,
                           recv_rows=0)
    assert lib.moe_ep_recv_rows_bound(ctypes.byref(dropless), ctypes.byref(ep1)) == 4 * 100 * 2
    ep1.n_local = 1     # a token picks an expert at most once
    assert lib.moe_ep_recv_rows_bound(ctypes.byref(dropless), ctypes.byref(ep1)) == 4 * 100 * 1
    for bad in (dict(world=0), dict(world=65), dict(rank=8), dict(rank=-1), dict(n_local=0),
                dict(n_local=257), dict(ranks_per_node=0)):
        e = _abi.MoeEpConfig(world=8, rank=3, ranks_per_node=1, n_local=32, expert_rank=None,
                             recv_rows=0)
        for key, val in bad.items():
            setattr(e, key, val)
        assert lib.moe_ep_recv_rows_bound(ctypes.byref(cfg), ctypes.byref(e)) == -2, bad
    # calls that would launch: a missing placement or buffer is refused on the host
    ep.recv_rows = 1024
    ws = ctypes.c_size_t(0)
    assert lib.moe_workspace_size(ctypes.byref(cfg), ctypes.byref(ws)) == 0
    st = lib.moe_ep_put_counts(ctypes.byref(cfg), ctypes.byref(ep), 16, 16, None)
    assert st == 1 and b"expert_rank" in lib.moe_last_error()
    ep.expert_rank = 16
    assert lib.moe_ep_put_counts(ctypes.byref(cfg), ctypes.byref(ep), None, 16, None) == 1
    assert lib.moe_ep_dispatch(ctypes.byref(cfg), ctypes.byref(ep), 17, 16, 16, 16, 256,
                               ws.value, None) == 1          # misaligned x
    assert lib.moe_ep_combine(ctypes.byref(cfg), ctypes.byref(ep), None, 16, 16, 16, 16, 256,
                              ws.value, None) == 1
    assert lib.moe_ep_stats(ctypes.byref(cfg), ctypes.byref(ep), None, 16, None, None) == 1
    assert lib.moe_ipc_handle(None, ctypes.create_string_buffer(64),
                              ctypes.byref(ctypes.c_int64())) == 1


def test_prototype_arity_matches_the_header():
    """Every ctypes prototype takes as many arguments as the header's declaration."""
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    decls = re.findall(r"\b(moe_[a-z0-9_]+)\s*\(([^;{)]*)\)\s*;", src)
    assert len(decls) == len(_abi.PROTOTYPES)
    for name, params in decls:
        params = " ".join(params.split())
        n = 0 if params in ("", "void") else params.count(",") + 1
        assert n == len(_abi.PROTOTYPES[name][1]), (name, n, len(_abi.PROTOTYPES[name][1]))


def test_ffn_kernel_choice_is_checked(lib):
    """moe_set_ffn_kernel takes the three schedules and refuses anything else (no GPU needed:
    the choice is host state read at the next launch)."""
    for kind in (1, 2, 0):                   # pairs, token-N, back to token-major (default)
        assert lib.moe_set_ffn_kernel(kind) == 0
    assert lib.moe_set_ffn_kernel(3) == 1    # MOE_ERR_INVALID_ARG
    assert lib.moe_set_ffn_kernel(-1) == 1
    assert b"moe_set_ffn_kernel" in lib.moe_last_error()


def test_router_split_sizes_and_checks(lib):
    """The split router weight: 2 E d bf16 values where the layer can take the tensor-core
    router (bf16, E > 32, d a multiple of 64; T does not matter), none otherwise; the
    argument checks run on the host before anything is enqueued."""
    L = lib
    big = M.make_config(256, 512, 128, 256, 8, dtype=M.BF16)
    small_t = M.make_config(16, 512, 128, 256, 8, dtype=M.BF16)
    assert M.router_split_size(big) == 2 * 256 * 512 * 2
    assert M.router_split_size(small_t) == M.router_split_size(big)
    for cfg in (M.make_config(256, 512, 128, 8, 2, dtype=M.BF16),      # E <= 32
                M.make_config(256, 512, 128, 256, 8, dtype=M.F32),     # fp32 layer
                M.make_config(256, 96, 128, 256, 8, dtype=M.BF16)):    # d % 64 != 0
        assert M.router_split_size(cfg) == 0
        st = L.moe_router_split(ctypes.byref(cfg), 16, 256, 1 << 20, None)
        assert st == 2 and b"tensor-core router" in L.moe_last_error()  # MOE_ERR_UNSUPPORTED
    n = M.router_split_size(big)
    assert L.moe_router_split(ctypes.byref(big), None, 256, n, None) == 1
    assert L.moe_router_split(ctypes.byref(big), 16, 258, n, None) == 1   # misaligned
    assert L.moe_router_split(ctypes.byref(big), 16, 256, n - 2, None) == 1
    assert b"split_bytes" in L.moe_last_error()
    ws_bytes = M.workspace_size(big)
    st = L.moe_route_ex(ctypes.byref(big), 16, 16, 258, None, 0, None, 16, 16, 256, ws_bytes,
                        None)
    assert st == 1 and b"w_router_split" in L.moe_last_error()
    st = L.moe_route_ex(ctypes.byref(big), 16, None, 256, None, 0, None, 16, 16, 256, ws_bytes,
                        None)
    assert st == 1   # w_router is required even with a split
