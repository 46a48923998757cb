"""Host-side rules of the library, checked in its own host code (no GPU): the tensor-core
router's split-K rule and the workspace layout.  Both are internal C++ functions of
libmoe.so, called here under their exported C++ names.

With fewer 128-token tiles than half the SMs, the router cuts each tile's K steps (2 d / 64:
x against the hi and then the lo term of W_r) into pieces, one block each, whose fp32 sums
the top-k kernel adds in piece order.  The rule lives in the library's host function
`moe::router_tc_splits` (exported by libmoe.so under its C++ name; without a GPU the library
takes 148 SMs, the B200's count).  Here it is called for every tile count and model width up
to 16384 and held to what the kernels need: an even number of K steps per piece (a piece
starts on a hi/lo chunk pair), no empty piece (an empty one would leave its accumulator
unwritten), at most 16 pieces of at least 4 steps, and no split once the tiles fill half the
GPU.  It must also agree with `moe_parity.router_tc_splits`, the rule the GPU tests use to
predict each layer's kernel launches.
"""
import ctypes

import pytest

import moe_parity as MP
from routing_dispatch_expert_warp_b200 import _abi, build as B
from routing_dispatch_expert_warp_b200 import workload as W

SMS = 148


class Shape(ctypes.Structure):
    """The library's checked layer shape (moe::Shape in csrc/moe_internal.h)."""
    _fields_ = [("T", ctypes.c_int64), ("d", ctypes.c_int64), ("f", ctypes.c_int64),
                ("E", ctypes.c_int), ("k", ctypes.c_int), ("gating", ctypes.c_int),
                ("layout", ctypes.c_int), ("dtype", ctypes.c_int), ("n_groups", ctypes.c_int),
                ("topk_groups", ctypes.c_int), ("bias_mode", ctypes.c_int),
                ("drop_policy", ctypes.c_int), ("C", ctypes.c_int64),
                ("max_rows", ctypes.c_int64), ("elem", ctypes.c_int64)]


@pytest.fixture(scope="module")
def host():
    B.build()
    lib = _abi.lib()
    splits = getattr(lib, "_ZN3moe16router_tc_splitsERKNS_5ShapeEPi")
    splits.argtypes = [ctypes.POINTER(Shape), ctypes.POINTER(ctypes.c_int)]
    splits.restype = ctypes.c_int
    uses = getattr(lib, "_ZN3moe24router_uses_tensor_coresERKNS_5ShapeE")
    uses.argtypes = [ctypes.POINTER(Shape)]
    uses.restype = ctypes.c_bool
    nbytes = getattr(lib, "_ZN3moe18router_split_bytesERKNS_5ShapeE")
    nbytes.argtypes = [ctypes.POINTER(Shape)]
    nbytes.restype = ctypes.c_size_t
    return splits, uses, nbytes


def _shape(T, d, E=256, k=8, dtype=1):
    return Shape(T=T, d=d, f=128, E=E, k=k, gating=1, layout=0, dtype=dtype, n_groups=0,
                 topk_groups=0, bias_mode=0, drop_policy=0, C=-1, max_rows=T * k,
                 elem=2 if dtype == 1 else 4)


def test_split_rule_over_every_tile_count_and_width(host):
    splits, _, _ = host
    per = ctypes.c_int(0)
    split_seen = 0
    for tiles in range(1, SMS // 2 + 3):
        for T in {128 * tiles - 127, 128 * tiles}:
            for d in range(64, 16384 + 1, 64):
                s = _shape(T, d)
                ks = splits(ctypes.byref(s), ctypes.byref(per))
                KB = 2 * d // 64
                if 2 * tiles >= SMS:
                    assert ks == 1, (T, d)
                if ks > 1:
                    split_seen += 1
                    p = per.value
                    assert p % 2 == 0 and p >= 4, (T, d, ks, p)
                    assert ks <= 16 and ks * tiles <= SMS, (T, d, ks)
                    assert (ks - 1) * p < KB <= ks * p, (T, d, ks, p)   # no empty piece
                shape = W.reduced(W.DSV3_PREFILL_ZIPF, T, d, 128)
                assert ks == MP.router_tc_splits(shape, SMS), (T, d)
    assert split_seen > 10000


def test_tensor_core_router_shapes_and_split_weight_size(host):
    _, uses, nbytes = host
    for T in (1, 128, 16384):
        for d in (64, 96, 7168):
            for E in (8, 32, 33, 256):
                for dtype in (0, 1):
                    s = _shape(T, d, E=E, k=min(8, E), dtype=dtype)
                    want = dtype == 1 and E > 32 and d % 64 == 0
                    assert uses(ctypes.byref(s)) == want, (T, d, E, dtype)
                    assert nbytes(ctypes.byref(s)) == (2 * E * d * 2 if want else 0)
                    shape = W.reduced(W.DSV3_PREFILL_ZIPF, T, d, 128).replace(
                        E=E, k=min(8, E), dtype=W.BF16 if dtype == 1 else W.F32)
                    assert MP.router_on_tensor_cores(shape) == want


class WsLayout(ctypes.Structure):
    """Offsets and sizes of the workspace sections (moe::WsLayout in csrc/moe_internal.h)."""
    _fields_ = [(n, ctypes.c_size_t) for n in (
        "status", "hist", "hist_bytes", "logits", "logits_bytes", "partials", "partials_bytes",
        "router_tc", "router_tc_bytes", "ep_base", "arrive", "score", "total")]


def test_workspace_sections_hold_what_the_kernels_index(host):
    """Every section of the workspace, as the library lays it out, is 256-byte aligned, does
    not overlap the next one, and holds what the kernels index in it: the status record, the
    per-256-token-block histograms (k planes under pick-rank drops), [T, E] fp32 logits, the
    router's scratch (lane-ordered W_r for E <= 32, the split-K partial sums [pieces, T, E]
    otherwise), the split router weight [E, 2 d] bf16, the EP send bases [E], the fused
    combine's counters [T, ceil(d / 256)], and 24 bytes per pick (plus per-expert tables) under
    score-priority drops.  The total is what moe_workspace_size reports."""
    import routing_dispatch_expert_warp_b200 as M
    splits, uses, _ = host
    lib = _abi.lib()
    layout = getattr(lib, "_ZN3moe16workspace_layoutERKNS_5ShapeE")
    layout.argtypes = [ctypes.POINTER(Shape)]
    layout.restype = WsLayout
    sgemm_splits = getattr(lib, "_ZN3moe13router_splitsERKNS_5ShapeE")
    sgemm_splits.argtypes = [ctypes.POINTER(Shape)]
    sgemm_splits.restype = ctypes.c_int
    per = ctypes.c_int(0)
    n = 0
    for T in (1, 127, 128, 4096, 9471, 9472, 16384):
        for d in (64, 96, 4096, 7168):
            for E in (1, 8, 16, 32, 33, 256):
                for k in sorted({1, min(2, E), min(8, E)}):
                    for dtype in (0, 1):
                        for policy in (0, 1, 2):
                            cfg = M.make_config(T, d, 128, E, k, dtype=dtype,
                                                capacity_factor=1.0, drop_policy=policy)
                            C = M.capacity(cfg)
                            s = Shape(T=T, d=d, f=128, E=E, k=k, gating=0, layout=0,
                                      dtype=dtype, n_groups=0, topk_groups=0, bias_mode=0,
                                      drop_policy=policy, C=C, max_rows=M.max_rows(cfg),
                                      elem=2 if dtype == 1 else 4)
                            w = layout(ctypes.byref(s))
                            assert w.total == M.workspace_size(cfg)
                            starts = [w.status, w.hist, w.logits, w.partials, w.router_tc,
                                      w.ep_base, w.arrive, w.score, w.total]
                            assert starts[0] == 0 and all(o % 256 == 0 for o in starts)
                            ext = [b - a for a, b in zip(starts, starts[1:])]
                            assert min(ext) >= 0
                            assert ext[0] >= 16                                  # DevStatus
                            planes = k if policy == 1 else 1
                            assert ext[1] >= -(-T // 256) * planes * E * 4
                            assert ext[2] >= T * E * 4
                            if E <= 32:
                                et = 8 if E <= 8 else (16 if E <= 16 else 32)
                                assert ext[3] >= -(-d // 256) * 256 * et * 4
                            else:
                                tc = uses(ctypes.byref(s))
                                parts = (splits(ctypes.byref(s), ctypes.byref(per)) if tc
                                         else sgemm_splits(ctypes.byref(s)))
                                if parts > 1:
                                    assert ext[3] >= parts * T * E * 4
                                if tc:
                                    assert ext[4] >= 2 * E * d * 2
                            assert ext[5] >= E * 4
                            assert ext[6] >= T * (-(-d // 256)) * 4
                            if policy == 2:
                                assert ext[7] >= T * k * (4 + 4 + 8) + E * (4 + 8) + (E + 1) * 4
                            n += 1
    assert n > 2000
