"""The tensor-core router's split-K rule, checked in the library's own host code (no GPU).

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
