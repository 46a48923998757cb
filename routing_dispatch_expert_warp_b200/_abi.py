"""ctypes mirror of include/moe.h: structs, prototypes and library loading.

Argument marshalling only.  The library is loaded from this package directory; if it is
missing or fails to load, every call raises -- there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
import threading

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe.so")

MOE_OK = 0
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED",
                3: "MOE_ERR_WORKSPACE", 4: "MOE_ERR_CUDA", 5: "MOE_ERR_TIMEOUT",
                6: "MOE_ERR_DEVICE_DATA"}
MOE_MAX_EXPERTS = 256
MOE_MAX_TOPK = 8

c_i32, c_i64, c_f32, c_f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_double
c_vp, c_sz = ctypes.c_void_p, ctypes.c_size_t


class MoeConfig(ctypes.Structure):
    _fields_ = [("T", c_i64), ("d_model", c_i64), ("d_ff", c_i64), ("E", c_i32), ("k", c_i32),
                ("gating", c_i32), ("layout", c_i32), ("dtype", c_i32),
                ("capacity_factor", c_f32), ("n_groups", c_i32), ("topk_groups", c_i32),
                ("bias_mode", c_i32), ("drop_policy", c_i32)]


class MoeLoadStats(ctypes.Structure):
    _fields_ = [("E", c_i32), ("k", c_i32), ("active_tokens", c_i64), ("capacity", c_i64),
                ("routed_total", c_i64), ("kept_total", c_i64), ("dropped", c_i64),
                ("tokens_with_drop", c_i64), ("tokens_fully_dropped", c_i64),
                ("p50", c_f64), ("p95", c_f64), ("p99", c_f64), ("max", c_f64),
                ("mean", c_f64), ("max_to_mean", c_f64), ("routed_max", c_f64),
                ("routed_max_to_mean", c_f64), ("top5pct_share", c_f64),
                ("dropped_by_rank", c_i64 * MOE_MAX_TOPK)]

    def as_dict(self) -> dict:
        d = {name: getattr(self, name) for name, _ in self._fields_}
        d["dropped_by_rank"] = list(self.dropped_by_rank)[: self.k]
        return d


class MoeLayerInputs(ctypes.Structure):
    _fields_ = [("x", c_vp), ("w_router", c_vp), ("logit_bias", c_vp),
                ("bias_row_stride", c_i64), ("w_gate", c_vp), ("w_up", c_vp), ("w_down", c_vp),
                ("w_router_split", c_vp)]


class MoeLayerBuffers(ctypes.Structure):
    _fields_ = [("logits", c_vp), ("topk_idx", c_vp), ("topk_w", c_vp),
                ("routed_counts", c_vp), ("kept_counts", c_vp), ("expert_offsets", c_vp),
                ("assign_row", c_vp), ("token_of_row", c_vp), ("x_perm", c_vp), ("h", c_vp),
                ("y_perm", c_vp), ("out", c_vp), ("stats", c_vp)]


class MoeEpConfig(ctypes.Structure):
    _fields_ = [("world", c_i32), ("rank", c_i32), ("ranks_per_node", c_i32),
                ("n_local", c_i32), ("expert_rank", c_vp), ("recv_rows", c_i64)]


MOE_MAX_RANKS = 64


class MoeEpStats(ctypes.Structure):
    _fields_ = [("world", c_i32), ("ranks_per_node", c_i32), ("nodes", c_i32),
                ("reserved", c_i32), ("total_assignments", c_i64),
                ("local_assignments", c_i64), ("remote_bytes", c_i64),
                ("cross_node_bytes", c_i64), ("local_fraction", c_f64),
                ("cross_node_fraction", c_f64), ("pair_bytes_p50", c_f64),
                ("pair_bytes_p99", c_f64), ("pair_bytes_max", c_f64),
                ("rank_load_max", c_f64), ("rank_load_mean", c_f64),
                ("rank_load_max_minus_mean", c_f64), ("rank_load_max_to_mean", c_f64),
                ("node_load_max_to_mean", c_f64),
                ("rank_load", c_i64 * MOE_MAX_RANKS), ("node_load", c_i64 * MOE_MAX_RANKS),
                ("bytes_sent", c_i64 * MOE_MAX_RANKS), ("bytes_recv", c_i64 * MOE_MAX_RANKS)]

    def as_dict(self) -> dict:
        d = {name: getattr(self, name) for name, _ in self._fields_}
        for key in ("rank_load", "bytes_sent", "bytes_recv"):
            d[key] = list(getattr(self, key))[: self.world]
        d["node_load"] = list(self.node_load)[: self.nodes]
        d.pop("reserved")
        return d


P = ctypes.POINTER
# name -> (restype, argtypes); every function declared in include/moe.h
PROTOTYPES = {
    "moe_workspace_size": (c_i32, [P(MoeConfig), P(c_sz)]),
    "moe_workspace_init": (c_i32, [c_vp, c_sz, c_vp]),
    "moe_capacity": (c_i64, [P(MoeConfig)]),
    "moe_max_rows": (c_i64, [P(MoeConfig)]),
    "moe_route": (c_i32, [P(MoeConfig), c_vp, c_vp, c_vp, c_i64, c_vp, c_vp, c_vp, c_vp, c_sz,
                          c_vp]),
    "moe_route_ex": (c_i32, [P(MoeConfig), c_vp, c_vp, c_vp, c_vp, c_i64, c_vp, c_vp, c_vp,
                             c_vp, c_sz, c_vp]),
    "moe_router_split_size": (c_i32, [P(MoeConfig), P(c_sz)]),
    "moe_router_split": (c_i32, [P(MoeConfig), c_vp, c_vp, c_sz, c_vp]),
    "moe_dispatch": (c_i32, [P(MoeConfig), c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp,
                             c_vp, c_sz, c_vp]),
    "moe_dispatch_scored": (c_i32, [P(MoeConfig), c_vp, c_vp, c_vp, c_vp, c_i64, c_vp, c_vp,
                                    c_vp, c_vp, c_vp, c_vp, c_vp, c_sz, c_vp]),
    "moe_dispatch_static_scratch": (c_i32, [P(MoeConfig), c_vp, c_vp, c_vp, c_vp, c_vp, c_vp,
                                            c_vp, c_vp, c_vp]),
    "moe_expert_ffn": (c_i32, [P(MoeConfig), c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp,
                               c_vp, c_sz, c_vp]),
    "moe_expert_ffn_gather": (c_i32, [P(MoeConfig), c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp,
                                      c_vp, c_vp, c_vp, c_sz, c_vp]),
    "moe_expert_ffn_combine": (c_i32, [P(MoeConfig), c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp,
                                       c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_sz, c_vp]),
    "moe_combine": (c_i32, [P(MoeConfig), c_vp, c_vp, c_vp, c_vp, c_vp]),
    "moe_load_stats": (c_i32, [P(MoeConfig), c_vp, c_vp, c_vp, c_vp, P(MoeLoadStats), c_vp]),
    "moe_pick_rank_counts": (c_i32, [P(MoeConfig), c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp,
                                     c_sz, c_vp]),
    "moe_load_stats_merge": (c_i32, [P(MoeConfig), c_vp, c_vp, c_vp, c_i32, c_vp,
                                     P(MoeLoadStats), c_vp]),
    "moe_layer_forward": (c_i32, [P(MoeConfig), P(MoeLayerInputs), P(MoeLayerBuffers), c_vp,
                                  c_sz, c_vp]),
    "moe_static_scratch_check": (c_i32, [c_vp]),
    "moe_check_device_error": (c_i32, [c_vp, c_sz, c_vp]),
    "moe_last_error": (ctypes.c_char_p, []),
    "moe_status_string": (ctypes.c_char_p, [c_i32]),
    "moe_set_wait_limit_ns": (None, [ctypes.c_uint64]),
    "moe_set_ffn_kernel": (c_i32, [c_i32]),
    "moe_selftest_bounded_wait": (c_i32, [c_vp, c_sz, c_vp]),
    "moe_ep_recv_rows_bound": (c_i64, [P(MoeConfig), P(MoeEpConfig)]),
    "moe_ep_put_counts": (c_i32, [P(MoeConfig), P(MoeEpConfig), c_vp, c_vp, c_vp]),
    "moe_ep_plan": (c_i32, [P(MoeConfig), P(MoeEpConfig), c_vp, c_vp, c_vp, c_vp, c_vp, c_vp,
                            c_vp, c_vp, c_sz, c_vp]),
    "moe_ep_dispatch": (c_i32, [P(MoeConfig), P(MoeEpConfig), c_vp, c_vp, c_vp, c_vp, c_vp,
                                c_sz, c_vp]),
    "moe_ep_expert_ffn": (c_i32, [P(MoeConfig), P(MoeEpConfig), c_vp, c_vp, c_vp, c_vp, c_vp,
                                  c_vp, c_vp, c_vp, c_vp, c_sz, c_vp]),
    "moe_ep_combine": (c_i32, [P(MoeConfig), P(MoeEpConfig), c_vp, c_vp, c_vp, c_vp, c_vp,
                               c_vp, c_sz, c_vp]),
    "moe_ep_stats": (c_i32, [P(MoeConfig), P(MoeEpConfig), c_vp, c_vp, P(MoeEpStats), c_vp]),
    "moe_ipc_handle": (c_i32, [c_vp, ctypes.c_char_p, P(c_i64)]),
    "moe_ipc_open": (c_i32, [ctypes.c_char_p, P(c_vp)]),
    "moe_ipc_close": (c_i32, [c_vp]),
    "moe_abi_version": (c_i32, []),
    "moe_kernel_launch_count": (ctypes.c_uint64, []),
}

_lib = None
_lock = threading.Lock()


class MoEError(RuntimeError):
    def __init__(self, status: int, message: str):
        self.status = status
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")


def lib() -> ctypes.CDLL:
    """The loaded libmoe.so.  Raises if the library has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(
                    f"{LIB_PATH} is missing: build it with "
                    "`python -m routing_dispatch_expert_warp_b200.build` (no fallback exists)")
            L = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in PROTOTYPES.items():
                fn = getattr(L, name)
                fn.restype = res
                fn.argtypes = args
            _lib = L
    return _lib


def check(status: int) -> None:
    if status != MOE_OK:
        msg = lib().moe_last_error().decode(errors="replace")
        raise MoEError(status, msg)
