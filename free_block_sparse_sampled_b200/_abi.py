"""ctypes mirror of include/sparsepr.h (argument marshalling only)."""

from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsparsepr.so")

SPARSEPR_OK = 0
STATUS_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "WORKSPACE_TOO_SMALL",
                4: "CUDA_ERROR", 5: "TIMEOUT", 6: "NUMERIC"}
BF16, F32 = 0, 1
FLAG_DEBUG_EXPORT = 1
FLAG_SIMT_ATTENTION = 2
FLAG_WARM_START = 4
FLAG_SEMANTIC_KEYS = 8
FLAG_SEMANTIC_QUERIES = 16
PROBES = {"stratified": 0, "random": 1, "uniform": 2}
CORRECTIONS = {"full": 0, "diagonal": 1, "scalar": 2, "mean": 3}

EXPORTED = ["sparsepr_status_string", "sparsepr_validate", "sparsepr_workspace_size",
            "sparsepr_partition", "sparsepr_route", "sparsepr_attention", "sparsepr_probe_fit",
            "sparsepr_apply", "sparsepr_call", "sparsepr_last_error_string", "sparsepr_get_device_status",
            "sparsepr_probe_fit_static", "sparsepr_partition_warm", "sparsepr_debug_stall_attention"]

# size of the static scratch array behind sparsepr_probe_fit_static
FIT_STATIC_SCRATCH_BYTES = 8 << 20

P = ctypes.c_void_p


class Params(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("N", ctypes.c_int32), ("d", ctypes.c_int32),
                ("T", ctypes.c_int32), ("Y", ctypes.c_int32), ("X", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("density", ctypes.c_double), ("M", ctypes.c_int32),
                ("Ms", ctypes.c_int32), ("lambda_", ctypes.c_double), ("Cq", ctypes.c_int32),
                ("Ck", ctypes.c_int32), ("rK", ctypes.c_int32), ("rQ", ctypes.c_int32),
                ("kmeans_iters", ctypes.c_int32), ("kmeans_tol", ctypes.c_double),
                ("seed", ctypes.c_uint64), ("block", ctypes.c_int32), ("eps_rms", ctypes.c_float),
                ("eps_std", ctypes.c_float), ("flags", ctypes.c_int32), ("probe_select", ctypes.c_int32),
                ("correction", ctypes.c_int32), ("residual_rank", ctypes.c_int32), ("Hkv", ctypes.c_int32)]


PARTITION_FIELDS = ["Qp", "Kp", "Vp", "q_label", "kv_label", "perm_q", "perm_kv", "pos_q", "q_offsets",
                    "kv_offsets", "n_groups", "kmeans_iters_run", "q_centroid", "k_centroid",
                    "v_centroid", "q_dist", "F_K", "F_Q", "phi_K", "phi_Q", "kv_centres", "q_centres",
                    "debug_kv_scores", "debug_q_scores", "debug_kv_hist", "debug_q_hist"]
ROUTE_FIELDS = ["score", "mask", "sel_count", "sel_groups", "pairs", "probe_idx", "probe_group",
                "probe_weight", "probe_alloc"]
FIT_FIELDS = ["B", "mu_x", "sigma", "mu_r"]


class PartitionOut(ctypes.Structure):
    _fields_ = [(n, P) for n in PARTITION_FIELDS]


WARM_FIELDS = ["F_K", "F_Q", "k_centroid", "q_centroid", "n_groups"]


class WarmState(ctypes.Structure):
    _fields_ = [(n, P) for n in WARM_FIELDS]


class RouteOut(ctypes.Structure):
    _fields_ = [(n, P) for n in ROUTE_FIELDS]


class FitOut(ctypes.Structure):
    _fields_ = [(n, P) for n in FIT_FIELDS]


class Stats(ctypes.Structure):
    _fields_ = [("ms_partition", ctypes.c_float), ("ms_route", ctypes.c_float),
                ("ms_attention", ctypes.c_float), ("ms_fit", ctypes.c_float),
                ("ms_apply", ctypes.c_float), ("ms_total", ctypes.c_float),
                ("pairs_route", ctypes.c_int64), ("pairs_exec", ctypes.c_int64),
                ("pairs_visited", ctypes.c_int64), ("rho_exec", ctypes.c_double),
                ("launches", ctypes.c_int64)]


_LIB = None


def lib() -> ctypes.CDLL:
    """The loaded C library; raises if it has not been built (no fallback)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"SparsePR CUDA library not built: {LIB_PATH} is missing "
                               "(run python -m free_block_sparse_sampled_b200.build)")
        L = ctypes.CDLL(LIB_PATH)
        L.sparsepr_status_string.restype = ctypes.c_char_p
        L.sparsepr_status_string.argtypes = [ctypes.c_int32]
        L.sparsepr_validate.restype = ctypes.c_int32
        L.sparsepr_validate.argtypes = [ctypes.POINTER(Params)]
        L.sparsepr_workspace_size.restype = ctypes.c_size_t
        L.sparsepr_workspace_size.argtypes = [ctypes.POINTER(Params)]
        L.sparsepr_partition.restype = ctypes.c_int32
        L.sparsepr_partition.argtypes = [ctypes.POINTER(Params), P, P, P, ctypes.POINTER(PartitionOut), P,
                                         ctypes.c_size_t, P]
        L.sparsepr_partition_warm.restype = ctypes.c_int32
        L.sparsepr_partition_warm.argtypes = [ctypes.POINTER(Params), P, P, P, ctypes.POINTER(WarmState),
                                              ctypes.POINTER(PartitionOut), P, ctypes.c_size_t, P]
        L.sparsepr_route.restype = ctypes.c_int32
        L.sparsepr_route.argtypes = [ctypes.POINTER(Params), ctypes.POINTER(PartitionOut),
                                     ctypes.POINTER(RouteOut), P, ctypes.c_size_t, P]
        L.sparsepr_attention.restype = ctypes.c_int32
        L.sparsepr_attention.argtypes = [ctypes.POINTER(Params), ctypes.POINTER(PartitionOut),
                                         ctypes.POINTER(RouteOut), P, P, P, P, ctypes.c_size_t, P]
        L.sparsepr_probe_fit.restype = ctypes.c_int32
        L.sparsepr_probe_fit.argtypes = [ctypes.POINTER(Params), ctypes.POINTER(PartitionOut),
                                         ctypes.POINTER(RouteOut), P, P, ctypes.POINTER(FitOut), P,
                                         ctypes.c_size_t, P]
        L.sparsepr_apply.restype = ctypes.c_int32
        L.sparsepr_apply.argtypes = [ctypes.POINTER(Params), ctypes.POINTER(PartitionOut),
                                     ctypes.POINTER(RouteOut), P, P, ctypes.POINTER(FitOut), P, P,
                                     ctypes.c_size_t, P]
        L.sparsepr_call.restype = ctypes.c_int32
        L.sparsepr_call.argtypes = [ctypes.POINTER(Params), P, P, P, P, ctypes.POINTER(Stats), P,
                                    ctypes.c_size_t, P]
        L.sparsepr_last_error_string.restype = ctypes.c_char_p
        L.sparsepr_last_error_string.argtypes = []
        L.sparsepr_get_device_status.restype = ctypes.c_int32
        L.sparsepr_get_device_status.argtypes = [P, P, ctypes.POINTER(ctypes.c_int32)]
        L.sparsepr_probe_fit_static.restype = ctypes.c_int32
        L.sparsepr_probe_fit_static.argtypes = [ctypes.POINTER(Params), ctypes.POINTER(PartitionOut),
                                                ctypes.POINTER(RouteOut), P, P, ctypes.POINTER(FitOut), P, P]
        L.sparsepr_debug_stall_attention.restype = None
        L.sparsepr_debug_stall_attention.argtypes = [ctypes.c_uint32]
        _LIB = L
    return _LIB


class SparsePRError(RuntimeError):
    def __init__(self, fn: str, status: int):
        msg = f"{fn} failed: {STATUS_NAMES.get(status, status)}"
        if status == 4 and _LIB is not None:
            msg += f" ({_LIB.sparsepr_last_error_string().decode()})"
        super().__init__(msg)
        self.status = status


def check(fn: str, status: int) -> None:
    if status != SPARSEPR_OK:
        raise SparsePRError(fn, status)
