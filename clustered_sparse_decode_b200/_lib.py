"""ctypes declarations of the C ABI in include/mpattn.h (argument marshalling only)."""
import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmpattn.so")

MP_OK, MP_EINVAL, MP_ENOSPC, MP_ECUDA, MP_EUNSUPPORTED, MP_EDEVICE = range(6)
MP_F32, MP_BF16 = 0, 1
MP_INIT_KMEANSPP, MP_INIT_STRIDE = 0, 1
MP_NO_APPROX = 1
MP_STATIC_SCRATCH_BYTES = 32 << 20

EXPORTS = ["mp_workspace_size", "mp_index_init", "mp_cluster_build", "mp_cluster_update", "mp_cluster_assign",
           "mp_decode", "mp_dense_decode",
           "mp_decode_static",
           "mp_index_export", "mp_index_import", "mp_check_device_error", "mp_decode_phases", "mp_status_str"]


class MpConfig(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("kv_heads", ctypes.c_int32), ("q_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("max_tokens", ctypes.c_int32),
                ("tokens_per_centroid", ctypes.c_int32), ("block_tokens", ctypes.c_int32),
                ("levels", ctypes.c_int32), ("coarse_tokens_per_centroid", ctypes.c_int32),
                ("kmeans_iters", ctypes.c_int32), ("update_interval", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("init", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("seed", ctypes.c_uint64)]


class MpIndex(ctypes.Structure):
    _fields_ = [("cfg", MpConfig), ("n_tokens", ctypes.c_int64), ("n_clustered", ctypes.c_int64),
                ("blocks_max", ctypes.c_int32), ("slots_per_block", ctypes.c_int32), ("slots", ctypes.c_int32),
                ("coarse_per_block", ctypes.c_int32), ("coarse_slots", ctypes.c_int32), ("device", ctypes.c_int32),
                ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
                ("layout", ctypes.c_uint64 * 24)]


class MpIndexView(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("Kc", "Vc", "off", "Kp", "Vp", "perm", "assign", "Kcc", "Vcc", "coff")]


class MpDecodeParams(ctypes.Structure):
    _fields_ = [("budget", ctypes.c_int32), ("coarse_budget", ctypes.c_int32), ("scale", ctypes.c_float),
                ("flags", ctypes.c_uint32), ("n_split", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("sel_mask_out", ctypes.c_void_p), ("coarse_sel_mask_out", ctypes.c_void_p),
                ("scores_out", ctypes.c_void_p), ("coarse_scores_out", ctypes.c_void_p),
                ("phase_events", ctypes.c_void_p), ("n_phase_events", ctypes.c_int32),
                ("reserved2", ctypes.c_int32)]


_lib = None


class MpError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__(f"{where}: {status_str(status)} (status {status})")


def load():
    """Load libmpattn.so (built by clustered_sparse_decode_b200.build); raise if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"CUDA library not built: {LIB_PATH} is missing "
                           "(run `python -m clustered_sparse_decode_b200.build`)")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    sig = {
        "mp_workspace_size": [P(MpConfig), P(sz), P(sz)],
        "mp_index_init": [P(MpConfig), vp, sz, P(MpIndex), vp],
        "mp_cluster_build": [P(MpIndex), vp, vp, i32, vp, vp],
        "mp_cluster_update": [P(MpIndex), vp, vp, i32, P(i32), vp],
        "mp_cluster_assign": [P(MpIndex), vp, i32, vp, vp],
        "mp_decode": [P(MpIndex), vp, vp, P(MpDecodeParams), vp, sz, vp],
        "mp_decode_static": [P(MpIndex), vp, vp, P(MpDecodeParams), vp],
        "mp_dense_decode": [P(MpConfig), vp, vp, i32, vp, vp, ctypes.c_float, vp],
        "mp_index_export": [P(MpIndex), P(MpIndexView)],
        "mp_index_import": [P(MpIndex), P(MpIndexView), i64, i64, vp],
        "mp_check_device_error": [P(MpIndex), P(i32), vp],
    }
    for name, args in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = ctypes.c_int
    lib.mp_decode_phases.argtypes = [P(MpIndex)]
    lib.mp_decode_phases.restype = ctypes.c_char_p
    lib.mp_status_str.argtypes = [ctypes.c_int]
    lib.mp_status_str.restype = ctypes.c_char_p
    _lib = lib
    return lib


def status_str(status):
    return load().mp_status_str(status).decode()


def check(status, where):
    if status != MP_OK:
        raise MpError(status, where)
