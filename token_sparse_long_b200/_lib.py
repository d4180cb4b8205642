"""ctypes declarations of the C ABI in include/jenga.h (argument marshalling only)."""
import ctypes
import os
from ctypes import POINTER, c_char_p, c_float, c_int, c_int64, c_size_t, c_uint32, c_uint64, c_void_p

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libjenga.so")


class JengaError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"{status_name(status)}: {msg}")
        self.status = status


STATUS = {0: "JENGA_OK", 1: "JENGA_EINVAL", 2: "JENGA_EUNSUPPORTED", 3: "JENGA_ECUDA", 4: "JENGA_ETIMEOUT",
          5: "JENGA_EWORKSPACE", 6: "JENGA_EINTERNAL"}
EINVAL, EUNSUPPORTED, ECUDA, ETIMEOUT, EWORKSPACE, EINTERNAL = 1, 2, 3, 4, 5, 6
F32, BF16 = 0, 1
SCORE_SOFTMAX_MASS, SCORE_PAPER_BLOCKMAX = 0, 1
SELECT_MEAN_GE, SELECT_TOPK_FRAC, SELECT_ABS_GE, SELECT_TOPK = 0, 1, 2, 3


def status_name(s):
    return STATUS.get(int(s), f"status {s}")


class LayerWeights(ctypes.Structure):
    _fields_ = [("hidden", c_int), ("heads", c_int), ("head_dim", c_int), ("ffn", c_int),
                ("rms_eps", c_float), ("rope_theta", c_float),
                ("attn_norm", c_void_p), ("mlp_norm", c_void_p),
                ("wq", c_void_p), ("wk", c_void_p), ("wv", c_void_p), ("wo", c_void_p),
                ("wg", c_void_p), ("wu", c_void_p), ("wd", c_void_p)]


class Lora(ctypes.Structure):
    _fields_ = [("rank", c_int), ("scale", c_float),
                ("aq", c_void_p), ("bq", c_void_p), ("av", c_void_p), ("bv", c_void_p)]


class LoraGrads(ctypes.Structure):
    _fields_ = [("daq", c_void_p), ("dbq", c_void_p), ("dav", c_void_p), ("dbv", c_void_p)]


# name -> (restype, argtypes)
_SIGS = {
    "jenga_status_string": (c_char_p, [c_int]),
    "jenga_last_error": (c_size_t, [c_char_p, c_size_t]),
    "jenga_check_device_status": (c_int, [c_void_p, POINTER(c_uint32)]),
    "jenga_set_wait_budget_ns": (c_int, [c_uint64]),
    "jenga_version": (c_char_p, []),
    "jenga_profile_enable": (c_int, [c_int]),
    "jenga_profile_report": (c_size_t, [c_char_p, c_size_t]),
    "jenga_score_workspace_bytes": (c_size_t, [c_int, c_int, c_int, c_int, c_int]),
    "jenga_score_blocks": (c_int, [c_void_p, c_int64, c_void_p, c_int64, c_int, c_int, c_int, c_int, c_int, c_int,
                                   c_int, c_int, c_void_p, c_void_p, c_size_t, c_void_p]),
    "jenga_score_blocks_noalloc_max_bytes": (c_size_t, []),
    "jenga_score_blocks_noalloc": (c_int, [c_void_p, c_int64, c_void_p, c_int64, c_int, c_int, c_int, c_int, c_int,
                                           c_int, c_int, c_int, c_void_p, c_void_p]),
    "jenga_select_workspace_bytes": (c_size_t, [c_int, c_int]),
    "jenga_select": (c_int, [c_void_p, c_int, c_int, c_int, c_float, c_void_p, c_void_p, c_void_p, c_void_p,
                             c_size_t, c_void_p]),
    "jenga_gather": (c_int, [c_void_p, c_int64, c_int, c_int, c_int, c_int, c_void_p, c_void_p, c_int, c_void_p,
                             c_int64, c_int, c_void_p]),
    "jenga_scatter_add": (c_int, [c_void_p, c_int64, c_void_p, c_int64, c_int, c_int, c_int, c_int, c_void_p,
                                  c_void_p, c_float, c_int, c_int, c_void_p]),
    "jenga_scale_rows": (c_int, [c_void_p, c_int64, c_int, c_int, c_int, c_void_p, c_int, c_float, c_int, c_void_p]),
    "jenga_layer_pack_bytes": (c_size_t, [POINTER(LayerWeights), POINTER(Lora)]),
    "jenga_layer_pack": (c_int, [POINTER(LayerWeights), POINTER(Lora), c_void_p, c_size_t, c_void_p]),
    "jenga_layer_score_qk_workspace_bytes": (c_size_t, [POINTER(LayerWeights), c_int, c_int]),
    "jenga_layer_score_qk": (c_int, [POINTER(LayerWeights), POINTER(Lora), c_void_p, c_void_p, c_int, c_int,
                                     c_void_p, c_void_p, c_size_t, c_void_p]),
    "jenga_layer_saved_bytes": (c_size_t, [POINTER(LayerWeights), c_int, c_int, c_int]),
    "jenga_layer_fwd_workspace_bytes": (c_size_t, [POINTER(LayerWeights), c_int, c_int, c_int]),
    "jenga_sparse_layer_fwd": (c_int, [POINTER(LayerWeights), POINTER(Lora), c_void_p, c_void_p, c_int, c_int, c_int,
                                       c_void_p, c_void_p, c_int, c_void_p, c_size_t, c_void_p, c_size_t, c_void_p]),
    "jenga_sparse_layer_fwd_qk": (c_int, [POINTER(LayerWeights), POINTER(Lora), c_void_p, c_void_p, c_int, c_int, c_int,
                                          c_void_p, c_void_p, c_int, c_void_p, c_int64, c_void_p, c_size_t, c_void_p,
                                          c_size_t, c_void_p]),
    "jenga_sparse_layer_fwd_mlp": (c_int, [POINTER(LayerWeights), POINTER(Lora), c_void_p, c_void_p, c_int, c_int,
                                           c_int, c_void_p, c_void_p, c_int, c_void_p, c_int64, c_int, c_float,
                                           c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p, c_size_t,
                                           c_void_p]),
    "jenga_layer_bwd_workspace_bytes": (c_size_t, [POINTER(LayerWeights), c_int, c_int, c_int, c_int]),
    "jenga_sparse_layer_bwd": (c_int, [POINTER(LayerWeights), POINTER(Lora), c_void_p, c_void_p, c_int, c_int, c_int,
                                       c_void_p, c_void_p, c_int, c_void_p, c_size_t, POINTER(LoraGrads), c_int,
                                       c_void_p, c_size_t, c_void_p]),
    "jenga_predict_workspace_bytes": (c_size_t, [c_int, c_int, c_int, c_int]),
    "jenga_lm_loss_workspace_bytes": (c_size_t, [c_int, c_int, c_int, c_int]),
    "jenga_mlp_block_scores": (c_int, [c_void_p, c_int64, c_int, c_int, c_void_p, c_int, c_void_p, c_void_p]),
    "jenga_compose_block_indices": (c_int, [c_void_p, c_int, c_void_p, c_void_p, c_int, c_void_p, c_void_p]),
    "jenga_predict_qk_workspace_bytes": (c_size_t, [c_int, c_int, c_int, c_int, c_int]),
    "jenga_predict_blocks_qk": (c_int, [c_void_p, c_int, c_int, c_int, c_int, c_void_p, c_void_p, c_void_p, c_void_p,
                                        c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_void_p, c_void_p, c_size_t,
                                        c_void_p]),
    "jenga_lm_loss_segmented": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_void_p, c_void_p,
                                        c_void_p, c_size_t, c_void_p]),
    "jenga_predict_blocks": (c_int, [c_void_p, c_int, c_int, c_int, c_int, c_void_p, c_void_p, c_void_p, c_void_p,
                                     c_int, c_void_p, c_void_p, c_size_t, c_void_p]),
    "jenga_test_gemm": (c_int, [c_void_p, c_int64, c_void_p, c_int64, c_int, c_int, c_int, c_void_p, c_int64, c_int,
                                c_int, c_void_p]),
    "jenga_test_exp2": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_void_p]),
    "jenga_test_wait_timeout": (c_int, [c_void_p]),
}

_lib = None


def load():
    """Load libjenga.so (built in-tree).  Raises if it is missing: there is no fallback."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m token_sparse_long_b200.build` "
                              "(nvcc, sm_100a); the library has no CPU or PyTorch fallback")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _lib = lib
    return _lib


def exported_symbols():
    return list(_SIGS)


def last_error():
    lib = load()
    buf = ctypes.create_string_buffer(2048)
    lib.jenga_last_error(buf, 2048)
    return buf.value.decode(errors="replace")


def check(status):
    if status != 0:
        raise JengaError(status, last_error())
