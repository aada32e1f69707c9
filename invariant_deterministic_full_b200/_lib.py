"""ctypes binding of libbi.so (include/bi.h).  Argument marshalling only.

Every function of the C ABI is exposed under its own name on `lib`; the thin
wrappers in ops.py take torch tensors and call these.  The library must have
been built (invariant_deterministic_full_b200/build.py, or
__graft_entry__.build()); if it is missing, importing this module raises:
there is no fallback path.
"""
import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libbi.so")

BI_OK, BI_ERR_INVALID_ARG, BI_ERR_UNSUPPORTED, BI_ERR_WORKSPACE, BI_ERR_CAPACITY, BI_ERR_CUDA = range(6)
MODE_BF16, MODE_LAYERCAST, MODE_FP32 = 0, 1, 2
VARIANT_INVARIANT, VARIANT_FAST = 0, 1
DTYPE_BF16, DTYPE_F32 = 0, 1
EPI_NONE, EPI_SWIGLU, EPI_ROPE_KV_APPEND = 0, 1, 2
GU_INTERLEAVE = 16
ATTN_CHUNK = 256
VOCAB_CHUNK = 256
_STATUS = {1: "BI_ERR_INVALID_ARG", 2: "BI_ERR_UNSUPPORTED", 3: "BI_ERR_WORKSPACE", 4: "BI_ERR_CAPACITY",
           5: "BI_ERR_CUDA"}


class BiError(RuntimeError):
    def __init__(self, status, fn, msg):
        super().__init__(f"{fn}: {_STATUS.get(status, status)}: {msg}")
        self.status = status


P = ctypes.c_void_p
I = ctypes.c_int
F = ctypes.c_float
D = ctypes.c_double
SZ = ctypes.c_size_t


class KvLayout(ctypes.Structure):
    _fields_ = [("k", P), ("v", P), ("n_slots", I), ("n_layers", I), ("n_kv_heads", I), ("capacity", I),
                ("head_dim", I), ("dtype", I)]


class EpiArgs(ctypes.Structure):
    _fields_ = [("rope", P), ("rope_max_pos", I), ("q_out", P), ("kv", ctypes.POINTER(KvLayout)), ("layer", I),
                ("slot", P), ("pos", P), ("n_heads", I)]


class ModelDesc(ctypes.Structure):
    _fields_ = [("n_layers", I), ("hidden", I), ("n_heads", I), ("n_kv_heads", I), ("head_dim", I), ("ffn", I),
                ("vocab", I), ("eps", F), ("mode", I), ("variant", I), ("margin_threshold", F)]


class Weights(ctypes.Structure):
    _fields_ = [("embed", P), ("lm_head", P), ("final_norm", P), ("attn_norm", P), ("ffn_norm", P), ("w_qkv", P),
                ("w_o", P), ("w_gu", P), ("w_down", P), ("rope", P), ("rope_max_pos", I)]


class Batch(ctypes.Structure):
    _fields_ = [("n_tokens", I), ("ids", P), ("slot", P), ("pos", P), ("slot_host", P), ("pos_host", P),
                ("lm_row", P), ("n_lm", I), ("target", P)]


class StepOut(ctypes.Structure):
    _fields_ = [("logprob", P), ("lse", P), ("argmax", P), ("margin", P), ("recomputed", P), ("logits", P),
                ("h", P)]


# name -> (restype, argtypes); the same list the header declares
SIGNATURES = {
    "bi_last_error": (ctypes.c_char_p, []),
    "bi_version": (I, []),
    "bi_device_error": (I, [ctypes.POINTER(ctypes.c_uint), I]),
    "bi_num_sms": (I, [I]),
    "bi_launch_count": (ctypes.c_longlong, []),
    "bi_selftest_wait_timeout": (I, [P]),
    "bi_gemm_workspace_size": (SZ, [I, I, I, I, I]),
    "bi_gemm": (I, [P, I, P, P, I, I, I, I, I, I, I, ctypes.POINTER(EpiArgs), I, I, P, SZ, P]),
    "bi_rmsnorm": (I, [P, P, P, P, P, P, I, I, F, I, P]),
    "bi_rope_table_fill": (I, [P, I, I, D, P]),
    "bi_rope_kv_append": (I, [P, P, I, P, ctypes.POINTER(KvLayout), I, P, P, I, I, I, I, P]),
    "bi_attention_workspace_size": (SZ, [I, I, I, I]),
    "bi_attention": (I, [P, ctypes.POINTER(KvLayout), I, P, P, P, P, P, I, I, F, I, I, P, SZ, P]),
    "bi_lmhead_workspace_size": (SZ, [I, I, I, I]),
    "bi_lmhead_logprob": (I, [P, P, P, I, I, I, F, I, P, P, P, P, P, P, P, SZ, P]),
    "bi_lmhead_logprob_noalloc": (I, [P, P, P, I, I, I, F, I, P, P, P, P, P, P, P]),
    "bi_lmhead_split": (I, [P, I, I, I, P, P]),
    "bi_lmhead_logits_workspace_size": (SZ, [I, I]),
    "bi_lmhead_from_logits": (I, [P, I, I, I, P, F, P, P, P, P, P, P, SZ, P]),
    "bi_ctx_create": (I, [ctypes.POINTER(ModelDesc), ctypes.POINTER(Weights), ctypes.POINTER(KvLayout),
                          ctypes.POINTER(P)]),
    "bi_ctx_destroy": (I, [P]),
    "bi_decode_workspace_size": (SZ, [P, I, I, I]),
    "bi_decode_step": (I, [P, ctypes.POINTER(Batch), ctypes.POINTER(StepOut), P, SZ, P]),
    "bi_greedy_advance": (I, [P, P, P, I, P]),
    "bi_embed": (I, [P, P, I, I, I, I, P, P]),
    "bi_synth_fill_bf16": (I, [P, ctypes.c_int64, ctypes.c_int64, ctypes.c_uint64, D, I, I, P]),
}


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libbi.so is not built ({LIB_PATH}); run invariant_deterministic_full_b200/build.py")
    so = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(so, name)
        fn.restype = res
        fn.argtypes = args
    return so


lib = _load()


def check(status, fn):
    if status != BI_OK:
        raise BiError(status, fn, lib.bi_last_error().decode(errors="replace"))
