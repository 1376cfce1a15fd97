"""ctypes view of libsta.so (include/sta.h).  Loading fails loudly when the
library has not been built: there is no other implementation."""
import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# STA_LIB=debug selects libsta_debug.so, the build whose kernels check every
# list entry, token index and TMEM column (build.py --debug)
DEBUG_LIB_PATH = os.path.join(_HERE, "libsta_debug.so")
LIB_PATH = DEBUG_LIB_PATH if os.environ.get("STA_LIB") == "debug" else os.path.join(
    _HERE, "libsta.so")

# sta_status
STA_OK = 0
STA_ERR_ARG = -1
STA_ERR_UNSUPPORTED = -2
STA_ERR_CAPACITY = -3
STA_ERR_CUDA = -4
STA_ERR_WORKSPACE = -5

# device status bits
STA_DEV_TIMEOUT = 0x1
STA_DEV_CAPACITY = 0x2
STA_DEV_EMPTY_ROW = 0x4
STA_DEV_BAD_INDEX = 0x8
STA_DEV_RANGE = 0x10
STA_DEV_DEBUG = 0x20

STA_BF16, STA_F32 = 0, 1
(STA_SEL_RADIAL, STA_SEL_ENTROPY, STA_SEL_IBCS_SIP, STA_SEL_ROUTED, STA_SEL_TRA_TOKEN,
 STA_SEL_DYNRAD) = 0, 1, 2, 3, 4, 5
STA_ATTN_LISTS, STA_ATTN_ROUTED = 0, 1


class Problem(ctypes.Structure):
    _fields_ = [("heads", ctypes.c_int), ("F", ctypes.c_int), ("H", ctypes.c_int),
                ("W", ctypes.c_int), ("d", ctypes.c_int), ("dtype", ctypes.c_int)]


class SelectorParams(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int), ("block_q", ctypes.c_int), ("kv_unit", ctypes.c_int),
                ("radial_w0", ctypes.c_int), ("radial_w_off", ctypes.c_int),
                ("radial_full_df", ctypes.c_int),
                ("ent_alpha", ctypes.c_float), ("ent_beta", ctypes.c_float),
                ("ent_r_lo", ctypes.c_int), ("ent_r_hi", ctypes.c_int),
                ("ent_tile_h", ctypes.c_int), ("ent_tile_w", ctypes.c_int),
                ("km_k", ctypes.c_int), ("km_iters", ctypes.c_int),
                ("sample_frac", ctypes.c_float), ("seed", ctypes.c_uint64),
                ("dense_frac", ctypes.c_float), ("win_f", ctypes.c_int),
                ("win_h", ctypes.c_int), ("win_w", ctypes.c_int),
                ("difficulty", ctypes.c_void_p),
                ("tra_tau", ctypes.c_float), ("tra_gamma", ctypes.c_float),
                ("tra_vote", ctypes.c_int), ("tra_entropy", ctypes.c_void_p),
                ("dyn_mode", ctypes.c_int), ("dyn_ratio", ctypes.c_float),
                ("dyn_threshold", ctypes.c_float),
                ("layout_tile_h", ctypes.c_int), ("layout_tile_w", ctypes.c_int)]


class BlockLists(ctypes.Structure):
    _fields_ = [("idx", ctypes.c_void_p), ("cnt", ctypes.c_void_p), ("logw", ctypes.c_void_p),
                ("cap", ctypes.c_int32), ("head_shared", ctypes.c_int32),
                ("required_cap", ctypes.c_void_p), ("routed_ids", ctypes.c_void_p),
                ("routed_flag", ctypes.c_void_p), ("n_routed", ctypes.c_int32),
                ("entropy", ctypes.c_void_p), ("radius", ctypes.c_void_p)]


class AttnParams(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int), ("block_q", ctypes.c_int), ("kv_unit", ctypes.c_int),
                ("scale", ctypes.c_float), ("win_f", ctypes.c_int), ("win_h", ctypes.c_int),
                ("win_w", ctypes.c_int)]


# every function include/sta.h declares, with its ctypes signature
SIGNATURES = {
    "sta_build_blocks_workspace": (ctypes.c_size_t, [ctypes.POINTER(Problem),
                                                     ctypes.POINTER(SelectorParams)]),
    "sta_build_blocks_rows": (ctypes.c_int, [ctypes.POINTER(Problem),
                                             ctypes.POINTER(SelectorParams)]),
    "sta_build_blocks": (ctypes.c_int, [ctypes.POINTER(Problem), ctypes.POINTER(SelectorParams),
                                        ctypes.c_void_p, ctypes.c_void_p,
                                        ctypes.POINTER(BlockLists), ctypes.c_void_p,
                                        ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p]),
    "sta_attn_workspace": (ctypes.c_size_t, [ctypes.POINTER(Problem)]),
    "sta_sparse_attn_fwd": (ctypes.c_int, [ctypes.POINTER(Problem), ctypes.POINTER(AttnParams),
                                           ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                           ctypes.POINTER(BlockLists), ctypes.c_void_p,
                                           ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p,
                                           ctypes.c_void_p]),
    "sta_sparse_attn_fwd_noalloc": (ctypes.c_int, [ctypes.POINTER(Problem),
                                                   ctypes.POINTER(AttnParams), ctypes.c_void_p,
                                                   ctypes.c_void_p, ctypes.c_void_p,
                                                   ctypes.POINTER(BlockLists), ctypes.c_void_p,
                                                   ctypes.c_void_p, ctypes.c_void_p]),
    "sta_dense_attn_fwd": (ctypes.c_int, [ctypes.POINTER(Problem), ctypes.c_void_p,
                                          ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float,
                                          ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                          ctypes.c_void_p, ctypes.c_void_p]),
    "sta_dense_attn_entropy_fwd": (ctypes.c_int, [ctypes.POINTER(Problem), ctypes.c_void_p,
                                                  ctypes.c_void_p, ctypes.c_void_p,
                                                  ctypes.c_float, ctypes.c_void_p,
                                                  ctypes.c_void_p, ctypes.c_void_p,
                                                  ctypes.c_size_t, ctypes.c_void_p,
                                                  ctypes.c_void_p]),
    "sta_permute_tokens": (ctypes.c_int, [ctypes.POINTER(Problem), ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                                          ctypes.c_void_p]),
    "sta_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "sta_dev_status_string": (ctypes.c_char_p, [ctypes.c_int32]),
    "sta_version": (ctypes.c_int, []),
    "sta_debug_build": (ctypes.c_int, []),
    "sta_selftest_index_check": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                                ctypes.c_void_p, ctypes.c_void_p]),
    "sta_last_cuda_error": (ctypes.c_char_p, []),
    "sta_selftest_bounded_wait": (ctypes.c_int, [ctypes.c_uint64, ctypes.c_void_p,
                                                 ctypes.c_void_p, ctypes.c_void_p]),
}

_lib = None


def load(path=LIB_PATH):
    """Load libsta.so and attach signatures.  Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        flag = " --debug" if path == DEBUG_LIB_PATH else ""
        raise ImportError(
            f"{path} is missing: build it with "
            f"`python sparse_spatiotemporal_attention_video_b200/build.py{flag}` (nvcc, sm_100a)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


class StaError(RuntimeError):
    def __init__(self, code, what):
        self.code = code
        lib = load()
        msg = f"{what}: {lib.sta_status_string(code).decode()} ({code})"
        if code == STA_ERR_CUDA:
            msg += f": {lib.sta_last_cuda_error().decode()}"
        super().__init__(msg)


def check(code, what):
    if code != STA_OK:
        raise StaError(code, what)
