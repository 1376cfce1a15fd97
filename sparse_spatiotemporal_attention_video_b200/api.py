"""Python binding of the C ABI: the same entry points, argument marshalling
only.  Tensors are passed as device pointers (tensor.data_ptr()), the stream
as torch's current CUDA stream unless one is given.  Every step of the path
runs in libsta.so's kernels; there is no other implementation."""
import ctypes

import torch

from . import _lib
from ._lib import AttnParams, BlockLists, Problem, SelectorParams, check


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if isinstance(x, torch.Tensor):
        # the library reads dense row-major buffers from the base pointer
        if not x.is_contiguous():
            raise ValueError("libsta takes contiguous tensors (got a strided view)")
        if x.device.type != "cuda":
            raise ValueError("libsta takes device tensors (got a host tensor)")
        return x.data_ptr()
    raise TypeError(f"expected a CUDA tensor or a pointer, got {type(x)}")


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def sta_version():
    return _lib.load().sta_version()


def sta_debug_build() -> bool:
    """True when the loaded library is libsta_debug.so (STA_LIB=debug)."""
    return bool(_lib.load().sta_debug_build())


def sta_selftest_index_check(buf, n, index, dev_status, stream=None):
    """Debug build: store 1 into buf[index] through the kernels' index check
    (an index outside [0, n) raises STA_DEV_DEBUG and stores nothing)."""
    lib = _lib.load()
    check(lib.sta_selftest_index_check(_ptr(buf), int(n), int(index), _ptr(dev_status),
                                       _stream(stream)), "sta_selftest_index_check")


def sta_build_blocks_workspace(prob: Problem, sel: SelectorParams) -> int:
    return _lib.load().sta_build_blocks_workspace(ctypes.byref(prob), ctypes.byref(sel))


def sta_build_blocks_rows(prob: Problem, sel: SelectorParams) -> int:
    return _lib.load().sta_build_blocks_rows(ctypes.byref(prob), ctypes.byref(sel))


def sta_build_blocks(prob, sel, q, k, out: BlockLists, workspace=None, workspace_bytes=0,
                     dev_status=None, stream=None):
    lib = _lib.load()
    if isinstance(workspace, torch.Tensor) and not workspace_bytes:
        workspace_bytes = workspace.numel() * workspace.element_size()
    check(lib.sta_build_blocks(ctypes.byref(prob), ctypes.byref(sel), _ptr(q), _ptr(k),
                               ctypes.byref(out), _ptr(workspace), workspace_bytes,
                               _ptr(dev_status), _stream(stream)), "sta_build_blocks")


def sta_attn_workspace(prob: Problem) -> int:
    return _lib.load().sta_attn_workspace(ctypes.byref(prob))


def sta_sparse_attn_fwd(prob, prm: AttnParams, q, k, v, lists: BlockLists, o, workspace=None,
                        workspace_bytes=0, dev_status=None, stream=None):
    lib = _lib.load()
    if isinstance(workspace, torch.Tensor) and not workspace_bytes:
        workspace_bytes = workspace.numel() * workspace.element_size()
    check(lib.sta_sparse_attn_fwd(ctypes.byref(prob), ctypes.byref(prm), _ptr(q), _ptr(k),
                                  _ptr(v), ctypes.byref(lists), _ptr(o), _ptr(workspace),
                                  workspace_bytes, _ptr(dev_status), _stream(stream)),
          "sta_sparse_attn_fwd")


def sta_sparse_attn_fwd_noalloc(prob, prm: AttnParams, q, k, v, lists: BlockLists, o,
                                dev_status=None, stream=None):
    """sta_sparse_attn_fwd without a workspace: fp32 inputs are staged in
    the library's fixed device array (see include/sta.h)."""
    lib = _lib.load()
    check(lib.sta_sparse_attn_fwd_noalloc(ctypes.byref(prob), ctypes.byref(prm), _ptr(q),
                                          _ptr(k), _ptr(v), ctypes.byref(lists), _ptr(o),
                                          _ptr(dev_status), _stream(stream)),
          "sta_sparse_attn_fwd_noalloc")


def sta_dense_attn_fwd(prob, q, k, v, scale, o, workspace=None, workspace_bytes=0,
                       dev_status=None, stream=None):
    lib = _lib.load()
    if isinstance(workspace, torch.Tensor) and not workspace_bytes:
        workspace_bytes = workspace.numel() * workspace.element_size()
    check(lib.sta_dense_attn_fwd(ctypes.byref(prob), _ptr(q), _ptr(k), _ptr(v),
                                 float(scale), _ptr(o), _ptr(workspace), workspace_bytes,
                                 _ptr(dev_status), _stream(stream)), "sta_dense_attn_fwd")


def sta_dense_attn_entropy_fwd(prob, q, k, v, scale, o, entropy, workspace=None,
                               workspace_bytes=0, dev_status=None, stream=None):
    """Dense attention plus each query's attention entropy (nats) into
    `entropy` [heads, N] float32: the dense warm-up of the token-level
    selector."""
    lib = _lib.load()
    if isinstance(workspace, torch.Tensor) and not workspace_bytes:
        workspace_bytes = workspace.numel() * workspace.element_size()
    check(lib.sta_dense_attn_entropy_fwd(ctypes.byref(prob), _ptr(q), _ptr(k), _ptr(v),
                                         float(scale), _ptr(o), _ptr(entropy), _ptr(workspace),
                                         workspace_bytes, _ptr(dev_status), _stream(stream)),
          "sta_dense_attn_entropy_fwd")


def sta_permute_tokens(prob, tile_h, tile_w, inverse, x, out, stream=None):
    """Raster <-> tile-major row permutation of a [heads][N][d] tensor (inverse=0:
    raster to tile-major, 1: back)."""
    lib = _lib.load()
    check(lib.sta_permute_tokens(ctypes.byref(prob), int(tile_h), int(tile_w), int(inverse),
                                 _ptr(x), _ptr(out), _stream(stream)), "sta_permute_tokens")


def sta_status_string(code: int) -> str:
    return _lib.load().sta_status_string(code).decode()


def sta_dev_status_string(bits: int) -> str:
    return _lib.load().sta_dev_status_string(bits).decode()
