"""ctypes binding of libgs (include/gs.h).  Argument marshalling only: every
step runs in the library's kernels.  Device buffers are torch CUDA tensors
(or raw device pointers); the stream is torch's current stream unless one
is given.

Importing this module loads libgs.so and raises if it is missing: there is
no fallback."""
from __future__ import annotations

import ctypes as C
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libgs.so")

GS_OK = 0
GS_WARN_BUDGET = 1
GS_ERR_ARG = -1
GS_ERR_CAPACITY = -2
GS_ERR_CUDA = -3
GS_ERR_TIMEOUT = -4
GS_ERR_BOUNDS = -5
GS_ERR_UNSUPPORTED = -6
GS_SORT_IOTA = 1
GS_SORT_ONESWEEP = 2
GS_RASTER_WS = 0x20
GS_COUNT_ON_DEVICE = -1
GS_SORT_TEST_STALL = 0x80000000
TILE = 16


class GsError(RuntimeError):
    def __init__(self, call, status, needed=None):
        self.status = status
        self.needed = needed
        super().__init__(f"{call} failed: {status} ({status_string(status)})"
                         + (f", needed={needed}" if needed is not None else ""))


class gs_camera(C.Structure):
    _fields_ = [("R", C.c_float * 9), ("t", C.c_float * 3), ("fx", C.c_float),
                ("fy", C.c_float), ("cx", C.c_float), ("cy", C.c_float),
                ("width", C.c_int32), ("height", C.c_int32)]


class gs_model(C.Structure):
    _fields_ = [("n", C.c_int64), ("n_pad", C.c_int64), ("sh_degree", C.c_int32),
                ("reserved", C.c_int32), ("params", C.c_void_p)]


class gs_proj(C.Structure):
    _fields_ = [("capacity", C.c_int64), ("n_cand", C.c_void_p), ("cand_idx", C.c_void_p),
                ("slot", C.c_void_p), ("rec", C.c_void_p), ("rect", C.c_void_p),
                ("depth_key", C.c_void_p), ("square_isect", C.c_void_p)]


class gs_rect(C.Structure):
    _fields_ = [("x0", C.c_int32), ("y0", C.c_int32), ("x1", C.c_int32), ("y1", C.c_int32)]


class gs_pixels(C.Structure):
    _fields_ = [("x0", C.c_int32), ("y0", C.c_int32), ("w", C.c_int32), ("h", C.c_int32),
                ("pitch", C.c_int64), ("plane", C.c_int64), ("img", C.c_void_p),
                ("T_final", C.c_void_p), ("last", C.c_void_p), ("dL_dimg", C.c_void_p),
                ("target", C.c_void_p), ("tx0", C.c_int32), ("ty0", C.c_int32),
                ("tpitch", C.c_int64), ("tplane", C.c_int64), ("loss_tiles", C.c_void_p),
                ("norm", C.c_double), ("counters", C.c_void_p)]


def pixels(x0, y0, w, h, img, T_final, last, dL, target=None, target_origin=(0, 0),
           target_pitch=None, target_plane=None, loss_tiles=None, norm=0.0, pitch=None,
           plane=None, counters=None) -> gs_pixels:
    """Descriptor of Leaf-local pixel buffers (pitch w, plane w*h by default)."""
    pitch = w if pitch is None else pitch
    plane = pitch * h if plane is None else plane
    p = gs_pixels()
    p.x0, p.y0, p.w, p.h, p.pitch, p.plane = x0, y0, w, h, pitch, plane
    p.img, p.T_final, p.last, p.dL_dimg = ptr(img), ptr(T_final), ptr(last), ptr(dL)
    p.target = ptr(target)
    p.tx0, p.ty0 = target_origin
    p.tpitch = target_pitch if target_pitch is not None else pitch
    p.tplane = target_plane if target_plane is not None else plane
    p.loss_tiles = ptr(loss_tiles)
    p.norm = norm
    p.counters = ptr(counters)
    return p


class gs_load_model(C.Structure):
    _fields_ = [("bytes_per_isect", C.c_int64), ("bytes_per_pixel", C.c_int64),
                ("bytes_per_tile", C.c_int64), ("fixed_bytes", C.c_int64), ("align", C.c_int64)]


class gs_adam_args(C.Structure):
    _fields_ = [("lr", C.c_double), ("beta1", C.c_double), ("beta2", C.c_double),
                ("eps", C.c_double), ("step", C.c_int32), ("reserved", C.c_int32)]


SYMBOLS = [
    "gs_version", "gs_status_string", "gs_check", "gs_launch_counter",
    "gs_project_workspace_size", "gs_project",
    "gs_sort_workspace_size", "gs_sort_keys", "gs_sort_keys32", "gs_sort_tiles",
    "gs_sort_keys32_noalloc",
    "gs_leaf_load_model", "gs_leaf_partition",
    "gs_depth_order_workspace_size", "gs_depth_order",
    "gs_bin_workspace_size", "gs_bin_tiles",
    "gs_block_sat_workspace_size", "gs_block_sat", "gs_bin_blocks_workspace_size",
    "gs_bin_blocks", "gs_expand_workspace_size", "gs_expand_tiles",
    "gs_tile_ranges", "gs_raster_fwd_blocks", "gs_upload_crop", "gs_project_region",
    "gs_grad_accumulate",
    "gs_raster_fwd", "gs_loss_l1", "gs_loss_total", "gs_ssim_workspace_size", "gs_loss_ssim",
    "gs_raster_bwd",
    "gs_project_bwd", "gs_adam",
]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libgs.so not built ({LIB_PATH}); run __graft_entry__.build()")
    L = C.CDLL(LIB_PATH)
    p, i64, i32, u32, sz = C.c_void_p, C.c_int64, C.c_int32, C.c_uint32, C.c_size_t
    P = C.POINTER
    sig = {
        "gs_version": (i32, []),
        "gs_launch_counter": (i64, []),
        "gs_status_string": (C.c_char_p, [i32]),
        "gs_check": (i32, [p, p]),
        "gs_project_workspace_size": (sz, [i64, i32, i32]),
        "gs_project": (i32, [P(gs_model), P(gs_camera), u32, P(gs_proj), p, p, sz, p, p]),
        "gs_project_region": (i32, [P(gs_model), P(gs_camera), u32, gs_rect, P(gs_proj), p, p, sz,
                                    p, p]),
        "gs_grad_accumulate": (i32, [p, i64, p, i64, i32, p, i64, p]),
        "gs_sort_workspace_size": (sz, [i64, i32, i32, i32]),
        "gs_sort_keys": (i32, [p, p, i64, i32, i32, p, sz, p, p]),
        "gs_sort_keys32": (i32, [p, p, p, i64, i32, i32, u32, p, sz, p, p]),
        "gs_sort_keys32_noalloc": (i32, [p, p, p, i64, i32, i32, u32, p, p]),
        "gs_sort_tiles": (i32, [p, p, i64, p, i64, p, sz, p, p]),
        "gs_leaf_load_model": (i32, [i32, i32, P(gs_load_model)]),
        "gs_leaf_partition": (i32, [p, i32, i32, i32, i32, P(gs_load_model), i64, p, p, p, p,
                                    i32, P(i32)]),
        "gs_bin_workspace_size": (sz, [i64]),
        "gs_depth_order_workspace_size": (sz, [i64]),
        "gs_depth_order": (i32, [P(gs_proj), i64, p, p, p, sz, p, p]),
        "gs_bin_tiles": (i32, [P(gs_proj), i64, p, p, gs_rect, i32, i32, p, i64, p, p, p, i64, p,
                               P(i64), p, sz, p, p]),
        "gs_block_sat_workspace_size": (sz, [i32, i32]),
        "gs_block_sat": (i32, [P(gs_proj), i32, i32, p, p, sz, p, p]),
        "gs_bin_blocks_workspace_size": (sz, [i64, i64, i32, i32]),
        "gs_bin_blocks": (i32, [P(gs_proj), i64, p, p, i32, i32, p, i64, p, i64, p, P(i64), p, sz,
                                p, p]),
        "gs_expand_workspace_size": (sz, [gs_rect, i64]),
        "gs_expand_tiles": (i32, [P(gs_proj), p, p, i64, gs_rect, i32, i32, p, i64, p, i64, p,
                                  P(i64), p, sz, p, p]),
        "gs_raster_fwd": (i32, [P(gs_proj), p, p, gs_rect, P(gs_camera), P(gs_pixels), u32, p, p]),
        "gs_tile_ranges": (i32, [p, i32, i32, gs_rect, p, p]),
        "gs_upload_crop": (i32, [p, i64, i64, i32, i32, i32, i32, i32, p, i64, i64, p]),
        "gs_raster_fwd_blocks": (i32, [P(gs_proj), p, p, gs_rect, P(gs_camera), P(gs_pixels), p,
                                       i64, i64, p, P(i64), u32, p, p]),
        "gs_loss_l1": (i32, [P(gs_pixels), gs_rect, P(gs_camera), p]),
        "gs_loss_total": (i32, [p, i64, p, p]),
        "gs_ssim_workspace_size": (sz, [gs_rect, P(gs_camera)]),
        "gs_loss_ssim": (i32, [P(gs_pixels), gs_rect, P(gs_camera), C.c_double, p, sz, p]),
        "gs_raster_bwd": (i32, [P(gs_proj), p, p, gs_rect, P(gs_camera), P(gs_pixels), p, u32, p,
                                p]),
        "gs_project_bwd": (i32, [P(gs_model), P(gs_camera), P(gs_proj), i64, p, p, i64, p, p,
                                 P(gs_adam_args), p, p]),
        "gs_adam": (i32, [p, p, p, p, i64, p, i64, i64, i32, P(gs_adam_args), p]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    return L


_L = _load()


def lib():
    return _L


def status_string(s: int) -> str:
    return _L.gs_status_string(s).decode()


def version() -> int:
    return _L.gs_version()


def gs_launch_counter() -> int:
    """Kernel launches the library has issued in this process."""
    return int(_L.gs_launch_counter())


def ptr(x) -> int | None:
    """Device pointer of a tensor (None for None; ints pass through)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _ok(name, st, needed=None):
    if st < 0:
        raise GsError(name, st, needed)
    return st


def camera_struct(cam) -> gs_camera:
    c = gs_camera()
    R = [float(v) for v in list(cam.R.reshape(-1))]
    for k in range(9):
        c.R[k] = R[k]
    for k in range(3):
        c.t[k] = float(cam.t.reshape(-1)[k])
    c.fx, c.fy, c.cx, c.cy = float(cam.fx), float(cam.fy), float(cam.cx), float(cam.cy)
    c.width, c.height = int(cam.width), int(cam.height)
    return c


# ---------------------------------------------------------------------------
# one wrapper per entry point, same names as the C ABI
# ---------------------------------------------------------------------------

def gs_check(dev_status, stream=None) -> int:
    return _L.gs_check(ptr(dev_status), _stream(stream))


def gs_project_workspace_size(n, width, height) -> int:
    return _L.gs_project_workspace_size(n, width, height)


def gs_project(model: gs_model, cam: gs_camera, proj: gs_proj, tile_sat, ws, dev_status,
               flags=0, stream=None):
    return _ok("gs_project", _L.gs_project(C.byref(model), C.byref(cam), flags, C.byref(proj),
                                           ptr(tile_sat), ptr(ws), ws.numel() * ws.element_size(),
                                           ptr(dev_status), _stream(stream)))


def gs_project_region(model: gs_model, cam: gs_camera, region, proj: gs_proj, tile_sat, ws,
                      dev_status, flags=0, stream=None):
    return _ok("gs_project_region", _L.gs_project_region(
        C.byref(model), C.byref(cam), flags, gs_rect(*[int(v) for v in region]), C.byref(proj),
        ptr(tile_sat), ptr(ws), ws.numel() * ws.element_size(), ptr(dev_status), _stream(stream)))


def gs_grad_accumulate(g3d, g3d_stride, cand_idx, n_cand, P, G, n_pad, stream=None):
    return _ok("gs_grad_accumulate", _L.gs_grad_accumulate(ptr(g3d), g3d_stride, ptr(cand_idx),
                                                           n_cand, P, ptr(G), n_pad,
                                                           _stream(stream)))


def gs_sort_workspace_size(n, key_bytes, begin_bit, end_bit) -> int:
    return _L.gs_sort_workspace_size(n, key_bytes, begin_bit, end_bit)


def gs_sort_keys(keys, vals, n, begin_bit, end_bit, ws, dev_status, stream=None):
    return _ok("gs_sort_keys", _L.gs_sort_keys(ptr(keys), ptr(vals), n, begin_bit, end_bit,
                                               ptr(ws), ws.numel() * ws.element_size(),
                                               ptr(dev_status), _stream(stream)))


def gs_sort_keys32(keys_in, keys, vals, n, begin_bit, end_bit, flags, ws, dev_status,
                   stream=None):
    return _ok("gs_sort_keys32", _L.gs_sort_keys32(ptr(keys_in), ptr(keys), ptr(vals), n,
                                                   begin_bit, end_bit, flags, ptr(ws),
                                                   ws.numel() * ws.element_size(),
                                                   ptr(dev_status), _stream(stream)))


def gs_sort_tiles(tile_keys, vals, n, ranges, n_tiles, ws, dev_status, stream=None):
    return _ok("gs_sort_tiles", _L.gs_sort_tiles(ptr(tile_keys), ptr(vals), n, ptr(ranges), n_tiles,
                                                 ptr(ws), ws.numel() * ws.element_size(),
                                                 ptr(dev_status), _stream(stream)))


SORT_NOALLOC_MAX_N = 1 << 18
SORT_NOALLOC_SCRATCH_BYTES = 3 << 20


def gs_sort_keys32_noalloc(keys_in, keys, vals, n, begin_bit, end_bit, flags, dev_status,
                           stream=None):
    """gs_sort_keys32 without a workspace (library-held scratch, n <= 2**18).
    Calls must not overlap on the GPU: they share that scratch."""
    return _ok("gs_sort_keys32_noalloc", _L.gs_sort_keys32_noalloc(
        ptr(keys_in), ptr(keys), ptr(vals), n, begin_bit, end_bit, flags, ptr(dev_status),
        _stream(stream)))


GS_PROJ_DENSE = 1
GS_BIN_SORT = 0
GS_BIN_EXPAND = 1
GS_LOAD_SSIM = 0x100
TILE_BLOCK = 8
SSIM_LAMBDA = 0.2


def gs_leaf_load_model(tile_bits, binning=GS_BIN_EXPAND) -> gs_load_model:
    lm = gs_load_model()
    _ok("gs_leaf_load_model", _L.gs_leaf_load_model(binning, tile_bits, C.byref(lm)))
    return lm


def gs_leaf_partition(sat_host, TW, TH, width, height, lm: gs_load_model, budget,
                      max_leaves=1 << 16):
    """sat_host: contiguous int64 numpy array (TH+1, TW+1).  Returns
    (status, leaves[n,4] int32, leaf_isect[n], leaf_bytes[n], over[n])."""
    import numpy as np
    sat_host = np.ascontiguousarray(sat_host, np.int64)
    while True:
        leaves = np.zeros((max_leaves, 4), np.int32)
        li = np.zeros(max_leaves, np.int64)
        lb = np.zeros(max_leaves, np.int64)
        ov = np.zeros(max_leaves, np.uint8)
        n = C.c_int32(0)
        st = _L.gs_leaf_partition(sat_host.ctypes.data, TW, TH, width, height, C.byref(lm),
                                  int(budget), leaves.ctypes.data, li.ctypes.data,
                                  lb.ctypes.data, ov.ctypes.data, max_leaves, C.byref(n))
        if st == GS_ERR_CAPACITY:
            max_leaves = n.value
            continue
        _ok("gs_leaf_partition", st)
        k = n.value
        return st, leaves[:k].copy(), li[:k].copy(), lb[:k].copy(), ov[:k].astype(bool)


def gs_depth_order_workspace_size(n_cand) -> int:
    return _L.gs_depth_order_workspace_size(n_cand)


def gs_depth_order(proj: gs_proj, n_cand, depth_order, depth_rect, ws, dev_status, stream=None):
    return _ok("gs_depth_order", _L.gs_depth_order(C.byref(proj), n_cand, ptr(depth_order),
                                                   ptr(depth_rect), ptr(ws),
                                                   ws.numel() * ws.element_size(),
                                                   ptr(dev_status), _stream(stream)))


def gs_bin_workspace_size(n_cand) -> int:
    return _L.gs_bin_workspace_size(n_cand)


def gs_bin_tiles(proj: gs_proj, n_cand, depth_order, depth_rect, leaf, TW, TH, tile_sat, n_isect,
                 tile_keys, vals, capacity, ranges, ws, dev_status, keys64=None, stream=None):
    needed = C.c_int64(0)
    st = _L.gs_bin_tiles(C.byref(proj), n_cand, ptr(depth_order), ptr(depth_rect),
                         gs_rect(*[int(v) for v in leaf]), TW, TH, ptr(tile_sat), n_isect,
                         ptr(tile_keys), ptr(vals), ptr(keys64), capacity, ptr(ranges),
                         C.byref(needed), ptr(ws), ws.numel() * ws.element_size(),
                         ptr(dev_status), _stream(stream))
    return _ok("gs_bin_tiles", st, needed.value if st == GS_ERR_CAPACITY else None)


def gs_block_sat_workspace_size(TW, TH) -> int:
    return _L.gs_block_sat_workspace_size(TW, TH)


def gs_block_sat(proj: gs_proj, TW, TH, block_sat, ws, dev_status, stream=None):
    return _ok("gs_block_sat", _L.gs_block_sat(C.byref(proj), TW, TH, ptr(block_sat), ptr(ws),
                                               ws.numel() * ws.element_size(), ptr(dev_status),
                                               _stream(stream)))


def gs_bin_blocks_workspace_size(n_cand, n_entries, TW, TH) -> int:
    return _L.gs_bin_blocks_workspace_size(n_cand, n_entries, TW, TH)


def gs_bin_blocks(proj: gs_proj, n_cand, depth_order, depth_rect, TW, TH, block_sat, n_entries,
                  block_vals, capacity, block_ranges, ws, dev_status, stream=None):
    needed = C.c_int64(0)
    st = _L.gs_bin_blocks(C.byref(proj), n_cand, ptr(depth_order), ptr(depth_rect), TW, TH,
                          ptr(block_sat), n_entries, ptr(block_vals), capacity, ptr(block_ranges),
                          C.byref(needed), ptr(ws), ws.numel() * ws.element_size(),
                          ptr(dev_status), _stream(stream))
    return _ok("gs_bin_blocks", st, needed.value if st == GS_ERR_CAPACITY else None)


def gs_expand_workspace_size(leaf, block_entries) -> int:
    return _L.gs_expand_workspace_size(gs_rect(*[int(v) for v in leaf]), int(block_entries))


def gs_expand_tiles(proj: gs_proj, block_vals, block_ranges, block_entries, leaf, TW, TH,
                    tile_sat, n_isect, vals, capacity, ranges, ws, dev_status, stream=None):
    needed = C.c_int64(0)
    st = _L.gs_expand_tiles(C.byref(proj), ptr(block_vals), ptr(block_ranges), int(block_entries),
                            gs_rect(*[int(v) for v in leaf]), TW, TH, ptr(tile_sat), n_isect,
                            ptr(vals), capacity, ptr(ranges), C.byref(needed), ptr(ws),
                            ws.numel() * ws.element_size(), ptr(dev_status), _stream(stream))
    return _ok("gs_expand_tiles", st, needed.value if st == GS_ERR_CAPACITY else None)


def block_entries(block_sat_host, leaf) -> int:
    """Summed block-list lengths of the blocks meeting a Leaf (host SAT)."""
    x0, y0, x1, y1 = (int(v) for v in leaf)
    bx0, by0 = x0 // TILE_BLOCK, y0 // TILE_BLOCK
    bx1, by1 = (x1 - 1) // TILE_BLOCK + 1, (y1 - 1) // TILE_BLOCK + 1
    S = block_sat_host
    return int(S[by1, bx1] - S[by0, bx1] - S[by1, bx0] + S[by0, bx0])


def local_tile_bits(leaf) -> int:
    """Bits of a Leaf's local tile index (the sort range for its entries)."""
    x0, y0, x1, y1 = (int(v) for v in leaf)
    nt = (x1 - x0) * (y1 - y0)
    return (nt - 1).bit_length() if nt > 1 else 0


def gs_raster_fwd(proj: gs_proj, vals, ranges, leaf, cam: gs_camera, px: gs_pixels, dev_status,
                  flags=0, stream=None):
    return _ok("gs_raster_fwd", _L.gs_raster_fwd(C.byref(proj), ptr(vals), ptr(ranges),
                                                 gs_rect(*[int(v) for v in leaf]), C.byref(cam),
                                                 C.byref(px), flags, ptr(dev_status),
                                                 _stream(stream)))


def gs_tile_ranges(tile_sat, TW, TH, leaf, ranges, stream=None):
    return _ok("gs_tile_ranges", _L.gs_tile_ranges(ptr(tile_sat), TW, TH,
                                                   gs_rect(*[int(v) for v in leaf]), ptr(ranges),
                                                   _stream(stream)))


def gs_raster_fwd_blocks(proj: gs_proj, block_vals, block_ranges, leaf, cam: gs_camera,
                         px: gs_pixels, vals, capacity, n_isect, ranges, dev_status, flags=0,
                         stream=None):
    needed = C.c_int64(0)
    st = _L.gs_raster_fwd_blocks(C.byref(proj), ptr(block_vals), ptr(block_ranges),
                                 gs_rect(*[int(v) for v in leaf]), C.byref(cam), C.byref(px),
                                 ptr(vals), capacity, n_isect, ptr(ranges), C.byref(needed), flags,
                                 ptr(dev_status), _stream(stream))
    return _ok("gs_raster_fwd_blocks", st, needed.value if st == GS_ERR_CAPACITY else None)


def gs_upload_crop(host, x0, y0, w, h, dev, stream=None):
    """Crop of a planar host image [C][H][W] (pinned for an async copy) into a
    contiguous device buffer [C][h][w]."""
    C_, H_, W_ = host.shape
    return _ok("gs_upload_crop", _L.gs_upload_crop(host.data_ptr(), W_, H_ * W_, x0, y0, w, h, C_,
                                                   ptr(dev), w, w * h, _stream(stream)))


def gs_loss_l1(px: gs_pixels, leaf, cam: gs_camera, stream=None):
    return _ok("gs_loss_l1", _L.gs_loss_l1(C.byref(px), gs_rect(*[int(v) for v in leaf]),
                                           C.byref(cam), _stream(stream)))


def gs_loss_total(loss_tiles, n, loss, stream=None):
    return _ok("gs_loss_total", _L.gs_loss_total(ptr(loss_tiles), n, ptr(loss), _stream(stream)))


def gs_ssim_workspace_size(leaf, cam: gs_camera) -> int:
    return int(_L.gs_ssim_workspace_size(gs_rect(*[int(v) for v in leaf]), C.byref(cam)))


def gs_loss_ssim(px: gs_pixels, leaf, cam: gs_camera, weight, ws=None, stream=None):
    """ws: a device byte buffer of gs_ssim_workspace_size bytes, or None for
    the loss only (no gradient)."""
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    return _ok("gs_loss_ssim", _L.gs_loss_ssim(C.byref(px), gs_rect(*[int(v) for v in leaf]),
                                               C.byref(cam), float(weight), ptr(ws), nbytes,
                                               _stream(stream)))


def gs_raster_bwd(proj: gs_proj, vals, ranges, leaf, cam: gs_camera, px: gs_pixels, g2d,
                  dev_status, flags=0, stream=None):
    return _ok("gs_raster_bwd", _L.gs_raster_bwd(C.byref(proj), ptr(vals), ptr(ranges),
                                                 gs_rect(*[int(v) for v in leaf]), C.byref(cam),
                                                 C.byref(px), ptr(g2d), flags, ptr(dev_status),
                                                 _stream(stream)))


def gs_project_bwd(model: gs_model, cam: gs_camera, proj: gs_proj, n_cand, g2d, g3d=None,
                   g3d_stride=0, adam_m=None, adam_v=None, fused: gs_adam_args | None = None,
                   dev_status=None, stream=None):
    return _ok("gs_project_bwd", _L.gs_project_bwd(
        C.byref(model), C.byref(cam), C.byref(proj), n_cand, ptr(g2d), ptr(g3d), g3d_stride,
        ptr(adam_m), ptr(adam_v), C.byref(fused) if fused is not None else None,
        ptr(dev_status), _stream(stream)))


def gs_adam(params, m, v, g, g_stride, slot, n, n_pad, P, args: gs_adam_args, stream=None):
    return _ok("gs_adam", _L.gs_adam(ptr(params), ptr(m), ptr(v), ptr(g), g_stride, ptr(slot), n,
                                     n_pad, P, C.byref(args), _stream(stream)))
