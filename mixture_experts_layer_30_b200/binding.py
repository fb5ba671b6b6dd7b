"""ctypes binding of libmoe_b200.so: argument marshalling only.

Every step of the layer runs in the CUDA library; this module checks tensor
placement/dtype/contiguity, passes raw device pointers and the current torch
stream, and turns status codes into exceptions.  There is no CPU fallback: if
the library is missing, every call raises.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_F32, MOE_BF16 = 0, 1
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED",
                3: "MOE_ERR_WORKSPACE", 4: "MOE_ERR_CUDA", 5: "MOE_ERR_DEVICE_STATUS"}
DEV_BAD_EXPERT_INDEX, DEV_COUNT_MISMATCH, DEV_BAD_OFFSETS, DEV_PIPELINE_TIMEOUT = 1, 2, 4, 8

# Every symbol of include/moe.h, with its ctypes signature.
_vp, _i32, _i64, _f32, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, \
    ctypes.c_size_t


WEIGHTS_ROW_MAJOR, WEIGHTS_TILED = 0, 1


class Shape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d", ctypes.c_int32), ("N", ctypes.c_int32),
                ("Z", ctypes.c_int32), ("K", ctypes.c_int32), ("I", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("weight_layout", ctypes.c_int32)]


_SP = ctypes.POINTER(Shape)
SIGNATURES = {
    "moe_pack_weights": (ctypes.c_int, [_i32, _i32, _i32, _i32, _vp, _vp, _vp]),
    "moe_quantize_weights_mxfp8": (ctypes.c_int, [_i32, _i32, _i32, _vp, _vp, _vp, _vp]),
    "moe_permute_mxfp8": (ctypes.c_int, [_SP, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz,
                                         _vp]),
    "moe_expert_gate_up_mxfp8": (ctypes.c_int, [_SP, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                                _vp, _sz, _vp]),
    "moe_expert_down_mxfp8": (ctypes.c_int, [_SP, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_workspace_bytes": (_sz, [_SP]),
    "moe_workspace_init": (ctypes.c_int, [_vp, _sz, _vp]),
    "moe_route": (ctypes.c_int,
                  [_SP, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_lb_stats": (ctypes.c_int, [_i32, _i32, _i32, _vp, _vp, _i64, _i32, _f32, _f32, _vp, _vp,
                                    _vp, _vp]),
    "moe_permute": (ctypes.c_int, [_SP, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_route_dispatch": (ctypes.c_int, [_SP, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                          _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_permute_noalloc": (ctypes.c_int, [_SP, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "moe_expert_gate_up": (ctypes.c_int, [_SP, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_expert_gate_up_gather": (ctypes.c_int,
                                  [_SP, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_expert_down": (ctypes.c_int, [_SP, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_expert_ffn": (ctypes.c_int, [_SP, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_combine": (ctypes.c_int, [_SP, _vp, _vp, _vp, _vp, _vp, _f32, _vp, _vp]),
    "moe_bias_update": (ctypes.c_int, [_i32, _i32, _vp, _i64, _i32, _f32, _f32, _vp, _vp]),
    "moe_backward_workspace_bytes": (_sz, [_SP]),
    "moe_expert_gate_up_save": (ctypes.c_int, [_SP, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_combine_backward": (ctypes.c_int, [_SP, _vp, _vp, _vp, _vp, _vp, _vp, _f32, _vp, _vp,
                                            _vp]),
    "moe_route_backward": (ctypes.c_int, [_SP, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _f32, _i64,
                                          _vp, _vp, _vp, _sz, _vp]),
    "moe_expert_ffn_backward": (ctypes.c_int, [_SP, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                               _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_permute_backward": (ctypes.c_int, [_SP, _vp, _vp, _vp, _vp, _vp, _vp, _f32, _vp, _vp]),
    "moe_get_device_status": (ctypes.c_int, [_vp, _vp, ctypes.POINTER(ctypes.c_uint32)]),
    "moe_last_error": (ctypes.c_char_p, []),
    "moe_kernel_launches": (ctypes.c_uint64, []),
    "moe_debug_set_pipeline": (ctypes.c_int, [ctypes.c_uint64, _i32]),
}

_lib = None


class MoEError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"{STATUS_NAMES.get(code, code)}: {msg}")
        self.code = code


def lib():
    """The loaded CUDA library (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"CUDA library {LIB_PATH} is missing; build it with "
                               "`python -m mixture_experts_layer_30_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype, fn.argtypes = res, args
        _lib = L
    return _lib


def _check(code):
    if code != 0:
        raise MoEError(code, lib().moe_last_error().decode())


def make_shape(T, d, N, Z, K, I, dtype, weight_layout=WEIGHTS_ROW_MAJOR) -> Shape:
    code = {"f32": MOE_F32, "bf16": MOE_BF16, torch.float32: MOE_F32,
            torch.bfloat16: MOE_BF16}[dtype]
    return Shape(T, d, N, Z, K, I, code, weight_layout)


def shape_of(cfg, T=None, weight_layout=WEIGHTS_ROW_MAJOR) -> Shape:
    return make_shape(cfg.T if T is None else T, cfg.d, cfg.N, cfg.Z, cfg.K, cfg.I, cfg.dtype,
                      weight_layout)


def pack_weights(w: torch.Tensor, out: torch.Tensor = None, stream=None) -> torch.Tensor:
    """MOE_WEIGHTS_TILED copy of bf16 weights [n, rows, cols] (or [rows, cols])."""
    if w.dim() == 2:
        w = w.unsqueeze(0)
    n, rows, cols = w.shape
    if out is None:
        out = torch.empty_like(w)
    _check(lib().moe_pack_weights(n, rows, cols, MOE_BF16, _p(w, torch.bfloat16, "w"),
                                  _p(out, torch.bfloat16, "out"), _stream(stream)))
    return out


def torch_dtype(shape: Shape):
    return torch.bfloat16 if shape.dtype == MOE_BF16 else torch.float32


def _p(t, dtype=None, name="tensor"):
    """Device pointer of a contiguous CUDA tensor (None -> NULL)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def quantize_weights_mxfp8(w: torch.Tensor, stream=None):
    """MXFP8 of bf16 weights [n, rows, cols] (reduction axis = cols): returns
    (codes uint8 [n*rows*cols] in 128x128 tiles, scales uint8 [n*rows*cols/32]
    in 512-byte atoms)."""
    if w.dim() == 2:
        w = w.unsqueeze(0)
    n, rows, cols = w.shape
    q = torch.empty(n * rows * cols, dtype=torch.uint8, device=w.device)
    sf = torch.empty(n * rows * cols // 32, dtype=torch.uint8, device=w.device)
    _check(lib().moe_quantize_weights_mxfp8(n, rows, cols, _p(w, torch.bfloat16, "w"), _p(q),
                                            _p(sf), _stream(stream)))
    return q, sf


def permute_mxfp8(shape, x, topk_idx, counts, offsets, row_token, slot_pos, x_perm_q, x_perm_sf,
                  ws, stream=None):
    _check(lib().moe_permute_mxfp8(ctypes.byref(shape), _p(x, torch.bfloat16, "x"),
                                   _p(topk_idx, torch.int32, "topk_idx"),
                                   _p(counts, torch.int32, "counts"),
                                   _p(offsets, torch.int32, "offsets"),
                                   _p(row_token, torch.int32, "row_token"),
                                   _p(slot_pos, torch.int32, "slot_pos"),
                                   _p(x_perm_q, torch.uint8, "x_perm_q"),
                                   _p(x_perm_sf, torch.uint8, "x_perm_sf"), _p(ws), ws.numel(),
                                   _stream(stream)))


def expert_gate_up_mxfp8(shape, x_perm_q, x_perm_sf, w1, w3, offsets, h_q, h_sf, ws,
                         stream=None):
    """w1, w3: (codes, scales) pairs from quantize_weights_mxfp8."""
    _check(lib().moe_expert_gate_up_mxfp8(
        ctypes.byref(shape), _p(x_perm_q, torch.uint8, "x_perm_q"),
        _p(x_perm_sf, torch.uint8, "x_perm_sf"), _p(w1[0]), _p(w1[1]), _p(w3[0]), _p(w3[1]),
        _p(offsets, torch.int32, "offsets"), _p(h_q, torch.uint8, "h_q"),
        _p(h_sf, torch.uint8, "h_sf"), _p(ws), ws.numel(), _stream(stream)))


def expert_down_mxfp8(shape, h_q, h_sf, w2, offsets, y_perm, ws, stream=None):
    _check(lib().moe_expert_down_mxfp8(
        ctypes.byref(shape), _p(h_q, torch.uint8, "h_q"), _p(h_sf, torch.uint8, "h_sf"),
        _p(w2[0]), _p(w2[1]), _p(offsets, torch.int32, "offsets"),
        _p(y_perm, torch.bfloat16, "y_perm"), _p(ws), ws.numel(), _stream(stream)))


class Mxfp8Buffers:
    """Routed-row buffers of the MXFP8 expert path for one shape."""

    def __init__(self, shape: Shape, device="cuda"):
        R = max(shape.T * shape.K, 1)
        kw = dict(dtype=torch.uint8, device=device)
        self.x_perm_q = torch.empty((R, shape.d), **kw)
        self.x_perm_sf = torch.empty((R, shape.d // 32), **kw)
        self.h_q = torch.empty((R, shape.I), **kw)
        self.h_sf = torch.empty((R, shape.I // 32), **kw)


def forward_mxfp8(buf: "LayerBuffers", fb: Mxfp8Buffers, x, w_router, w1, w3, w2, bias,
                  gamma=1.0, logit_offset=None, stream=None):
    """The layer with MXFP8 experts: w1, w3, w2 are (codes, scales) pairs."""
    s = buf.shape
    route(s, x, w_router, bias, buf.ws, buf.topk_idx, buf.topk_gate, buf.counts, buf.n_ffn,
          logit_offset=logit_offset, probs_out=buf.probs, stream=stream)
    permute_mxfp8(s, x, buf.topk_idx, buf.counts, buf.offsets, buf.row_token, buf.slot_pos,
                  fb.x_perm_q, fb.x_perm_sf, buf.ws, stream=stream)
    expert_gate_up_mxfp8(s, fb.x_perm_q, fb.x_perm_sf, w1, w3, buf.offsets, fb.h_q, fb.h_sf,
                         buf.ws, stream=stream)
    expert_down_mxfp8(s, fb.h_q, fb.h_sf, w2, buf.offsets, buf.y_perm, buf.ws, stream=stream)
    combine(s, x, buf.y_perm, buf.topk_idx, buf.topk_gate, buf.slot_pos, gamma, buf.out,
            stream=stream)
    return buf.out


def workspace_bytes(shape: Shape) -> int:
    n = lib().moe_workspace_bytes(ctypes.byref(shape))
    if n == 0:
        raise MoEError(1, "invalid shape")
    return n


def new_workspace(shape: Shape, device="cuda", stream=None) -> torch.Tensor:
    ws = torch.empty(workspace_bytes(shape), dtype=torch.uint8, device=device)
    _check(lib().moe_workspace_init(_p(ws), ws.numel(), _stream(stream)))
    return ws


def route(shape, x, w_router, bias, ws, topk_idx, topk_gate, counts, n_ffn,
          logit_offset=None, probs_out=None, prob_sum=None, stream=None):
    dt = torch_dtype(shape)
    _check(lib().moe_route(ctypes.byref(shape), _p(x, dt, "x"), _p(w_router, dt, "w_router"),
                           _p(bias, torch.float32, "bias"),
                           _p(logit_offset, torch.float32, "logit_offset"),
                           _p(topk_idx, torch.int32, "topk_idx"),
                           _p(topk_gate, torch.float32, "topk_gate"),
                           _p(counts, torch.int32, "counts"), _p(n_ffn, torch.uint8, "n_ffn"),
                           _p(probs_out, torch.float32, "probs_out"),
                           _p(prob_sum, torch.float32, "prob_sum"), _p(ws), ws.numel(),
                           _stream(stream)))


def route_dispatch(shape, x, w_router, bias, ws, topk_idx, topk_gate, counts, n_ffn, offsets,
                   row_token, slot_pos, logit_offset=None, probs_out=None, prob_sum=None,
                   stream=None):
    """route followed by the dispatch layout (permute with x_perm=None), one call."""
    dt = torch_dtype(shape)
    _check(lib().moe_route_dispatch(ctypes.byref(shape), _p(x, dt, "x"),
                                    _p(w_router, dt, "w_router"), _p(bias, torch.float32, "bias"),
                                    _p(logit_offset, torch.float32, "logit_offset"),
                                    _p(topk_idx, torch.int32, "topk_idx"),
                                    _p(topk_gate, torch.float32, "topk_gate"),
                                    _p(counts, torch.int32, "counts"),
                                    _p(n_ffn, torch.uint8, "n_ffn"),
                                    _p(probs_out, torch.float32, "probs_out"),
                                    _p(prob_sum, torch.float32, "prob_sum"),
                                    _p(offsets, torch.int32, "offsets"),
                                    _p(row_token, torch.int32, "row_token"),
                                    _p(slot_pos, torch.int32, "slot_pos"), _p(ws), ws.numel(),
                                    _stream(stream)))


def lb_stats(N, Z, D, counts, prob_sum, T, K, K_e, alpha, f, P, loss=None, stream=None):
    """Eq. (3)-(5) statistics from the route's counts and probability sums."""
    _check(lib().moe_lb_stats(N, Z, D, _p(counts, torch.int32, "counts"),
                              _p(prob_sum, torch.float32, "prob_sum"), int(T), K, float(K_e),
                              float(alpha), _p(f, torch.float32, "f"),
                              _p(P, torch.float32, "P"), _p(loss, torch.float32, "loss"),
                              _stream(stream)))


def permute(shape, x, topk_idx, counts, offsets, row_token, slot_pos, x_perm, ws, stream=None):
    """x_perm=None builds the layout only (no copy of the token rows)."""
    dt = torch_dtype(shape)
    _check(lib().moe_permute(ctypes.byref(shape), _p(x, dt, "x"),
                             _p(topk_idx, torch.int32, "topk_idx"),
                             _p(counts, torch.int32, "counts"),
                             _p(offsets, torch.int32, "offsets"),
                             _p(row_token, torch.int32, "row_token"),
                             _p(slot_pos, torch.int32, "slot_pos"), _p(x_perm, dt, "x_perm"),
                             _p(ws), ws.numel(), _stream(stream)))


def permute_noalloc(shape, x, topk_idx, counts, offsets, row_token, slot_pos, x_perm,
                    stream=None):
    """moe_permute for callers that cannot provide a workspace: the dispatch
    scratch lives in a fixed 4 MiB device array owned by the library."""
    dt = torch_dtype(shape)
    _check(lib().moe_permute_noalloc(ctypes.byref(shape), _p(x, dt, "x"),
                                     _p(topk_idx, torch.int32, "topk_idx"),
                                     _p(counts, torch.int32, "counts"),
                                     _p(offsets, torch.int32, "offsets"),
                                     _p(row_token, torch.int32, "row_token"),
                                     _p(slot_pos, torch.int32, "slot_pos"),
                                     _p(x_perm, dt, "x_perm"), _stream(stream)))


def expert_gate_up(shape, x_perm, w1, w3, offsets, h, ws, stream=None):
    dt = torch_dtype(shape)
    _check(lib().moe_expert_gate_up(ctypes.byref(shape), _p(x_perm, dt, "x_perm"),
                                    _p(w1, dt, "w1"), _p(w3, dt, "w3"),
                                    _p(offsets, torch.int32, "offsets"), _p(h, dt, "h"),
                                    _p(ws), ws.numel(), _stream(stream)))


def expert_gate_up_gather(shape, x, row_token, w1, w3, offsets, h, ws, stream=None):
    dt = torch_dtype(shape)
    _check(lib().moe_expert_gate_up_gather(ctypes.byref(shape), _p(x, dt, "x"),
                                           _p(row_token, torch.int32, "row_token"),
                                           _p(w1, dt, "w1"), _p(w3, dt, "w3"),
                                           _p(offsets, torch.int32, "offsets"), _p(h, dt, "h"),
                                           _p(ws), ws.numel(), _stream(stream)))


def expert_down(shape, h, w2, offsets, y_perm, ws, stream=None):
    dt = torch_dtype(shape)
    _check(lib().moe_expert_down(ctypes.byref(shape), _p(h, dt, "h"), _p(w2, dt, "w2"),
                                 _p(offsets, torch.int32, "offsets"),
                                 _p(y_perm, dt, "y_perm"), _p(ws), ws.numel(),
                                 _stream(stream)))


def expert_ffn(shape, x_perm, w1, w3, w2, offsets, y_perm, ws, stream=None):
    dt = torch_dtype(shape)
    _check(lib().moe_expert_ffn(ctypes.byref(shape), _p(x_perm, dt, "x_perm"), _p(w1, dt, "w1"),
                                _p(w3, dt, "w3"), _p(w2, dt, "w2"),
                                _p(offsets, torch.int32, "offsets"), _p(y_perm, dt, "y_perm"),
                                _p(ws), ws.numel(), _stream(stream)))


def combine(shape, x, y_perm, topk_idx, topk_gate, slot_pos, gamma, out, stream=None):
    dt = torch_dtype(shape)
    _check(lib().moe_combine(ctypes.byref(shape), _p(x, dt, "x"), _p(y_perm, dt, "y_perm"),
                             _p(topk_idx, torch.int32, "topk_idx"),
                             _p(topk_gate, torch.float32, "topk_gate"),
                             _p(slot_pos, torch.int32, "slot_pos"), float(gamma),
                             _p(out, dt, "out"), _stream(stream)))


def bias_update(N, Z, counts, T_all, K, K_e, mu, bias, stream=None):
    _check(lib().moe_bias_update(N, Z, _p(counts, torch.int32, "counts"), int(T_all), K,
                                 float(K_e), float(mu), _p(bias, torch.float32, "bias"),
                                 _stream(stream)))


def kernel_launches() -> int:
    """Kernels the library has launched in this process."""
    return int(lib().moe_kernel_launches())


def device_status(ws, stream=None) -> int:
    """Synchronises, returns the workspace status bits and clears them."""
    v = ctypes.c_uint32(0)
    code = lib().moe_get_device_status(_p(ws), _stream(stream), ctypes.byref(v))
    if code not in (0, 5):
        _check(code)
    return int(v.value)


def set_pipeline_wait(limit_ns=0, stall_first_fill=False):
    """Time limit of the GEMMs' bounded pipeline waits (0: the 4 s default);
    stall_first_fill is for tests of the timeout path only."""
    _check(lib().moe_debug_set_pipeline(int(limit_ns), 1 if stall_first_fill else 0))


class LayerBuffers:
    """Every buffer one forward pass of a shape needs, allocated once by torch."""

    def __init__(self, shape: Shape, device="cuda", with_probs=False):
        T, K, d, I, E = shape.T, shape.K, shape.d, shape.I, shape.N + shape.Z
        dt = torch_dtype(shape)
        R = max(T * K, 1)
        kw = dict(device=device)
        self.shape = shape
        self.ws = new_workspace(shape, device)
        self.topk_idx = torch.empty((T, K), dtype=torch.int32, **kw)
        self.topk_gate = torch.empty((T, K), dtype=torch.float32, **kw)
        self.counts = torch.empty(E, dtype=torch.int32, **kw)
        self.n_ffn = torch.empty(T, dtype=torch.uint8, **kw)
        self.probs = torch.empty((T, E), dtype=torch.float32, **kw) if with_probs else None
        self.offsets = torch.empty(shape.N + 1, dtype=torch.int32, **kw)
        self.row_token = torch.empty(R, dtype=torch.int32, **kw)
        self.slot_pos = torch.empty((T, K), dtype=torch.int32, **kw)
        self.x_perm = torch.empty((R, d), dtype=dt, **kw)
        self.h = torch.empty((R, I), dtype=dt, **kw)
        self.y_perm = torch.empty((R, d), dtype=dt, **kw)
        self.out = torch.empty((T, d), dtype=dt, **kw)


def forward(buf: LayerBuffers, x, w_router, w1, w3, w2, bias, gamma=1.0, logit_offset=None,
            stream=None, split_ffn=False, fused_gather=False):
    """route -> permute -> expert FFN -> combine; returns buf.out.

    split_ffn: gate/up and down as two calls (h in buf.h); fused_gather: no
    x_perm copy -- route_dispatch builds the layout with the selection and the
    gate/up GEMM reads x through row_token."""
    s = buf.shape
    if fused_gather:
        route_dispatch(s, x, w_router, bias, buf.ws, buf.topk_idx, buf.topk_gate, buf.counts,
                       buf.n_ffn, buf.offsets, buf.row_token, buf.slot_pos,
                       logit_offset=logit_offset, probs_out=buf.probs, stream=stream)
    else:
        route(s, x, w_router, bias, buf.ws, buf.topk_idx, buf.topk_gate, buf.counts, buf.n_ffn,
              logit_offset=logit_offset, probs_out=buf.probs, stream=stream)
        permute(s, x, buf.topk_idx, buf.counts, buf.offsets, buf.row_token, buf.slot_pos,
                buf.x_perm, buf.ws, stream=stream)
    if fused_gather:
        expert_gate_up_gather(s, x, buf.row_token, w1, w3, buf.offsets, buf.h, buf.ws,
                              stream=stream)
        expert_down(s, buf.h, w2, buf.offsets, buf.y_perm, buf.ws, stream=stream)
    elif split_ffn:
        expert_gate_up(s, buf.x_perm, w1, w3, buf.offsets, buf.h, buf.ws, stream=stream)
        expert_down(s, buf.h, w2, buf.offsets, buf.y_perm, buf.ws, stream=stream)
    else:
        expert_ffn(s, buf.x_perm, w1, w3, w2, buf.offsets, buf.y_perm, buf.ws, stream=stream)
    combine(s, x, buf.y_perm, buf.topk_idx, buf.topk_gate, buf.slot_pos, gamma, buf.out,
            stream=stream)
    return buf.out


# ---------------------------------------------------------------------------
# Backward pass
# ---------------------------------------------------------------------------

def backward_workspace_bytes(shape: Shape) -> int:
    n = lib().moe_backward_workspace_bytes(ctypes.byref(shape))
    if n == 0:
        raise MoEError(1, "invalid shape")
    return n


def new_backward_workspace(shape: Shape, device="cuda", stream=None) -> torch.Tensor:
    ws = torch.empty(backward_workspace_bytes(shape), dtype=torch.uint8, device=device)
    _check(lib().moe_workspace_init(_p(ws), ws.numel(), _stream(stream)))
    return ws


def expert_gate_up_save(shape, x_perm, w1, w3, offsets, h, au, ws, stream=None):
    dt = torch_dtype(shape)
    _check(lib().moe_expert_gate_up_save(ctypes.byref(shape), _p(x_perm, dt, "x_perm"),
                                         _p(w1, dt, "w1"), _p(w3, dt, "w3"),
                                         _p(offsets, torch.int32, "offsets"), _p(h, dt, "h"),
                                         _p(au, dt, "au"), _p(ws), ws.numel(), _stream(stream)))


def combine_backward(shape, x, y_perm, topk_idx, topk_gate, slot_pos, dout, gamma, dy_perm,
                     dgate, stream=None):
    dt = torch_dtype(shape)
    _check(lib().moe_combine_backward(ctypes.byref(shape), _p(x, dt, "x"),
                                      _p(y_perm, dt, "y_perm"),
                                      _p(topk_idx, torch.int32, "topk_idx"),
                                      _p(topk_gate, torch.float32, "topk_gate"),
                                      _p(slot_pos, torch.int32, "slot_pos"), _p(dout, dt, "dout"),
                                      float(gamma), _p(dy_perm, dt, "dy_perm"),
                                      _p(dgate, torch.float32, "dgate"), _stream(stream)))


def route_backward(shape, x, w_router, probs, topk_idx, dgate, dw_router, dx_router, bws,
                   lb=None, stream=None):
    """lb = (f, D, alpha, tokens): add the load-balance loss gradient (f [D+1]
    from lb_stats)."""
    dt = torch_dtype(shape)
    lb_f, lb_D, lb_alpha, lb_T = lb if lb is not None else (None, 0, 0.0, 0)
    _check(lib().moe_route_backward(ctypes.byref(shape), _p(x, dt, "x"),
                                    _p(w_router, dt, "w_router"),
                                    _p(probs, torch.float32, "probs"),
                                    _p(topk_idx, torch.int32, "topk_idx"),
                                    _p(dgate, torch.float32, "dgate"),
                                    _p(lb_f, torch.float32, "lb_f"), int(lb_D), float(lb_alpha),
                                    int(lb_T), _p(dw_router, dt, "dw_router"),
                                    _p(dx_router, torch.float32, "dx_router"), _p(bws),
                                    bws.numel(), _stream(stream)))


def expert_ffn_backward(shape, x_perm, w1, w3, w2, offsets, h, au, dy_perm, dx_perm, dw1, dw3,
                        dw2, bws, stream=None):
    dt = torch_dtype(shape)
    _check(lib().moe_expert_ffn_backward(
        ctypes.byref(shape), _p(x_perm, dt, "x_perm"), _p(w1, dt, "w1"), _p(w3, dt, "w3"),
        _p(w2, dt, "w2"), _p(offsets, torch.int32, "offsets"), _p(h, dt, "h"), _p(au, dt, "au"),
        _p(dy_perm, dt, "dy_perm"), _p(dx_perm, dt, "dx_perm"), _p(dw1, dt, "dw1"),
        _p(dw3, dt, "dw3"), _p(dw2, dt, "dw2"), _p(bws), bws.numel(), _stream(stream)))


def permute_backward(shape, dout, topk_idx, topk_gate, slot_pos, dx_perm, dx_router, gamma, dx,
                     stream=None):
    dt = torch_dtype(shape)
    _check(lib().moe_permute_backward(ctypes.byref(shape), _p(dout, dt, "dout"),
                                      _p(topk_idx, torch.int32, "topk_idx"),
                                      _p(topk_gate, torch.float32, "topk_gate"),
                                      _p(slot_pos, torch.int32, "slot_pos"),
                                      _p(dx_perm, dt, "dx_perm"),
                                      _p(dx_router, torch.float32, "dx_router"), float(gamma),
                                      _p(dx, dt, "dx"), _stream(stream)))


class BackwardBuffers:
    """Buffers of one training step (forward intermediates kept for the
    backward pass, and every gradient) for a shape, allocated once by torch."""

    def __init__(self, shape: Shape, device="cuda"):
        T, K, d, I, N, E = shape.T, shape.K, shape.d, shape.I, shape.N, shape.N + shape.Z
        dt = torch_dtype(shape)
        R = max(T * K, 1)
        kw = dict(device=device)
        self.bws = new_backward_workspace(shape, device)
        self.au = torch.empty((R, 2 * I), dtype=dt, **kw)
        self.dy_perm = torch.empty((R, d), dtype=dt, **kw)
        self.dgate = torch.empty((T, K), dtype=torch.float32, **kw)
        self.dx_router = torch.empty((T, d), dtype=torch.float32, **kw)
        self.dx_perm = torch.empty((R, d), dtype=dt, **kw)
        self.dx = torch.empty((T, d), dtype=dt, **kw)
        self.dw_router = torch.empty((E, d), dtype=dt, **kw)
        self.dw1 = torch.empty((N, I, d), dtype=dt, **kw)
        self.dw3 = torch.empty((N, I, d), dtype=dt, **kw)
        self.dw2 = torch.empty((N, d, I), dtype=dt, **kw)


def forward_train(buf: LayerBuffers, bb: BackwardBuffers, x, w_router, w1, w3, w2, bias,
                  gamma=1.0, logit_offset=None, prob_sum=None, stream=None):
    """The forward pass keeping what the backward pass needs (probs, x_perm,
    h, and the pre-activations a | u in bb.au); returns buf.out.  prob_sum [E]:
    also the probability column sums for lb_stats."""
    s = buf.shape
    if buf.probs is None:
        raise ValueError("forward_train needs LayerBuffers(with_probs=True)")
    route(s, x, w_router, bias, buf.ws, buf.topk_idx, buf.topk_gate, buf.counts, buf.n_ffn,
          logit_offset=logit_offset, probs_out=buf.probs, prob_sum=prob_sum, stream=stream)
    permute(s, x, buf.topk_idx, buf.counts, buf.offsets, buf.row_token, buf.slot_pos,
            buf.x_perm, buf.ws, stream=stream)
    expert_gate_up_save(s, buf.x_perm, w1, w3, buf.offsets, buf.h, bb.au, buf.ws, stream=stream)
    expert_down(s, buf.h, w2, buf.offsets, buf.y_perm, buf.ws, stream=stream)
    combine(s, x, buf.y_perm, buf.topk_idx, buf.topk_gate, buf.slot_pos, gamma, buf.out,
            stream=stream)
    return buf.out


def backward(buf: LayerBuffers, bb: BackwardBuffers, x, w_router, w1, w3, w2, dout, gamma=1.0,
             lb=None, stream=None):
    """Gradients of the layer for upstream gradient dout, after forward_train:
    bb.dx, bb.dw_router, bb.dw1, bb.dw3, bb.dw2 (the selection held fixed);
    lb = (f, D, alpha, tokens) adds the load-balance loss."""
    s = buf.shape
    combine_backward(s, x, buf.y_perm, buf.topk_idx, buf.topk_gate, buf.slot_pos, dout, gamma,
                     bb.dy_perm, bb.dgate, stream=stream)
    route_backward(s, x, w_router, buf.probs, buf.topk_idx, bb.dgate, bb.dw_router,
                   bb.dx_router, bb.bws, lb=lb, stream=stream)
    expert_ffn_backward(s, buf.x_perm, w1, w3, w2, buf.offsets, buf.h, bb.au, bb.dy_perm,
                        bb.dx_perm, bb.dw1, bb.dw3, bb.dw2, bb.bws, stream=stream)
    permute_backward(s, dout, buf.topk_idx, buf.topk_gate, buf.slot_pos, bb.dx_perm,
                     bb.dx_router, gamma, bb.dx, stream=stream)
