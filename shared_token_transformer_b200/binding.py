"""ctypes binding of libtileshare.so (include/tileshare.h, include/tileshare_ops.h).

Argument marshalling only: tensors are passed as device pointers with the current
CUDA stream, structs are filled field by field, and a non-zero status raises
TileShareError with the library's own message.  Every step of the computation
runs in the library's CUDA kernels.  The library must have been built
(``python -m shared_token_transformer_b200.build``); loading raises otherwise.
"""

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtileshare.so")

# ---------------------------------------------------------------------------
# C types
# ---------------------------------------------------------------------------
TS_OK = 0
TS_BLEND_LINEAR_RAMP = 0
TS_BLEND_HARD_STITCH = 1
TS_SHARE_QKV, TS_SHARE_OUT, TS_SHARE_MLP = 1, 2, 4
TS_F32, TS_BF16, TS_FP8_E4M3 = 0, 1, 2
TS_ROWS_SHARED, TS_ROWS_TILED = 0, 1
TS_EPI_BIAS, TS_EPI_BIAS_GELU, TS_EPI_BIAS_RESID, TS_EPI_BIAS_SWIGLU = 0, 1, 2, 3
TS_BLOCK_LN_GELU, TS_BLOCK_RMS_SWIGLU = 0, 1
BLOCKS = {"ln_gelu": TS_BLOCK_LN_GELU, "rms_swiglu": TS_BLOCK_RMS_SWIGLU}
DTYPES = {"f32": TS_F32, "bf16": TS_BF16, "fp8": TS_FP8_E4M3}

_int3 = ctypes.c_int * 3
_cp = ctypes.c_void_p


class PlanDesc(ctypes.Structure):
    _fields_ = [("grid", _int3), ("win", _int3), ("stride", _int3),
                ("T", ctypes.c_int), ("U", ctypes.c_int), ("Nw", ctypes.c_int), ("N", ctypes.c_int),
                ("nnz", ctypes.c_int), ("max_cover", ctypes.c_int), ("device", ctypes.c_int),
                ("run", ctypes.c_int),
                ("origins", ctypes.POINTER(ctypes.c_int)), ("tile_tok", ctypes.POINTER(ctypes.c_int)),
                ("slot_pos", ctypes.POINTER(ctypes.c_int)), ("tok_ptr", ctypes.POINTER(ctypes.c_int)),
                ("tok_ent", ctypes.POINTER(ctypes.c_int)), ("wbar", ctypes.POINTER(ctypes.c_float)),
                ("R", ctypes.c_int)]


class ModelDesc(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int), ("heads", ctypes.c_int), ("mlp", ctypes.c_int), ("dtype", ctypes.c_int),
                ("eps_ln", ctypes.c_float), ("eps_qk", ctypes.c_float), ("rope_base", ctypes.c_float),
                ("rope_dims", _int3), ("block", ctypes.c_int)]


_WEIGHT_FIELDS = ["ln1_g", "ln1_b", "w_qkv", "b_qkv", "q_g", "k_g", "w_o", "b_o", "ln2_g", "ln2_b",
                  "w_1", "b_1", "w_2", "b_2", "s_qkv", "s_o", "s_1", "s_2"]


class LayerWeights(ctypes.Structure):
    _fields_ = [(n, _cp) for n in _WEIGHT_FIELDS]


class TraceEntry(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 48), ("launches", ctypes.c_int), ("timed", ctypes.c_int),
                ("ms", ctypes.c_double), ("flops", ctypes.c_double), ("bytes", ctypes.c_double)]


class TileShareError(RuntimeError):
    def __init__(self, fn, status, msg):
        super().__init__(f"{fn} -> status {status}: {msg}")
        self.status = status


# ---------------------------------------------------------------------------
# library loading
# ---------------------------------------------------------------------------
_lib = None

_SIGS = {
    "ts_plan_create": [ctypes.POINTER(ctypes.c_int)] * 3 + [ctypes.c_int, ctypes.POINTER(_cp)],
    "ts_plan_create_host": [ctypes.POINTER(ctypes.c_int)] * 3 + [ctypes.c_int, ctypes.POINTER(_cp)],
    "ts_plan_create_registers": [ctypes.POINTER(ctypes.c_int)] * 3 + [ctypes.c_int, ctypes.c_int, ctypes.POINTER(_cp)],
    "ts_plan_create_host_registers": [ctypes.POINTER(ctypes.c_int)] * 3 + [ctypes.c_int, ctypes.c_int,
                                                                            ctypes.POINTER(_cp)],
    "ts_plan_info": [_cp, ctypes.POINTER(PlanDesc)],
    "ts_plan_destroy": [_cp],
    "ts_workspace_size": [_cp, ctypes.POINTER(ModelDesc), ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_size_t)],
    "ts_block_tiled": [_cp, ctypes.POINTER(ModelDesc), ctypes.POINTER(LayerWeights), _cp, _cp, ctypes.c_size_t, _cp],
    "ts_block_shared": [_cp, ctypes.POINTER(ModelDesc), ctypes.POINTER(LayerWeights), _cp, _cp, ctypes.c_size_t, _cp],
    "ts_block_shared_noalloc": [_cp, ctypes.POINTER(ModelDesc), ctypes.POINTER(LayerWeights), _cp, _cp],
    "ts_block_partial": [_cp, ctypes.POINTER(ModelDesc), ctypes.POINTER(LayerWeights), ctypes.c_uint, _cp, _cp,
                         ctypes.c_size_t, _cp],
    "ts_decode_stack": [_cp, ctypes.POINTER(ModelDesc), ctypes.POINTER(LayerWeights), ctypes.c_int, ctypes.c_int,
                        _cp, _cp, _cp, _cp, ctypes.c_size_t, _cp],
    "ts_quantize_rows_e4m3": [_cp, ctypes.c_int, ctypes.c_int, _cp, _cp, _cp],
    "ts_gather_tiles": [_cp, ctypes.POINTER(ModelDesc), _cp, _cp, _cp, _cp],
    "ts_trace_begin": [ctypes.c_int],
    "ts_trace_end": [ctypes.POINTER(TraceEntry), ctypes.c_int, ctypes.POINTER(ctypes.c_int)],
    "ts_launch_count": [],
    "ts_device_status": [],
    "ts_selftest_bounded_wait": [ctypes.c_longlong, _cp, _cp],
    "ts_status_string": [ctypes.c_int],
    "ts_last_error": [],
    "ts_op_layernorm": [ctypes.POINTER(ModelDesc), _cp, ctypes.c_int, _cp, _cp, _cp, _cp],
    "ts_op_linear": [ctypes.POINTER(ModelDesc), _cp, ctypes.c_int, ctypes.c_int, _cp, _cp, ctypes.c_int, _cp,
                     ctypes.c_int, _cp, _cp, _cp],
    "ts_op_qkv": [_cp, ctypes.POINTER(ModelDesc), ctypes.POINTER(LayerWeights), ctypes.c_int, _cp, _cp, _cp, _cp],
    "ts_op_attention": [_cp, ctypes.POINTER(ModelDesc), ctypes.c_int, _cp, _cp, _cp],
    "ts_op_merge": [_cp, ctypes.POINTER(ModelDesc), _cp, ctypes.c_int, _cp, _cp],
}


def lib():
    """Load libtileshare.so once; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m shared_token_transformer_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, args in _SIGS.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = None if name == "ts_plan_destroy" else ctypes.c_int
        L.ts_launch_count.restype = ctypes.c_longlong
        L.ts_status_string.restype = ctypes.c_char_p
        L.ts_last_error.restype = ctypes.c_char_p
        _lib = L
    return _lib


def exported_symbols():
    return list(_SIGS)


def _check(name, status):
    if status != TS_OK:
        raise TileShareError(name, status, lib().ts_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


# ---------------------------------------------------------------------------
# plan
# ---------------------------------------------------------------------------
class Plan:
    """ts_plan_t with its host arrays as NumPy views (copied)."""

    def __init__(self, grid, win, stride, host_only=False, rule=TS_BLEND_LINEAR_RAMP, registers=1):
        g, w, s = _int3(*grid), _int3(*win), _int3(*stride)
        h = _cp()
        fn = "ts_plan_create_host_registers" if host_only else "ts_plan_create_registers"
        _check(fn, getattr(lib(), fn)(g, w, s, rule, int(registers), ctypes.byref(h)))
        self.handle = h
        d = PlanDesc()
        _check("ts_plan_info", lib().ts_plan_info(h, ctypes.byref(d)))
        self.desc = d
        self.T, self.U, self.Nw, self.N, self.nnz = d.T, d.U, d.Nw, d.N, d.nnz
        self.max_cover, self.device, self.run, self.R = d.max_cover, d.device, d.run, d.R

        def arr(p, n, dt):
            return np.ctypeslib.as_array(p, shape=(n,)).astype(dt).copy()

        self.origins = arr(d.origins, 3 * d.T, np.int64).reshape(d.T, 3)
        self.tile_tok = arr(d.tile_tok, d.T * d.Nw, np.int64).reshape(d.T, d.Nw)
        self.slot_pos = arr(d.slot_pos, 3 * d.Nw, np.int64).reshape(d.Nw, 3)
        self.tok_ptr = arr(d.tok_ptr, d.U + 1, np.int64)
        self.tok_ent = arr(d.tok_ent, d.nnz, np.int64)
        self.wbar = arr(d.wbar, d.nnz, np.float32)

    def close(self):
        if self.handle is not None and self.handle.value:
            lib().ts_plan_destroy(self.handle)
        self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# ---------------------------------------------------------------------------
# model / weights
# ---------------------------------------------------------------------------
def model_desc(d, heads, mlp, dtype, rope_dims, eps_ln=1e-6, eps_qk=1e-6, rope_base=10000.0, block="ln_gelu"):
    return ModelDesc(d, heads, mlp, DTYPES[dtype] if isinstance(dtype, str) else dtype, eps_ln, eps_qk, rope_base,
                     _int3(*rope_dims), BLOCKS[block] if isinstance(block, str) else block)


def layer_weights(tensors):
    """ts_layer_weights from a dict of device tensors (missing names -> NULL).

    The struct keeps a reference to the tensors: their device memory stays
    allocated for as long as the struct is alive."""
    w = LayerWeights()
    for n in _WEIGHT_FIELDS:
        t = tensors.get(n)
        setattr(w, n, None if t is None else t.data_ptr())
    w._tensors = dict(tensors)
    return w


def workspace_size(plan, model, L=0, k=0):
    n = ctypes.c_size_t()
    _check("ts_workspace_size", lib().ts_workspace_size(plan.handle, ctypes.byref(model), L, k, ctypes.byref(n)))
    return n.value


# ---------------------------------------------------------------------------
# compute calls (device tensors, current stream)
# ---------------------------------------------------------------------------
def block_tiled(plan, model, weights, X, ws, stream=None):
    _check("ts_block_tiled", lib().ts_block_tiled(plan.handle, ctypes.byref(model), ctypes.byref(weights), _ptr(X),
                                                  _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def block_shared(plan, model, weights, S, ws, stream=None):
    _check("ts_block_shared", lib().ts_block_shared(plan.handle, ctypes.byref(model), ctypes.byref(weights), _ptr(S),
                                                    _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def block_partial(plan, model, weights, shared_ops, X, ws, stream=None):
    """ts_block_partial: per-tile states X, the TS_SHARE_* operations in shared_ops once per token."""
    _check("ts_block_partial", lib().ts_block_partial(plan.handle, ctypes.byref(model), ctypes.byref(weights),
                                                      int(shared_ops), _ptr(X), _ptr(ws),
                                                      ws.numel() * ws.element_size(), _stream(stream)))


def block_shared_noalloc(plan, model, weights, S, stream=None):
    """ts_block_shared with the library's static scratch instead of a workspace (allocates nothing)."""
    _check("ts_block_shared_noalloc", lib().ts_block_shared_noalloc(plan.handle, ctypes.byref(model),
                                                                    ctypes.byref(weights), _ptr(S), _stream(stream)))


def decode_stack(plan, model, weights_list, k, S0, G0, out, ws, stream=None):
    L = len(weights_list)
    arr = (LayerWeights * L)(*weights_list)      # copies of the structs; the originals keep the tensors alive
    _check("ts_decode_stack", lib().ts_decode_stack(plan.handle, ctypes.byref(model), arr, L, k, _ptr(S0), _ptr(G0),
                                                    _ptr(out), _ptr(ws), ws.numel() * ws.element_size(),
                                                    _stream(stream)))


def gather_tiles(plan, model, S0, G0, X, stream=None):
    _check("ts_gather_tiles", lib().ts_gather_tiles(plan.handle, ctypes.byref(model), _ptr(S0), _ptr(G0), _ptr(X),
                                                    _stream(stream)))


def trace_begin(max_launches=100000):
    _check("ts_trace_begin", lib().ts_trace_begin(max_launches))


def trace_end():
    """Per kernel class: dict name -> {launches, timed, ms, flops, bytes} (synchronises)."""
    cap = 64
    arr = (TraceEntry * cap)()
    n = ctypes.c_int()
    _check("ts_trace_end", lib().ts_trace_end(arr, cap, ctypes.byref(n)))
    return {arr[i].name.decode(): {"launches": arr[i].launches, "timed": arr[i].timed, "ms": arr[i].ms,
                                   "flops": arr[i].flops, "bytes": arr[i].bytes} for i in range(min(n.value, cap))}


def launch_count():
    return int(lib().ts_launch_count())


def quantize_rows_e4m3(x, q, scale, stream=None):
    rows, cols = x.shape
    _check("ts_quantize_rows_e4m3", lib().ts_quantize_rows_e4m3(_ptr(x), rows, cols, _ptr(q), _ptr(scale),
                                                                _stream(stream)))


def device_status():
    _check("ts_device_status", lib().ts_device_status())


def selftest_bounded_wait(limit_ns, done, stream=None):
    """ts_selftest_bounded_wait: a wait that nothing satisfies must time out (device int32 done[2])."""
    _check("ts_selftest_bounded_wait", lib().ts_selftest_bounded_wait(int(limit_ns), _ptr(done), _stream(stream)))


def op_layernorm(model, x, g, b, y, stream=None):
    _check("ts_op_layernorm", lib().ts_op_layernorm(ctypes.byref(model), _ptr(x), x.shape[0], _ptr(g), _ptr(b),
                                                    _ptr(y), _stream(stream)))


def op_linear(model, x, W, bias, y, epi=TS_EPI_BIAS, w_scale=None, scratch=None, stream=None):
    rows, K = x.shape
    N = W.shape[0] // 2 if epi == TS_EPI_BIAS_SWIGLU else W.shape[0]     # output width
    _check("ts_op_linear", lib().ts_op_linear(ctypes.byref(model), _ptr(x), rows, K, _ptr(W), _ptr(w_scale), N,
                                              _ptr(bias), epi, _ptr(y), _ptr(scratch), _stream(stream)))


def op_qkv(plan, model, weights, mode, state, qkv, scratch, stream=None):
    _check("ts_op_qkv", lib().ts_op_qkv(plan.handle, ctypes.byref(model), ctypes.byref(weights), mode, _ptr(state),
                                        _ptr(qkv), _ptr(scratch), _stream(stream)))


def op_attention(plan, model, mode, qkv, O, stream=None):
    _check("ts_op_attention", lib().ts_op_attention(plan.handle, ctypes.byref(model), mode, _ptr(qkv), _ptr(O),
                                                    _stream(stream)))


def op_merge(plan, model, P, rows, A, stream=None):
    _check("ts_op_merge", lib().ts_op_merge(plan.handle, ctypes.byref(model), _ptr(P), rows, _ptr(A),
                                            _stream(stream)))
