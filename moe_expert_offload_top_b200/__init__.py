"""Python binding of libftmoe.so: a routed mixture-of-experts layer stack run
against a shared LRU cache of expert slots in GPU memory (NVIDIA B200, sm_100a).

Argument marshalling only: every entry point has the name of its C function
(include/ftmoe.h) and forwards to it.  Tensors (torch or anything with
``data_ptr()``) and ints are accepted wherever the C call takes a pointer;
torch streams are accepted wherever it takes a stream.  Every step of the
computation runs in the library's CUDA kernels; there is no other path.  The
import fails if the library has not been built
(``python moe_expert_offload_top_b200/build.py``).
"""
import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libftmoe.so")

if not os.path.exists(LIB_PATH):
    raise ImportError("libftmoe.so is not built: run `python moe_expert_offload_top_b200/build.py`")

_lib = ctypes.CDLL(LIB_PATH)

FT_OK, FT_ERR_INVALID, FT_ERR_OOM, FT_ERR_CUDA, FT_ERR_CAPACITY, FT_ERR_BUSY, FT_ERR_TIMEOUT, \
    FT_ERR_DEVICE_CHECK = range(8)
FT_W_F32, FT_W_BF16, FT_W_INT4_G128, FT_W_NVFP4 = 0, 1, 2, 3
FT_GATE_SOFTMAX, FT_GATE_SIGMOID = 0, 1
FT_ROUTED, FT_PREFETCH = 0, 1
FT_INJECT_COPY_FAIL, FT_INJECT_ROUTE_TIMEOUT, FT_INJECT_FUSED_WAIT = 1, 2, 3
FT_POLICY_LRU, FT_POLICY_STATIC = 0, 1
FT_MAX_EXPERTS, FT_MAX_TOPK = 256, 16
WDTYPE = {"f32": FT_W_F32, "bf16": FT_W_BF16, "int4": FT_W_INT4_G128, "nvfp4": FT_W_NVFP4}
GATING = {"softmax": FT_GATE_SOFTMAX, "sigmoid": FT_GATE_SIGMOID}


class ft_cache_stats_t(ctypes.Structure):
    _fields_ = [("routed", ctypes.c_longlong), ("hits", ctypes.c_longlong),
                ("misses", ctypes.c_longlong), ("evictions", ctypes.c_longlong),
                ("prefetch", ctypes.c_longlong), ("prefetch_hits", ctypes.c_longlong),
                ("prefetch_misses", ctypes.c_longlong), ("h2d_bytes", ctypes.c_longlong),
                ("h2d_seconds", ctypes.c_double), ("resident", ctypes.c_int),
                ("capacity", ctypes.c_int)]

    def as_dict(self):
        return {f: getattr(self, f) for f, _ in self._fields_}


class ft_perf_t(ctypes.Structure):
    _fields_ = [("forwards", ctypes.c_longlong), ("kernel_launches", ctypes.c_longlong),
                ("timed_forwards", ctypes.c_longlong), ("router_ms", ctypes.c_double),
                ("permute_ms", ctypes.c_double), ("ffn_gate_up_ms", ctypes.c_double),
                ("ffn_down_ms", ctypes.c_double), ("combine_ms", ctypes.c_double),
                ("ffn_gate_up_bytes", ctypes.c_double), ("ffn_down_bytes", ctypes.c_double),
                ("ffn_flops", ctypes.c_double), ("host_wait_ms", ctypes.c_double),
                ("ffn_fused_ms", ctypes.c_double), ("ffn_fused_bytes", ctypes.c_double),
                ("ffn_fused_launches", ctypes.c_longlong), ("ffn_gate_up_launches", ctypes.c_longlong),
                ("host_issue_ms", ctypes.c_double)]

    def as_dict(self):
        return {f: getattr(self, f) for f, _ in self._fields_}


class ft_access_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in
                ("call", "layer", "expert", "kind", "hit", "slot", "ev_layer", "ev_expert")]


_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
_SIGS = {
    "ft_moe_create": ([_i, _i, _i, _i, _i, _i], _vp),
    "ft_moe_set_layers": ([_vp, _i, _i, _i], _i),
    "ft_moe_blob_bytes": ([_vp], _sz),
    "ft_moe_pool_ptr": ([_vp, _i, _i], _vp),
    "ft_moe_set_shared": ([_vp, _i, _vp], _i),
    "ft_moe_set_mode": ([_vp, _i], _i),
    "ft_moe_reserve": ([_vp, _i], _i),
    "ft_moe_forward": ([_vp, _i, _vp, _i, _vp, _vp, _vp], _i),
    "ft_moe_last_routing": ([_vp, _vp, _vp, ctypes.POINTER(_i)], _i),
    "ft_cache_resize": ([_vp, _i], _i),
    "ft_cache_stats": ([_vp, ctypes.POINTER(ft_cache_stats_t)], _i),
    "ft_cache_clear": ([_vp], _i),
    "ft_cache_reset_stats": ([_vp], _i),
    "ft_cache_trace": ([_vp, _vp, _i, ctypes.POINTER(_i)], _i),
    "ft_cache_set_trace": ([_vp, _i], _i),
    "ft_cache_slot_of": ([_vp, _i, _i], _i),
    "ft_cache_slot_ptr": ([_vp, _i], _vp),
    "ft_moe_set_timeout_ms": ([_vp, _i], _i),
    "ft_last_error": ([_vp], ctypes.c_char_p),
    "ft_moe_destroy": ([_vp], None),
    "ft_router_topk": ([_vp, _i, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp], _i),
    "ft_permute": ([_vp, _i, _i, _i, _vp, _vp, _vp, _vp, _vp], _i),
    "ft_route_decode": ([_vp, _i, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp], _i),
    "ft_expert_ffn_decode": ([_vp, _i, _i, _i, _i, _i, _vp, _vp, _i, _i, _vp, _vp, _vp, _vp, _vp], _i),
    "ft_combine": ([_vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _vp], _i),
    "ft_expert_ffn_prefill": ([_vp, _i, _i, _i, _i, _vp, _i, _vp, _vp, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp],
                              _i),
    "ft_expert_ffn_decode_noalloc": ([_vp, _i, _i, _i, _i, _i, _vp, _vp, _i, _i, _vp, _vp, _vp, _vp, _i,
                                      _vp, _vp], _i),
    "ft_version": ([], ctypes.c_char_p),
    "ft_moe_set_stage_timing": ([_vp, _i], _i),
    "ft_moe_sync": ([_vp], _i),
    "ft_moe_set_gemm_threshold": ([_vp, _i], _i),
    "ft_moe_debug_inject": ([_vp, _i, _i], _i),
    "ft_moe_set_fused_routing": ([_vp, _i], _i),
    "ft_moe_set_fused_ffn": ([_vp, _i], _i),
    "ft_moe_set_int4_tensor_cores": ([_vp, _i], _i),
    "ft_debug_device_wait_selftest": ([_i, _vp], _i),
    "ft_moe_perf": ([_vp, ctypes.POINTER(ft_perf_t)], _i),
    "ft_moe_reset_perf": ([_vp], _i),
    "ft_cache_simulate_policy": ([_i, _i, _i, _i, _vp, _i, _vp, _i, ctypes.POINTER(_i),
                                  ctypes.POINTER(ft_cache_stats_t), ctypes.POINTER(_i)], _i),
    "ft_probe_host_link": ([_sz, _i, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double)], _i),
    "ft_probe_host_memory": ([_sz, _i, _i, ctypes.POINTER(ctypes.c_double)], _i),
    "ft_cache_simulate": ([_i, _i, _i, _vp, _i, _vp, _i, ctypes.POINTER(_i),
                           ctypes.POINTER(ft_cache_stats_t), ctypes.POINTER(_i)], _i),
}
for _name, (_args, _res) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = _res

EXPORTED = tuple(_SIGS)


class FtError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__("%s (status %d)" % (msg, code))
        self.code = code


def _p(a):
    """Pointer of a tensor / array / int / None."""
    if a is None:
        return None
    if isinstance(a, int):
        return a
    if hasattr(a, "data_ptr"):
        return a.data_ptr()
    if hasattr(a, "ctypes"):
        return a.ctypes.data
    raise TypeError("cannot take the address of %r" % type(a))


def _s(stream):
    if stream is None:
        return None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(h, rc):
    if rc != FT_OK:
        raise FtError(rc, _lib.ft_last_error(h).decode())
    return rc


def _int_array(xs):
    return (ctypes.c_int * len(xs))(*xs)


# ------------------------------------------------------------ cache level --

def ft_moe_create(num_experts, top_k, hidden, inter, wdtype, cache_slots):
    h = _lib.ft_moe_create(num_experts, top_k, hidden, inter, WDTYPE.get(wdtype, wdtype), cache_slots)
    if not h:
        raise FtError(FT_ERR_INVALID, _lib.ft_last_error(None).decode())
    return h


def ft_moe_set_layers(h, num_layers, gating, has_shared_expert):
    return _check(h, _lib.ft_moe_set_layers(h, num_layers, GATING.get(gating, gating), int(has_shared_expert)))


def ft_moe_blob_bytes(h):
    return _lib.ft_moe_blob_bytes(h)


def ft_moe_pool_ptr(h, layer, expert):
    p = _lib.ft_moe_pool_ptr(h, layer, expert)
    if not p:
        raise FtError(FT_ERR_INVALID, "ft_moe_pool_ptr: bad index or pool allocation failed")
    return p


def ft_moe_set_shared(h, layer, host_blob):
    return _check(h, _lib.ft_moe_set_shared(h, layer, _p(host_blob)))


def ft_moe_set_mode(h, prefill):
    return _check(h, _lib.ft_moe_set_mode(h, int(prefill)))


def ft_moe_reserve(h, max_tokens):
    return _check(h, _lib.ft_moe_reserve(h, max_tokens))


def ft_moe_forward(h, layer, x, n_tokens, router_w, out, stream=None):
    return _check(h, _lib.ft_moe_forward(h, layer, _p(x), n_tokens, _p(router_w), _p(out), _s(stream)))


def ft_moe_last_routing(h, ids=None, gates=None):
    n = ctypes.c_int(0)
    _check(h, _lib.ft_moe_last_routing(h, _p(ids), _p(gates), ctypes.byref(n)))
    return n.value


def ft_cache_resize(h, slots):
    return _check(h, _lib.ft_cache_resize(h, slots))


def ft_cache_clear(h):
    return _check(h, _lib.ft_cache_clear(h))


def ft_cache_stats(h):
    st = ft_cache_stats_t()
    _check(h, _lib.ft_cache_stats(h, ctypes.byref(st)))
    return st.as_dict()


def ft_cache_reset_stats(h):
    return _check(h, _lib.ft_cache_reset_stats(h))


def ft_cache_trace(h):
    n = ctypes.c_int(0)
    _check(h, _lib.ft_cache_trace(h, None, 0, ctypes.byref(n)))
    buf = (ft_access_t * max(n.value, 1))()
    _check(h, _lib.ft_cache_trace(h, ctypes.cast(buf, ctypes.c_void_p), n.value, ctypes.byref(n)))
    return [tuple(getattr(buf[i], f) for f, _ in ft_access_t._fields_) for i in range(n.value)]


def ft_cache_set_trace(h, enabled):
    return _check(h, _lib.ft_cache_set_trace(h, int(enabled)))


def ft_cache_slot_of(h, layer, expert):
    return _lib.ft_cache_slot_of(h, layer, expert)


def ft_cache_slot_ptr(h, slot):
    return _lib.ft_cache_slot_ptr(h, slot)


def ft_moe_set_timeout_ms(h, ms):
    return _check(h, _lib.ft_moe_set_timeout_ms(h, ms))


def ft_moe_sync(h):
    return _check(h, _lib.ft_moe_sync(h))


def ft_moe_set_gemm_threshold(h, min_avg_pairs):
    return _check(h, _lib.ft_moe_set_gemm_threshold(h, min_avg_pairs))


def ft_moe_set_fused_routing(h, enabled):
    return _check(h, _lib.ft_moe_set_fused_routing(h, int(enabled)))


def ft_moe_set_fused_ffn(h, enabled):
    return _check(h, _lib.ft_moe_set_fused_ffn(h, int(enabled)))


def ft_moe_set_int4_tensor_cores(h, enabled):
    return _check(h, _lib.ft_moe_set_int4_tensor_cores(h, int(enabled)))


def ft_moe_debug_inject(h, what, countdown):
    return _check(h, _lib.ft_moe_debug_inject(h, what, countdown))


def ft_debug_device_wait_selftest(limit_us, stream=None):
    """Returns the status code (FT_ERR_DEVICE_CHECK expected) without raising."""
    return _lib.ft_debug_device_wait_selftest(limit_us, _s(stream))


def ft_moe_set_stage_timing(h, enabled):
    return _check(h, _lib.ft_moe_set_stage_timing(h, int(enabled)))


def ft_moe_perf(h):
    p = ft_perf_t()
    _check(h, _lib.ft_moe_perf(h, ctypes.byref(p)))
    return p.as_dict()


def ft_moe_reset_perf(h):
    return _check(h, _lib.ft_moe_reset_perf(h))


def ft_last_error(h=None):
    return _lib.ft_last_error(h).decode()


def ft_moe_destroy(h):
    _lib.ft_moe_destroy(h)


# ------------------------------------------------------------- step level --

def ft_router_topk(x, x_is_bf16, router_w, T, H, E, top_k, gating, logits, ids, gates, stream=None):
    return _check(None, _lib.ft_router_topk(_p(x), int(x_is_bf16), _p(router_w), T, H, E, top_k,
                                            GATING.get(gating, gating), _p(logits), _p(ids), _p(gates),
                                            _s(stream)))


def ft_route_decode(x, x_is_bf16, router_w, T, H, E, top_k, gating, logits, ids, gates, counts, offsets, perm,
                    inv, ticket, stream=None):
    return _check(None, _lib.ft_route_decode(_p(x), int(x_is_bf16), _p(router_w), T, H, E, top_k,
                                             GATING.get(gating, gating), _p(logits), _p(ids), _p(gates),
                                             _p(counts), _p(offsets), _p(perm), _p(inv), _p(ticket), _s(stream)))


def ft_permute(ids, T, top_k, E, counts, offsets, perm, inv=None, stream=None):
    return _check(None, _lib.ft_permute(_p(ids), T, top_k, E, _p(counts), _p(offsets), _p(perm),
                                        _p(inv), _s(stream)))


def ft_expert_ffn_decode(x, T, H, I, top_k, wdtype, blobs, experts, max_pairs_per_expert, offsets,
                         perm, h, y, stream=None):
    n = len(experts)
    bl = (ctypes.c_void_p * max(n, 1))(*[_p(b) for b in blobs])
    ex = _int_array(list(experts) or [0])
    return _check(None, _lib.ft_expert_ffn_decode(
        _p(x), T, H, I, top_k, WDTYPE.get(wdtype, wdtype), ctypes.cast(bl, ctypes.c_void_p),
        ctypes.cast(ex, ctypes.c_void_p), n, max_pairs_per_expert, _p(offsets), _p(perm), _p(h), _p(y),
        _s(stream)))


def ft_expert_ffn_prefill(x, T, H, I, top_k, weights, n_slots, experts, slots, offsets, perm, a_rows, h, y, err,
                          stream=None):
    n = len(experts)
    ex = _int_array(list(experts) or [0])
    sl = _int_array(list(slots) or [0])
    return _check(None, _lib.ft_expert_ffn_prefill(
        _p(x), T, H, I, top_k, _p(weights), n_slots, ctypes.cast(ex, ctypes.c_void_p),
        ctypes.cast(sl, ctypes.c_void_p), n, _p(offsets), _p(perm), _p(a_rows), _p(h), _p(y), _p(err),
        _s(stream)))


def ft_combine(y, gates, inv, T, H, top_k, has_shared, out_is_bf16, out, stream=None):
    return _check(None, _lib.ft_combine(_p(y), _p(gates), _p(inv), T, H, top_k, int(has_shared),
                                        int(out_is_bf16), _p(out), _s(stream)))


def ft_cache_simulate(num_layers, num_experts, capacity, ops):
    """ops: flat int list (see include/ftmoe.h).  Returns (trace tuples, stats dict, n_capacity_errors)."""
    arr = _int_array(list(ops) or [0])
    n = ctypes.c_int(0)
    nerr = ctypes.c_int(0)
    st = ft_cache_stats_t()
    _check(None, _lib.ft_cache_simulate(num_layers, num_experts, capacity, ctypes.cast(arr, ctypes.c_void_p),
                                        len(ops), None, 0, ctypes.byref(n), None, None))
    buf = (ft_access_t * max(n.value, 1))()
    _check(None, _lib.ft_cache_simulate(num_layers, num_experts, capacity, ctypes.cast(arr, ctypes.c_void_p),
                                        len(ops), ctypes.cast(buf, ctypes.c_void_p), n.value, ctypes.byref(n),
                                        ctypes.byref(st), ctypes.byref(nerr)))
    trace = [tuple(getattr(buf[i], f) for f, _ in ft_access_t._fields_) for i in range(n.value)]
    return trace, st.as_dict(), nerr.value


FT_NOALLOC_SCRATCH_FLOATS = 3 * 1024 * 1024


def ft_expert_ffn_decode_noalloc(x, T, H, I, top_k, wdtype, blobs, experts, max_pairs_per_expert, offsets,
                                 perm, gates, inv, has_shared, out, stream=None):
    """Decode FFN + combine with the library's static device scratch (no allocation)."""
    n = len(experts)
    bl = (ctypes.c_void_p * max(n, 1))(*[_p(b) for b in blobs])
    ex = _int_array(list(experts) or [0])
    return _check(None, _lib.ft_expert_ffn_decode_noalloc(
        _p(x), T, H, I, top_k, WDTYPE.get(wdtype, wdtype), ctypes.cast(bl, ctypes.c_void_p),
        ctypes.cast(ex, ctypes.c_void_p), n, max_pairs_per_expert, _p(offsets), _p(perm), _p(gates), _p(inv),
        int(has_shared), _p(out), _s(stream)))


def ft_cache_simulate_policy(policy, num_layers, num_experts, capacity, ops):
    """Like ft_cache_simulate under FT_POLICY_LRU or FT_POLICY_STATIC."""
    arr = _int_array(list(ops) or [0])
    n = ctypes.c_int(0)
    nerr = ctypes.c_int(0)
    st = ft_cache_stats_t()
    _check(None, _lib.ft_cache_simulate_policy(policy, num_layers, num_experts, capacity,
                                               ctypes.cast(arr, ctypes.c_void_p), len(ops), None, 0,
                                               ctypes.byref(n), None, None))
    buf = (ft_access_t * max(n.value, 1))()
    _check(None, _lib.ft_cache_simulate_policy(policy, num_layers, num_experts, capacity,
                                               ctypes.cast(arr, ctypes.c_void_p), len(ops),
                                               ctypes.cast(buf, ctypes.c_void_p), n.value, ctypes.byref(n),
                                               ctypes.byref(st), ctypes.byref(nerr)))
    trace = [tuple(getattr(buf[i], f) for f, _ in ft_access_t._fields_) for i in range(n.value)]
    return trace, st.as_dict(), nerr.value


def ft_probe_host_link(bytes_, iters=5):
    a, b = ctypes.c_double(0), ctypes.c_double(0)
    _check(None, _lib.ft_probe_host_link(bytes_, iters, ctypes.byref(a), ctypes.byref(b)))
    return a.value, b.value


def ft_probe_host_memory(bytes_, threads=1, iters=3):
    g = ctypes.c_double(0)
    _check(None, _lib.ft_probe_host_memory(bytes_, threads, iters, ctypes.byref(g)))
    return g.value


def ft_version():
    return _lib.ft_version().decode()
