"""ctypes binding of libmoe_b200.so -- argument marshalling only.

Every function has the name and argument order of the C entry point in
include/moe.h.  Array arguments are torch CUDA tensors (or None for a nullable
pointer); `stream` defaults to torch's current stream.  Each call returns the
integer moe_status; ``check`` turns a non-zero status into an exception.

The shared library is loaded on first use.  If it is missing the binding raises
(there is no fallback implementation); build it with
``python -m mixture_experts_sparse_b200.build``.
"""
import ctypes
import os

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, MOE_ERR_TIMEOUT = range(6)
MOE_F32, MOE_BF16 = 0, 1
MOE_RELU, MOE_SWIGLU = 0, 1

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe_b200.so")


class MoeConfig(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d_model", ctypes.c_int32), ("d_ff", ctypes.c_int32),
                ("n_experts", ctypes.c_int32), ("top_k", ctypes.c_int32), ("capacity", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("act", ctypes.c_int32), ("alpha", ctypes.c_float),
                ("priority", ctypes.c_int32)]


class MoeError(RuntimeError):
    def __init__(self, status):
        self.status = status
        super().__init__(f"moe status {status}: {moe_status_string(status)}")


_lib = None
_P = ctypes.c_void_p
_SIGS = {
    "moe_capacity": ([ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, ctypes.c_double], ctypes.c_int32),
    "moe_workspace_bytes": ([ctypes.POINTER(MoeConfig)], ctypes.c_size_t),
    "moe_status_string": ([ctypes.c_int32], ctypes.c_char_p),
    "moe_workspace_init": ([_P, ctypes.c_size_t, _P], ctypes.c_int32),
    "moe_route": ([ctypes.POINTER(MoeConfig)] + [_P] * 10 + [ctypes.c_size_t, _P], ctypes.c_int32),
    "moe_route_z": ([ctypes.POINTER(MoeConfig)] + [_P] * 11 + [ctypes.c_size_t, _P], ctypes.c_int32),
    "moe_dispatch_ntlb": ([ctypes.POINTER(MoeConfig)] + [_P] * 13 + [ctypes.c_size_t, _P], ctypes.c_int32),
    "moe_router_backward": ([ctypes.POINTER(MoeConfig)] + [_P] * 12 + [ctypes.c_size_t, _P], ctypes.c_int32),
    "moe_gate_grad": ([ctypes.POINTER(MoeConfig)] + [_P] * 8, ctypes.c_int32),
    "moe_dispatch": ([ctypes.POINTER(MoeConfig)] + [_P] * 12 + [ctypes.c_size_t, _P], ctypes.c_int32),
    "moe_expert_ffn": ([ctypes.POINTER(MoeConfig)] + [_P] * 10 + [ctypes.c_size_t, _P], ctypes.c_int32),
    "moe_combine": ([ctypes.POINTER(MoeConfig)] + [_P] * 8, ctypes.c_int32),
    "moe_combine_shard": ([ctypes.POINTER(MoeConfig)] + [_P] * 10, ctypes.c_int32),
    "moe_forward": ([ctypes.POINTER(MoeConfig)] + [_P] * 21 + [ctypes.c_size_t, _P], ctypes.c_int32),
    "moe_forward_events": ([ctypes.POINTER(MoeConfig)] + [_P] * 21 + [ctypes.c_size_t, _P, _P], ctypes.c_int32),
    "moe_dispatch_noalloc": ([ctypes.POINTER(MoeConfig)] + [_P] * 13, ctypes.c_int32),
    "moe_dispatch_shard": ([ctypes.POINTER(MoeConfig)] + [_P] * 13 + [ctypes.c_size_t, _P], ctypes.c_int32),
    "moe_expert_counts": ([ctypes.POINTER(MoeConfig), _P, _P, _P], ctypes.c_int32),
    "moe_claim_base": ([_P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, _P, _P], ctypes.c_int32),
    "moe_aux_shards": ([ctypes.c_int32, ctypes.c_int32, _P, _P, _P, ctypes.c_float, _P, _P, _P, _P],
                       ctypes.c_int32),
    "moe_ep_recv_rows": ([ctypes.POINTER(MoeConfig), ctypes.c_int32], ctypes.c_int64),
    "moe_ep_workspace_bytes": ([ctypes.POINTER(MoeConfig), ctypes.c_int32], ctypes.c_size_t),
    "moe_ep_layout": ([ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, _P, _P, _P, _P], ctypes.c_int32),
    "moe_ep_dispatch": ([ctypes.POINTER(MoeConfig), ctypes.c_int32, ctypes.c_int32] + [_P] * 12, ctypes.c_int32),
    "moe_ep_expert_ffn": ([ctypes.POINTER(MoeConfig), ctypes.c_int32] + [_P] * 13 + [ctypes.c_size_t, _P],
                          ctypes.c_int32),
    "moe_expert_backward_workspace_bytes": ([ctypes.POINTER(MoeConfig)], ctypes.c_size_t),
    "moe_expert_backward": ([ctypes.POINTER(MoeConfig)] + [_P] * 21 + [ctypes.c_size_t, _P], ctypes.c_int32),
    "moe_read_device_status": ([_P, _P], ctypes.c_int32),
    "moe_test_lookback_timeout": ([_P, ctypes.c_size_t, ctypes.c_int64, _P], ctypes.c_int32),
}


def lib():
    """Load the library (raises OSError if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise OSError(f"{LIB_PATH} is missing: build it with python -m mixture_experts_sparse_b200.build")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            fn = getattr(handle, name)
            fn.argtypes = args
            fn.restype = res
        _lib = handle
    return _lib


MOE_ORDER_TOKEN, MOE_ORDER_PRIORITY, MOE_ORDER_NTLB = 0, 1, 2


def config(T, d_model, d_ff, n_experts, top_k, capacity, dtype="bf16", act="relu", alpha=1e-2, priority=False):
    """moe_config.  priority: False/MOE_ORDER_TOKEN, True/MOE_ORDER_PRIORITY
    (batch priority) or MOE_ORDER_NTLB (No-Token-Left-Behind re-routing)."""
    order = MOE_ORDER_PRIORITY if priority is True else (MOE_ORDER_TOKEN if priority is False else int(priority))
    return MoeConfig(int(T), int(d_model), int(d_ff), int(n_experts), int(top_k), int(capacity),
                     MOE_BF16 if dtype in ("bf16", MOE_BF16) else MOE_F32,
                     MOE_SWIGLU if act in ("swiglu", MOE_SWIGLU) else MOE_RELU, float(alpha), order)


def _p(t):
    if t is None:
        return None
    if isinstance(t, int):
        return ctypes.c_void_p(t)
    return ctypes.c_void_p(t.data_ptr())


def _s(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _nbytes(ws):
    return ws.numel() * ws.element_size()


def check(status):
    if status != MOE_OK:
        raise MoeError(status)
    return status


def moe_capacity(T, n_experts, top_k, capacity_factor):
    return int(lib().moe_capacity(int(T), int(n_experts), int(top_k), float(capacity_factor)))


def moe_workspace_bytes(cfg):
    return int(lib().moe_workspace_bytes(ctypes.byref(cfg)))


def moe_workspace_init(ws, stream=None):
    return lib().moe_workspace_init(_p(ws), _nbytes(ws), _s(stream))


def new_workspace(cfg, device="cuda", stream=None):
    """Allocate (torch) and initialise a workspace for `cfg`."""
    import torch
    nbytes = moe_workspace_bytes(cfg)
    if nbytes == 0:
        raise ValueError("invalid layer configuration")
    ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
    check(moe_workspace_init(ws, stream))
    return ws


def moe_status_string(status):
    return lib().moe_status_string(int(status)).decode()


def moe_route(cfg, x, w_r, b_r, idx, gate, probs, f, P, aux, ws, stream=None):
    return lib().moe_route(ctypes.byref(cfg), _p(x), _p(w_r), _p(b_r), _p(idx), _p(gate), _p(probs),
                           _p(f), _p(P), _p(aux), _p(ws), _nbytes(ws), _s(stream))


def moe_route_z(cfg, x, w_r, b_r, idx, gate, probs, f, P, aux, z_loss, ws, stream=None):
    return lib().moe_route_z(ctypes.byref(cfg), _p(x), _p(w_r), _p(b_r), _p(idx), _p(gate), _p(probs),
                             _p(f), _p(P), _p(aux), _p(z_loss), _p(ws), _nbytes(ws), _s(stream))


def moe_gate_grad(cfg, dout, ye, idx, pos, drop, offsets, dgate, stream=None):
    return lib().moe_gate_grad(ctypes.byref(cfg), _p(dout), _p(ye), _p(idx), _p(pos), _p(drop), _p(offsets),
                               _p(dgate), _s(stream))


def moe_router_backward(cfg, x, w_r, probs, idx, gate, f, dgate, dh, dw_r, db_r, dx, ws, stream=None):
    return lib().moe_router_backward(ctypes.byref(cfg), _p(x), _p(w_r), _p(probs), _p(idx), _p(gate), _p(f),
                                     _p(dgate), _p(dh), _p(dw_r), _p(db_r), _p(dx), _p(ws), _nbytes(ws), _s(stream))


def moe_dispatch_ntlb(cfg, x, probs, expert, gate, pos, drop, counts, kept, offsets, row_token, row_gate, xe, ws,
                      stream=None):
    return lib().moe_dispatch_ntlb(ctypes.byref(cfg), _p(x), _p(probs), _p(expert), _p(gate), _p(pos), _p(drop),
                                   _p(counts), _p(kept), _p(offsets), _p(row_token), _p(row_gate), _p(xe), _p(ws),
                                   _nbytes(ws), _s(stream))


def moe_dispatch(cfg, x, idx, gate, pos, drop, counts, kept, offsets, row_token, row_gate, xe, ws,
                 stream=None):
    return lib().moe_dispatch(ctypes.byref(cfg), _p(x), _p(idx), _p(gate), _p(pos), _p(drop), _p(counts),
                              _p(kept), _p(offsets), _p(row_token), _p(row_gate), _p(xe), _p(ws),
                              _nbytes(ws), _s(stream))


def moe_dispatch_noalloc(cfg, x, idx, gate, pos, drop, counts, kept, offsets, row_token, row_gate, xe, status,
                         stream=None):
    return lib().moe_dispatch_noalloc(ctypes.byref(cfg), _p(x), _p(idx), _p(gate), _p(pos), _p(drop), _p(counts),
                                      _p(kept), _p(offsets), _p(row_token), _p(row_gate), _p(xe), _p(status),
                                      _s(stream))


def moe_expert_counts(cfg, idx, counts, stream=None):
    return lib().moe_expert_counts(ctypes.byref(cfg), _p(idx), _p(counts), _s(stream))


def moe_claim_base(shard_counts, n_shards, shard, top_k, n_experts, claim_base, stream=None):
    return lib().moe_claim_base(_p(shard_counts), int(n_shards), int(shard), int(top_k), int(n_experts),
                                _p(claim_base), _s(stream))


def moe_dispatch_shard(cfg, x, idx, gate, claim_base, pos, drop, counts, kept, offsets, row_token, row_gate, xe,
                       ws, stream=None):
    return lib().moe_dispatch_shard(ctypes.byref(cfg), _p(x), _p(idx), _p(gate), _p(claim_base), _p(pos), _p(drop),
                                    _p(counts), _p(kept), _p(offsets), _p(row_token), _p(row_gate), _p(xe), _p(ws),
                                    _nbytes(ws), _s(stream))


def moe_aux_shards(n_shards, n_experts, shard_tokens, f_all, P_all, alpha, f, P, aux, stream=None):
    return lib().moe_aux_shards(int(n_shards), int(n_experts), _p(shard_tokens), _p(f_all), _p(P_all),
                                float(alpha), _p(f), _p(P), _p(aux), _s(stream))


def moe_expert_ffn(cfg, xe, offsets, w1, b1, w3, b3, w2, b2, ye, ws, stream=None):
    return lib().moe_expert_ffn(ctypes.byref(cfg), _p(xe), _p(offsets), _p(w1), _p(b1), _p(w3), _p(b3),
                                _p(w2), _p(b2), _p(ye), _p(ws), _nbytes(ws), _s(stream))


def moe_combine(cfg, ye, idx, pos, drop, gate, offsets, out, stream=None):
    return lib().moe_combine(ctypes.byref(cfg), _p(ye), _p(idx), _p(pos), _p(drop), _p(gate), _p(offsets),
                             _p(out), _s(stream))


def moe_combine_shard(cfg, ye, idx, pos, drop, gate, offsets, claim_base, counts, out, stream=None):
    return lib().moe_combine_shard(ctypes.byref(cfg), _p(ye), _p(idx), _p(pos), _p(drop), _p(gate),
                                   _p(offsets), _p(claim_base), _p(counts), _p(out), _s(stream))


def moe_forward(cfg, x, w_r, b_r, w1, b1, w3, b3, w2, b2, out, idx=None, gate=None, pos=None, drop=None,
                counts=None, kept=None, offsets=None, f=None, P=None, aux=None, ws=None, stream=None):
    return lib().moe_forward(ctypes.byref(cfg), _p(x), _p(w_r), _p(b_r), _p(w1), _p(b1), _p(w3), _p(b3),
                             _p(w2), _p(b2), _p(out), _p(idx), _p(gate), _p(pos), _p(drop), _p(counts),
                             _p(kept), _p(offsets), _p(f), _p(P), _p(aux), _p(ws), _nbytes(ws), _s(stream))


def moe_forward_events(cfg, x, w_r, b_r, w1, b1, w3, b3, w2, b2, out, idx=None, gate=None, pos=None,
                       drop=None, counts=None, kept=None, offsets=None, f=None, P=None, aux=None, ws=None,
                       stream=None, events=None):
    """events: a sequence of 6 raw cudaEvent_t handles (int or ctypes.c_void_p; entries may be None)."""
    arr = None
    if events is not None:
        arr = (ctypes.c_void_p * 6)(*[None if e is None else (e.value if isinstance(e, ctypes.c_void_p) else e)
                                      for e in events])
    return lib().moe_forward_events(ctypes.byref(cfg), _p(x), _p(w_r), _p(b_r), _p(w1), _p(b1), _p(w3), _p(b3),
                                    _p(w2), _p(b2), _p(out), _p(idx), _p(gate), _p(pos), _p(drop), _p(counts),
                                    _p(kept), _p(offsets), _p(f), _p(P), _p(aux), _p(ws), _nbytes(ws),
                                    _s(stream), arr)


def moe_read_device_status(ws, stream=None):
    return lib().moe_read_device_status(_p(ws), _s(stream))


def moe_test_lookback_timeout(ws, limit_ns, stream=None):
    return lib().moe_test_lookback_timeout(_p(ws), _nbytes(ws), int(limit_ns), _s(stream))


# ---- expert parallelism (pointer tables are device int64 tensors of addresses)

def moe_ep_recv_rows(cfg, n_ranks):
    return int(lib().moe_ep_recv_rows(ctypes.byref(cfg), int(n_ranks)))


def moe_ep_workspace_bytes(cfg, n_ranks):
    return int(lib().moe_ep_workspace_bytes(ctypes.byref(cfg), int(n_ranks)))


def moe_ep_layout(n_ranks, rank, n_experts, kept_all, dst_start, recv_offsets, stream=None):
    return lib().moe_ep_layout(int(n_ranks), int(rank), int(n_experts), _p(kept_all), _p(dst_start),
                               _p(recv_offsets), _s(stream))


def moe_ep_dispatch(cfg, n_ranks, rank, x, offsets, row_token, row_gate, drop, dst_start, recv_x, recv_rank,
                    recv_row, recv_gate, out, stream=None):
    return lib().moe_ep_dispatch(ctypes.byref(cfg), int(n_ranks), int(rank), _p(x), _p(offsets), _p(row_token),
                                 _p(row_gate), _p(drop), _p(dst_start), _p(recv_x), _p(recv_rank), _p(recv_row),
                                 _p(recv_gate), _p(out), _s(stream))


def moe_ep_expert_ffn(cfg, n_ranks, recv_x, recv_offsets, w1, b1, w3, b3, w2, b2, recv_rank, recv_row, recv_gate,
                      out_ptrs, ws, stream=None):
    return lib().moe_ep_expert_ffn(ctypes.byref(cfg), int(n_ranks), _p(recv_x), _p(recv_offsets), _p(w1), _p(b1),
                                   _p(w3), _p(b3), _p(w2), _p(b2), _p(recv_rank), _p(recv_row), _p(recv_gate),
                                   _p(out_ptrs), _p(ws), _nbytes(ws), _s(stream))


def moe_expert_backward_workspace_bytes(cfg):
    return int(lib().moe_expert_backward_workspace_bytes(ctypes.byref(cfg)))


def moe_expert_backward(cfg, xe, offsets, row_token, row_gate, idx, pos, drop, dout, w1, b1, w3, b3, w2, dx, dw1,
                        db1, dw3, db3, dw2, db2, ws, stream=None):
    return lib().moe_expert_backward(ctypes.byref(cfg), _p(xe), _p(offsets), _p(row_token), _p(row_gate), _p(idx),
                                     _p(pos), _p(drop), _p(dout), _p(w1), _p(b1), _p(w3), _p(b3), _p(w2), _p(dx),
                                     _p(dw1), _p(db1), _p(dw3), _p(db3), _p(dw2), _p(db2), _p(ws), _nbytes(ws),
                                     _s(stream))
