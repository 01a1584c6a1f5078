"""Python binding of libbytecross (the C ABI in include/bytecross.h).

Argument marshalling only: every step of the decode path runs in the CUDA
kernels of libbytecross.so.  PyTorch is used for device memory and streams.
There is no fallback: if the shared library is missing the import fails.
Build it with ``python activation_kv_sparsity_b200/build.py``.
"""
from __future__ import annotations

import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbytecross.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python activation_kv_sparsity_b200/build.py`")
_lib = C.CDLL(LIB_PATH)

# ------------------------------------------------------------------ enums
BC_OK, BC_EINVAL, BC_ENOMEM, BC_ECAPACITY, BC_ECUDA, BC_ETIMEOUT = range(6)
BC_DENSE, BC_ACT, BC_KV, BC_BOTH, BC_SNAP, BC_MASKED = range(6)
MODES = {"dense": BC_DENSE, "act": BC_ACT, "kv": BC_KV, "both": BC_BOTH, "snap": BC_SNAP, "masked": BC_MASKED}
(BC_TRACE_XN, BC_TRACE_SEL_QKV, BC_TRACE_Q, BC_TRACE_ATTN, BC_TRACE_SEL_O, BC_TRACE_XN2,
 BC_TRACE_SEL_GU, BC_TRACE_H, BC_TRACE_SEL_D, BC_TRACE_X, BC_TRACE_PAGE_SCORES, BC_TRACE_PAGES,
 BC_TRACE_QKV, BC_TRACE_SNAP_SCORES, BC_TRACE_SNAP_PAGES) = range(15)


class bc_config(C.Structure):
    _fields_ = [(n, C.c_int) for n in ("n_layers", "hidden", "intermediate", "n_heads", "n_kv_heads",
                                       "head_dim", "vocab", "max_ctx", "page")] + \
               [("rms_eps", C.c_float), ("rope_theta", C.c_float)]


class bc_weights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("embed", "lm_head", "final_norm", "attn_norm", "mlp_norm",
                                          "wqkv_t", "wo_t", "wgu_t", "wd_t")]


class bc_bytes(C.Structure):
    _fields_ = [(n, C.c_double) for n in (
        "weight_bytes", "head_bytes", "kv_bytes_per_token", "dense_bytes", "saved_bytes", "bound",
        "n_star", "n_star_ff", "impl_weight_bytes", "impl_head_bytes", "impl_kv_read_bytes",
        "impl_meta_read_bytes", "impl_kv_write_bytes", "impl_other_bytes", "impl_total_bytes")] + \
        [("pages_total", C.c_longlong), ("pages_kept", C.c_longlong)]


_P = C.c_void_p
_SIGS = {
    "bc_kv_pool_bytes": (C.c_size_t, [C.POINTER(bc_config)]),
    "bc_meta_pool_bytes": (C.c_size_t, [C.POINTER(bc_config)]),
    "bc_workspace_bytes": (C.c_size_t, [C.POINTER(bc_config)]),
    "bc_model_create": (C.c_int, [C.POINTER(bc_config), C.POINTER(bc_weights), _P, _P, _P, C.c_size_t, _P,
                                  C.POINTER(_P)]),
    "bc_model_destroy": (C.c_int, [_P]),
    "bc_set_stream": (C.c_int, [_P, _P]),
    "bc_set_graphs": (C.c_int, [_P, C.c_int]),
    "bc_kv_length": (C.c_int, [_P]),
    "bc_launch_count": (C.c_longlong, [_P]),
    "bc_kv_reset": (C.c_int, [_P, C.c_int]),
    "bc_kv_append": (C.c_int, [_P, _P, _P, C.c_int]),
    "bc_kv_snap_select": (C.c_int, [_P, _P, C.c_int, C.c_double, C.c_int, C.c_int]),
    "bc_decode_step": (C.c_int, [_P, C.c_int, C.c_int, C.c_double, C.c_double, C.c_int, C.c_int, C.c_int, _P]),
    "bc_decode_step_host": (C.c_int, [_P, C.c_int, C.c_int, C.c_double, C.c_double, C.c_int, C.c_int, C.c_int, _P]),
    "bc_trace": (C.c_int, [_P, C.c_int, C.c_int, C.POINTER(_P), C.POINTER(C.c_int), C.POINTER(C.c_int)]),
    "bc_gemv_scratch_bytes": (C.c_size_t, [C.c_int]),
    "bc_gemv": (C.c_int, [_P, C.c_int, C.c_int, _P, _P, C.c_int, _P, _P, C.c_size_t, _P]),
    "bc_gemv_noalloc_max_dout": (C.c_int, []),
    "bc_gemv_noalloc": (C.c_int, [_P, C.c_int, C.c_int, _P, _P, C.c_int, _P, _P]),
    "bc_gemv_batch_scratch_bytes": (C.c_size_t, [C.c_int, C.c_int, C.c_int]),
    "bc_gemv_batch": (C.c_int, [_P, C.c_int, C.c_int, _P, _P, C.c_int, C.c_int, _P, _P, _P, C.c_size_t, _P]),
    "bc_select_topk": (C.c_int, [_P, C.c_int, C.c_int, _P, _P]),
    "bc_attention_scratch_bytes": (C.c_size_t, [C.c_int, C.c_int]),
    "bc_attention": (C.c_int, [_P, _P, C.c_int, C.c_int, C.c_int, C.c_int, _P, C.c_int, C.c_int, _P, _P,
                               C.c_size_t, _P]),
    "bc_byte_account": (C.c_int, [C.POINTER(bc_config), C.c_int, C.c_double, C.c_double, C.c_longlong, C.c_int,
                                  C.c_int, C.c_int, C.POINTER(bc_bytes)]),
    "bc_crossover_batch": (C.c_int, [C.POINTER(bc_config), C.c_double, C.c_double, C.c_int,
                                     C.POINTER(C.c_double)]),
    "bc_batch_workspace_bytes": (C.c_size_t, [C.POINTER(bc_config), C.c_int]),
    "bc_batch_create": (C.c_int, [C.POINTER(bc_config), C.POINTER(bc_weights), C.c_int, _P, _P, _P, C.c_size_t, _P,
                                  C.POINTER(_P)]),
    "bc_batch_destroy": (C.c_int, [_P]),
    "bc_batch_set_graphs": (C.c_int, [_P, C.c_int]),
    "bc_batch_length": (C.c_int, [_P]),
    "bc_batch_launch_count": (C.c_longlong, [_P]),
    "bc_batch_reset": (C.c_int, [_P, C.c_int]),
    "bc_batch_append": (C.c_int, [_P, _P, _P, C.c_int]),
    "bc_batch_step": (C.c_int, [_P, C.POINTER(C.c_int), C.c_int, C.c_double, C.c_double, C.c_int, C.c_int, C.c_int,
                                _P]),
    "bc_batch_trace": (C.c_int, [_P, C.c_int, C.c_int, C.c_int, C.POINTER(_P), C.POINTER(C.c_int),
                                 C.POINTER(C.c_int)]),
    "bc_last_error": (C.c_char_p, []),
    "bc_status_string": (C.c_char_p, [C.c_int]),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args
    globals()[_name] = _f


class BCError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        msg = bc_last_error().decode(errors="replace")
        super().__init__(f"{where}: {bc_status_string(status).decode()} ({status}): {msg}")


def check(status, where=""):
    if status != BC_OK:
        raise BCError(status, where)


def config(d: dict, max_ctx: int) -> bc_config:
    return bc_config(d["n_layers"], d["hidden"], d["intermediate"], d["n_heads"], d["n_kv_heads"],
                     d["head_dim"], d["vocab"], max_ctx, d.get("page", 16), d.get("rms_eps", 1e-5),
                     d.get("rope_theta", 5e5))


def byte_account(cfg: dict, mode: str, n_ctx: int, rp=1.0, rkv=1.0, sinks=1, recent=16) -> dict:
    c = config(cfg, max(n_ctx + 1, 1))
    out = bc_bytes()
    check(bc_byte_account(C.byref(c), MODES[mode], rp, rkv, n_ctx, sinks, recent, c.page, C.byref(out)),
          "bc_byte_account")
    return {name: getattr(out, name) for name, _ in bc_bytes._fields_}


def crossover_batch(cfg: dict, union_keep: float, rkv: float, batch: int) -> float:
    """bc_crossover_batch: the batch byte crossover, in tokens."""
    c = config(cfg, 1)
    out = C.c_double()
    check(bc_crossover_batch(C.byref(c), union_keep, rkv, batch, C.byref(out)), "bc_crossover_batch")
    return out.value


def _stream_ptr(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


class Model:
    """Owns the device buffers (allocated with torch) and the bc_model handle."""

    def __init__(self, cfg: dict, weights: dict, max_ctx: int, stream=None):
        import torch
        self.cfg = cfg
        self.c = config(cfg, max_ctx)
        self.weights = weights           # keep the tensors alive
        dev = weights["embed"].device
        self.stream = stream if stream is not None else torch.cuda.current_stream(dev)
        kvb = bc_kv_pool_bytes(C.byref(self.c))
        mb = bc_meta_pool_bytes(C.byref(self.c))
        wsb = bc_workspace_bytes(C.byref(self.c))
        if not (kvb and mb and wsb):
            raise ValueError("bad config for libbytecross")
        self.kv_pool = torch.empty(kvb, dtype=torch.uint8, device=dev)
        self.meta_pool = torch.empty(mb, dtype=torch.uint8, device=dev)
        self.workspace = torch.zeros(wsb, dtype=torch.uint8, device=dev)
        w = bc_weights(*(C.c_void_p(weights[k].data_ptr()) for k in (
            "embed", "lm_head", "final_norm", "attn_norm", "mlp_norm", "wqkv_t", "wo_t", "wgu_t", "wd_t")))
        h = C.c_void_p()
        check(bc_model_create(C.byref(self.c), C.byref(w), C.c_void_p(self.kv_pool.data_ptr()),
                              C.c_void_p(self.meta_pool.data_ptr()), C.c_void_p(self.workspace.data_ptr()),
                              wsb, C.c_void_p(self.stream.cuda_stream), C.byref(h)), "bc_model_create")
        self.h = h

    def close(self):
        if getattr(self, "h", None):
            bc_model_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __len__(self):
        return bc_kv_length(self.h)

    def set_graphs(self, enable: bool):
        check(bc_set_graphs(self.h, 1 if enable else 0), "bc_set_graphs")

    def launches(self) -> int:
        return bc_launch_count(self.h)

    def reset(self, n_ctx: int):
        check(bc_kv_reset(self.h, n_ctx), "bc_kv_reset")

    def append(self, k, v):
        """k, v: bf16 device tensors [L][Hkv][n][hd]."""
        k, v = k.contiguous(), v.contiguous()
        check(bc_kv_append(self.h, C.c_void_p(k.data_ptr()), C.c_void_p(v.data_ptr()), k.shape[2]),
              "bc_kv_append")

    def snap_select(self, q_obs, rkv, sinks=1, recent=16):
        """Once-after-prefill page selection; q_obs: f32 device tensor
        [L][n_obs][Hq][hd] of rotated observation queries."""
        q_obs = q_obs.contiguous()
        check(bc_kv_snap_select(self.h, C.c_void_p(q_obs.data_ptr()), q_obs.shape[1], rkv, sinks, recent),
              "bc_kv_snap_select")

    def step(self, token: int, mode: str, logits, rp=1.0, rkv=1.0, sinks=1, recent=16):
        check(bc_decode_step(self.h, int(token), MODES[mode], rp, rkv, sinks, recent, self.c.page,
                             C.c_void_p(logits.data_ptr())), "bc_decode_step")

    def step_host(self, token: int, mode: str, logits_host, rp=1.0, rkv=1.0, sinks=1, recent=16):
        check(bc_decode_step_host(self.h, int(token), MODES[mode], rp, rkv, sinks, recent, self.c.page,
                                  C.c_void_p(logits_host.data_ptr())), "bc_decode_step_host")

    def trace(self, layer: int, kind: int):
        """Device tensor view of a per-layer trace from the last step."""
        import torch
        ptr, cnt, stride = C.c_void_p(), C.c_int(), C.c_int()
        check(bc_trace(self.h, layer, kind, C.byref(ptr), C.byref(cnt), C.byref(stride)), "bc_trace")
        off = ptr.value - self.workspace.data_ptr()
        is_int = kind in (BC_TRACE_SEL_QKV, BC_TRACE_SEL_O, BC_TRACE_SEL_GU, BC_TRACE_SEL_D, BC_TRACE_PAGES,
                          BC_TRACE_SNAP_PAGES)
        dt = torch.int32 if is_int else torch.float32
        if stride.value:
            rows = self.cfg["n_kv_heads"]
            t = self.workspace[off:off + 4 * rows * stride.value].view(dt).view(rows, stride.value)
            return t[:, :cnt.value]
        return self.workspace[off:off + 4 * cnt.value].view(dt)


_INT_TRACES = (BC_TRACE_SEL_QKV, BC_TRACE_SEL_O, BC_TRACE_SEL_GU, BC_TRACE_SEL_D, BC_TRACE_PAGES, BC_TRACE_SNAP_PAGES)


class Batch:
    """A batch of sequences decoding in lock step (bc_batch_*): owns the
    sequences' KV and bound pools and the workspace (allocated with torch)."""

    def __init__(self, cfg: dict, weights: dict, batch: int, max_ctx: int, stream=None):
        import torch
        self.cfg = cfg
        self.B = batch
        self.c = config(cfg, max_ctx)
        self.weights = weights
        dev = weights["embed"].device
        self.stream = stream if stream is not None else torch.cuda.current_stream(dev)
        kvb = bc_kv_pool_bytes(C.byref(self.c))
        mb = bc_meta_pool_bytes(C.byref(self.c))
        wsb = bc_batch_workspace_bytes(C.byref(self.c), batch)
        if not (kvb and mb and wsb):
            raise ValueError("bad config or batch size for a libbytecross batch")
        self.kv_pool = torch.empty(batch * kvb, dtype=torch.uint8, device=dev)
        self.meta_pool = torch.empty(batch * mb, dtype=torch.uint8, device=dev)
        self.workspace = torch.zeros(wsb, dtype=torch.uint8, device=dev)
        w = bc_weights(*(C.c_void_p(weights[k].data_ptr()) for k in (
            "embed", "lm_head", "final_norm", "attn_norm", "mlp_norm", "wqkv_t", "wo_t", "wgu_t", "wd_t")))
        h = C.c_void_p()
        check(bc_batch_create(C.byref(self.c), C.byref(w), batch, C.c_void_p(self.kv_pool.data_ptr()),
                              C.c_void_p(self.meta_pool.data_ptr()), C.c_void_p(self.workspace.data_ptr()), wsb,
                              C.c_void_p(self.stream.cuda_stream), C.byref(h)), "bc_batch_create")
        self.h = h

    def close(self):
        if getattr(self, "h", None):
            bc_batch_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __len__(self):
        return bc_batch_length(self.h)

    def set_graphs(self, enable: bool):
        check(bc_batch_set_graphs(self.h, 1 if enable else 0), "bc_batch_set_graphs")

    def launches(self) -> int:
        return bc_batch_launch_count(self.h)

    def reset(self, n_ctx: int):
        check(bc_batch_reset(self.h, n_ctx), "bc_batch_reset")

    def append(self, k, v):
        """k, v: bf16 device tensors [batch][L][Hkv][n][hd]."""
        k, v = k.contiguous(), v.contiguous()
        check(bc_batch_append(self.h, C.c_void_p(k.data_ptr()), C.c_void_p(v.data_ptr()), k.shape[3]),
              "bc_batch_append")

    def step(self, tokens, mode: str, logits, rp=1.0, rkv=1.0, sinks=1, recent=16):
        """tokens: B ints; logits: f32 device tensor [B][vocab]."""
        toks = (C.c_int * self.B)(*[int(t) for t in tokens])
        check(bc_batch_step(self.h, toks, MODES[mode], rp, rkv, sinks, recent, self.c.page,
                            C.c_void_p(logits.data_ptr())), "bc_batch_step")

    def seq(self, b: int):
        """A view of sequence b with the trace() of a Model."""
        return _BatchSeq(self, b)


class _BatchSeq:
    def __init__(self, batch: Batch, b: int):
        self.batch, self.b, self.cfg = batch, b, batch.cfg

    def trace(self, layer: int, kind: int):
        import torch
        bt = self.batch
        ptr, cnt, stride = C.c_void_p(), C.c_int(), C.c_int()
        check(bc_batch_trace(bt.h, self.b, layer, kind, C.byref(ptr), C.byref(cnt), C.byref(stride)),
              "bc_batch_trace")
        off = ptr.value - bt.workspace.data_ptr()
        dt = torch.int32 if kind in _INT_TRACES else torch.float32
        if stride.value:
            rows = self.cfg["n_kv_heads"]
            t = bt.workspace[off:off + 4 * rows * stride.value].view(dt).view(rows, stride.value)
            return t[:, :cnt.value]
        return bt.workspace[off:off + 4 * cnt.value].view(dt)


# ------------------------------------------------------------------ single kernels

def gemv(W, x, idx, y, scratch, stream=None):
    d_in, d_out = W.shape
    k = d_in if idx is None else idx.numel()
    check(bc_gemv(C.c_void_p(W.data_ptr()), d_in, d_out, C.c_void_p(x.data_ptr()),
                  C.c_void_p(idx.data_ptr()) if idx is not None else None, k, C.c_void_p(y.data_ptr()),
                  C.c_void_p(scratch.data_ptr()), scratch.numel() * scratch.element_size(),
                  _stream_ptr(stream)), "bc_gemv")


def gemv_noalloc(W, x, idx, y, stream=None):
    """bc_gemv without a scratch argument (scratch is a static device array)."""
    d_in, d_out = W.shape
    k = d_in if idx is None else idx.numel()
    check(bc_gemv_noalloc(C.c_void_p(W.data_ptr()), d_in, d_out, C.c_void_p(x.data_ptr()),
                          C.c_void_p(idx.data_ptr()) if idx is not None else None, k, C.c_void_p(y.data_ptr()),
                          _stream_ptr(stream)), "bc_gemv_noalloc")


def gemv_batch(W, x, idx, y, scratch, n_union=None, stream=None):
    """bc_gemv_batch: x [B][d_in] f32, idx [B][k] int32 (or None for all
    channels), y [B][d_out] f32, n_union an int32 tensor of one element or None."""
    d_in, d_out = W.shape
    B = x.shape[0]
    k = d_in if idx is None else idx.shape[1]
    check(bc_gemv_batch(C.c_void_p(W.data_ptr()), d_in, d_out, C.c_void_p(x.data_ptr()),
                        C.c_void_p(idx.data_ptr()) if idx is not None else None, k, B,
                        C.c_void_p(y.data_ptr()), C.c_void_p(n_union.data_ptr()) if n_union is not None else None,
                        C.c_void_p(scratch.data_ptr()), scratch.numel() * scratch.element_size(),
                        _stream_ptr(stream)), "bc_gemv_batch")


def select_topk(v, k, idx, stream=None):
    check(bc_select_topk(C.c_void_p(v.data_ptr()), v.numel(), k, C.c_void_p(idx.data_ptr()),
                         _stream_ptr(stream)), "bc_select_topk")


def attention(q, kv, n_kv_heads, group, head_dim, Pmax, pages, n_pages, n_tok, out, scratch, stream=None):
    check(bc_attention(C.c_void_p(q.data_ptr()), C.c_void_p(kv.data_ptr()), n_kv_heads, group, head_dim, Pmax,
                       C.c_void_p(pages.data_ptr()) if pages is not None else None, n_pages, n_tok,
                       C.c_void_p(out.data_ptr()), C.c_void_p(scratch.data_ptr()),
                       scratch.numel() * scratch.element_size(), _stream_ptr(stream)), "bc_attention")
