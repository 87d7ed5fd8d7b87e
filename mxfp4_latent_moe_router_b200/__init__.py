"""Python binding of libmoe_b200.so, the B200 latent-MoE decode block.

Argument marshalling only: every step of the block runs in the CUDA kernels
behind the C ABI declared in ``include/moe.h``.  The functions below carry the
C names; ``MoePlan`` bundles them for convenience.  PyTorch provides device
memory and streams.  There is no CPU fallback: if the shared library is
missing or has no device to run on, the calls raise.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_OK = 0
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED",
                3: "MOE_ERR_NOT_LOADED", 4: "MOE_ERR_OOM", 5: "MOE_ERR_CUDA",
                6: "MOE_ERR_TIMEOUT", 7: "MOE_ERR_RANGE"}
MOE_SCORE_SOFTMAX = 0
MOE_SCORE_SIGMOID = 1
MOE_DBG_LOGITS, MOE_DBG_Z, MOE_DBG_H, MOE_DBG_Y, MOE_DBG_HS = range(5)

# every entry point include/moe.h declares
ABI_SYMBOLS = ["moe_plan_create", "moe_load_weights", "moe_forward", "moe_forward_host",
               "moe_last_routing", "moe_debug_fetch", "moe_sync_status", "moe_get_plan_info",
               "moe_plan_destroy", "moe_status_str", "moe_set_profiling", "moe_get_profile",
               "moe_route_noalloc", "moe_debug_trace", "moe_debug_geometry",
               "moe_debug_expire_wait", "moe_set_next_layer"]
# launch slots: the four kernels a forward runs (the dense front kernel
# streams the router, latent-projection and shared-expert gate/up rows and
# runs top-k), then the single fused launch that MOE_FUSED=1 selects for
# forwards of at most 8 tokens
KERNEL_NAMES = ["dense_front", "expert_gate_up", "expert_down", "latent_tail", "fused_block",
                "shared_front", "shared_tail"]


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__("%s: %s" % (where, STATUS_NAMES.get(status, str(status))))


class moe_config(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("latent", ctypes.c_int32),
                ("num_experts", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("expert_inter", ctypes.c_int32), ("shared_inter", ctypes.c_int32),
                ("max_tokens", ctypes.c_int32), ("score_fn", ctypes.c_int32),
                ("renormalize", ctypes.c_int32), ("routed_scale", ctypes.c_float),
                ("shared_sms", ctypes.c_int32)]


class moe_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "router_w", "router_bias", "w_in", "w_out", "gu_codes", "gu_scales", "dn_codes",
        "dn_scales", "sh_gate", "sh_up", "sh_down")]


class moe_plan_info(ctypes.Structure):
    _fields_ = [("device", ctypes.c_int32), ("num_sms", ctypes.c_int32),
                ("front_ctas", ctypes.c_int32), ("expert_ctas", ctypes.c_int32),
                ("packed_bytes", ctypes.c_int64), ("workspace_bytes", ctypes.c_int64),
                ("dense_weight_bytes", ctypes.c_int64), ("expert_weight_bytes", ctypes.c_int64),
                ("kernels_per_forward", ctypes.c_int32)]


class moe_geometry(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("grid", ctypes.c_int32), ("ctas_per_sm", ctypes.c_int32),
                ("token_tiles", ctypes.c_int32), ("max_piece_tokens", ctypes.c_int32),
                ("stages", ctypes.c_int32), ("stage_bytes", ctypes.c_int32),
                ("pieces_per_row_block", ctypes.c_int32), ("smem_bytes", ctypes.c_int64),
                ("partial_floats_needed", ctypes.c_int64),
                ("partial_floats_capacity", ctypes.c_int64),
                ("route_logit_floats", ctypes.c_int32), ("resident_tail_bytes", ctypes.c_int32)]


_lib = None


def load_library():
    """Load the shared library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError("libmoe_b200.so is not built (python -m mxfp4_latent_moe_router_b200.build)")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.c_void_p
    lib.moe_plan_create.argtypes = [ctypes.POINTER(moe_config), ctypes.c_int, ctypes.POINTER(P)]
    lib.moe_load_weights.argtypes = [P, ctypes.POINTER(moe_weights), P]
    lib.moe_forward.argtypes = [P, P, ctypes.c_int32, P, P]
    lib.moe_forward_host.argtypes = [P, P, ctypes.c_int32, P, P]
    lib.moe_last_routing.argtypes = [P, P, P, ctypes.c_int32]
    lib.moe_debug_fetch.argtypes = [P, ctypes.c_int32, ctypes.c_int32, P, ctypes.c_int64]
    lib.moe_sync_status.argtypes = [P]
    lib.moe_debug_expire_wait.argtypes = [P, ctypes.c_int32, P]
    lib.moe_get_plan_info.argtypes = [P, ctypes.POINTER(moe_plan_info)]
    lib.moe_plan_destroy.argtypes = [P]
    lib.moe_set_next_layer.argtypes = [P, P, ctypes.c_int64]
    lib.moe_plan_destroy.restype = None
    lib.moe_route_noalloc.argtypes = [P, P, P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                      ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                      ctypes.c_float, P, P, P]
    lib.moe_set_profiling.argtypes = [P, ctypes.c_int32]
    lib.moe_debug_trace.argtypes = [P, P, ctypes.c_int64]
    lib.moe_get_profile.argtypes = [P, P, P]
    lib.moe_debug_geometry.argtypes = [ctypes.POINTER(moe_config), ctypes.c_int32, ctypes.c_int32,
                                       ctypes.POINTER(moe_geometry)]
    lib.moe_status_str.argtypes = [ctypes.c_int]
    lib.moe_status_str.restype = ctypes.c_char_p
    for n in ABI_SYMBOLS:
        if n not in ("moe_plan_destroy", "moe_status_str"):
            getattr(lib, n).restype = ctypes.c_int
    _lib = lib
    return lib


def _check(st: int, where: str):
    if st != MOE_OK:
        raise MoeError(st, where)


def _ptr(t) -> int | None:
    if t is None:
        return None
    if hasattr(t, "data_ptr"):
        return t.data_ptr()
    return t.ctypes.data  # numpy


def _stream_ptr(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if hasattr(stream, "cuda_stream"):
        return stream.cuda_stream
    return int(stream)


# ---- C names -------------------------------------------------------------

def moe_status_str(status: int) -> str:
    return load_library().moe_status_str(status).decode()


def moe_plan_create(cfg: moe_config, device: int = 0) -> int:
    h = ctypes.c_void_p()
    _check(load_library().moe_plan_create(ctypes.byref(cfg), device, ctypes.byref(h)), "moe_plan_create")
    return h.value


def moe_load_weights(plan: int, w: moe_weights, stream=None) -> None:
    _check(load_library().moe_load_weights(plan, ctypes.byref(w), _stream_ptr(stream)), "moe_load_weights")


def moe_forward(plan: int, x, num_tokens: int, out, stream=None) -> int:
    return load_library().moe_forward(plan, _ptr(x), num_tokens, _ptr(out), _stream_ptr(stream))


def moe_forward_host(plan: int, x_host, num_tokens: int, out_host, stream=None) -> int:
    return load_library().moe_forward_host(plan, _ptr(x_host), num_tokens, _ptr(out_host),
                                           _stream_ptr(stream))


def moe_last_routing(plan: int, ids_host, w_host, num_tokens: int) -> None:
    _check(load_library().moe_last_routing(plan, _ptr(ids_host), _ptr(w_host), num_tokens),
           "moe_last_routing")


def moe_debug_fetch(plan: int, what: int, num_tokens: int, host) -> None:
    _check(load_library().moe_debug_fetch(plan, what, num_tokens, _ptr(host), host.size),
           "moe_debug_fetch")


def moe_sync_status(plan: int) -> int:
    return load_library().moe_sync_status(plan)


def moe_debug_expire_wait(plan: int, limit_polls: int, stream=None) -> int:
    """Test of the timeout path: a bounded wait that runs out (see include/moe.h)."""
    return load_library().moe_debug_expire_wait(plan, limit_polls, _stream_ptr(stream))


def moe_get_plan_info(plan: int) -> moe_plan_info:
    info = moe_plan_info()
    _check(load_library().moe_get_plan_info(plan, ctypes.byref(info)), "moe_get_plan_info")
    return info


def moe_set_profiling(plan: int, enable: bool) -> None:
    _check(load_library().moe_set_profiling(plan, int(enable)), "moe_set_profiling")


def moe_get_profile(plan: int):
    """-> (milliseconds per kernel kind as a dict, number of profiled forwards)."""
    ms = (ctypes.c_float * len(KERNEL_NAMES))()
    n = ctypes.c_int32()
    _check(load_library().moe_get_profile(plan, ms, ctypes.byref(n)), "moe_get_profile")
    return dict(zip(KERNEL_NAMES, list(ms))), n.value


def moe_route_noalloc(x, router_w, router_bias, num_tokens: int, hidden: int, num_experts: int,
                      top_k: int, score_fn: int, renormalize: int, routed_scale: float, ids, weights,
                      stream=None) -> int:
    """Router + top-k without any allocation (device tensors in, device tensors out)."""
    return load_library().moe_route_noalloc(_ptr(x), _ptr(router_w), _ptr(router_bias), num_tokens,
                                            hidden, num_experts, top_k, score_fn, renormalize,
                                            routed_scale, _ptr(ids), _ptr(weights),
                                            _stream_ptr(stream))


def moe_debug_trace(plan: int, num_sms: int):
    """Per-CTA timeline of the last forward: uint64 array [7 launch slots][num_sms][24]."""
    import numpy as np
    a = np.zeros((len(KERNEL_NAMES), num_sms, 24), np.uint64)
    _check(load_library().moe_debug_trace(plan, a.ctypes.data, a.size), "moe_debug_trace")
    return a


def moe_debug_geometry(cfg: moe_config, num_sms: int, num_tokens: int) -> list:
    """Launch geometry of the four kernels for a forward of num_tokens tokens on
    num_sms SMs, with default settings (host only: no device needed)."""
    out = (moe_geometry * 6)()
    _check(load_library().moe_debug_geometry(ctypes.byref(cfg), num_sms, num_tokens, out),
           "moe_debug_geometry")
    return [{f[0]: getattr(g, f[0]) for f in moe_geometry._fields_} for g in out]


def moe_set_next_layer(plan: int, next_plan, nbytes: int) -> int:
    """Cross-layer prefetch of next_plan's front weights (see include/moe.h)."""
    return load_library().moe_set_next_layer(plan, next_plan, nbytes)


def moe_plan_destroy(plan: int) -> None:
    if plan:
        load_library().moe_plan_destroy(plan)


# ---- convenience wrapper ---------------------------------------------------

def config_from_shape(shape, max_tokens: int | None = None, shared_sms: int = 0) -> moe_config:
    return moe_config(shape.hidden, shape.latent, shape.num_experts, shape.top_k,
                      shape.expert_inter, shape.shared_inter,
                      shape.tokens if max_tokens is None else max_tokens, shape.score_fn,
                      shape.renormalize, float(shape.routed_scale), shared_sms)


def weights_to_device(w: dict, device: str = "cuda"):
    """numpy canonical weights -> dict of torch device tensors (raw bits)."""
    import numpy as np
    import torch
    out = {}
    for k, v in w.items():
        if v is None:
            out[k] = None
            continue
        a = np.ascontiguousarray(v)
        if a.dtype == np.uint16:
            a = a.view(np.int16)
        out[k] = torch.from_numpy(a).to(device)
    return out


class MoePlan:
    """One plan = one layer's packed weights + workspace on one device."""

    def __init__(self, cfg: moe_config, device: int = 0):
        self.cfg = cfg
        self.device = device
        self.handle = moe_plan_create(cfg, device)

    def load(self, dev_w: dict, stream=None):
        w = moe_weights(**{f[0]: _ptr(dev_w.get(f[0])) for f in moe_weights._fields_})
        moe_load_weights(self.handle, w, stream)

    def forward(self, x, out, stream=None):
        st = moe_forward(self.handle, x, x.shape[0], out, stream)
        _check(st, "moe_forward")

    def forward_host(self, x_host, out_host, stream=None):
        st = moe_forward_host(self.handle, x_host, x_host.shape[0], out_host, stream)
        _check(st, "moe_forward_host")

    def routing(self, B: int):
        import numpy as np
        ids = np.zeros((B, self.cfg.top_k), np.int32)
        w = np.zeros((B, self.cfg.top_k), np.float32)
        moe_last_routing(self.handle, ids, w, B)
        return ids, w

    def fetch(self, what: int, B: int):
        import numpy as np
        c = self.cfg
        shape = {MOE_DBG_LOGITS: (B, c.num_experts), MOE_DBG_Z: (B, c.latent),
                 MOE_DBG_H: (B, c.top_k, c.expert_inter), MOE_DBG_Y: (B, c.top_k, c.latent),
                 MOE_DBG_HS: (B, c.shared_inter)}[what]
        a = np.zeros(shape, np.float32)
        moe_debug_fetch(self.handle, what, B, a)
        return a

    def sync_status(self) -> int:
        return moe_sync_status(self.handle)

    def set_next_layer(self, nxt, nbytes: int):
        """Pull nbytes of nxt's front weights into L2 during each forward
        (nxt None: off)."""
        st = moe_set_next_layer(self.handle, nxt.handle if nxt is not None else None, nbytes)
        _check(st, "moe_set_next_layer")

    def info(self) -> moe_plan_info:
        return moe_get_plan_info(self.handle)

    def close(self):
        if self.handle:
            moe_plan_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
