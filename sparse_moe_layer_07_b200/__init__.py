"""B200-native forward pass of a Grok-1-style top-2 sparse MoE SwiGLU layer.

Thin ctypes binding over ``libmoe_b200.so`` (C ABI declared in
``include/moe.h``).  The functions below carry the same names as the C entry
points without the ``moe_`` prefix; they only check and marshal arguments
(tensor pointers, the current CUDA stream) and allocate output tensors with
PyTorch when the caller does not pass them.  Every step of the layer runs in
the library's CUDA kernels: there is no fallback of any kind, and importing
this package fails if the library has not been built
(``python sparse_moe_layer_07_b200/build.py``).
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

__all__ = [
    "MoEError", "Config", "LIB_PATH", "lib", "abi_version", "capacity", "workspace_size",
    "dispatch_workspace_size", "router_topk", "dispatch", "expert_ffn", "expert_gate_up",
    "expert_down", "combine", "layer_forward", "layer_forward_host", "get_device_error",
    "STATUS", "DEVERR", "ExpertUtilization", "dispatch_noalloc", "NOALLOC_MAX_TOKENS", "quantize_int8", "expert_ffn_w8",
    "layer_forward_w8", "QuantizedExperts", "w8_workspace_views", "expert_down_combine",
    "layer_forward_host_batches", "workspace_size_host_batches",
    "workspace_size_train", "layer_forward_train", "layer_backward", "route_counts", "dispatch_shard", "gather_rows",
    "EP_MAX_WORLD", "EpPeers", "ep_dispatch_peers", "ep_expert_ffn_peers", "ep_combine_peers", "peer_export",
    "peer_import", "peer_release",
    "GEMM_TILES", "set_gemm_tiles", "gemm_tiles", "PHASES", "profile_phases", "profile_read",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe_b200.so")

STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_WORKSPACE",
          4: "MOE_ERR_CUDA", 5: "MOE_ERR_DEVICE_CHECK", 6: "MOE_ERR_TIMEOUT"}
DEVERR = {"EXPERT_INDEX": 0x1, "SLOT_INDEX": 0x2, "OFFSETS": 0x4, "TIMEOUT": 0x8}
_DTYPES = {"f32": 0, "bf16": 1}
NOALLOC_MAX_TOKENS = 1 << 20
_TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {STATUS.get(status, status)}")
        self.status = status


class _CConfig(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("d", ctypes.c_int64), ("f", ctypes.c_int64),
                ("E", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("capacity_factor", ctypes.c_double), ("dtype", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


EP_MAX_WORLD = 8


class _CEpPeers(ctypes.Structure):
    _fields_ = [("world", ctypes.c_int32), ("rank", ctypes.c_int32),
                ("x_grp", ctypes.c_void_p * EP_MAX_WORLD), ("src", ctypes.c_void_p * EP_MAX_WORLD),
                ("scale", ctypes.c_void_p * EP_MAX_WORLD), ("sums", ctypes.c_void_p * EP_MAX_WORLD)]


class _CPeerHandle(ctypes.Structure):
    _fields_ = [("ipc", ctypes.c_uint8 * 64), ("offset", ctypes.c_uint64)]


_BUILD_HINT = "build it with `python sparse_moe_layer_07_b200/build.py`"


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: {_BUILD_HINT}")
    L = ctypes.CDLL(LIB_PATH)
    P = ctypes.c_void_p
    cfgp = ctypes.POINTER(_CConfig)
    sz = ctypes.c_size_t
    sig = {
        "moe_abi_version": ([], ctypes.c_int32),
        "moe_status_string": ([ctypes.c_int], ctypes.c_char_p),
        "moe_capacity": ([cfgp], ctypes.c_int64),
        "moe_dispatch_workspace_size": ([cfgp], sz),
        "moe_expert_ffn_workspace_size": ([cfgp], sz),
        "moe_workspace_size": ([cfgp], sz),
        "moe_router_topk": ([cfgp, P, P, P, P, P, P, P], ctypes.c_int),
        "moe_dispatch": ([cfgp, P, P, P, P, P, P, P, P, P, P, P, sz, P], ctypes.c_int),
        "moe_expert_ffn": ([cfgp, P, P, P, P, P, P, P, P, P, sz, P], ctypes.c_int),
        "moe_expert_gate_up": ([cfgp, P, P, P, P, P, P], ctypes.c_int),
        "moe_expert_down": ([cfgp, P, P, P, P, P, P, sz, P], ctypes.c_int),
        "moe_combine": ([cfgp, P, P, P, ctypes.c_int32, P, P], ctypes.c_int),
        "moe_layer_forward": ([cfgp, P, P, P, P, P, P, P, P, P, sz, P], ctypes.c_int),
        "moe_layer_forward_host": ([cfgp, P, P, P, P, P, P, P, P, sz, P], ctypes.c_int),
        "moe_workspace_size_host_batches": ([cfgp], sz),
        "moe_expert_down_combine_workspace_size": ([cfgp], sz),
        "moe_workspace_size_train": ([cfgp], sz),
        "moe_route_counts": ([cfgp, P, P, P], ctypes.c_int),
        "moe_gather_rows": ([P, ctypes.c_int64, P, ctypes.c_int64, ctypes.c_int64, P, P], ctypes.c_int),
        "moe_check_bounded_wait": ([ctypes.c_int64, P], ctypes.c_int),
        "moe_dispatch_shard": ([cfgp, ctypes.c_int64, P, ctypes.c_int32, ctypes.c_int32, P, P, P, P, P, P, P, P, P,
                                P, P, sz, P], ctypes.c_int),
        "moe_layer_forward_train": ([cfgp, P, P, P, P, P, P, P, P, sz, P], ctypes.c_int),
        "moe_layer_backward": ([cfgp, P, P, P, P, P, P, P, P, P, P, P, P, P, sz, P], ctypes.c_int),
        "moe_expert_down_combine": ([cfgp, P, P, P, P, P, P, P, sz, P], ctypes.c_int),
        "moe_layer_forward_host_batches": ([cfgp, ctypes.c_int64, P, P, P, P, P, P, P, P, sz, P], ctypes.c_int),
        "moe_get_device_error": ([ctypes.POINTER(ctypes.c_int32), ctypes.c_int32], ctypes.c_int),
        "moe_set_gemm_tiles": ([ctypes.c_int32, ctypes.POINTER(ctypes.c_int32)], ctypes.c_int),
        "moe_dispatch_noalloc": ([cfgp, P, P, P, P, P, P, P, P, P, P, P], ctypes.c_int),
        "moe_quantize_int8": ([cfgp, P, ctypes.c_int64, ctypes.c_int64, P, P, P], ctypes.c_int),
        "moe_expert_ffn_w8_workspace_size": ([cfgp], sz),
        "moe_workspace_size_w8": ([cfgp], sz),
        "moe_expert_ffn_w8": ([cfgp, P, P, P, P, P, P, P, P, P, P, P, sz, P], ctypes.c_int),
        "moe_layer_forward_w8": ([cfgp, P, P, P, P, P, P, P, P, P, P, P, P, sz, P], ctypes.c_int),
        "moe_expert_utilization": ([P, ctypes.c_int32, P, P, P], ctypes.c_int),
        "moe_profile_phases": ([ctypes.c_int32], ctypes.c_int),
        "moe_profile_read": ([P, P, ctypes.c_int32], ctypes.c_int),
        "moe_ep_dispatch_peers": ([cfgp, ctypes.POINTER(_CEpPeers), P, P, P, P, P, P, P], ctypes.c_int),
        "moe_ep_expert_ffn_peers": ([cfgp, ctypes.POINTER(_CEpPeers), P, P, P, P, P, P], ctypes.c_int),
        "moe_ep_combine_peers": ([cfgp, ctypes.POINTER(_CEpPeers), P, P], ctypes.c_int),
        "moe_peer_export": ([P, ctypes.POINTER(_CPeerHandle)], ctypes.c_int),
        "moe_peer_import": ([ctypes.POINTER(_CPeerHandle), ctypes.POINTER(ctypes.c_void_p)], ctypes.c_int),
        "moe_peer_release": ([P, ctypes.POINTER(_CPeerHandle)], ctypes.c_int),
    }
    for name, (args, res) in sig.items():
        try:
            fn = getattr(L, name)
        except AttributeError as exc:
            raise ImportError(f"{LIB_PATH} lacks {name} (out of date): {_BUILD_HINT}") from exc
        fn.argtypes = args
        fn.restype = res
    return L


lib = _load()


class Config:
    """Layer hyper-parameters (``moe_config_t``)."""

    def __init__(self, T: int, d: int, f: int, E: int = 8, top_k: int = 2,
                 capacity_factor: float = 1.25, dtype: str = "bf16"):
        if dtype not in _DTYPES:
            raise ValueError(f"dtype must be one of {sorted(_DTYPES)}")
        self.T, self.d, self.f, self.E, self.top_k = int(T), int(d), int(f), int(E), int(top_k)
        self.capacity_factor = float(capacity_factor)
        self.dtype = dtype
        self._c = _CConfig(self.T, self.d, self.f, self.E, self.top_k, self.capacity_factor,
                           _DTYPES[dtype], 0)

    @property
    def torch_dtype(self):
        return _TORCH_DTYPE[self.dtype]

    @property
    def ref(self):
        return ctypes.byref(self._c)

    def __repr__(self):
        return (f"Config(T={self.T}, d={self.d}, f={self.f}, E={self.E}, top_k={self.top_k}, "
                f"capacity_factor={self.capacity_factor}, dtype={self.dtype!r})")


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _dev_ptr(t):
    if t is not None and not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    return _ptr(t)


def _stream(stream, device=None):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _check(status: int, where: str):
    if status != 0:
        raise MoEError(status, where)


def _expect(name, t, numel, dtype):
    """Host-side check of what the C ABI cannot see: element count and type."""
    if t is None:
        return
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if t.numel() != numel:
        raise ValueError(f"{name} must hold {numel} elements, got {t.numel()}")


def _expect_layer(cfg, x=None, w_router=None, w_gate=None, w_up=None, w_down=None, logit_bias=None, out=None):
    if cfg.T == 0:
        return
    dt = cfg.torch_dtype
    _expect("x", x, cfg.T * cfg.d, dt)
    _expect("w_router", w_router, cfg.E * cfg.d, dt)
    _expect("w_gate", w_gate, cfg.E * cfg.d * cfg.f, dt)
    _expect("w_up", w_up, cfg.E * cfg.d * cfg.f, dt)
    _expect("w_down", w_down, cfg.E * cfg.f * cfg.d, dt)
    _expect("logit_bias", logit_bias, cfg.E, torch.float32)
    _expect("out", out, cfg.T * cfg.d, dt)


def _empty(shape, dtype, like):
    return torch.empty(shape, dtype=dtype, device=like.device)


def abi_version() -> int:
    return lib.moe_abi_version()


def capacity(cfg: Config) -> int:
    return lib.moe_capacity(cfg.ref)


def workspace_size(cfg: Config) -> int:
    return lib.moe_workspace_size(cfg.ref)


def dispatch_workspace_size(cfg: Config) -> int:
    return lib.moe_dispatch_workspace_size(cfg.ref)


def router_topk(cfg: Config, x, w_router, logit_bias=None, logits=None, topk_idx=None, topk_w=None,
                want_logits: bool = False, stream=None):
    """Router logits, top-2 experts and their softmax weights.  Returns (idx, w, logits|None)."""
    _expect_layer(cfg, x=x, w_router=w_router, logit_bias=logit_bias)
    if topk_idx is None:
        topk_idx = _empty((cfg.T, cfg.top_k), torch.int32, x)
    if topk_w is None:
        topk_w = _empty((cfg.T, cfg.top_k), torch.float32, x)
    if logits is None and want_logits:
        logits = _empty((cfg.T, cfg.E), torch.float32, x)
    _check(lib.moe_router_topk(cfg.ref, _dev_ptr(x), _dev_ptr(w_router), _dev_ptr(logit_bias), _dev_ptr(logits),
                               _dev_ptr(topk_idx), _dev_ptr(topk_w), _stream(stream, x.device)), "moe_router_topk")
    return topk_idx, topk_w, logits


def dispatch(cfg: Config, x, topk_idx, topk_w, gather: bool = True, out=None, ws=None, stream=None):
    """Capacity dispatch.  Returns a dict of counts_raw, counts_kept, offsets, perm, slot_of,
    row_scale and x_perm (None when gather is False)."""
    dev = topk_idx
    rows = cfg.T * cfg.top_k
    o = dict(out or {})
    o.setdefault("counts_raw", _empty((cfg.E,), torch.int32, dev))
    o.setdefault("counts_kept", _empty((cfg.E,), torch.int32, dev))
    o.setdefault("offsets", _empty((cfg.E + 1,), torch.int32, dev))
    o.setdefault("perm", _empty((rows,), torch.int32, dev))
    o.setdefault("slot_of", _empty((cfg.T, cfg.top_k), torch.int32, dev))
    o.setdefault("row_scale", _empty((rows,), torch.float32, dev))
    if gather:
        o.setdefault("x_perm", _empty((rows, cfg.d), cfg.torch_dtype, dev))
    else:
        o["x_perm"] = None
    nbytes = dispatch_workspace_size(cfg)
    if ws is None:
        ws = _empty((max(nbytes, 1),), torch.uint8, dev)
    _check(lib.moe_dispatch(cfg.ref, _dev_ptr(x), _dev_ptr(topk_idx), _dev_ptr(topk_w), _dev_ptr(o["counts_raw"]),
                            _dev_ptr(o["counts_kept"]), _dev_ptr(o["offsets"]), _dev_ptr(o["perm"]),
                            _dev_ptr(o["slot_of"]), _dev_ptr(o["row_scale"]), _dev_ptr(o["x_perm"]),
                            _dev_ptr(ws), ws.numel(), _stream(stream, dev.device)), "moe_dispatch")
    return o


def gather_rows(src, idx, out=None, stream=None):
    """out[i] = src[idx[i]] along dim 0 (moe_gather_rows); rows of a multiple of 16 bytes."""
    n = idx.numel()
    row_bytes = src[0].numel() * src.element_size() if src.shape[0] else src.stride(0) * src.element_size()
    if out is None:
        out = torch.empty((n,) + tuple(src.shape[1:]), dtype=src.dtype, device=src.device)
    if idx.dtype != torch.int32:
        raise ValueError("idx must be int32")
    _check(lib.moe_gather_rows(_dev_ptr(src), src.shape[0], _dev_ptr(idx), n, row_bytes, _dev_ptr(out),
                               _stream(stream, src.device)), "moe_gather_rows")
    return out


def route_counts(cfg: Config, topk_idx, counts=None, stream=None):
    """counts[e] = assignments routed to expert e (device int32 [E])."""
    if counts is None:
        counts = _empty((cfg.E,), torch.int32, topk_idx)
    _check(lib.moe_route_counts(cfg.ref, _dev_ptr(topk_idx), _dev_ptr(counts), _stream(stream, topk_idx.device)),
           "moe_route_counts")
    return counts


def dispatch_shard(cfg: Config, capacity: int, shard_counts, shard: int, x, topk_idx, topk_w, gather: bool = True,
                   out=None, ws=None, stream=None):
    """Dispatch of token shard `shard` of a larger batch under the global capacity:
    shard_counts [n_shards, E] holds every shard's route_counts in shard order.
    Returns the same dict as dispatch()."""
    dev = topk_idx
    rows = cfg.T * cfg.top_k
    o = dict(out or {})
    o.setdefault("counts_raw", _empty((cfg.E,), torch.int32, dev))
    o.setdefault("counts_kept", _empty((cfg.E,), torch.int32, dev))
    o.setdefault("offsets", _empty((cfg.E + 1,), torch.int32, dev))
    o.setdefault("perm", _empty((rows,), torch.int32, dev))
    o.setdefault("slot_of", _empty((cfg.T, cfg.top_k), torch.int32, dev))
    o.setdefault("row_scale", _empty((rows,), torch.float32, dev))
    if gather:
        o.setdefault("x_perm", _empty((rows, cfg.d), cfg.torch_dtype, dev))
    else:
        o["x_perm"] = None
    if ws is None:
        ws = _empty((max(dispatch_workspace_size(cfg), 1),), torch.uint8, dev)
    if shard_counts.dtype != torch.int32 or shard_counts.dim() != 2 or shard_counts.shape[1] != cfg.E:
        raise ValueError("shard_counts must be int32 [n_shards, E]")
    _check(lib.moe_dispatch_shard(cfg.ref, int(capacity), _dev_ptr(shard_counts), shard_counts.shape[0], int(shard),
                                  _dev_ptr(x), _dev_ptr(topk_idx), _dev_ptr(topk_w), _dev_ptr(o["counts_raw"]),
                                  _dev_ptr(o["counts_kept"]), _dev_ptr(o["offsets"]), _dev_ptr(o["perm"]),
                                  _dev_ptr(o["slot_of"]), _dev_ptr(o["row_scale"]), _dev_ptr(o["x_perm"]),
                                  _dev_ptr(ws), ws.numel(), _stream(stream, dev.device)), "moe_dispatch_shard")
    return o


def dispatch_noalloc(cfg: Config, x, topk_idx, topk_w, gather: bool = True, out=None, stream=None):
    """moe_dispatch_noalloc: the same outputs as dispatch(), with the library's own fixed
    scratch instead of a caller workspace (for callers that cannot allocate device memory).
    Output tensors are allocated here only when the caller does not pass them in `out`."""
    dev = topk_idx
    rows = cfg.T * cfg.top_k
    o = dict(out or {})
    o.setdefault("counts_raw", _empty((cfg.E,), torch.int32, dev))
    o.setdefault("counts_kept", _empty((cfg.E,), torch.int32, dev))
    o.setdefault("offsets", _empty((cfg.E + 1,), torch.int32, dev))
    o.setdefault("perm", _empty((rows,), torch.int32, dev))
    o.setdefault("slot_of", _empty((cfg.T, cfg.top_k), torch.int32, dev))
    o.setdefault("row_scale", _empty((rows,), torch.float32, dev))
    if gather:
        o.setdefault("x_perm", _empty((rows, cfg.d), cfg.torch_dtype, dev))
    else:
        o["x_perm"] = None
    _check(lib.moe_dispatch_noalloc(cfg.ref, _dev_ptr(x), _dev_ptr(topk_idx), _dev_ptr(topk_w),
                                    _dev_ptr(o["counts_raw"]), _dev_ptr(o["counts_kept"]), _dev_ptr(o["offsets"]),
                                    _dev_ptr(o["perm"]), _dev_ptr(o["slot_of"]), _dev_ptr(o["row_scale"]),
                                    _dev_ptr(o["x_perm"]), _stream(stream, dev.device)), "moe_dispatch_noalloc")
    return o


def expert_gate_up(cfg: Config, x_perm, offsets, w_gate, w_up, h=None, stream=None):
    if h is None:
        h = _empty((cfg.T * cfg.top_k, cfg.f), cfg.torch_dtype, x_perm)
    _check(lib.moe_expert_gate_up(cfg.ref, _dev_ptr(x_perm), _dev_ptr(offsets), _dev_ptr(w_gate), _dev_ptr(w_up),
                                  _dev_ptr(h), _stream(stream, x_perm.device)), "moe_expert_gate_up")
    return h


def expert_down(cfg: Config, h, offsets, w_down, row_scale=None, y=None, ws=None, stream=None):
    if y is None:
        y = _empty((cfg.T * cfg.top_k, cfg.d), torch.float32, h)
    _check(lib.moe_expert_down(cfg.ref, _dev_ptr(h), _dev_ptr(offsets), _dev_ptr(w_down), _dev_ptr(row_scale),
                               _dev_ptr(y), _dev_ptr(ws), 0 if ws is None else ws.numel(),
                               _stream(stream, h.device)), "moe_expert_down")
    return y


def expert_ffn(cfg: Config, x_perm, offsets, w_gate, w_up, w_down, row_scale=None, h=None, y=None, ws=None,
               stream=None):
    """SwiGLU experts over the grouped rows.  Returns (h, y)."""
    if h is None:
        h = _empty((cfg.T * cfg.top_k, cfg.f), cfg.torch_dtype, x_perm)
    if y is None:
        y = _empty((cfg.T * cfg.top_k, cfg.d), torch.float32, x_perm)
    _check(lib.moe_expert_ffn(cfg.ref, _dev_ptr(x_perm), _dev_ptr(offsets), _dev_ptr(w_gate), _dev_ptr(w_up),
                              _dev_ptr(w_down), _dev_ptr(row_scale), _dev_ptr(h), _dev_ptr(y), _dev_ptr(ws),
                              0 if ws is None else ws.numel(), _stream(stream, x_perm.device)), "moe_expert_ffn")
    return h, y


def expert_down_combine(cfg: Config, h, offsets, w_down, row_scale, perm, out=None, ws=None, stream=None):
    """down x routing weight summed straight into token order (down + combine, no y)."""
    if out is None:
        out = _empty((cfg.T, cfg.d), cfg.torch_dtype, h)
    if ws is None:
        ws = _empty((max(lib.moe_expert_down_combine_workspace_size(cfg.ref), 1),), torch.uint8, h)
    _check(lib.moe_expert_down_combine(cfg.ref, _dev_ptr(h), _dev_ptr(offsets), _dev_ptr(w_down), _dev_ptr(row_scale),
                                       _dev_ptr(perm), _dev_ptr(out), _dev_ptr(ws), ws.numel(),
                                       _stream(stream, h.device)), "moe_expert_down_combine")
    return out


class EpPeers:
    """``moe_ep_peers_t``: every rank's exchange buffers as addresses valid in
    this process.  ``addrs[q]`` = (x_grp, src, scale, sums) device addresses of
    rank q (this process's own tensors, or another rank's mapped with
    ``peer_import``); ``world`` ranks, this one ``rank``."""

    def __init__(self, world: int, rank: int, addrs):
        if not 1 <= world <= EP_MAX_WORLD or not 0 <= rank < world or len(addrs) != world:
            raise ValueError(f"world {world}, rank {rank}, {len(addrs)} address sets")
        self.world, self.rank = int(world), int(rank)
        self._c = _CEpPeers()
        self._c.world, self._c.rank = self.world, self.rank
        for q, (xg, src, sc, sums) in enumerate(addrs):
            self._c.x_grp[q], self._c.src[q], self._c.scale[q], self._c.sums[q] = xg, src, sc, sums

    @property
    def ref(self):
        return ctypes.byref(self._c)


def ep_dispatch_peers(cfg: Config, peers: EpPeers, table, x, disp, grp_offsets=None, stream=None):
    """Zero this rank's sums and store its kept rows (x[perm]) into the owners'
    grouped buffers (moe_ep_dispatch_peers).  table [world, E] int32 on the
    device; disp: this rank's dispatch() result.  Returns grp_offsets [E + 1]."""
    if grp_offsets is None:
        grp_offsets = _empty((cfg.E + 1,), torch.int32, table)
    _expect("table", table, peers.world * cfg.E, torch.int32)
    _check(lib.moe_ep_dispatch_peers(cfg.ref, peers.ref, _dev_ptr(table), _dev_ptr(x), _dev_ptr(disp["offsets"]),
                                     _dev_ptr(disp["perm"]), _dev_ptr(disp["row_scale"]), _dev_ptr(grp_offsets),
                                     _stream(stream, table.device)), "moe_ep_dispatch_peers")
    return grp_offsets


def ep_expert_ffn_peers(cfg: Config, peers: EpPeers, grp_offsets, w_gate, w_up, w_down, h, stream=None):
    """This rank's experts over the rows it received; the weighted outputs are
    added into the source ranks' sums (moe_ep_expert_ffn_peers).  h: scratch of
    world * T * top_k rows of f."""
    _expect("h", h, peers.world * cfg.T * cfg.top_k * cfg.f, cfg.torch_dtype)
    _check(lib.moe_ep_expert_ffn_peers(cfg.ref, peers.ref, _dev_ptr(grp_offsets), _dev_ptr(w_gate), _dev_ptr(w_up),
                                       _dev_ptr(w_down), _dev_ptr(h), _stream(stream, h.device)),
           "moe_ep_expert_ffn_peers")


def ep_combine_peers(cfg: Config, peers: EpPeers, out, stream=None):
    """out [T, d] = this rank's sums rounded once (moe_ep_combine_peers)."""
    _expect("out", out, cfg.T * cfg.d, cfg.torch_dtype)
    _check(lib.moe_ep_combine_peers(cfg.ref, peers.ref, _dev_ptr(out), _stream(stream, out.device)),
           "moe_ep_combine_peers")
    return out


def peer_export(t) -> bytes:
    """Handle (72 bytes) that lets another process map the allocation holding t."""
    h = _CPeerHandle()
    _check(lib.moe_peer_export(_dev_ptr(t), ctypes.byref(h)), "moe_peer_export")
    return bytes(h)


def peer_import(handle: bytes) -> int:
    """Maps another process's exported allocation; returns the address matching its tensor."""
    h = _CPeerHandle.from_buffer_copy(handle)
    p = ctypes.c_void_p()
    _check(lib.moe_peer_import(ctypes.byref(h), ctypes.byref(p)), "moe_peer_import")
    return int(p.value)


def peer_release(addr: int, handle: bytes):
    h = _CPeerHandle.from_buffer_copy(handle)
    _check(lib.moe_peer_release(ctypes.c_void_p(addr), ctypes.byref(h)), "moe_peer_release")


def combine(cfg: Config, y, slot_of, topk_w=None, weights_applied: bool = True, out=None, stream=None):
    if out is None:
        out = _empty((cfg.T, cfg.d), cfg.torch_dtype, y)
    _check(lib.moe_combine(cfg.ref, _dev_ptr(y), _dev_ptr(slot_of), _dev_ptr(topk_w), int(bool(weights_applied)),
                           _dev_ptr(out), _stream(stream, y.device)), "moe_combine")
    return out


def layer_forward(cfg: Config, x, w_router, w_gate, w_up, w_down, logit_bias=None, out=None, stats=None,
                  ws=None, stream=None):
    """The whole layer; returns out [T, d] (stats, if given, is filled on the device)."""
    _expect_layer(cfg, x, w_router, w_gate, w_up, w_down, logit_bias, out)
    if out is None:
        out = _empty((cfg.T, cfg.d), cfg.torch_dtype, x)
    if ws is None:
        ws = _empty((max(workspace_size(cfg), 1),), torch.uint8, x)
    _check(lib.moe_layer_forward(cfg.ref, _dev_ptr(x), _dev_ptr(w_router), _dev_ptr(logit_bias), _dev_ptr(w_gate),
                                 _dev_ptr(w_up), _dev_ptr(w_down), _dev_ptr(out), _dev_ptr(stats), _dev_ptr(ws),
                                 ws.numel(), _stream(stream, x.device)), "moe_layer_forward")
    return out


def layer_forward_host(cfg: Config, x_host, w_router, w_gate, w_up, w_down, out_host, ws, logit_bias=None,
                       stream=None):
    """The layer with x and out in (preferably pinned) host memory; returns when out_host is filled."""
    if x_host.is_cuda or out_host.is_cuda:
        raise ValueError("x_host and out_host must be host tensors")
    _expect_layer(cfg, x_host, w_router, w_gate, w_up, w_down, logit_bias, out_host)
    _check(lib.moe_layer_forward_host(cfg.ref, _ptr(x_host), _dev_ptr(w_router), _dev_ptr(logit_bias),
                                      _dev_ptr(w_gate), _dev_ptr(w_up), _dev_ptr(w_down), _ptr(out_host),
                                      _dev_ptr(ws), ws.numel(), _stream(stream, w_router.device)),
           "moe_layer_forward_host")
    return out_host


def workspace_size_host_batches(cfg: Config) -> int:
    return lib.moe_workspace_size_host_batches(cfg.ref)


def layer_forward_host_batches(cfg: Config, x_hosts, w_router, w_gate, w_up, w_down, out_hosts, ws, logit_bias=None,
                               stream=None):
    """The layer over several host-resident batches, copies overlapped with compute
    (``moe_layer_forward_host_batches``); returns when every out_hosts[i] is filled."""
    if len(x_hosts) != len(out_hosts):
        raise ValueError("x_hosts and out_hosts must have the same length")
    if any(t.is_cuda for t in list(x_hosts) + list(out_hosts)):
        raise ValueError("x_hosts and out_hosts must be host tensors")
    for t in list(x_hosts) + list(out_hosts):
        if t.dtype != cfg.torch_dtype or t.numel() != cfg.T * cfg.d:
            raise ValueError(f"host batches must be [T, d] = [{cfg.T}, {cfg.d}] of {cfg.dtype}")
    _expect_layer(cfg, None, w_router, w_gate, w_up, w_down, logit_bias)
    n = len(x_hosts)
    xs = (ctypes.c_void_p * max(n, 1))(*[_ptr(t) for t in x_hosts])
    outs = (ctypes.c_void_p * max(n, 1))(*[_ptr(t) for t in out_hosts])
    _check(lib.moe_layer_forward_host_batches(cfg.ref, n, ctypes.cast(xs, ctypes.c_void_p), _dev_ptr(w_router),
                                              _dev_ptr(logit_bias), _dev_ptr(w_gate), _dev_ptr(w_up),
                                              _dev_ptr(w_down), ctypes.cast(outs, ctypes.c_void_p), _dev_ptr(ws),
                                              ws.numel(), _stream(stream, w_router.device)),
           "moe_layer_forward_host_batches")
    return out_hosts


def workspace_size_train(cfg: Config) -> int:
    return lib.moe_workspace_size_train(cfg.ref)


def layer_forward_train(cfg: Config, x, w_router, w_gate, w_up, w_down, ws, logit_bias=None, out=None, stream=None):
    """The layer forward that keeps the backward's inputs in ws (moe_workspace_size_train bytes)."""
    _expect_layer(cfg, x, w_router, w_gate, w_up, w_down, logit_bias, out)
    if out is None:
        out = _empty((cfg.T, cfg.d), cfg.torch_dtype, x)
    _check(lib.moe_layer_forward_train(cfg.ref, _dev_ptr(x), _dev_ptr(w_router), _dev_ptr(logit_bias),
                                       _dev_ptr(w_gate), _dev_ptr(w_up), _dev_ptr(w_down), _dev_ptr(out),
                                       _dev_ptr(ws), ws.numel(), _stream(stream, x.device)), "moe_layer_forward_train")
    return out


def layer_backward(cfg: Config, x, w_router, w_gate, w_up, w_down, dout, ws, grads=None, want_dbias=True,
                   stream=None):
    """Gradients of sum(out * dout) after layer_forward_train on the same ws.  Returns a dict of
    dx (layer dtype) and fp32 dw_router, dbias (or None), dw_gate, dw_up, dw_down."""
    _expect_layer(cfg, x, w_router, w_gate, w_up, w_down)
    _expect("dout", dout, cfg.T * cfg.d if cfg.T else dout.numel(), cfg.torch_dtype)
    E, d, f = cfg.E, cfg.d, cfg.f
    g = dict(grads or {})
    g.setdefault("dx", _empty((cfg.T, d), cfg.torch_dtype, x))
    g.setdefault("dw_router", _empty((E, d), torch.float32, x))
    if want_dbias:
        g.setdefault("dbias", _empty((E,), torch.float32, x))
    else:
        g["dbias"] = None
    g.setdefault("dw_gate", _empty((E, d, f), torch.float32, x))
    g.setdefault("dw_up", _empty((E, d, f), torch.float32, x))
    g.setdefault("dw_down", _empty((E, f, d), torch.float32, x))
    _check(lib.moe_layer_backward(cfg.ref, _dev_ptr(x), _dev_ptr(w_router), _dev_ptr(w_gate), _dev_ptr(w_up),
                                  _dev_ptr(w_down), _dev_ptr(dout), _dev_ptr(g["dx"]), _dev_ptr(g["dw_router"]),
                                  _dev_ptr(g["dbias"]), _dev_ptr(g["dw_gate"]), _dev_ptr(g["dw_up"]),
                                  _dev_ptr(g["dw_down"]), _dev_ptr(ws), ws.numel(), _stream(stream, x.device)),
           "moe_layer_backward")
    return g


def quantize_int8(cfg: Config, w, q=None, scale=None, stream=None):
    """Per-output-channel int8 codes and fp32 scales of expert weights w [E, K, N] (bf16)."""
    E, K, N = w.shape
    if q is None:
        q = torch.empty((E, K, N), dtype=torch.int8, device=w.device)
    if scale is None:
        scale = torch.empty((E, N), dtype=torch.float32, device=w.device)
    _check(lib.moe_quantize_int8(cfg.ref, _dev_ptr(w), K, N, _dev_ptr(q), _dev_ptr(scale), _stream(stream, w.device)),
           "moe_quantize_int8")
    return q, scale


class QuantizedExperts:
    """int8 expert weights of one layer: codes and per-channel scales of gate, up and down."""

    def __init__(self, cfg: Config, w_gate, w_up, w_down, stream=None):
        self.q_gate, self.s_gate = quantize_int8(cfg, w_gate, stream=stream)
        self.q_up, self.s_up = quantize_int8(cfg, w_up, stream=stream)
        self.q_down, self.s_down = quantize_int8(cfg, w_down, stream=stream)

    def ptrs(self):
        return [_dev_ptr(t) for t in (self.q_gate, self.s_gate, self.q_up, self.s_up, self.q_down, self.s_down)]


def _round256(n):
    return (n + 255) // 256 * 256


def _W8_PARTS(cfg: Config) -> int:
    """Partial buffers the 8-bit down pass may use (up to 8 K splits at decode sizes)."""
    return 1 if cfg.T * cfg.top_k > 64 * cfg.E else 8


def w8_workspace_views(cfg: Config, ws):
    """Named views into the scratch of expert_ffn_w8 (layout stated in include/moe.h)."""
    rows, d, f = cfg.T * cfg.top_k, cfg.d, cfg.f
    spec = [("x_hi", rows * d, torch.int8, (rows, d)), ("x_lo", rows * d, torch.int8, (rows, d)),
            ("x_scale", rows * 4, torch.float32, (rows,)), ("h", rows * f * 4, torch.float32, (rows, f)),
            ("h_hi", rows * f, torch.int8, (rows, f)), ("h_lo", rows * f, torch.int8, (rows, f)),
            ("h_scale", rows * 4, torch.float32, (rows,)),
            ("y_parts", _W8_PARTS(cfg) * rows * d * 4, torch.float32, (_W8_PARTS(cfg), rows, d))]
    views, o = {}, 0
    for name, nbytes, dt, shape in spec:
        views[name] = ws[o:o + nbytes].view(dt).view(shape)
        o += _round256(nbytes)
    return views


def expert_ffn_w8(cfg: Config, x_perm, offsets, qw: QuantizedExperts, row_scale=None, y=None, ws=None,
                  stream=None):
    """SwiGLU experts with int8 weights over the grouped rows.  Returns (y, ws)."""
    if y is None:
        y = _empty((cfg.T * cfg.top_k, cfg.d), torch.float32, x_perm)
    if ws is None:
        ws = _empty((max(lib.moe_expert_ffn_w8_workspace_size(cfg.ref), 1),), torch.uint8, x_perm)
    _check(lib.moe_expert_ffn_w8(cfg.ref, _dev_ptr(x_perm), _dev_ptr(offsets), *qw.ptrs(), _dev_ptr(row_scale),
                                 _dev_ptr(y), _dev_ptr(ws), ws.numel(), _stream(stream, x_perm.device)),
           "moe_expert_ffn_w8")
    return y, ws


def layer_forward_w8(cfg: Config, x, w_router, qw: QuantizedExperts, logit_bias=None, out=None, stats=None, ws=None,
                     stream=None):
    """The whole layer with int8 expert weights; returns out [T, d]."""
    _expect_layer(cfg, x=x, w_router=w_router, logit_bias=logit_bias, out=out)
    if out is None:
        out = _empty((cfg.T, cfg.d), cfg.torch_dtype, x)
    if ws is None:
        ws = _empty((max(lib.moe_workspace_size_w8(cfg.ref), 1),), torch.uint8, x)
    _check(lib.moe_layer_forward_w8(cfg.ref, _dev_ptr(x), _dev_ptr(w_router), _dev_ptr(logit_bias), *qw.ptrs(),
                                    _dev_ptr(out), _dev_ptr(stats), _dev_ptr(ws), ws.numel(),
                                    _stream(stream, x.device)), "moe_layer_forward_w8")
    return out


class ExpertUtilization:
    """Router utilisation over many layer calls ("Training dynamics: expert
    specialization": assignments per expert normalised so that a balanced
    router gives 1.0 for every expert).  Feed it the stats array that
    layer_forward fills (counts_raw in its first E entries); the running
    counts stay on the device until utilization() is read."""

    def __init__(self, E: int = 8, device="cuda"):
        self.E = E
        self.counts = torch.zeros(E, dtype=torch.int64, device=device)
        self.util = torch.zeros(E, dtype=torch.float32, device=device)
        self.calls = 0

    def add(self, stats, stream=None):
        """moe_expert_utilization: counts += stats[:E] and the normalised statistic, on the device."""
        _check(lib.moe_expert_utilization(_dev_ptr(stats), self.E, _dev_ptr(self.counts), _dev_ptr(self.util),
                                          _stream(stream, stats.device)), "moe_expert_utilization")
        self.calls += 1

    def utilization(self):
        """The statistic after the last add() (a copy of the device array)."""
        return self.util.cpu().tolist()


GEMM_TILES = {"auto": 0, "single": 1, "pair": 2}


def set_gemm_tiles(mode: str) -> str:
    """Tile shape of the bf16 grouped GEMMs for later calls (``moe_set_gemm_tiles``):
    "auto", "single" (one CTA per 128-row tile) or "pair" (2-SM CTA pairs per
    256-row tile).  Returns the previous mode."""
    if mode not in GEMM_TILES:
        raise ValueError(f"mode must be one of {sorted(GEMM_TILES)}")
    prev = ctypes.c_int32(0)
    st = lib.moe_set_gemm_tiles(GEMM_TILES[mode], ctypes.byref(prev))
    if st != 0:
        raise MoEError(st, "moe_set_gemm_tiles")
    return {v: k for k, v in GEMM_TILES.items()}[prev.value]


class gemm_tiles:
    """Context manager: ``with gemm_tiles("pair"): ...`` restores the previous mode on exit."""

    def __init__(self, mode: str):
        self.mode = mode
        self.prev = None

    def __enter__(self):
        self.prev = set_gemm_tiles(self.mode)
        return self

    def __exit__(self, *exc):
        set_gemm_tiles(self.prev)
        return False


PHASES = ("fwd_router", "fwd_dispatch", "fwd_gather", "fwd_gate_up", "fwd_down", "fwd_combine",
          "bwd_gather", "bwd_dh", "bwd_zero", "bwd_dx", "bwd_router", "bwd_wg_down", "bwd_wg_gate", "bwd_wg_up")


def profile_phases(enable: bool) -> None:
    """moe_profile_phases: record CUDA events around each kernel of the training pair."""
    _check(lib.moe_profile_phases(int(bool(enable))), "moe_profile_phases")


def profile_read() -> dict:
    """moe_profile_read: {phase: (summed ms, calls)} since the previous read (waits for the events)."""
    n = len(PHASES)
    ms = (ctypes.c_float * n)()
    calls = (ctypes.c_int32 * n)()
    _check(lib.moe_profile_read(ms, calls, n), "moe_profile_read")
    return {PHASES[i]: (float(ms[i]), int(calls[i])) for i in range(n)}


def get_device_error(clear: bool = True) -> int:
    code = ctypes.c_int32(0)
    st = lib.moe_get_device_error(ctypes.byref(code), int(bool(clear)))
    if st not in (0, 5):
        raise MoEError(st, "moe_get_device_error")
    return int(code.value)
