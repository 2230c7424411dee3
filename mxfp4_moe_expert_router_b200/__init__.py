"""Python binding of the MXFP4 MoE expert feed-forward C ABI (``include/moe_mxfp4.h``).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of ``libmoe_mxfp4.so``.  PyTorch supplies device memory and streams.
Importing this package fails loudly when the library has not been built
(``python mxfp4_moe_expert_router_b200/build.py``); there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe_mxfp4.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED_SHAPE, MOE_ERR_OOM, MOE_ERR_CUDA, \
    MOE_ERR_TIMEOUT, MOE_ERR_DEVICE = range(7)

EXPORTS = ("mxfp4_quantize", "moe_mxfp4_create", "moe_route", "moe_forward", "moe_forward_host",
           "moe_status", "moe_set_timeout_ns", "moe_engine_grid", "moe_mxfp4_destroy",
           "moe_status_str", "moe_route_static", "moe_route_static_status", "moe_phase_ns",
           "moe_stream_profile", "moe_set_large_kind", "moe_forward_host_async", "moe_host_join",
           "moe_forward_ops", "spec_verify_workspace_bytes", "spec_verify", "spec_verify_status",
           "spec_exp", "moe_forward_partial", "moe_round_bf16", "moe_ishard_region", "moe_ishard_ipc_handle",
           "moe_ishard_ipc_open", "moe_ishard_ipc_close", "moe_ishard_attach", "moe_forward_ishard")

MOE_OPS_PDL = 1
MOE_ROUTE_STATIC_SCRATCH_BYTES = 8 << 20  # the header's static working memory of moe_route_static
MOE_IPC_HANDLE_BYTES = 64
AR_MAX_RANKS, AR_FLAG_BYTES = 8, 256  # layout of an I-shard region: epoch words, then two fp32 slots


class MoeConfig(ctypes.Structure):
    """Mirror of ``moe_config_t``."""
    _fields_ = [("hidden", ctypes.c_int32), ("inter", ctypes.c_int32),
                ("num_experts", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("max_tokens", ctypes.c_int32), ("num_layers", ctypes.c_int32),
                ("rms_eps", ctypes.c_float)]


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_str(status)} ({status})")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python mxfp4_moe_expert_router_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, u64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64
    pp = ctypes.POINTER(ctypes.c_void_p)
    sig = {
        "mxfp4_quantize": (i32, [vp, i64, i64, vp, vp, vp]),
        "moe_mxfp4_create": (i32, [ctypes.POINTER(MoeConfig), pp, pp, pp, pp, pp, pp, pp, pp, vp,
                                   ctypes.POINTER(vp)]),
        "moe_route": (i32, [vp, i32, vp, i32, vp, vp, vp, vp, vp, vp, vp]),
        "moe_forward": (i32, [vp, vp, i32, vp, vp, vp]),
        "moe_forward_host": (i32, [vp, vp, i32, vp, vp]),
        "moe_forward_ops": (i32, [vp, vp, i32, vp, vp, i32, vp]),
        "moe_forward_partial": (i32, [vp, vp, i32, vp, vp]),
        "moe_round_bf16": (i32, [vp, vp, i64, vp]),
        "moe_ishard_region": (i32, [vp, ctypes.POINTER(vp), ctypes.POINTER(u64)]),
        "moe_ishard_ipc_handle": (i32, [vp, vp]),
        "moe_ishard_ipc_open": (i32, [vp, ctypes.POINTER(vp)]),
        "moe_ishard_ipc_close": (i32, [vp]),
        "moe_ishard_attach": (i32, [vp, i32, i32, pp]),
        "moe_forward_ishard": (i32, [vp, vp, i32, vp, vp]),
        "moe_forward_host_async": (i32, [vp, vp, i32, vp, vp]),
        "moe_host_join": (i32, [vp, vp]),
        "moe_status": (i32, [vp, vp]),
        "moe_set_timeout_ns": (i32, [vp, u64]),
        "moe_set_large_kind": (i32, [vp, i32]),
        "moe_engine_grid": (i32, [vp]),
        "moe_mxfp4_destroy": (None, [vp]),
        "moe_status_str": (ctypes.c_char_p, [i32]),
        "moe_stream_profile": (i32, [vp, i32, ctypes.POINTER(ctypes.c_uint64), i32, vp]),
        "moe_phase_ns": (i32, [vp, ctypes.POINTER(ctypes.c_uint64), i32, vp]),
        "moe_route_static": (i32, [vp, i32, i32, vp, vp, i32, i32, vp, vp, vp, vp, vp, vp, vp]),
        "moe_route_static_status": (i32, [vp]),
        "spec_verify_workspace_bytes": (i64, [i32, i32, i32]),
        "spec_verify": (i32, [vp, vp, vp, vp, vp, i32, i32, i32, vp, vp, vp, i64, vp]),
        "spec_verify_status": (i32, [vp, vp]),
        "spec_exp": (i32, [vp, vp, i64, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


def status_str(status: int) -> str:
    return lib.moe_status_str(int(status)).decode()


def _check(status: int, where: str):
    if status != MOE_OK:
        raise MoeError(status, where)


def _stream(stream=None):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def mxfp4_quantize(w, stream=None):
    """bf16 ``w`` [rows][K] (CUDA) -> (codes uint8 [rows][K/2], scales uint8 [rows][K/32])."""
    import torch
    assert w.dtype == torch.bfloat16 and w.is_cuda and w.dim() == 2 and w.is_contiguous()
    rows, K = w.shape
    codes = torch.empty((rows, K // 2), dtype=torch.uint8, device=w.device)
    scales = torch.empty((rows, K // 32), dtype=torch.uint8, device=w.device)
    _check(lib.mxfp4_quantize(_ptr(w), rows, K, _ptr(codes), _ptr(scales), _stream(stream)),
           "mxfp4_quantize")
    return codes, scales


@dataclass
class LayerMX:
    """One layer's canonical MXFP4 tensors on the device (see ``moe_mxfp4_create``)."""
    gate_codes: object
    gate_scales: object
    up_codes: object
    up_scales: object
    down_codes: object
    down_scales: object
    router_w: object
    router_b: object = None


class Moe:
    """Owner of a ``moe_mxfp4_t`` handle."""

    def __init__(self, hidden, inter, num_experts, top_k, max_tokens, layers, rms_eps=1e-6,
                 stream=None):
        self.cfg = MoeConfig(hidden, inter, num_experts, top_k, max_tokens, len(layers), rms_eps)
        self.handle = ctypes.c_void_p(0)
        n = len(layers)

        def arr(get):
            a = (ctypes.c_void_p * n)()
            for i, lw in enumerate(layers):
                v = get(lw)
                a[i] = v.data_ptr() if v is not None else 0
            return ctypes.cast(a, ctypes.POINTER(ctypes.c_void_p)), a

        keep = [arr(lambda l, f=f: getattr(l, f)) for f in
                ("gate_codes", "gate_scales", "up_codes", "up_scales", "down_codes",
                 "down_scales", "router_w", "router_b")]
        _check(lib.moe_mxfp4_create(ctypes.byref(self.cfg), *[k[0] for k in keep], _stream(stream),
                                    ctypes.byref(self.handle)), "moe_mxfp4_create")

    # -- the C entry points, same names -------------------------------------------------------
    def moe_route(self, x, layer=0, stream=None):
        import torch
        T = x.shape[0]
        K, E = self.cfg.top_k, self.cfg.num_experts
        dev = x.device
        out = dict(topk_idx=torch.empty((T, K), dtype=torch.int32, device=dev),
                   topk_w=torch.empty((T, K), dtype=torch.float32, device=dev),
                   counts=torch.empty((E,), dtype=torch.int32, device=dev),
                   offsets=torch.empty((E + 1,), dtype=torch.int32, device=dev),
                   perm=torch.empty((T * K,), dtype=torch.int32, device=dev),
                   inv_perm=torch.empty((T * K,), dtype=torch.int32, device=dev))
        _check(lib.moe_route(self.handle, layer, _ptr(x), T, *[_ptr(out[k]) for k in
                             ("topk_idx", "topk_w", "counts", "offsets", "perm", "inv_perm")],
                             _stream(stream)), "moe_route")
        return out

    def moe_forward(self, x, y=None, layer_io=None, stream=None):
        import torch
        T = x.shape[0]
        if y is None:
            y = torch.empty((T, self.cfg.hidden), dtype=torch.bfloat16, device=x.device)
        _check(lib.moe_forward(self.handle, _ptr(x), T, _ptr(y), _ptr(layer_io), _stream(stream)),
               "moe_forward")
        return y

    def moe_forward_ops(self, x, y=None, layer_io=None, pdl=True, stream=None):
        """moe_forward as six launches per layer (one per operator); pdl: programmatic
        dependent launches."""
        import torch
        T = x.shape[0]
        if y is None:
            y = torch.empty((T, self.cfg.hidden), dtype=torch.bfloat16, device=x.device)
        _check(lib.moe_forward_ops(self.handle, _ptr(x), T, _ptr(y), _ptr(layer_io),
                                   MOE_OPS_PDL if pdl else 0, _stream(stream)), "moe_forward_ops")
        return y

    def moe_forward_partial(self, x, y_f32=None, stream=None):
        """One layer's fp32 output before the bf16 rounding: a rank's share of an
        I-sharded layer (see ``shard_layer_i``)."""
        import torch
        T = x.shape[0]
        if y_f32 is None:
            y_f32 = torch.empty((T, self.cfg.hidden), dtype=torch.float32, device=x.device)
        _check(lib.moe_forward_partial(self.handle, _ptr(x), T, _ptr(y_f32), _stream(stream)),
               "moe_forward_partial")
        return y_f32

    # -- I-sharded layer with the fused all-reduce ----------------------------------------------
    def moe_ishard_region(self):
        """(device address, bytes) of this handle's all-reduce region (allocated on first use)."""
        base, n = ctypes.c_void_p(0), ctypes.c_uint64(0)
        _check(lib.moe_ishard_region(self.handle, ctypes.byref(base), ctypes.byref(n)), "moe_ishard_region")
        return int(base.value), int(n.value)

    def moe_ishard_ipc_handle(self) -> bytes:
        buf = ctypes.create_string_buffer(MOE_IPC_HANDLE_BYTES)
        _check(lib.moe_ishard_ipc_handle(self.handle, buf), "moe_ishard_ipc_handle")
        return buf.raw

    def moe_ishard_attach(self, rank: int, world: int, regions):
        """Every rank's region (device addresses as this GPU sees them; own at `rank`)."""
        arr = (ctypes.c_void_p * world)(*[int(r) for r in regions])
        _check(lib.moe_ishard_attach(self.handle, rank, world, ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p))),
               "moe_ishard_attach")

    def moe_forward_ishard(self, x, y=None, stream=None):
        import torch
        T = x.shape[0]
        if y is None:
            y = torch.empty((T, self.cfg.hidden), dtype=torch.bfloat16, device=x.device)
        _check(lib.moe_forward_ishard(self.handle, _ptr(x), T, _ptr(y), _stream(stream)), "moe_forward_ishard")
        return y

    def moe_forward_host(self, x_host, y_host=None, stream=None):
        import torch
        T = x_host.shape[0]
        if y_host is None:
            y_host = torch.empty((T, self.cfg.hidden), dtype=torch.bfloat16, pin_memory=True)
        _check(lib.moe_forward_host(self.handle, _ptr(x_host), T, _ptr(y_host), _stream(stream)),
               "moe_forward_host")
        return y_host

    def moe_forward_host_async(self, x_host, y_host, stream=None):
        """Enqueue H2D of x_host, the layers, D2H into y_host (pinned); no synchronisation."""
        _check(lib.moe_forward_host_async(self.handle, _ptr(x_host), x_host.shape[0], _ptr(y_host),
                                          _stream(stream)), "moe_forward_host_async")
        return y_host

    def moe_host_join(self, stream=None):
        """Make `stream` wait for every enqueued output copy of moe_forward_host_async."""
        _check(lib.moe_host_join(self.handle, _stream(stream)), "moe_host_join")

    def moe_status(self, stream=None):
        _check(lib.moe_status(self.handle, _stream(stream)), "moe_status")

    def moe_phase_ns(self, stream=None):
        """Durations (ns) of the last forward's phases as CTA 0 saw them, 7 per layer:
        router logits, x term images, routing wait, top-k or table copy, permutation,
        weight stream, combine."""
        n = self.cfg.num_layers * 7
        arr = (ctypes.c_uint64 * n)()
        _check(lib.moe_phase_ns(self.handle, arr, n, _stream(stream)), "moe_phase_ns")
        return [int(v) for v in arr]

    PROFILE_KEYS = ("prod_wait_empty", "prod_wait_ready", "prod_total", "stages",
                    "mma_wait_full", "mma_issue", "mma_wait_acc", "epi_wait_acc", "epi_work",
                    "epi_total", "jobs")

    def moe_stream_profile(self, enable=True, stream=None):
        """Counters since the previous call (dict), then counting switched on/off."""
        n = len(self.PROFILE_KEYS)
        arr = (ctypes.c_uint64 * n)()
        _check(lib.moe_stream_profile(self.handle, int(bool(enable)), arr, n, _stream(stream)),
               "moe_stream_profile")
        return dict(zip(self.PROFILE_KEYS, (int(v) for v in arr)))

    def moe_set_timeout_ns(self, ns: int):
        _check(lib.moe_set_timeout_ns(self.handle, int(ns)), "moe_set_timeout_ns")

    LARGE_MXF4, LARGE_F16, LARGE_MXF8 = 1, 2, 3

    def moe_set_large_kind(self, kind: int):
        """Weight stream for many positions per expert: LARGE_MXF4 (default), LARGE_F16 or LARGE_MXF8."""
        _check(lib.moe_set_large_kind(self.handle, int(kind)), "moe_set_large_kind")

    @property
    def grid(self) -> int:
        return lib.moe_engine_grid(self.handle)

    def moe_mxfp4_destroy(self):
        if self.handle and self.handle.value:
            lib.moe_mxfp4_destroy(self.handle)
            self.handle = ctypes.c_void_p(0)

    close = moe_mxfp4_destroy

    def __del__(self):
        try:
            self.moe_mxfp4_destroy()
        except Exception:
            pass


def moe_route_static(x, router_w, router_b, top_k, stream=None):
    """Routing without a handle or any device allocation (see ``moe_route_static`` in the header).

    ``x`` bf16 [T][H], ``router_w`` fp32 [E][H], ``router_b`` fp32 [E] or None, all CUDA.
    Returns the same dict as ``Moe.moe_route``.
    """
    import torch
    T, H = x.shape
    E = router_w.shape[0]
    dev = x.device
    out = dict(topk_idx=torch.empty((T, top_k), dtype=torch.int32, device=dev),
               topk_w=torch.empty((T, top_k), dtype=torch.float32, device=dev),
               counts=torch.empty((E,), dtype=torch.int32, device=dev),
               offsets=torch.empty((E + 1,), dtype=torch.int32, device=dev),
               perm=torch.empty((T * top_k,), dtype=torch.int32, device=dev),
               inv_perm=torch.empty((T * top_k,), dtype=torch.int32, device=dev))
    _check(lib.moe_route_static(_ptr(x), T, H, _ptr(router_w), _ptr(router_b), E, top_k,
                                *[_ptr(out[k]) for k in ("topk_idx", "topk_w", "counts", "offsets",
                                                         "perm", "inv_perm")], _stream(stream)),
           "moe_route_static")
    return out


def moe_route_static_status(stream=None) -> int:
    """Synchronise the stream; MOE_OK, or MOE_ERR_TIMEOUT (then cleared) if the last
    ``moe_route_static`` call on the current device ran out of its wait bound."""
    return int(lib.moe_route_static_status(_stream(stream)))


def moe_ishard_ipc_open(handle: bytes) -> int:
    """Map a peer's all-reduce region (its 64-byte IPC handle) on the current device."""
    base = ctypes.c_void_p(0)
    _check(lib.moe_ishard_ipc_open(ctypes.create_string_buffer(bytes(handle), MOE_IPC_HANDLE_BYTES),
                                   ctypes.byref(base)), "moe_ishard_ipc_open")
    return int(base.value)


def moe_ishard_ipc_close(base: int):
    _check(lib.moe_ishard_ipc_close(ctypes.c_void_p(base)), "moe_ishard_ipc_close")


class _DeviceSpan:
    """A raw device address range seen through __cuda_array_interface__ (no copy)."""

    def __init__(self, ptr: int, shape, typestr: str):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr, "data": (int(ptr), False),
                                         "version": 2, "strides": None}


def region_views(base: int, max_tokens: int, hidden: int):
    """Torch views of an I-shard region: (epoch words as int32 [8], partial slots fp32 [2][T][H])."""
    import torch
    flags = torch.as_tensor(_DeviceSpan(base, (AR_MAX_RANKS,), "<i4"), device="cuda")
    parts = torch.as_tensor(_DeviceSpan(base + AR_FLAG_BYTES, (2, max_tokens, hidden), "<f4"), device="cuda")
    return flags, parts


def exchange_ipc_handles(handle: bytes, group=None) -> list:
    """All ranks' IPC handles, in rank order (torch.distributed all-gather of the bytes)."""
    import torch.distributed as dist
    out = [None] * dist.get_world_size(group)
    dist.all_gather_object(out, bytes(handle), group=group)
    return [bytes(h) for h in out]


def connect_ishard(m: "Moe", group=None, opener=None):
    """Attach handle `m` (this rank's I-slice) to every rank's region: export this
    rank's region, gather all handles, map the peers' regions (``opener``: the
    mapping call, moe_ishard_ipc_open by default).  Returns the mapped peer
    addresses (to close with moe_ishard_ipc_close when done)."""
    import torch.distributed as dist
    opener = opener or moe_ishard_ipc_open
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    own, _ = m.moe_ishard_region()
    handles = exchange_ipc_handles(m.moe_ishard_ipc_handle(), group)
    regions, opened = [], []
    for r, h in enumerate(handles):
        if r == rank:
            regions.append(own)
        else:
            b = opener(h)
            opened.append(b)
            regions.append(b)
    m.moe_ishard_attach(rank, world, regions)
    dist.barrier(group)  # every rank's epoch words are cleared before any rank publishes
    return opened


def moe_mxfp4_create(hidden, inter, num_experts, top_k, max_tokens, layers, rms_eps=1e-6,
                     stream=None) -> Moe:
    return Moe(hidden, inter, num_experts, top_k, max_tokens, layers, rms_eps, stream)


class SpecVerify:
    """The speculative-verify acceptance step (``spec_verify`` in include/spec_verify.h)
    for up to ``max_blocks`` verify blocks of ``gamma`` drafts over ``vocab`` tokens.
    Owns the zero-filled device workspace."""

    def __init__(self, max_blocks: int, gamma: int, vocab: int, device="cuda"):
        import torch
        self.max_blocks, self.gamma, self.vocab = max_blocks, gamma, vocab
        nbytes = lib.spec_verify_workspace_bytes(max_blocks, gamma, vocab)
        if nbytes < 0:
            raise MoeError(MOE_ERR_INVALID_ARG, "spec_verify_workspace_bytes")
        self.workspace = torch.zeros(nbytes, dtype=torch.uint8, device=device)

    def __call__(self, target_logits, draft_logits, draft_tokens, r_accept, u_sample, n_out=None,
                 tokens_out=None, stream=None):
        """target_logits fp32 [B][G+1][V], draft_logits fp32 [B][G][V], draft_tokens
        int32 [B][G], r_accept fp64 [B][G], u_sample fp64 [B] (CUDA) ->
        (n_accepted int32 [B], tokens int32 [B][G+1])."""
        import torch
        B = target_logits.shape[0]
        if B > self.max_blocks:
            raise MoeError(MOE_ERR_INVALID_ARG, "spec_verify (more blocks than the workspace holds)")
        dev = target_logits.device
        if n_out is None:
            n_out = torch.empty((B,), dtype=torch.int32, device=dev)
        if tokens_out is None:
            tokens_out = torch.empty((B, self.gamma + 1), dtype=torch.int32, device=dev)
        _check(lib.spec_verify(_ptr(target_logits), _ptr(draft_logits), _ptr(draft_tokens), _ptr(r_accept),
                               _ptr(u_sample), B, self.gamma, self.vocab, _ptr(n_out), _ptr(tokens_out),
                               _ptr(self.workspace), self.workspace.numel(), _stream(stream)), "spec_verify")
        return n_out, tokens_out

    def status(self, stream=None):
        _check(lib.spec_verify_status(_ptr(self.workspace), _stream(stream)), "spec_verify_status")


def spec_exp(x, stream=None):
    """The verify step's fp64 exp on a CUDA fp64 tensor (for accuracy tests)."""
    import torch
    y = torch.empty_like(x)
    _check(lib.spec_exp(_ptr(x), _ptr(y), x.numel(), _stream(stream)), "spec_exp")
    return y


def round_bf16(y_f32, out=None, stream=None):
    """bf16(y_f32), round to nearest even, on the device (``moe_round_bf16``)."""
    import torch
    if out is None:
        out = torch.empty(y_f32.shape, dtype=torch.bfloat16, device=y_f32.device)
    _check(lib.moe_round_bf16(_ptr(y_f32), _ptr(out), y_f32.numel(), _stream(stream)), "moe_round_bf16")
    return out


def shard_layer_i(layer: "LayerMX", rank: int, world: int) -> "LayerMX":
    """Rank `rank` of `world`'s share of an I-sharded layer: rows [r*I/N, (r+1)*I/N)
    of every expert's gate and up matrices, the same columns of its down matrix,
    with their block scales; the router is replicated.  I/N must be a multiple of
    128 (the engine's tiling)."""
    E, I = layer.gate_codes.shape[0], layer.gate_codes.shape[1]
    if world < 1 or not 0 <= rank < world or I % world or (I // world) % 128:
        raise ValueError(f"cannot shard I = {I} over {world} ranks into multiples of 128")
    i0, i1 = rank * I // world, (rank + 1) * I // world
    rows = lambda t: t[:, i0:i1].contiguous()
    return LayerMX(rows(layer.gate_codes), rows(layer.gate_scales), rows(layer.up_codes), rows(layer.up_scales),
                   layer.down_codes[:, :, i0 // 2:i1 // 2].contiguous(),
                   layer.down_scales[:, :, i0 // 32:i1 // 32].contiguous(), layer.router_w, layer.router_b)
