"""Python binding of the B200 W4A8 routed-expert MoE library (``libw4a8.so``).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  PyTorch supplies device memory and the current stream.  The
functions carry the names of the C entry points in ``include/w4a8.h``.
There is no CPU fallback: without the built library, or without a CUDA
device, the calls raise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional, Sequence

import torch

__all__ = ["W4A8Error", "lib", "LIB_PATH", "NUM_STAGES", "STAGE_NAMES", "w4a8_abi_version",
           "w4a8_status_string", "w4a8_pack_int4", "w4a8_quant_act_fp8_per_token",
           "w4a8_moe_route_workspace_size", "w4a8_moe_route_permute",
           "w4a8_moe_route_permute_noalloc", "w4a8_moe_workspace_size",
           "w4a8_moe_forward", "w4a8_check_device_error", "W4A8MoELayer",
           "w4a8_quant_fp8_block", "w4a8_quant_act_fp8_group", "w4a8_shared_expert_forward",
           "w4a8_moe_forward_shared", "SharedExpertFP8", "SHARED_STAGE_NAMES",
           "w4a8_moe_route_topk", "w4a8_moe_experts_workspace_size", "w4a8_moe_forward_experts",
           "w4a8_cast_f32_bf16", "w4a8_ep_dispatch_plan", "w4a8_ep_gather_rows",
           "w4a8_ep_combine_rows", "capture_graph"]

# W4A8_LIBRARY=debug selects the bounds-checking build (see build.py); an
# absolute path to a .so selects that build of the library instead
_lib_choice = os.environ.get("W4A8_LIBRARY", "")
LIB_PATH = (_lib_choice if os.path.isabs(_lib_choice) and _lib_choice.endswith(".so") else
            os.path.join(os.path.dirname(os.path.abspath(__file__)),
                         "libw4a8_debug.so" if _lib_choice == "debug" else "libw4a8.so"))
NUM_STAGES = 6
STAGE_NAMES = ["act_quant", "route_permute", "gemm_gate_up", "inter_quant", "gemm_down",
               "combine"]
SHARED_STAGE_NAMES = ["shared_act_quant", "shared_gemm_gate_up", "shared_inter_quant",
                      "shared_gemm_down"]

_lib = None


class W4A8Error(RuntimeError):
    """A library call returned a non-zero status."""

    def __init__(self, func: str, status: int, message: str):
        self.status = status
        super().__init__(f"{func}: {_status_name(status)}: {message}")


class MoEAux(ctypes.Structure):
    _fields_ = [("topk_ids", ctypes.c_void_p), ("topk_w", ctypes.c_void_p),
                ("expert_offsets", ctypes.c_void_p), ("sorted_token_ids", ctypes.c_void_p),
                ("row_of", ctypes.c_void_p), ("act_codes", ctypes.c_void_p),
                ("act_scales", ctypes.c_void_p), ("inter_h", ctypes.c_void_p),
                ("inter_codes", ctypes.c_void_p), ("inter_scales", ctypes.c_void_p),
                ("y_rows", ctypes.c_void_p), ("stage_events", ctypes.c_void_p)]


class SharedAux(ctypes.Structure):
    _fields_ = [("act_codes", ctypes.c_void_p), ("act_scales", ctypes.c_void_p),
                ("h", ctypes.c_void_p), ("h_codes", ctypes.c_void_p),
                ("h_scales", ctypes.c_void_p), ("stage_events", ctypes.c_void_p)]


def _declare(L):
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    sig = {
        "w4a8_abi_version": (i32, []),
        "w4a8_build_flags": (i32, []),
        "w4a8_status_string": (ctypes.c_char_p, [i32]),
        "w4a8_last_error": (ctypes.c_char_p, []),
        "w4a8_check_device_error": (i32, [vp]),
        "w4a8_selftest_wait_timeout": (i32, [ctypes.c_uint64, vp]),
        "w4a8_pack_int4": (i32, [vp, i64, i64, i32, vp, vp, vp]),
        "w4a8_pack_int4_mse_clip": (i32, [vp, i64, i64, i32, vp, vp, vp]),
        "w4a8_prepare_experts_b200": (i32, [vp, vp, i64, i64, i64, vp, vp, vp]),
        "w4a8_quant_act_fp8_per_token": (i32, [vp, i64, i64, vp, vp, vp]),
        "w4a8_moe_route_workspace_size": (sz, [i64, i32]),
        "w4a8_moe_route_permute": (i32, [vp, i64, i32, i32, vp, vp, vp, vp, vp, vp, sz, vp]),
        "w4a8_moe_route_permute_noalloc": (i32, [vp, i64, i32, i32, vp, vp, vp, vp, vp, vp]),
        "w4a8_moe_workspace_size": (sz, [i64, i64, i64, i32, i32]),
        "w4a8_moe_forward_launches": (i32, [i64, i32, i32]),
        "w4a8_moe_forward": (i32, [vp, vp, vp, vp, vp, vp, i64, i64, i64, i32, i32, vp, vp, sz,
                                   vp, vp]),
        "w4a8_pack_int4_channel": (i32, [vp, i64, i64, vp, vp, vp]),
        "w4a8_prepare_experts_channel_b200": (i32, [vp, i64, i64, i64, vp, vp, vp]),
        "w4a8_moe_forward_channel_int8": (i32, [vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64,
                                                i32, i32, vp, vp, sz, vp, vp]),
        "w4a8_quant_fp8_block": (i32, [vp, i64, i64, vp, vp, vp]),
        "w4a8_quant_act_fp8_group": (i32, [vp, i64, i64, vp, vp, vp]),
        "w4a8_shared_expert_workspace_size": (sz, [i64, i64, i64]),
        "w4a8_shared_expert_forward": (i32, [vp, vp, vp, vp, vp, i64, i64, i64, vp, vp, sz, vp,
                                             vp]),
        "w4a8_moe_shared_workspace_size": (sz, [i64, i64, i64, i32, i32, i64]),
        "w4a8_moe_forward_shared": (i32, [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64,
                                          i64, i32, i32, vp, vp, sz, vp, vp, vp]),
        "w4a8_moe_route_topk": (i32, [vp, i64, i32, i32, vp, vp, vp]),
        "w4a8_moe_experts_workspace_size": (sz, [i64, i64, i64, i32, i32]),
        "w4a8_moe_forward_experts": (i32, [vp, vp, vp, vp, i64, i64, i64, i32, i32, i32, i32,
                                           vp, vp, vp, vp, vp, vp, sz, vp]),
        "w4a8_cast_f32_bf16": (i32, [vp, i64, vp, vp]),
        "w4a8_ep_dispatch_plan": (i32, [vp, i64, i32, i32, i32, vp, vp, i64, vp, vp]),
        "w4a8_ep_gather_rows": (i32, [vp, vp, vp, vp, i64, i64, i32, vp, i64, vp, vp, vp, vp,
                                      vp]),
        "w4a8_ep_combine_rows": (i32, [vp, i64, i64, vp, i64, i32, vp, vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args


def lib():
    """The loaded ``libw4a8.so`` (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                               "`python -m w4a8_quantized_moe_b200.build` (add "
                               "--debug-bounds for the checking build)")
        L = ctypes.CDLL(LIB_PATH)
        _declare(L)
        _lib = L
    return _lib


def _status_name(status: int) -> str:
    try:
        return lib().w4a8_status_string(status).decode()
    except Exception:  # pragma: no cover - only reached while reporting another error
        return f"status {status}"


def _check(func: str, status: int):
    if status != 0:
        raise W4A8Error(func, status, lib().w4a8_last_error().decode())


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, ndim: int):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (the library has no CPU path)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got shape {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def w4a8_abi_version() -> int:
    return int(lib().w4a8_abi_version())


def w4a8_build_flags() -> int:
    """Bit 0: the loaded library is the bounds-checking build."""
    return int(lib().w4a8_build_flags())


def w4a8_status_string(status: int) -> str:
    return lib().w4a8_status_string(status).decode()


def w4a8_check_device_error(device=None):
    """Synchronise the current stream and raise if a bounded in-kernel wait ran out."""
    dev = torch.device("cuda") if device is None else torch.device(device)
    _check("w4a8_check_device_error", lib().w4a8_check_device_error(_stream(dev)))


def w4a8_selftest_wait_timeout(timeout_s: float = 0.05, device=None):
    """Launch a bounded wait that nothing satisfies; the next
    ``w4a8_check_device_error`` then raises W4A8_ERR_DEVICE_TIMEOUT."""
    dev = torch.device("cuda") if device is None else torch.device(device)
    _check("w4a8_selftest_wait_timeout",
           lib().w4a8_selftest_wait_timeout(int(timeout_s * 1e9), _stream(dev)))


def w4a8_pack_int4(w: torch.Tensor, group: int = 128, packed: Optional[torch.Tensor] = None,
                   scales: Optional[torch.Tensor] = None, mse_clip: bool = False):
    """INT4 group-128 quantisation + uint4b8 packing of bf16 ``w`` [..., K].

    ``mse_clip=False``: round-to-nearest with scale absmax / 7
    (``w4a8_pack_int4``); ``True``: the per-group MSE clip search over 11
    shrink ratios (``w4a8_pack_int4_mse_clip``).  Returns
    ``(packed int32 [..., K/8], scales bf16 [..., K/128])``.
    """
    if w.dim() < 2:
        raise ValueError("w must have at least 2 dims")
    lead, K = tuple(w.shape[:-1]), w.shape[-1]
    w2 = w.reshape(-1, K)
    _need(w2, "w", torch.bfloat16, 2)
    R = w2.shape[0]
    if packed is None:
        packed = torch.empty(*lead, K // 8, dtype=torch.int32, device=w.device)
    if scales is None:
        scales = torch.empty(*lead, max(K // group, 0), dtype=torch.bfloat16, device=w.device)
    name = "w4a8_pack_int4_mse_clip" if mse_clip else "w4a8_pack_int4"
    _check(name, getattr(lib(), name)(_p(w2), R, K, group, _p(packed), _p(scales),
                                      _stream(w.device)))
    return packed, scales


def w4a8_prepare_experts_b200(packed: torch.Tensor, scales: torch.Tensor,
                              packed_out: Optional[torch.Tensor] = None,
                              scales_out: Optional[torch.Tensor] = None):
    """Lay out ``w4a8_pack_int4`` output the way ``w4a8_moe_forward`` reads it.

    ``packed`` int32 [E, rows, K/8] and ``scales`` bf16 [E, rows, K/128] ->
    ``(packed_out [E, rows, K/8], scales_out [E, K/128, rows])``: nibbles
    interleaved inside each word, scales group-major.  ``packed_out`` may be
    ``packed`` itself (in place).
    """
    _need(packed, "packed", torch.int32, 3)
    _need(scales, "scales", torch.bfloat16, 3)
    E, rows, k8 = packed.shape
    K = k8 * 8
    if scales.shape != (E, rows, K // 128):
        raise ValueError("scales must be [E, rows, K/128] for packed [E, rows, K/8]")
    if packed_out is None:
        packed_out = torch.empty_like(packed)
    if scales_out is None:
        scales_out = torch.empty(E, K // 128, rows, dtype=torch.bfloat16, device=packed.device)
    _need(packed_out, "packed_out", torch.int32, 3)
    _need(scales_out, "scales_out", torch.bfloat16, 3)
    if packed_out.shape != packed.shape or scales_out.shape != (E, K // 128, rows):
        raise ValueError("packed_out must match packed; scales_out must be [E, K/128, rows]")
    _check("w4a8_prepare_experts_b200",
           lib().w4a8_prepare_experts_b200(_p(packed), _p(scales), E, rows, K, _p(packed_out),
                                           _p(scales_out), _stream(packed.device)))
    return packed_out, scales_out


def w4a8_quant_act_fp8_per_token(x: torch.Tensor, codes: Optional[torch.Tensor] = None,
                                 scales: Optional[torch.Tensor] = None):
    """Per-token dynamic E4M3 quantisation of bf16 ``x`` [T, H] -> (uint8 codes, f32 scales)."""
    _need(x, "x", torch.bfloat16, 2)
    T, H = x.shape
    if codes is None:
        codes = torch.empty(T, H, dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(T, dtype=torch.float32, device=x.device)
    _check("w4a8_quant_act_fp8_per_token",
           lib().w4a8_quant_act_fp8_per_token(_p(x), T, H, _p(codes), _p(scales),
                                              _stream(x.device)))
    return codes, scales


def w4a8_moe_route_workspace_size(T: int, E: int) -> int:
    return int(lib().w4a8_moe_route_workspace_size(T, E))


def w4a8_moe_route_permute(logits: torch.Tensor, k: int,
                           workspace: Optional[torch.Tensor] = None) -> Dict[str, torch.Tensor]:
    """Top-k routing + stable permutation by expert (see include/w4a8.h)."""
    _need(logits, "logits", torch.float32, 2)
    T, E = logits.shape
    dev = logits.device
    out = dict(topk_ids=torch.empty(T, k, dtype=torch.int32, device=dev),
               topk_w=torch.empty(T, k, dtype=torch.float32, device=dev),
               expert_offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
               sorted_token_ids=torch.empty(T * k, dtype=torch.int32, device=dev),
               row_of=torch.empty(T, k, dtype=torch.int32, device=dev))
    need = w4a8_moe_route_workspace_size(T, E)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    _check("w4a8_moe_route_permute",
           lib().w4a8_moe_route_permute(_p(logits), T, E, k, _p(out["topk_ids"]),
                                        _p(out["topk_w"]), _p(out["expert_offsets"]),
                                        _p(out["sorted_token_ids"]), _p(out["row_of"]),
                                        _p(workspace), workspace.numel(), _stream(dev)))
    return out


def w4a8_moe_route_permute_noalloc(logits: torch.Tensor, k: int,
                                   out: Optional[Dict[str, torch.Tensor]] = None
                                   ) -> Dict[str, torch.Tensor]:
    """Routing + permutation without a workspace, for callers that cannot
    allocate device memory at call time (see include/w4a8.h).  The library
    allocates nothing; pass ``out`` (the five output tensors) to allocate
    nothing here either."""
    _need(logits, "logits", torch.float32, 2)
    T, E = logits.shape
    dev = logits.device
    if out is None:
        out = dict(topk_ids=torch.empty(T, k, dtype=torch.int32, device=dev),
                   topk_w=torch.empty(T, k, dtype=torch.float32, device=dev),
                   expert_offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
                   sorted_token_ids=torch.empty(T * k, dtype=torch.int32, device=dev),
                   row_of=torch.empty(T, k, dtype=torch.int32, device=dev))
    _check("w4a8_moe_route_permute_noalloc",
           lib().w4a8_moe_route_permute_noalloc(_p(logits), T, E, k, _p(out["topk_ids"]),
                                                _p(out["topk_w"]), _p(out["expert_offsets"]),
                                                _p(out["sorted_token_ids"]), _p(out["row_of"]),
                                                _stream(dev)))
    return out


def w4a8_moe_workspace_size(T: int, H: int, I: int, E: int, k: int) -> int:
    return int(lib().w4a8_moe_workspace_size(T, H, I, E, k))


def w4a8_moe_forward_launches(T: int, E: int, k: int) -> int:
    """Kernels one forward launches for these sizes (see include/w4a8.h)."""
    return int(lib().w4a8_moe_forward_launches(T, E, k))


_AUX_FIELDS = ["topk_ids", "topk_w", "expert_offsets", "sorted_token_ids", "row_of", "act_codes",
               "act_scales", "inter_h", "inter_codes", "inter_scales", "y_rows"]


def _aux_struct(aux, stage_events):
    """The w4a8_moe_aux of a dict of caller buffers and optional stage events
    (None when neither is given), plus the objects that must outlive the call."""
    if not aux and not stage_events:
        return None, []
    st, keep = MoEAux(), []
    for name, t in (aux or {}).items():
        if name not in _AUX_FIELDS:
            raise KeyError(f"unknown aux buffer {name!r}")
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"aux[{name!r}] must be a contiguous CUDA tensor")
        setattr(st, name, t.data_ptr())
    if stage_events:
        if len(stage_events) != 2 * NUM_STAGES:
            raise ValueError(f"need {2 * NUM_STAGES} events")
        arr = (ctypes.c_void_p * (2 * NUM_STAGES))(*[e.cuda_event for e in stage_events])
        keep.append(arr)
        st.stage_events = ctypes.cast(arr, ctypes.c_void_p)
    return st, keep


def w4a8_moe_forward(hidden: torch.Tensor, logits: torch.Tensor, w13_packed: torch.Tensor,
                     w13_scales: torch.Tensor, w2_packed: torch.Tensor, w2_scales: torch.Tensor,
                     k: int, out: Optional[torch.Tensor] = None,
                     workspace: Optional[torch.Tensor] = None,
                     aux: Optional[Dict[str, torch.Tensor]] = None,
                     stage_events: Optional[Sequence[torch.cuda.Event]] = None) -> torch.Tensor:
    """One W4A8 MoE layer: returns bf16 [T, H].

    ``aux`` maps names of ``w4a8_moe_aux`` members to caller tensors that then
    receive the intermediates; ``stage_events`` (2 * NUM_STAGES timing-enabled
    CUDA events) are recorded around the stages.
    """
    _need(hidden, "hidden", torch.bfloat16, 2)
    _need(logits, "logits", torch.float32, 2)
    _need(w13_packed, "w13_packed", torch.int32, 3)
    _need(w13_scales, "w13_scales", torch.bfloat16, 3)
    _need(w2_packed, "w2_packed", torch.int32, 3)
    _need(w2_scales, "w2_scales", torch.bfloat16, 3)
    T, H = hidden.shape
    E = logits.shape[1]
    I = w2_packed.shape[2] * 8
    if w13_scales.shape == (E, 2 * I, H // 128) and w13_scales.shape != (E, H // 128, 2 * I):
        raise ValueError("w13_scales is in the pack-quantized layout [E, 2I, H/128]; "
                         "w4a8_moe_forward reads experts laid out by "
                         "w4a8_prepare_experts_b200 (or W4A8MoELayer.from_packed)")
    if logits.shape[0] != T or w13_packed.shape != (E, 2 * I, H // 8) or \
            w2_packed.shape != (E, H, I // 8) or w13_scales.shape != (E, H // 128, 2 * I) or \
            w2_scales.shape != (E, I // 128, H):
        raise ValueError("inconsistent shapes: hidden [T,H], logits [T,E], w13 [E,2I,H/8], "
                         "w2 [E,H,I/8], w13_scales [E,H/128,2I], w2_scales [E,I/128,H]")
    dev = hidden.device
    if out is None:
        out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    need = w4a8_moe_workspace_size(T, H, I, E, k)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    aux_struct, keep = _aux_struct(aux, stage_events)
    _check("w4a8_moe_forward",
           lib().w4a8_moe_forward(_p(hidden), _p(logits), _p(w13_packed), _p(w13_scales),
                                  _p(w2_packed), _p(w2_scales), T, H, I, E, k, _p(out),
                                  _p(workspace), workspace.numel(),
                                  None if aux_struct is None else ctypes.byref(aux_struct),
                                  _stream(dev)))
    return out


def capture_graph(fn, warmup: int = 2) -> "torch.cuda.CUDAGraph":
    """Capture ``fn()`` -- calls of this library on fixed tensors, e.g. one
    layer forward with its inputs, output and workspace already allocated -- as
    a CUDA graph; ``graph.replay()`` then reruns those kernels on whatever the
    buffers hold, without the per-call host work (argument checks, tensor-map
    encoding, launches).  ``fn`` runs ``warmup`` times first on a side stream
    (one-time set-up such as kernel attributes happens there, not during
    capture).  The calls must not allocate: pass ``out`` and a workspace."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(warmup):
            fn()
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


class W4A8MoELayer:
    """A layer with packed experts resident on the device and a reusable workspace.

    ``W4A8MoELayer.from_bf16(w13, w2, k)`` packs bf16 ``w13`` [E, 2I, H] and
    ``w2`` [E, H, I] with ``w4a8_pack_int4`` and lays them out with
    ``w4a8_prepare_experts_b200``; the ``w13_*`` / ``w2_*`` attributes hold
    that layout.  Calling the layer runs ``w4a8_moe_forward``.
    """

    def __init__(self, w13_packed, w13_scales, w2_packed, w2_scales, k: int):
        self.w13_packed, self.w13_scales = w13_packed, w13_scales
        self.w2_packed, self.w2_scales = w2_packed, w2_scales
        self.k = k
        self.E, twoI, h8 = w13_packed.shape
        self.H, self.I = h8 * 8, twoI // 2
        self._ws = None

    @classmethod
    def from_bf16(cls, w13: torch.Tensor, w2: torch.Tensor, k: int,
                  mse_clip: bool = False) -> "W4A8MoELayer":
        p13, s13 = w4a8_pack_int4(w13, mse_clip=mse_clip)
        p2, s2 = w4a8_pack_int4(w2, mse_clip=mse_clip)
        return cls.from_packed(p13, s13, p2, s2, k, in_place=True)

    @classmethod
    def from_packed(cls, w13_packed: torch.Tensor, w13_scales: torch.Tensor,
                    w2_packed: torch.Tensor, w2_scales: torch.Tensor, k: int,
                    in_place: bool = False) -> "W4A8MoELayer":
        """A layer from experts in the pages' compressed-tensors format, as
        ``w4a8_pack_int4`` writes it (uint4b8 words [E, rows, K/8], little-endian
        nibbles; bf16 scales [E, rows, K/128]): ``w4a8_prepare_experts_b200``
        lays them out for ``w4a8_moe_forward`` (in place if ``in_place``)."""
        p13, s13 = w4a8_prepare_experts_b200(w13_packed, w13_scales,
                                             packed_out=w13_packed if in_place else None)
        p2, s2 = w4a8_prepare_experts_b200(w2_packed, w2_scales,
                                           packed_out=w2_packed if in_place else None)
        return cls(p13, s13, p2, s2, k)

    def workspace(self, T: int) -> torch.Tensor:
        need = max(w4a8_moe_workspace_size(T, self.H, self.I, self.E, self.k), 1)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=self.w13_packed.device)
        return self._ws

    def __call__(self, hidden: torch.Tensor, logits: torch.Tensor,
                 out: Optional[torch.Tensor] = None, **kw) -> torch.Tensor:
        return w4a8_moe_forward(hidden, logits, self.w13_packed, self.w13_scales, self.w2_packed,
                                self.w2_scales, self.k, out=out,
                                workspace=self.workspace(hidden.shape[0]), **kw)


# ---------------------------------------------------------------- per-channel INT4 x INT8

def w4a8_pack_int4_channel(w: torch.Tensor, packed: Optional[torch.Tensor] = None,
                           scales: Optional[torch.Tensor] = None):
    """Per-channel INT4 RTN of bf16 ``w`` [..., K] -> (packed int32 [..., K/8], scales bf16 [...])."""
    if w.dim() < 2:
        raise ValueError("w must have at least 2 dims")
    lead, K = tuple(w.shape[:-1]), w.shape[-1]
    w2 = w.reshape(-1, K)
    _need(w2, "w", torch.bfloat16, 2)
    if packed is None:
        packed = torch.empty(*lead, K // 8, dtype=torch.int32, device=w.device)
    if scales is None:
        scales = torch.empty(*lead, dtype=torch.bfloat16, device=w.device)
    _check("w4a8_pack_int4_channel",
           lib().w4a8_pack_int4_channel(_p(w2), w2.shape[0], K, _p(packed), _p(scales),
                                        _stream(w.device)))
    return packed, scales


def w4a8_prepare_experts_channel_b200(packed: torch.Tensor, packed_out: Optional[torch.Tensor] = None):
    """``packed`` int32 [E, rows, K/8] -> (packed_out in the GEMM's word layout,
    nibble_sums int32 [E, rows]).  ``packed_out`` may be ``packed`` (in place)."""
    _need(packed, "packed", torch.int32, 3)
    E, rows, k8 = packed.shape
    if packed_out is None:
        packed_out = torch.empty_like(packed)
    sums = torch.empty(E, rows, dtype=torch.int32, device=packed.device)
    _check("w4a8_prepare_experts_channel_b200",
           lib().w4a8_prepare_experts_channel_b200(_p(packed), E, rows, k8 * 8, _p(packed_out),
                                                   _p(sums), _stream(packed.device)))
    return packed_out, sums


def w4a8_moe_forward_channel_int8(hidden, logits, w13_packed, w13_scales, w13_sums, w2_packed,
                                  w2_scales, w2_sums, k: int, out=None, workspace=None,
                                  aux: Optional[Dict[str, torch.Tensor]] = None,
                                  stage_events: Optional[Sequence[torch.cuda.Event]] = None
                                  ) -> torch.Tensor:
    """The per-channel INT4 x per-token INT8 layer; bf16 [T, H].  aux codes are offset-binary."""
    _need(hidden, "hidden", torch.bfloat16, 2)
    _need(logits, "logits", torch.float32, 2)
    _need(w13_packed, "w13_packed", torch.int32, 3)
    _need(w2_packed, "w2_packed", torch.int32, 3)
    _need(w13_scales, "w13_scales", torch.bfloat16, 2)
    _need(w2_scales, "w2_scales", torch.bfloat16, 2)
    _need(w13_sums, "w13_sums", torch.int32, 2)
    _need(w2_sums, "w2_sums", torch.int32, 2)
    T, H = hidden.shape
    E = logits.shape[1]
    I = w2_packed.shape[2] * 8
    if logits.shape[0] != T or w13_packed.shape != (E, 2 * I, H // 8) or \
            w2_packed.shape != (E, H, I // 8) or w13_scales.shape != (E, 2 * I) or \
            w2_scales.shape != (E, H) or w13_sums.shape != (E, 2 * I) or w2_sums.shape != (E, H):
        raise ValueError("inconsistent shapes")
    dev = hidden.device
    if out is None:
        out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    need = w4a8_moe_workspace_size(T, H, I, E, k)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    aux_struct, keep = _aux_struct(aux, stage_events)
    _check("w4a8_moe_forward_channel_int8",
           lib().w4a8_moe_forward_channel_int8(
               _p(hidden), _p(logits), _p(w13_packed), _p(w13_scales), _p(w13_sums),
               _p(w2_packed), _p(w2_scales), _p(w2_sums), T, H, I, E, k, _p(out), _p(workspace),
               workspace.numel(), None if aux_struct is None else ctypes.byref(aux_struct),
               _stream(dev)))
    return out


class W4A8ChannelInt8Layer:
    """Per-channel INT4 experts with per-token INT8 activations (resident, prepared)."""

    def __init__(self, w13_packed, w13_scales, w13_sums, w2_packed, w2_scales, w2_sums, k: int):
        self.w13 = (w13_packed, w13_scales, w13_sums)
        self.w2 = (w2_packed, w2_scales, w2_sums)
        self.k = k
        self.E, twoI, h8 = w13_packed.shape
        self.H, self.I = h8 * 8, twoI // 2
        self._ws = None

    @classmethod
    def from_bf16(cls, w13: torch.Tensor, w2: torch.Tensor, k: int) -> "W4A8ChannelInt8Layer":
        p13, s13 = w4a8_pack_int4_channel(w13)
        p2, s2 = w4a8_pack_int4_channel(w2)
        p13, n13 = w4a8_prepare_experts_channel_b200(p13, packed_out=p13)
        p2, n2 = w4a8_prepare_experts_channel_b200(p2, packed_out=p2)
        return cls(p13, s13, n13, p2, s2, n2, k)

    def workspace(self, T: int) -> torch.Tensor:
        need = max(w4a8_moe_workspace_size(T, self.H, self.I, self.E, self.k), 1)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=self.w13[0].device)
        return self._ws

    def __call__(self, hidden, logits, out=None, aux=None, stage_events=None) -> torch.Tensor:
        return w4a8_moe_forward_channel_int8(hidden, logits, *self.w13, *self.w2, self.k, out=out,
                                             workspace=self.workspace(hidden.shape[0]), aux=aux,
                                             stage_events=stage_events)


# ---------------------------------------------------------------- FP8-block shared expert

def w4a8_quant_fp8_block(w: torch.Tensor):
    """bf16 ``w`` [R, K] -> (E4M3 codes uint8 [R, K], float32 scales [R/128, K/128])."""
    _need(w, "w", torch.bfloat16, 2)
    R, K = w.shape
    codes = torch.empty(R, K, dtype=torch.uint8, device=w.device)
    scales = torch.empty(R // 128, K // 128, dtype=torch.float32, device=w.device)
    _check("w4a8_quant_fp8_block",
           lib().w4a8_quant_fp8_block(_p(w), R, K, _p(codes), _p(scales), _stream(w.device)))
    return codes, scales


def w4a8_quant_act_fp8_group(x: torch.Tensor):
    """bf16 ``x`` [T, H] -> (E4M3 codes uint8 [T, H], float32 scales [T, H/128])."""
    _need(x, "x", torch.bfloat16, 2)
    T, H = x.shape
    codes = torch.empty(T, H, dtype=torch.uint8, device=x.device)
    scales = torch.empty(T, H // 128, dtype=torch.float32, device=x.device)
    _check("w4a8_quant_act_fp8_group",
           lib().w4a8_quant_act_fp8_group(_p(x), T, H, _p(codes), _p(scales), _stream(x.device)))
    return codes, scales


_SHARED_AUX_FIELDS = ["act_codes", "act_scales", "h", "h_codes", "h_scales"]


def _shared_aux_struct(aux, stage_events):
    if not aux and not stage_events:
        return None, []
    st, keep = SharedAux(), []
    for name, t in (aux or {}).items():
        if name not in _SHARED_AUX_FIELDS:
            raise KeyError(f"unknown shared aux buffer {name!r}")
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"shared aux[{name!r}] must be a contiguous CUDA tensor")
        setattr(st, name, t.data_ptr())
    if stage_events:
        if len(stage_events) != 8:
            raise ValueError("need 8 events")
        arr = (ctypes.c_void_p * 8)(*[e.cuda_event for e in stage_events])
        keep.append(arr)
        st.stage_events = ctypes.cast(arr, ctypes.c_void_p)
    return st, keep


def _check_shared_weights(w13_codes, w13_scales, w2_codes, w2_scales, H):
    _need(w13_codes, "w13_codes", torch.uint8, 2)
    _need(w13_scales, "w13_scales", torch.float32, 2)
    _need(w2_codes, "w2_codes", torch.uint8, 2)
    _need(w2_scales, "w2_scales", torch.float32, 2)
    I = w2_codes.shape[1]
    if w13_codes.shape != (2 * I, H) or w2_codes.shape != (H, I) or \
            w13_scales.shape != (2 * I // 128, H // 128) or w2_scales.shape != (H // 128, I // 128):
        raise ValueError("shared expert: w13 [2I, H], w2 [H, I], scales [2I/128, H/128] and "
                         "[H/128, I/128]")
    return I


def w4a8_shared_expert_forward(hidden, w13_codes, w13_scales, w2_codes, w2_scales, y=None,
                               workspace=None, aux=None, stage_events=None) -> torch.Tensor:
    """The FP8-block shared expert alone: float32 [T, H] (see include/w4a8.h)."""
    _need(hidden, "hidden", torch.bfloat16, 2)
    T, H = hidden.shape
    I = _check_shared_weights(w13_codes, w13_scales, w2_codes, w2_scales, H)
    dev = hidden.device
    if y is None:
        y = torch.empty(T, H, dtype=torch.float32, device=dev)
    need = int(lib().w4a8_shared_expert_workspace_size(T, H, I))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    st, keep = _shared_aux_struct(aux, stage_events)
    _check("w4a8_shared_expert_forward",
           lib().w4a8_shared_expert_forward(
               _p(hidden), _p(w13_codes), _p(w13_scales), _p(w2_codes), _p(w2_scales), T, H, I,
               _p(y), _p(workspace), workspace.numel(), None if st is None else ctypes.byref(st),
               _stream(dev)))
    return y


def w4a8_moe_forward_shared(hidden, logits, w13_packed, w13_scales, w2_packed, w2_scales,
                            shared, k: int, out=None, workspace=None, aux=None, stage_events=None,
                            shared_aux=None, shared_stage_events=None) -> torch.Tensor:
    """The W4A8 layer plus the FP8-block shared expert ``shared`` = (w13_codes,
    w13_scales, w2_codes, w2_scales): bf16 [T, H]."""
    _need(hidden, "hidden", torch.bfloat16, 2)
    _need(logits, "logits", torch.float32, 2)
    T, H = hidden.shape
    E = logits.shape[1]
    I = w2_packed.shape[2] * 8
    Is = _check_shared_weights(*shared, H)
    if logits.shape[0] != T or w13_packed.shape != (E, 2 * I, H // 8) or \
            w2_packed.shape != (E, H, I // 8) or w13_scales.shape != (E, H // 128, 2 * I) or \
            w2_scales.shape != (E, I // 128, H):
        raise ValueError("inconsistent routed-expert shapes")
    dev = hidden.device
    if out is None:
        out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    need = int(lib().w4a8_moe_shared_workspace_size(T, H, I, E, k, Is))
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    ast, keep = _aux_struct(aux, stage_events)
    sst, keep2 = _shared_aux_struct(shared_aux, shared_stage_events)
    _check("w4a8_moe_forward_shared",
           lib().w4a8_moe_forward_shared(
               _p(hidden), _p(logits), _p(w13_packed), _p(w13_scales), _p(w2_packed),
               _p(w2_scales), *[_p(t) for t in shared], T, H, I, Is, E, k, _p(out),
               _p(workspace), workspace.numel(), None if ast is None else ctypes.byref(ast),
               None if sst is None else ctypes.byref(sst), _stream(dev)))
    return out


class SharedExpertFP8:
    """The shared expert's E4M3 weights and 128 x 128 block scales, resident."""

    def __init__(self, w13_codes, w13_scales, w2_codes, w2_scales):
        self.weights = (w13_codes, w13_scales, w2_codes, w2_scales)
        self.H, self.I = w2_codes.shape

    @classmethod
    def from_bf16(cls, w13: torch.Tensor, w2: torch.Tensor) -> "SharedExpertFP8":
        return cls(*w4a8_quant_fp8_block(w13), *w4a8_quant_fp8_block(w2))

    def __call__(self, hidden, **kw) -> torch.Tensor:
        return w4a8_shared_expert_forward(hidden, *self.weights, **kw)


class W4A8MoELayerShared(W4A8MoELayer):
    """``W4A8MoELayer`` plus an FP8-block shared expert, in one forward call."""

    def __init__(self, w13_packed, w13_scales, w2_packed, w2_scales, k: int,
                 shared: SharedExpertFP8):
        super().__init__(w13_packed, w13_scales, w2_packed, w2_scales, k)
        self.shared = shared

    @classmethod
    def from_bf16_with_shared(cls, w13, w2, k: int, ws13, ws2,
                              mse_clip: bool = False) -> "W4A8MoELayerShared":
        base = W4A8MoELayer.from_bf16(w13, w2, k, mse_clip=mse_clip)
        return cls(base.w13_packed, base.w13_scales, base.w2_packed, base.w2_scales, k,
                   SharedExpertFP8.from_bf16(ws13, ws2))

    def workspace(self, T: int) -> torch.Tensor:
        need = max(int(lib().w4a8_moe_shared_workspace_size(T, self.H, self.I, self.E, self.k,
                                                             self.shared.I)), 1)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=self.w13_packed.device)
        return self._ws

    def __call__(self, hidden, logits, out=None, **kw) -> torch.Tensor:
        return w4a8_moe_forward_shared(hidden, logits, self.w13_packed, self.w13_scales,
                                       self.w2_packed, self.w2_scales, self.shared.weights,
                                       self.k, out=out, workspace=self.workspace(hidden.shape[0]),
                                       **kw)


# ---------------------------------------------------------------- expert parallelism

def w4a8_moe_route_topk(logits: torch.Tensor, k: int, topk_ids: Optional[torch.Tensor] = None,
                        topk_w: Optional[torch.Tensor] = None):
    """Top-k ids and softmax-renormalised weights only: (int32 [T, k], float32 [T, k])."""
    _need(logits, "logits", torch.float32, 2)
    T, E = logits.shape
    dev = logits.device
    if topk_ids is None:
        topk_ids = torch.empty(T, k, dtype=torch.int32, device=dev)
    if topk_w is None:
        topk_w = torch.empty(T, k, dtype=torch.float32, device=dev)
    _need(topk_ids, "topk_ids", torch.int32, 2)
    _need(topk_w, "topk_w", torch.float32, 2)
    if topk_ids.shape != (T, k) or topk_w.shape != (T, k):
        raise ValueError("topk_ids / topk_w must be [T, k]")
    _check("w4a8_moe_route_topk",
           lib().w4a8_moe_route_topk(_p(logits), T, E, k, _p(topk_ids), _p(topk_w),
                                     _stream(dev)))
    return topk_ids, topk_w


def w4a8_moe_experts_workspace_size(T: int, H: int, I: int, e_count: int, k: int) -> int:
    return int(lib().w4a8_moe_experts_workspace_size(T, H, I, e_count, k))


def w4a8_moe_forward_experts(act_codes: torch.Tensor, act_scales: torch.Tensor,
                             topk_ids: torch.Tensor, topk_w: torch.Tensor, E: int, e_begin: int,
                             w13_packed: torch.Tensor, w13_scales: torch.Tensor,
                             w2_packed: torch.Tensor, w2_scales: torch.Tensor,
                             out: Optional[torch.Tensor] = None,
                             workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The local experts' share of the layer (expert parallelism): float32
    partial sums [T, H] over the slots routed to experts e_begin ..
    e_begin + e_count - 1, whose prepared weights ``w13_*`` / ``w2_*`` hold
    those experts only (see include/w4a8.h)."""
    _need(act_codes, "act_codes", torch.uint8, 2)
    _need(act_scales, "act_scales", torch.float32, 1)
    _need(topk_ids, "topk_ids", torch.int32, 2)
    _need(topk_w, "topk_w", torch.float32, 2)
    _need(w13_packed, "w13_packed", torch.int32, 3)
    _need(w13_scales, "w13_scales", torch.bfloat16, 3)
    _need(w2_packed, "w2_packed", torch.int32, 3)
    _need(w2_scales, "w2_scales", torch.bfloat16, 3)
    T, H = act_codes.shape
    k = topk_ids.shape[1]
    e_count = w13_packed.shape[0]
    I = w2_packed.shape[2] * 8
    if act_scales.shape != (T,) or topk_ids.shape[0] != T or topk_w.shape != (T, k) or \
            w13_packed.shape != (e_count, 2 * I, H // 8) or \
            w2_packed.shape != (e_count, H, I // 8) or \
            w13_scales.shape != (e_count, H // 128, 2 * I) or \
            w2_scales.shape != (e_count, I // 128, H):
        raise ValueError("inconsistent shapes: codes [T,H], scales [T], ids/w [T,k], local "
                         "w13 [e,2I,H/8], w2 [e,H,I/8], scales group-major")
    dev = act_codes.device
    if out is None:
        out = torch.empty(T, H, dtype=torch.float32, device=dev)
    _need(out, "out", torch.float32, 2)
    need = w4a8_moe_experts_workspace_size(T, H, I, e_count, k)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    _check("w4a8_moe_forward_experts",
           lib().w4a8_moe_forward_experts(
               _p(act_codes), _p(act_scales), _p(topk_ids), _p(topk_w), T, H, I, E, k, e_begin,
               e_count, _p(w13_packed), _p(w13_scales), _p(w2_packed), _p(w2_scales), _p(out),
               _p(workspace), workspace.numel(), _stream(dev)))
    return out


def w4a8_cast_f32_bf16(x: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """bf16 copy of float32 ``x`` (round to nearest even); numel % 8 == 0."""
    if not isinstance(x, torch.Tensor) or not x.is_cuda or x.dtype != torch.float32 or \
            not x.is_contiguous():
        raise ValueError("x must be a contiguous float32 CUDA tensor")
    if out is None:
        out = torch.empty(x.shape, dtype=torch.bfloat16, device=x.device)
    if out.shape != x.shape or out.dtype != torch.bfloat16 or not out.is_contiguous() or \
            not out.is_cuda:
        raise ValueError("out must be a contiguous bf16 CUDA tensor of x's shape")
    _check("w4a8_cast_f32_bf16",
           lib().w4a8_cast_f32_bf16(_p(x), x.numel(), _p(out), _stream(x.device)))
    return out


def w4a8_ep_dispatch_plan(topk_ids: torch.Tensor, E: int, n_ranks: int):
    """The all-to-all(v) dispatch plan of a rank's routed tokens:
    (send_counts int32 [n_ranks], send_rows int32 [T * min(k, n_ranks)] (the
    first sum(send_counts) entries used), pos int32 [T, n_ranks])."""
    _need(topk_ids, "topk_ids", torch.int32, 2)
    T, k = topk_ids.shape
    dev = topk_ids.device
    counts = torch.empty(n_ranks, dtype=torch.int32, device=dev)
    rows = torch.empty(max(T * min(k, n_ranks), 1), dtype=torch.int32, device=dev)
    pos = torch.empty(T, n_ranks, dtype=torch.int32, device=dev)
    _check("w4a8_ep_dispatch_plan",
           lib().w4a8_ep_dispatch_plan(_p(topk_ids), T, k, E, n_ranks, _p(counts), _p(rows),
                                       rows.numel(), _p(pos), _stream(dev)))
    return counts, rows, pos


def w4a8_ep_gather_rows(codes: torch.Tensor, scales: torch.Tensor, topk_ids: torch.Tensor,
                        topk_w: torch.Tensor, send_rows: torch.Tensor, n_rows: int):
    """Rows ``send_rows[:n_rows]`` of a rank's codes, scales, ids and weights:
    (uint8 [n, H], float32 [n], int32 [n, k], float32 [n, k])."""
    _need(codes, "codes", torch.uint8, 2)
    _need(scales, "scales", torch.float32, 1)
    _need(topk_ids, "topk_ids", torch.int32, 2)
    _need(topk_w, "topk_w", torch.float32, 2)
    _need(send_rows, "send_rows", torch.int32, 1)
    T, H = codes.shape
    k = topk_ids.shape[1]
    if scales.shape != (T,) or topk_ids.shape[0] != T or topk_w.shape != (T, k) or \
            not 0 <= n_rows <= send_rows.numel():
        raise ValueError("inconsistent shapes: codes [T,H], scales [T], ids/w [T,k], "
                         "n_rows <= len(send_rows)")
    dev = codes.device
    out = (torch.empty(n_rows, H, dtype=torch.uint8, device=dev),
           torch.empty(n_rows, dtype=torch.float32, device=dev),
           torch.empty(n_rows, k, dtype=torch.int32, device=dev),
           torch.empty(n_rows, k, dtype=torch.float32, device=dev))
    _check("w4a8_ep_gather_rows",
           lib().w4a8_ep_gather_rows(_p(codes), _p(scales), _p(topk_ids), _p(topk_w), T, H, k,
                                     _p(send_rows), n_rows, *(_p(o) for o in out), _stream(dev)))
    return out


def w4a8_ep_combine_rows(back: torch.Tensor, pos: torch.Tensor,
                         out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """bf16 [T, H]: each token's returned partial-sum rows ``back[pos[t, r]]``
    summed in rank order (float32) and rounded once."""
    _need(back, "back", torch.float32, 2)
    _need(pos, "pos", torch.int32, 2)
    n_rows, H = back.shape
    T, n_ranks = pos.shape
    dev = pos.device
    if out is None:
        out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, 2)
    if out.shape != (T, H):
        raise ValueError("out must be [T, H]")
    _check("w4a8_ep_combine_rows",
           lib().w4a8_ep_combine_rows(_p(back), n_rows, H, _p(pos), T, n_ranks, _p(out),
                                      _stream(dev)))
    return out
