"""MoE expert-MLP + Split-LoRA layer for NVIDIA B200 (sm_100a).

A thin ctypes binding over the C ABI in include/moelora.h (libmoelora.so, built
in-tree by `python -m mixture_experts_lora_b200.build`).  The functions below
carry the ABI's names and only marshal arguments: PyTorch provides device
memory and the current stream; every step of the layer runs in the library's
CUDA kernels.  There is no CPU or PyTorch fallback: if the library is missing
or was not built, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoelora.so")

# status codes (include/moelora.h)
MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_WORKSPACE = 3
MOE_ERR_CUDA = 4
MOE_ERR_DEVICE_INDEX = 5
MOE_ERR_TIMEOUT = 6
MOE_ERR_DEVICE_CHECK = 7

EXPORTED = (
    "moe_workspace_bytes", "moe_route_topk", "moe_permute", "moe_grouped_gemm_lora_fwd",
    "moe_grouped_gemm_lora_bwd", "moe_unpermute_combine", "moe_get_device_error",
    "moe_status_string", "moe_profile_enable", "moe_profile_select", "moe_profile_read",
    "moe_permute_noalloc", "moe_router_backward", "moe_grouped_gemm_full_bwd",
    "moe_check_permutation", "moe_selftest_bounded_wait", "moe_route_permute",
)


class MoEError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn}: {msg} (status {status})")
        self.status = status


class moe_dims_t(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("m", ctypes.c_int32), ("n", ctypes.c_int32),
                ("E", ctypes.c_int32), ("k", ctypes.c_int32), ("r", ctypes.c_int32),
                ("scale", ctypes.c_float)]


_lib_handle = None


def lib() -> ctypes.CDLL:
    """Load libmoelora.so (raises if it was not built)."""
    global _lib_handle
    if _lib_handle is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m mixture_experts_lora_b200.build`")
        h = ctypes.CDLL(LIB_PATH)
        P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        D = ctypes.POINTER(moe_dims_t)
        h.moe_workspace_bytes.argtypes = [D]
        h.moe_workspace_bytes.restype = SZ
        h.moe_route_topk.argtypes = [P, I64, I32, I32, P, P, P]
        h.moe_permute.argtypes = [P, I64, I32, I32, P, P, P, P, P, SZ, P]
        h.moe_permute_noalloc.argtypes = [P, I64, I32, I32, P, P, P, P, P]
        h.moe_route_permute.argtypes = [P, I64, I32, I32, P, P, P, P, P, P, P, SZ, P]
        h.moe_check_permutation.argtypes = [P, I64, I32, I32, P, P, P, P, P]
        h.moe_grouped_gemm_lora_fwd.argtypes = [D] + [P] * 16 + [SZ, P]
        h.moe_grouped_gemm_lora_bwd.argtypes = [D] + [P] * 21 + [SZ, P]
        h.moe_grouped_gemm_full_bwd.argtypes = [D] + [P] * 23 + [SZ, P]
        h.moe_unpermute_combine.argtypes = [P, P, P, I64, I32, I32, P, P]
        h.moe_router_backward.argtypes = [P, P, P, P, P, I64, I32, I32, I32, P, P]
        h.moe_selftest_bounded_wait.argtypes = [ctypes.c_uint64, P, P]
        h.moe_get_device_error.argtypes = [P]
        h.moe_status_string.argtypes = [ctypes.c_int]
        h.moe_status_string.restype = ctypes.c_char_p
        h.moe_profile_enable.argtypes = [ctypes.c_int]
        h.moe_profile_enable.restype = None
        h.moe_profile_select.argtypes = [ctypes.c_char_p]
        h.moe_profile_read.argtypes = [ctypes.c_int, ctypes.c_char_p, ctypes.c_int,
                                       ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_double)]
        for name in EXPORTED:
            if name not in ("moe_workspace_bytes", "moe_status_string", "moe_profile_enable"):
                getattr(h, name).restype = ctypes.c_int
        _lib_handle = h
    return _lib_handle


def status_string(status: int) -> str:
    return lib().moe_status_string(int(status)).decode()


def debug_checks() -> bool:
    """True when the environment variable MOE_CHECK is set (and not "0"): every call
    then synchronises and reads the device error word, and every permutation is
    checked on the device (moe_check_permutation).  For eager debugging; calls made
    while a CUDA graph is being captured are not checked."""
    return os.environ.get("MOE_CHECK", "") not in ("", "0")


def _check(fn: str, status: int):
    if status != MOE_OK:
        raise MoEError(fn, status, status_string(status))
    if debug_checks() and not torch.cuda.is_current_stream_capturing():
        torch.cuda.synchronize()
        st = int(lib().moe_get_device_error(_stream()))
        if st != MOE_OK:
            raise MoEError(fn, st, status_string(st))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def make_dims(T, m, n, E, k, r, scale) -> moe_dims_t:
    return moe_dims_t(int(T), int(m), int(n), int(E), int(k), int(r), float(scale))


# ---------------------------------------------------------------- ABI calls
def moe_workspace_bytes(dims: moe_dims_t) -> int:
    return int(lib().moe_workspace_bytes(ctypes.byref(dims)))


def moe_route_topk(logits, k, topk_ids, topk_w, stream=None):
    T, E = logits.shape
    _check("moe_route_topk", lib().moe_route_topk(_ptr(logits), T, E, int(k), _ptr(topk_ids),
                                                  _ptr(topk_w), _stream(stream)))


def moe_permute(topk_ids, E, counts, offsets, sorted_pairs, pair_pos, ws, stream=None):
    T, k = topk_ids.shape
    _check("moe_permute", lib().moe_permute(_ptr(topk_ids), T, k, int(E), _ptr(counts),
                                            _ptr(offsets), _ptr(sorted_pairs), _ptr(pair_pos),
                                            _ptr(ws), ws.numel() * ws.element_size(),
                                            _stream(stream)))
    if debug_checks():
        moe_check_permutation(topk_ids, E, counts, offsets, sorted_pairs, pair_pos, stream)


def moe_route_permute(logits, k, topk_ids, topk_w, counts, offsets, sorted_pairs, pair_pos, ws,
                      stream=None):
    """moe_route_topk and moe_permute in one call (one cooperative launch)."""
    T, E = logits.shape
    _check("moe_route_permute", lib().moe_route_permute(
        _ptr(logits), T, E, int(k), _ptr(topk_ids), _ptr(topk_w), _ptr(counts), _ptr(offsets),
        _ptr(sorted_pairs), _ptr(pair_pos), _ptr(ws), ws.numel() * ws.element_size(),
        _stream(stream)))
    if debug_checks():
        moe_check_permutation(topk_ids, E, counts, offsets, sorted_pairs, pair_pos, stream)


def moe_check_permutation(topk_ids, E, counts, offsets, sorted_pairs, pair_pos, stream=None):
    """Device check of every invariant moe_permute promises; a violation sets
    MOE_ERR_DEVICE_CHECK in the device error word (see moe_get_device_error)."""
    T, k = topk_ids.shape
    _check("moe_check_permutation", lib().moe_check_permutation(
        _ptr(topk_ids), T, k, int(E), _ptr(counts), _ptr(offsets), _ptr(sorted_pairs),
        _ptr(pair_pos), _stream(stream)))


def moe_permute_noalloc(topk_ids, E, counts, offsets, sorted_pairs, pair_pos, stream=None):
    """moe_permute without a workspace (scratch built into the library)."""
    T, k = topk_ids.shape
    _check("moe_permute_noalloc", lib().moe_permute_noalloc(
        _ptr(topk_ids), T, k, int(E), _ptr(counts), _ptr(offsets), _ptr(sorted_pairs),
        _ptr(pair_pos), _stream(stream)))
    if debug_checks():
        moe_check_permutation(topk_ids, E, counts, offsets, sorted_pairs, pair_pos, stream)


def moe_grouped_gemm_lora_fwd(dims, X, sorted_pairs, offsets, W_gu, W_d, A_gu, B_gu, A_d, B_d,
                              Y_sorted, save_Xs, save_GU, save_H, save_XA, save_HA, ws, stream=None):
    args = [X, sorted_pairs, offsets, W_gu, W_d, A_gu, B_gu, A_d, B_d, Y_sorted, save_Xs, save_GU,
            save_H, save_XA, save_HA, ws]
    _check("moe_grouped_gemm_lora_fwd", lib().moe_grouped_gemm_lora_fwd(
        ctypes.byref(dims), *[_ptr(a) for a in args], ws.numel() * ws.element_size(),
        _stream(stream)))


def moe_grouped_gemm_lora_bwd(dims, dY, topk_w, sorted_pairs, offsets, W_gu, W_d, A_gu, B_gu,
                              A_d, B_d, save_Xs, save_GU, save_H, save_XA, save_HA, dX_sorted, dA_gu,
                              dB_gu, dA_d, dB_d, ws, stream=None):
    args = [dY, topk_w, sorted_pairs, offsets, W_gu, W_d, A_gu, B_gu, A_d, B_d, save_Xs, save_GU,
            save_H, save_XA, save_HA, dX_sorted, dA_gu, dB_gu, dA_d, dB_d, ws]
    _check("moe_grouped_gemm_lora_bwd", lib().moe_grouped_gemm_lora_bwd(
        ctypes.byref(dims), *[_ptr(a) for a in args], ws.numel() * ws.element_size(),
        _stream(stream)))


def moe_grouped_gemm_full_bwd(dims, dY, topk_w, sorted_pairs, offsets, W_gu, W_d, A_gu, B_gu,
                              A_d, B_d, save_Xs, save_GU, save_H, save_XA, save_HA, dX_sorted, dW_gu,
                              dW_d, dA_gu=None, dB_gu=None, dA_d=None, dB_d=None, ws=None,
                              stream=None):
    """Backward with the expert-weight gradients dW_gu [E, m, 2n] and dW_d [E, n, m]
    (full fine-tuning); the adapter gradients are computed when all four are given."""
    if ws is None:
        raise ValueError("moe_grouped_gemm_full_bwd needs the workspace")
    args = [dY, topk_w, sorted_pairs, offsets, W_gu, W_d, A_gu, B_gu, A_d, B_d, save_Xs, save_GU,
            save_H, save_XA, save_HA, dX_sorted, dW_gu, dW_d, dA_gu, dB_gu, dA_d, dB_d, ws]
    _check("moe_grouped_gemm_full_bwd", lib().moe_grouped_gemm_full_bwd(
        ctypes.byref(dims), *[_ptr(a) for a in args], ws.numel() * ws.element_size(),
        _stream(stream)))


def moe_unpermute_combine(Y_sorted, topk_w, pair_pos, T, k, m, Y, stream=None):
    _check("moe_unpermute_combine", lib().moe_unpermute_combine(
        _ptr(Y_sorted), _ptr(topk_w), _ptr(pair_pos), int(T), int(k), int(m), _ptr(Y),
        _stream(stream)))


def moe_router_backward(dY, Y_sorted, topk_ids, topk_w, pair_pos, E: int, dlogits, stream=None):
    """dlogits [T, E] fp32: gradient into the router logits (see include/moelora.h)."""
    T, m = dY.shape
    k = topk_ids.shape[1]
    _check("moe_router_backward", lib().moe_router_backward(
        _ptr(dY), _ptr(Y_sorted), _ptr(topk_ids), _ptr(topk_w), _ptr(pair_pos), int(T), int(k),
        int(E), int(m), _ptr(dlogits), _stream(stream)))


def moe_selftest_bounded_wait(limit_ns: int, done, stream=None):
    """Run one bounded wait that nothing ends (see include/moelora.h); afterwards
    moe_get_device_error() reports MOE_ERR_TIMEOUT and done[0] == 1."""
    st = lib().moe_selftest_bounded_wait(int(limit_ns), _ptr(done), _stream(stream))
    if st != MOE_OK:
        raise MoEError("moe_selftest_bounded_wait", st, status_string(st))


def moe_get_device_error(stream=None) -> int:
    return int(lib().moe_get_device_error(_stream(stream)))


def moe_profile_enable(on: bool = True):
    lib().moe_profile_enable(1 if on else 0)


def moe_profile_select(kinds=None) -> int:
    """Trace only the named kernel kinds (a list or comma-separated string); None = all."""
    if kinds is not None and not isinstance(kinds, str):
        kinds = ",".join(kinds)
    n = lib().moe_profile_select(None if not kinds else kinds.encode())
    if n < 0:
        raise ValueError(f"unknown kernel kind in {kinds!r}")
    return n


def moe_profile_read() -> dict:
    """{kernel name: (launches, total ms)} since the last read (waits for the GPU)."""
    n, L = 32, 48
    names = ctypes.create_string_buffer(n * L)
    cnt = (ctypes.c_int * n)()
    ms = (ctypes.c_double * n)()
    w = lib().moe_profile_read(n, names, L, cnt, ms)
    return {names.raw[i * L:(i + 1) * L].split(b"\0", 1)[0].decode(): (cnt[i], ms[i])
            for i in range(w)}


# ---------------------------------------------------------------- whole layer
@dataclass
class LayerBuffers:
    """Device buffers of one layer step (allocated once with PyTorch, reused)."""
    ids: torch.Tensor
    w: torch.Tensor
    counts: torch.Tensor
    offsets: torch.Tensor
    sorted_pairs: torch.Tensor
    pair_pos: torch.Tensor
    Y_sorted: torch.Tensor
    save_Xs: torch.Tensor
    save_GU: torch.Tensor
    save_H: torch.Tensor
    save_XA: torch.Tensor
    save_HA: torch.Tensor
    Y: torch.Tensor
    dX_sorted: torch.Tensor
    dX: torch.Tensor
    dA_gu: torch.Tensor
    dB_gu: torch.Tensor
    dA_d: torch.Tensor
    dB_d: torch.Tensor
    ws: torch.Tensor


def alloc_buffers(T, m, n, E, k, r, scale, device="cuda") -> LayerBuffers:
    P = T * k
    bf = dict(dtype=torch.bfloat16, device=device)
    i32 = dict(dtype=torch.int32, device=device)
    wsb = moe_workspace_bytes(make_dims(T, m, n, E, k, r, scale))
    if wsb == 0:
        raise MoEError("moe_workspace_bytes", MOE_ERR_UNSUPPORTED, "unsupported shape")
    return LayerBuffers(
        ids=torch.empty(T, k, **i32), w=torch.empty(T, k, dtype=torch.float32, device=device),
        counts=torch.empty(E, **i32), offsets=torch.empty(E + 1, **i32),
        sorted_pairs=torch.empty(P, **i32), pair_pos=torch.empty(P, **i32),
        Y_sorted=torch.empty(P, m, **bf), save_Xs=torch.empty(P, m, **bf),
        save_GU=torch.empty(P, 2 * n, **bf),
        save_H=torch.empty(P, n, **bf), save_XA=torch.empty(P, r, **bf),
        save_HA=torch.empty(P, r, **bf), Y=torch.empty(T, m, **bf),
        dX_sorted=torch.empty(P, m, **bf), dX=torch.empty(T, m, **bf),
        dA_gu=torch.empty(E, m, r, **bf), dB_gu=torch.empty(E, r, 2 * n, **bf),
        dA_d=torch.empty(E, n, r, **bf), dB_d=torch.empty(E, r, m, **bf),
        ws=torch.empty(wsb, dtype=torch.uint8, device=device))


def layer_forward(inp: dict, k: int, scale: float, buf: LayerBuffers, stream=None):
    """route -> permute -> grouped GEMMs -> combine; fills buf.Y (and the saves)."""
    T, m = inp["X"].shape
    E, _, n2 = inp["W_gu"].shape
    r = inp["A_gu"].shape[2]
    dims = make_dims(T, m, n2 // 2, E, k, r, scale)
    moe_route_permute(inp["logits"], k, buf.ids, buf.w, buf.counts, buf.offsets, buf.sorted_pairs,
                      buf.pair_pos, buf.ws, stream)
    moe_grouped_gemm_lora_fwd(dims, inp["X"], buf.sorted_pairs, buf.offsets, inp["W_gu"],
                              inp["W_d"], inp["A_gu"], inp["B_gu"], inp["A_d"], inp["B_d"],
                              buf.Y_sorted, buf.save_Xs, buf.save_GU, buf.save_H, buf.save_XA,
                              buf.save_HA, buf.ws, stream)
    moe_unpermute_combine(buf.Y_sorted, buf.w, buf.pair_pos, T, k, m, buf.Y, stream)
    return buf.Y


def layer_backward(inp: dict, dY, k: int, scale: float, buf: LayerBuffers, stream=None):
    """grouped GEMM backward -> unweighted combine; fills buf.dX and the adapter grads."""
    T, m = inp["X"].shape
    E, _, n2 = inp["W_gu"].shape
    r = inp["A_gu"].shape[2]
    dims = make_dims(T, m, n2 // 2, E, k, r, scale)
    moe_grouped_gemm_lora_bwd(dims, dY, buf.w, buf.sorted_pairs, buf.offsets,
                              inp["W_gu"], inp["W_d"], inp["A_gu"], inp["B_gu"], inp["A_d"],
                              inp["B_d"], buf.save_Xs, buf.save_GU, buf.save_H, buf.save_XA,
                              buf.save_HA,
                              buf.dX_sorted, buf.dA_gu, buf.dB_gu, buf.dA_d, buf.dB_d, buf.ws,
                              stream)
    moe_unpermute_combine(buf.dX_sorted, None, buf.pair_pos, T, k, m, buf.dX, stream)
    return buf.dX


def layer_backward_full(inp: dict, dY, k: int, scale: float, buf: LayerBuffers, dW_gu, dW_d,
                        adapters: bool = True, stream=None):
    """layer_backward plus the expert-weight gradients (full fine-tuning) into dW_gu
    [E, m, 2n] and dW_d [E, n, m]; adapters=False skips the adapter gradients."""
    T, m = inp["X"].shape
    E, _, n2 = inp["W_gu"].shape
    r = inp["A_gu"].shape[2]
    dims = make_dims(T, m, n2 // 2, E, k, r, scale)
    lora = (buf.dA_gu, buf.dB_gu, buf.dA_d, buf.dB_d) if adapters else (None,) * 4
    moe_grouped_gemm_full_bwd(dims, dY, buf.w, buf.sorted_pairs, buf.offsets,
                              inp["W_gu"], inp["W_d"], inp["A_gu"], inp["B_gu"], inp["A_d"],
                              inp["B_d"], buf.save_Xs, buf.save_GU, buf.save_H, buf.save_XA,
                              buf.save_HA,
                              buf.dX_sorted, dW_gu, dW_d, *lora, ws=buf.ws, stream=stream)
    moe_unpermute_combine(buf.dX_sorted, None, buf.pair_pos, T, k, m, buf.dX, stream)
    return buf.dX


def layer_step(inp: dict, k: int, scale: float, buf: LayerBuffers, stream=None):
    """One pass of the whole hot path: forward then backward against inp['dY']."""
    layer_forward(inp, k, scale, buf, stream)
    layer_backward(inp, inp["dY"], k, scale, buf, stream)
    return buf


def shared_expert_step(inp: dict, scale: float, buf: LayerBuffers, stream=None):
    """Shared expert: a dense SwiGLU MLP with LoRA applied to every token, whose output
    the caller adds to the routed experts' Y (and its dX to theirs).  It is this layer
    with one expert, k = 1 and routing weight 1: `inp` holds X, dY and the six weight
    tensors with a leading expert dimension of 1, plus logits [T, 1] (any values; the
    softmax over one picked logit is 1).  Outputs land in buf.Y, buf.dX and the
    adapter gradients like layer_step; `buf` comes from alloc_buffers(T, m, n, 1, 1, r, scale)."""
    if inp["W_gu"].shape[0] != 1 or inp["logits"].shape[1] != 1:
        raise ValueError("a shared expert has exactly one expert and logits of width 1")
    return layer_step(inp, 1, scale, buf, stream)


# ---------------------------------------------------------------- adapter variants
class SplitGateUpAdapters:
    """Separate gate and up adapters (rank r each) held in the library's fused layout.

    gate_up carries one adapter of rank 2r with A_gu = [A_g | A_u] and
    B_gu = [[B_g, 0], [0, B_u]]; the down adapter is zero-padded to the same rank
    (the library uses one rank for both projections).  The result is exactly the
    layer with separate adapters.  The attributes A_g, B_g, A_u, B_u, A_d, B_d are
    views into the packed tensors: write them, or let an optimizer update them, in
    place.  Nothing ever writes the off-diagonal blocks or the padding, so those
    stay zero.  Pass A_gu, B_gu, A_d_packed and B_d_packed to the layer with rank 2r
    and the scale of one adapter (alpha / r, or alpha / sqrt(r) for rsLoRA)."""

    def __init__(self, E: int, m: int, n: int, r: int, device="cuda"):
        if 2 * r > 128:
            raise ValueError("separate gate/up adapters need 2r <= 128")
        bf = dict(dtype=torch.bfloat16, device=device)
        self.r, self.n = r, n
        self.A_gu = torch.zeros(E, m, 2 * r, **bf)
        self.B_gu = torch.zeros(E, 2 * r, 2 * n, **bf)
        self.A_d_packed = torch.zeros(E, n, 2 * r, **bf)
        self.B_d_packed = torch.zeros(E, 2 * r, m, **bf)
        self.A_g, self.A_u = self.A_gu[:, :, :r], self.A_gu[:, :, r:]
        self.B_g, self.B_u = self.B_gu[:, :r, :n], self.B_gu[:, r:, n:]
        self.A_d, self.B_d = self.A_d_packed[:, :, :r], self.B_d_packed[:, :r, :]

    def layer_inputs(self, inp: dict) -> dict:
        """inp (X, logits, dY, W_gu, W_d) completed with the packed adapters."""
        out = dict(inp)
        out.update(A_gu=self.A_gu, B_gu=self.B_gu, A_d=self.A_d_packed, B_d=self.B_d_packed)
        return out

    def grads(self, buf: LayerBuffers) -> dict:
        """Views of the separate adapters' gradients in a rank-2r LayerBuffers."""
        r, n = self.r, self.n
        return {"dA_g": buf.dA_gu[:, :, :r], "dA_u": buf.dA_gu[:, :, r:],
                "dB_g": buf.dB_gu[:, :r, :n], "dB_u": buf.dB_gu[:, r:, n:],
                "dA_d": buf.dA_d[:, :, :r], "dB_d": buf.dB_d[:, :r, :]}
