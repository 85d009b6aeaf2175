"""Python binding of the verifier hot-path library (libvgv.so, include/vgv.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of libvgv.so. The functions carry the C names and take torch tensors
(device memory, any stream) or ``None``; they return nothing and raise
``VgError`` on a non-OK status. There is no CPU fallback: if the library is not
built, the first call raises.

    import greedy_speculative_verify_b200 as vgv
    ws = torch.empty(vgv.vg_moe_workspace_bytes(vgv.MOE_DIMS, T), dtype=torch.uint8, device="cuda")
    vgv.vg_moe_ffn(vgv.MOE_DIMS, T, x, router_w, None, expert_w, shared_w, 1, out, None, ws)
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libvgv.so")

VG_OK = 0
STATUS_NAMES = {0: "VG_OK", 1: "VG_ERR_INVALID_ARG", 2: "VG_ERR_UNSUPPORTED", 3: "VG_ERR_WORKSPACE",
                4: "VG_ERR_CUDA", 5: "VG_ERR_TIMEOUT", 6: "VG_ERR_DEVICE_BOUNDS"}

# every symbol include/vgv.h declares
EXPORTS = (
    "vg_status_string", "vg_abi_version", "vg_moe_workspace_bytes", "vg_moe_ffn",
    "vg_moe_stack_workspace_bytes", "vg_moe_ffn_stack", "vg_verify_workspace_bytes",
    "vg_verify_greedy", "vg_get_device_status", "vg_set_wait_timeout_ns", "vg_debug_wait_flag", "vg_debug_wait_site",
    "vg_profile_set_events", "vg_profile_count", "vg_verify_greedy_noalloc",
    "vg_embed_rows", "vg_spec_rows", "vg_spec_commit", "vg_spec_rows_given",
    "vg_mtp_workspace_bytes", "vg_mtp_draft", "vg_attn_workspace_bytes", "vg_attn_verify",
    "vg_verify_step_small_workspace_bytes", "vg_verify_step_small",
)

# vg_kernel
VG_KERNEL_ROUTER, VG_KERNEL_GROUPING, VG_KERNEL_EXPERTS = 0, 1, 2
VG_KERNEL_COMBINE, VG_KERNEL_LM_HEAD, VG_KERNEL_ACCEPT = 3, 4, 5
VG_KERNEL_ATTENTION = 6


class VgError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


class vg_moe_dims(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("intermediate", ctypes.c_int32), ("n_routed", ctypes.c_int32),
                ("n_shared", ctypes.c_int32), ("top_k", ctypes.c_int32)]


class vg_moe_taps(ctypes.Structure):
    _fields_ = [("topk_idx", ctypes.c_void_p), ("topk_weight", ctypes.c_void_p),
                ("expert_offsets", ctypes.c_void_p), ("perm", ctypes.c_void_p), ("inv_perm", ctypes.c_void_p),
                ("act", ctypes.c_void_p), ("expert_out", ctypes.c_void_p)]


class vg_spec_state(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("K", ctypes.c_int32), ("V", ctypes.c_int32),
                ("last", ctypes.c_void_p), ("pos", ctypes.c_void_p), ("committed", ctypes.c_void_p),
                ("cap", ctypes.c_int32), ("ref", ctypes.c_void_p), ("ref_len", ctypes.c_int32),
                ("p", ctypes.c_float), ("seed", ctypes.c_uint64), ("step", ctypes.c_void_p),
                ("tokens", ctypes.c_void_p), ("drafts", ctypes.c_void_p)]


class vg_mtp_weights(ctypes.Structure):
    _fields_ = [("proj", ctypes.c_void_p), ("ffn", ctypes.c_void_p), ("gamma_h", ctypes.c_void_p),
                ("gamma_e", ctypes.c_void_p), ("gamma_f", ctypes.c_void_p), ("emb", ctypes.c_void_p),
                ("lm_head", ctypes.c_void_p), ("V", ctypes.c_int32)]


MOE_DIMS = vg_moe_dims(1280, 896, 64, 2, 6)

_lib = None


def load():
    """Loads libvgv.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with greedy_speculative_verify_b200.build.build()")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, u64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_uint64, ctypes.c_size_t
    dims_p = ctypes.POINTER(vg_moe_dims)
    sig = {
        "vg_status_string": (ctypes.c_char_p, [i32]),
        "vg_abi_version": (i32, []),
        "vg_moe_workspace_bytes": (sz, [dims_p, i32]),
        "vg_moe_ffn": (i32, [dims_p, i32, vp, vp, vp, vp, vp, i32, vp, ctypes.POINTER(vg_moe_taps), vp, sz, vp]),
        "vg_moe_stack_workspace_bytes": (sz, [dims_p, i32]),
        "vg_moe_ffn_stack": (i32, [dims_p, i32, i32, vp, ctypes.POINTER(vp), ctypes.POINTER(vp), ctypes.POINTER(vp),
                                   ctypes.POINTER(vp), vp, vp, sz, vp]),
        "vg_verify_workspace_bytes": (sz, [i32, i32, i32, i32]),
        "vg_verify_greedy": (i32, [i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "vg_get_device_status": (i32, [vp, ctypes.POINTER(i32)]),
        "vg_set_wait_timeout_ns": (i32, [u64]),
        "vg_debug_wait_flag": (i32, [vp, i32, u64, vp]),
        "vg_debug_wait_site": (i32, [i32, vp, u64, vp]),
        "vg_profile_set_events": (i32, [i32, ctypes.POINTER(vp), ctypes.POINTER(vp), i32]),
        "vg_profile_count": (ctypes.c_int64, [i32]),
        "vg_verify_greedy_noalloc": (i32, [i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp]),
        "vg_embed_rows": (i32, [vp, i32, vp, i32, i32, vp, vp]),
        "vg_spec_rows": (i32, [ctypes.POINTER(vg_spec_state), vp]),
        "vg_spec_commit": (i32, [ctypes.POINTER(vg_spec_state), vp, vp, vp]),
        "vg_spec_rows_given": (i32, [ctypes.POINTER(vg_spec_state), vp]),
        "vg_mtp_workspace_bytes": (sz, [i32, i32]),
        "vg_mtp_draft": (i32, [i32, i32, ctypes.POINTER(vg_mtp_weights), vp, i32, vp, vp, vp, vp, vp, sz, vp]),
        "vg_attn_workspace_bytes": (sz, [i32, i32, i32]),
        "vg_attn_verify": (i32, [i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "vg_verify_step_small_workspace_bytes": (sz, []),
        "vg_verify_step_small": (i32, [dims_p, i32, i32, i32, vp, ctypes.POINTER(vp), ctypes.POINTER(vp),
                                       ctypes.POINTER(vp), ctypes.POINTER(vp), vp, i32, vp, vp, vp, vp, vp, vp,
                                       vp, sz, vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch

        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _check(st: int, where: str):
    if st != VG_OK:
        raise VgError(st, where)


def vg_abi_version() -> int:
    return load().vg_abi_version()


def vg_status_string(s: int) -> str:
    return load().vg_status_string(s).decode()


def vg_moe_workspace_bytes(dims: vg_moe_dims, T_max: int) -> int:
    return load().vg_moe_workspace_bytes(ctypes.byref(dims), T_max)


def vg_moe_stack_workspace_bytes(dims: vg_moe_dims, T_max: int) -> int:
    return load().vg_moe_stack_workspace_bytes(ctypes.byref(dims), T_max)


def vg_verify_workspace_bytes(B: int, K: int, H: int, V: int) -> int:
    return load().vg_verify_workspace_bytes(B, K, H, V)


def make_taps(topk_idx=None, topk_weight=None, expert_offsets=None, perm=None, inv_perm=None, act=None,
              expert_out=None) -> vg_moe_taps:
    return vg_moe_taps(*(None if t is None else t.data_ptr()
                         for t in (topk_idx, topk_weight, expert_offsets, perm, inv_perm, act, expert_out)))


def vg_moe_ffn(dims, T, x, router_w, router_bias, expert_w, shared_w, add_residual, out, taps, workspace,
               stream=None):
    st = load().vg_moe_ffn(ctypes.byref(dims), T, _ptr(x), _ptr(router_w), _ptr(router_bias), _ptr(expert_w),
                           _ptr(shared_w), int(add_residual), _ptr(out),
                           None if taps is None else ctypes.byref(taps), _ptr(workspace),
                           0 if workspace is None else workspace.numel() * workspace.element_size(),
                           _stream(stream))
    _check(st, "vg_moe_ffn")


def vg_moe_ffn_stack(dims, n_layers, T, x, router_w, router_bias, expert_w, shared_w, out, workspace, stream=None):
    """router_w, expert_w, shared_w: sequences of n_layers tensors; router_bias:
    None or a sequence of tensors/None."""
    arr = ctypes.c_void_p * n_layers
    rw = arr(*(t.data_ptr() for t in router_w))
    ew = arr(*(t.data_ptr() for t in expert_w))
    sw = arr(*(t.data_ptr() for t in shared_w))
    rb = None if router_bias is None else arr(*(None if t is None else t.data_ptr() for t in router_bias))
    st = load().vg_moe_ffn_stack(ctypes.byref(dims), n_layers, T, _ptr(x), rw, rb, ew, sw, _ptr(out),
                                 _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "vg_moe_ffn_stack")


def vg_verify_greedy(B, K, H, V, h, lm_head, drafts, argmax, accepted, out_tokens, workspace, stream=None):
    st = load().vg_verify_greedy(B, K, H, V, _ptr(h), _ptr(lm_head), _ptr(drafts), _ptr(argmax), _ptr(accepted),
                                 _ptr(out_tokens), _ptr(workspace),
                                 0 if workspace is None else workspace.numel() * workspace.element_size(),
                                 _stream(stream))
    _check(st, "vg_verify_greedy")


def vg_verify_step_small_workspace_bytes() -> int:
    return load().vg_verify_step_small_workspace_bytes()


def vg_verify_step_small(dims, n_layers, B, K, x, router_w, router_bias, expert_w, shared_w, lm_head, V, drafts,
                         argmax, accepted, out_tokens, workspace, states_out=None, topk_idx_out=None, stream=None):
    """The whole verify step (n_layers MoE layers, LM-head argmax, accept) for
    B (K+1) <= 16 rows in one launch. Sequences of n_layers tensors as in
    vg_moe_ffn_stack."""
    arr = ctypes.c_void_p * n_layers
    rw = arr(*(t.data_ptr() for t in router_w))
    ew = arr(*(t.data_ptr() for t in expert_w))
    sw = arr(*(t.data_ptr() for t in shared_w))
    rb = None if router_bias is None else arr(*(None if t is None else t.data_ptr() for t in router_bias))
    st = load().vg_verify_step_small(ctypes.byref(dims), n_layers, B, K, _ptr(x), rw, rb, ew, sw, _ptr(lm_head), V,
                                     _ptr(drafts), _ptr(argmax), _ptr(accepted), _ptr(out_tokens),
                                     _ptr(states_out), _ptr(topk_idx_out), _ptr(workspace),
                                     workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "vg_verify_step_small")


def vg_get_device_status(stream=None) -> tuple[int, int]:
    """(status code, site) of the first fault recorded on the current device; clears it."""
    info = ctypes.c_int32(0)
    st = load().vg_get_device_status(_stream(stream), ctypes.byref(info))
    return st, info.value


def vg_set_wait_timeout_ns(ns: int):
    _check(load().vg_set_wait_timeout_ns(ns), "vg_set_wait_timeout_ns")


def vg_debug_wait_flag(flag, expect: int, max_ns: int, stream=None):
    _check(load().vg_debug_wait_flag(_ptr(flag), expect, max_ns, _stream(stream)), "vg_debug_wait_flag")


VG_WAIT_MBARRIER, VG_WAIT_GRID_BARRIER = 1, 2


def vg_debug_wait_site(which: int, ctr, max_ns: int, stream=None):
    _check(load().vg_debug_wait_site(which, _ptr(ctr), max_ns, _stream(stream)), "vg_debug_wait_site")


def vg_profile_set_events(kind: int, starts, stops):
    """starts/stops: sequences of torch.cuda.Event (enable_timing=True); empty clears."""
    n = len(starts)
    arr = ctypes.c_void_p * max(n, 1)
    a = arr(*(e.cuda_event for e in starts))
    b = arr(*(e.cuda_event for e in stops))
    _check(load().vg_profile_set_events(kind, a, b, n), "vg_profile_set_events")


def vg_profile_count(kind: int) -> int:
    return load().vg_profile_count(kind)


NOALLOC_SCRATCH_KEYS = (2 << 20) // 8


def vg_verify_greedy_noalloc(B, K, H, V, h, lm_head, drafts, argmax, accepted, out_tokens, stream=None):
    """vg_verify_greedy without a workspace, for callers that cannot allocate
    device memory; see include/vgv.h for the scratch limit and its sharing."""
    st = load().vg_verify_greedy_noalloc(B, K, H, V, _ptr(h), _ptr(lm_head), _ptr(drafts), _ptr(argmax),
                                         _ptr(accepted), _ptr(out_tokens), _stream(stream))
    _check(st, "vg_verify_greedy_noalloc")


# ------------------------------------------------------------ decode loop
def vg_embed_rows(tokens, emb, out, stream=None):
    """out[i] = emb[tokens[i]] (bf16 rows)."""
    _check(load().vg_embed_rows(_ptr(tokens), tokens.numel(), _ptr(emb), emb.shape[0], emb.shape[1], _ptr(out),
                                _stream(stream)), "vg_embed_rows")


def make_spec_state(B, K, V, last, pos, committed, ref, p, seed, step, tokens, drafts):
    """vg_spec_state over caller-owned device tensors (ref may be None); every
    tensor is read as dense rows, so each must be contiguous."""
    for t in (last, pos, committed, ref, step, tokens, drafts):
        if t is not None and not t.is_contiguous():
            raise ValueError("vg_spec_state tensors must be contiguous")
    return vg_spec_state(B, K, V, last.data_ptr(), pos.data_ptr(), committed.data_ptr(), committed.shape[1],
                         None if ref is None else ref.data_ptr(), 0 if ref is None else ref.shape[1],
                         float(p), int(seed), step.data_ptr(), tokens.data_ptr(),
                         None if drafts is None else drafts.data_ptr())


def vg_spec_rows(state, stream=None):
    _check(load().vg_spec_rows(ctypes.byref(state), _stream(stream)), "vg_spec_rows")


def vg_spec_commit(state, accepted, out_tokens, stream=None):
    _check(load().vg_spec_commit(ctypes.byref(state), _ptr(accepted), _ptr(out_tokens), _stream(stream)),
           "vg_spec_commit")


def vg_spec_rows_given(state, stream=None):
    _check(load().vg_spec_rows_given(ctypes.byref(state), _stream(stream)), "vg_spec_rows_given")


# ------------------------------------------------------------ draft block
def make_mtp_weights(proj, ffn, gamma_h, gamma_e, gamma_f, emb, lm_head):
    """vg_mtp_weights over caller-owned device tensors (fp32 gammas, bf16 rest)."""
    for t in (proj, ffn, gamma_h, gamma_e, gamma_f, emb, lm_head):
        if not t.is_contiguous():
            raise ValueError("vg_mtp_weights tensors must be contiguous")
    return vg_mtp_weights(proj.data_ptr(), ffn.data_ptr(), gamma_h.data_ptr(), gamma_e.data_ptr(),
                          gamma_f.data_ptr(), emb.data_ptr(), lm_head.data_ptr(), lm_head.shape[0])


def vg_mtp_workspace_bytes(B, V):
    return load().vg_mtp_workspace_bytes(B, V)


def vg_mtp_draft(B, K, weights, h, rows_per_seq, accepted, y0, drafts, workspace, hidden_out=None, stream=None):
    _check(load().vg_mtp_draft(B, K, ctypes.byref(weights), _ptr(h), rows_per_seq, _ptr(accepted), _ptr(y0),
                               _ptr(drafts), _ptr(hidden_out), _ptr(workspace), workspace.numel(), _stream(stream)),
           "vg_mtp_draft")


# ------------------------------------------------------------ verifier attention
def vg_attn_workspace_bytes(B, K, L_max):
    return load().vg_attn_workspace_bytes(B, K, L_max)


def vg_attn_verify(B, K, x, w_qkv, w_o, kv_cache, lens, out, workspace, o_out=None, stream=None):
    """One attention layer of a verify step; kv_cache [B, 2, L_max, H] (its
    third dimension is passed as L_max, so it must be that dense shape)."""
    if kv_cache.dim() != 4 or kv_cache.shape[0] != B or kv_cache.shape[1] != 2 or not kv_cache.is_contiguous():
        raise ValueError("kv_cache must be a contiguous [B, 2, L_max, H] tensor")
    _check(load().vg_attn_verify(B, K, kv_cache.shape[2], _ptr(x), _ptr(w_qkv), _ptr(w_o), _ptr(kv_cache), _ptr(lens),
                                 _ptr(out), _ptr(o_out), _ptr(workspace), workspace.numel(), _stream(stream)),
           "vg_attn_verify")
