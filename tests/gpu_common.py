"""Helpers shared by the GPU parity tests: running the library through its
binding on device tensors, and the comparison rules.

Comparison rules (the tolerances of the parity bar):
* integer outputs (routing ids, offsets, permutation, accepted lengths,
  committed tokens): bit-exact;
* activations: per row, max_h |gpu - ref| / max_h |ref| <= 1e-2 (ref = fp64
  oracle on the same bf16 inputs), maximum over rows;
* argmax: equal to the oracle's, except rows where the two candidates are a
  certified near-tie: z64[ref] - z64[gpu] <= 2^-14 * (A[ref] + A[gpu]), with
  z64 the fp64 logit and A = sum_h |hid_h * LM_vh|, a bound on the error of any
  fp32 summation order over 1280 terms.
"""
import os

import numpy as np
import torch

import greedy_speculative_verify_b200 as vgv
import oracle
import synth_inputs as si
from greedy_speculative_verify_b200 import build as vbuild

D = si.FULL
ACT_TOL = 1e-2
TIE_EPS = 2.0 ** -14


def ensure_lib():
    """Builds and loads the library; VG_TEST_LIB names another build of it to
    test instead (the bounds-checking debug build, tests/test_gpu_zy_debug_bounds.py)."""
    vbuild.build()
    other = os.environ.get("VG_TEST_LIB")
    if other:
        vgv.LIB_PATH = other
    vgv.load()


def dev(bits):
    return si.bits_to_torch(bits, "cuda")


def f32(bits):
    return si.bf16_bits_to_f32(bits).astype(np.float64)


def row_rel_err(gpu, ref):
    gpu = np.asarray(gpu, dtype=np.float64).reshape(ref.shape[0], -1)
    ref = np.asarray(ref, dtype=np.float64).reshape(ref.shape[0], -1)
    den = np.maximum(np.abs(ref).max(axis=1), 1e-30)
    return float((np.abs(gpu - ref).max(axis=1) / den).max())


GUARD_BYTES = 4096  # canary region on each side of every output buffer
_CANARY = 0xA5


class Guarded:
    """Output tensors carved from the middle of larger buffers whose guard
    regions (GUARD_BYTES on each side) hold a canary byte pattern; check()
    asserts that no kernel wrote outside the tensors it was given. A stand-in
    for a memory checker, which is not available on these GPUs."""

    def __init__(self):
        self.bufs = []

    def empty(self, shape, dtype, fill=None):
        n = 1
        for d in shape:
            n *= d
        nbytes = n * torch.empty((), dtype=dtype).element_size()
        raw = torch.full((nbytes + 2 * GUARD_BYTES,), _CANARY, dtype=torch.uint8, device="cuda")
        t = raw[GUARD_BYTES:GUARD_BYTES + nbytes].view(dtype).view(*shape)
        if fill is not None:
            t.fill_(fill)
        self.bufs.append((raw, nbytes))
        return t

    def check(self):
        torch.cuda.synchronize()
        for raw, nbytes in self.bufs:
            head, tail = raw[:GUARD_BYTES], raw[GUARD_BYTES + nbytes:]
            assert bool((head == _CANARY).all()) and bool((tail == _CANARY).all()), "write outside an output buffer"


def assert_device_ok():
    st, info = vgv.vg_get_device_status()
    assert st == 0, f"device status {vgv.STATUS_NAMES.get(st, st)} at site {info}"


def run_moe(x_bits, lw, bias=None, add_residual=True, xdev=None):
    """One layer through vg_moe_ffn with every intermediate tapped."""
    T = x_bits.shape[0] if xdev is None else xdev.shape[0]
    cuda = torch.device("cuda")
    x = xdev if xdev is not None else dev(x_bits)
    rw = lw["router_w"] if torch.is_tensor(lw["router_w"]) else dev(lw["router_w"])
    ew = lw["expert_w"] if torch.is_tensor(lw["expert_w"]) else dev(lw["expert_w"])
    sw = lw["shared_w"] if torch.is_tensor(lw["shared_w"]) else dev(lw["shared_w"])
    b = None if bias is None else torch.from_numpy(np.asarray(bias, dtype=np.float32)).to(cuda)
    N = T * D.k
    gd = Guarded()
    out = gd.empty((T, D.H), torch.bfloat16)
    idx = gd.empty((T, D.k), torch.int32, fill=-1)
    w = gd.empty((T, D.k), torch.float32)
    off = gd.empty((D.E + 1,), torch.int32)
    perm = gd.empty((N,), torch.int32)
    inv = gd.empty((N,), torch.int32)
    act = gd.empty(((D.k + D.S) * T, D.I), torch.bfloat16)
    eo = gd.empty(((D.k + D.S) * T, D.H), torch.bfloat16)
    taps = vgv.make_taps(idx, w, off, perm, inv, act, eo)
    ws = gd.empty((vgv.vg_moe_workspace_bytes(vgv.MOE_DIMS, T),), torch.uint8)
    vgv.vg_moe_ffn(vgv.MOE_DIMS, T, x, rw, b, ew, sw, int(add_residual), out, taps, ws)
    torch.cuda.synchronize()
    assert_device_ok()
    gd.check()
    return {
        "out": f32(si.torch_to_bits(out)), "idx": idx.cpu().numpy(), "g": w.cpu().numpy(),
        "offsets": off.cpu().numpy(), "perm": perm.cpu().numpy(), "inv": inv.cpu().numpy(),
        "act": f32(si.torch_to_bits(act)), "expert_out": f32(si.torch_to_bits(eo)),
    }


def run_verify(h, lm, drafts, B, K, V=None):
    """vg_verify_greedy on device tensors h [B(K+1),H] bf16, lm [V,H] bf16,
    drafts [B,K] int32 (numpy or tensor)."""
    cuda = torch.device("cuda")
    V = lm.shape[0] if V is None else V
    R = B * (K + 1)
    d = None
    if K > 0:
        d = drafts if torch.is_tensor(drafts) else torch.from_numpy(np.ascontiguousarray(drafts, dtype=np.int32)).to(cuda)
    gd = Guarded()
    am = gd.empty((max(R, 1),), torch.int32, fill=-7)
    acc = gd.empty((max(B, 1),), torch.int32, fill=-7)
    ot = gd.empty((max(B, 1), K + 1), torch.int32, fill=-7)
    ws = gd.empty((max(1, vgv.vg_verify_workspace_bytes(B, K, D.H, V)),), torch.uint8, fill=0)
    vgv.vg_verify_greedy(B, K, D.H, V, h, lm, d, am, acc, ot, ws)
    torch.cuda.synchronize()
    assert_device_ok()
    gd.check()
    assert int(ws.count_nonzero()) == 0  # the call leaves its workspace zero-filled
    return am.cpu().numpy(), acc.cpu().numpy(), ot.cpu().numpy()


def check_argmax(gpu_arg, ref_arg, hid_bits, lm_bits, rows=None):
    """Bit-exact argmax except certified near-ties; returns the number of
    certified near-ties."""
    gpu_arg = np.asarray(gpu_arg)
    ref_arg = np.asarray(ref_arg)
    rows = np.arange(len(ref_arg)) if rows is None else np.asarray(rows)
    bad = np.nonzero(gpu_arg[rows] != ref_arg[rows])[0]
    ties = 0
    for i in bad:
        r = rows[i]
        g, a = int(gpu_arg[r]), int(ref_arg[r])
        assert 0 <= g < lm_bits.shape[0], f"row {r}: argmax {g} out of range"
        z, amag = oracle.logit_fp64(hid_bits, lm_bits, [r, r], [a, g])
        assert z[0] - z[1] <= TIE_EPS * (amag[0] + amag[1]), f"row {r}: gpu {g} vs oracle {a}, margin {z[0] - z[1]}"
        ties += 1
    return ties
