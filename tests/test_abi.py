"""The C-ABI library builds, loads and exports what include/vgv.h declares;
host-side validation rejects bad arguments before any CUDA call (CPU only)."""
import ctypes
import os
import re
import subprocess

import pytest

import greedy_speculative_verify_b200 as vgv
from greedy_speculative_verify_b200 import build as vbuild


@pytest.fixture(scope="module")
def lib():
    vbuild.build()
    return vgv.load()


def _header_functions(root):
    src = open(os.path.join(root, "include", "vgv.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return set(re.findall(r"\b(vg_[a-z_0-9]+)\s*\(", src))


def test_exports_match_header(lib, root_dir):
    declared = _header_functions(root_dir)
    assert declared == set(vgv.EXPORTS)
    out = subprocess.run(["nm", "-D", "--defined-only", vgv.LIB_PATH], capture_output=True, text=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T vg_" in l}
    assert declared <= exported


def test_status_strings_and_version(lib):
    assert vgv.vg_abi_version() == 2
    for code, name in vgv.STATUS_NAMES.items():
        assert vgv.vg_status_string(code) == name


def test_workspace_queries(lib):
    d = vgv.MOE_DIMS
    w128 = vgv.vg_moe_workspace_bytes(d, 128)
    N = 128 * 6
    # routing tables, permutation, gathered rows (at 64-token tiles also 64 rows
    # for the first tile of each of the 64 routed experts), activations, expert
    # outputs; above that only small scratch (logits, per-CTA counts, counters)
    floor = 4 * N * 4 + (N + 64 * 64) * 1280 * 2 + 8 * 128 * 896 * 2 + 8 * 128 * 1280 * 2
    assert floor <= w128 < floor + 160 * 1024
    assert vgv.vg_moe_workspace_bytes(d, 256) > w128
    assert vgv.vg_moe_stack_workspace_bytes(d, 128) >= w128 + 2 * 128 * 1280 * 2
    assert vgv.vg_moe_workspace_bytes(vgv.vg_moe_dims(1280, 896, 64, 2, 8), 128) == 0
    assert vgv.vg_moe_workspace_bytes(d, -1) == 0
    # one running argmax key per verify row, then the CTA counter
    assert vgv.vg_verify_workspace_bytes(32, 3, 1280, 129280) == 128 * 8 + 256
    assert vgv.vg_verify_workspace_bytes(1, 0, 1280, 129280) == 256 + 256
    assert vgv.vg_verify_workspace_bytes(32, 3, 1024, 129280) == 0
    assert vgv.vg_verify_workspace_bytes(32, -1, 1280, 129280) == 0
    assert vgv.vg_verify_workspace_bytes(1 << 22, 3, 1280, 129280) == 0


def _moe_call(lib, dims, T, ptrs, ws_bytes, taps=None):
    x, rw, ew, sw, out, ws = ptrs
    return lib.vg_moe_ffn(ctypes.byref(dims), T, x, rw, None, ew, sw, 1, out, taps, ws, ws_bytes, None)


def test_moe_validation_before_launch(lib):
    d = vgv.MOE_DIMS
    A = 1 << 40  # fake, aligned, never dereferenced: validation fails first
    ok = [A, A + (1 << 30), A + (2 << 30), A + (3 << 30), A + (4 << 30), A + (5 << 30)]
    need = vgv.vg_moe_workspace_bytes(d, 16)
    assert _moe_call(lib, d, 0, ok, need) == 0                          # T = 0: no-op
    assert _moe_call(lib, d, -1, ok, need) == 1                         # negative T
    assert _moe_call(lib, vgv.vg_moe_dims(1024, 896, 64, 2, 6), 16, ok, need) == 2
    bad = list(ok); bad[0] = None
    assert _moe_call(lib, d, 16, bad, need) == 1                        # null x
    bad = list(ok); bad[2] = A + 8
    assert _moe_call(lib, d, 16, bad, need) == 1                        # misaligned weights
    assert _moe_call(lib, d, 16, ok, need - 1) == 3                     # short workspace
    bad = list(ok); bad[5] = None
    assert _moe_call(lib, d, 16, bad, need) == 3                        # no workspace
    bad = list(ok); bad[4] = ok[0] + 64
    assert _moe_call(lib, d, 16, bad, need) == 1                        # out overlaps x


def test_verify_validation_before_launch(lib):
    A = 1 << 40
    h, lm, dr, am, ac, ot, ws = (A + (i << 30) for i in range(7))
    need = vgv.vg_verify_workspace_bytes(4, 3, 1280, 129280)
    f = lib.vg_verify_greedy
    assert f(0, 3, 1280, 129280, h, lm, dr, am, ac, ot, ws, need, None) == 0      # B = 0
    assert f(-1, 3, 1280, 129280, h, lm, dr, am, ac, ot, ws, need, None) == 1
    assert f(4, -1, 1280, 129280, h, lm, dr, am, ac, ot, ws, need, None) == 1
    assert f(4, 3, 1280, 0, h, lm, dr, am, ac, ot, ws, need, None) == 1
    assert f(4, 3, 1024, 129280, h, lm, dr, am, ac, ot, ws, need, None) == 2
    assert f(4, 3, 1280, 129280, h, lm, None, am, ac, ot, ws, need, None) == 1    # drafts needed for K > 0
    assert f(4, 3, 1280, 129280, h, None, dr, am, ac, ot, ws, need, None) == 1
    assert f(4, 3, 1280, 129280, h, lm, dr, am, ac, ot, ws, need - 1, None) == 3
    assert f(4, 3, 1280, 129280, h + 4, lm, dr, am, ac, ot, ws, need, None) == 1  # misaligned h


def test_stack_validation_before_launch(lib):
    d = vgv.MOE_DIMS
    arr = ctypes.c_void_p * 2
    A = 1 << 40
    rw, ew, sw = arr(A, A), arr(A, A), arr(A, None)
    need = vgv.vg_moe_stack_workspace_bytes(d, 8)
    f = lib.vg_moe_ffn_stack
    assert f(ctypes.byref(d), 0, 8, A, rw, None, ew, sw, A + (1 << 30), A + (2 << 30), need, None) == 1
    assert f(ctypes.byref(d), 2, 8, A, rw, None, ew, sw, A + (1 << 30), A + (2 << 30), need, None) == 1  # null layer ptr
    sw = arr(A, A)
    assert f(ctypes.byref(d), 2, 8, A, rw, None, ew, sw, A + (1 << 30), A + (2 << 30), need - 1, None) == 3
    assert f(ctypes.byref(d), 2, 0, A, rw, None, ew, sw, A + (1 << 30), A + (2 << 30), need, None) == 0


def test_binding_has_no_fallback(tmp_path, monkeypatch):
    """Without the shared library the binding raises instead of computing."""
    monkeypatch.setattr(vgv, "_lib", None)
    monkeypatch.setattr(vgv, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError):
        vgv.vg_abi_version()


def test_decode_loop_validation_before_launch(lib):
    A = 1 << 40
    # embedding gather: bad sizes, null pointers, misaligned rows
    assert lib.vg_embed_rows(A, 0, A, 10, 1280, A + (1 << 30), None) == 0          # n = 0: no-op
    assert lib.vg_embed_rows(A, -1, A, 10, 1280, A + (1 << 30), None) == 1
    assert lib.vg_embed_rows(A, 4, A, 10, 1281, A + (1 << 30), None) == 1          # H not a multiple of 8
    assert lib.vg_embed_rows(None, 4, A, 10, 1280, A + (1 << 30), None) == 1
    assert lib.vg_embed_rows(A, 4, A + 8, 10, 1280, A + (1 << 30), None) == 1      # misaligned table
    assert lib.vg_embed_rows(A, 4, A, 10, 1280, A + 64, None) == 1                 # out overlaps the table
    # speculative-loop state
    mk = lambda **kw: vgv.vg_spec_state(**{**dict(B=2, K=3, V=100, last=A, pos=A, committed=A, cap=8, ref=None,
                                                  ref_len=0, p=0.5, seed=1, step=A, tokens=A, drafts=A), **kw})
    f_rows, f_commit = lib.vg_spec_rows, lib.vg_spec_commit
    assert f_rows(None, None) == 1
    assert f_rows(ctypes.byref(mk(p=1.5)), None) == 1
    assert f_rows(ctypes.byref(mk(K=3, drafts=None)), None) == 1                   # drafts needed for K > 0
    assert f_rows(ctypes.byref(mk(ref_len=4)), None) == 1                          # ref_len without ref
    assert f_rows(ctypes.byref(mk(B=0)), None) == 0                                # B = 0: no-op
    assert f_commit(ctypes.byref(mk()), None, A, None) == 1                        # accepted needed
    assert f_commit(ctypes.byref(mk(B=0)), None, None, None) == 0


def test_draft_block_validation_before_launch(lib):
    A = 1 << 40
    w = vgv.vg_mtp_weights(A, A, A, A, A, A, A, 1000)
    need = vgv.vg_mtp_workspace_bytes(4, 1000)
    assert need > 0 and vgv.vg_mtp_workspace_bytes(-1, 1000) == 0 and vgv.vg_mtp_workspace_bytes(4, 0) == 0
    f = lib.vg_mtp_draft
    assert f(4, 0, ctypes.byref(w), A, 4, None, A, A, None, A, need, None) == 0       # K = 0: no-op
    assert f(0, 3, ctypes.byref(w), A, 4, None, A, A, None, A, need, None) == 0       # B = 0: no-op
    assert f(-1, 3, ctypes.byref(w), A, 4, None, A, A, None, A, need, None) == 1
    assert f(4, 3, None, A, 4, None, A, A, None, A, need, None) == 1
    assert f(4, 3, ctypes.byref(w), A, 0, None, A, A, None, A, need, None) == 1       # rows_per_seq >= 1
    assert f(4, 3, ctypes.byref(w), None, 4, None, A, A, None, A, need, None) == 1    # h needed
    assert f(4, 3, ctypes.byref(w), A + 8, 4, None, A, A, None, A, need, None) == 1   # misaligned h
    assert f(4, 3, ctypes.byref(w), A, 4, None, A, A, None, A, need - 1, None) == 3   # short workspace
    assert f(4, 3, ctypes.byref(w), A, 4, None, A, A, None, A + 8, need, None) == 3   # misaligned workspace
    bad = vgv.vg_mtp_weights(A, None, A, A, A, A, A, 1000)
    assert f(4, 3, ctypes.byref(bad), A, 4, None, A, A, None, A, need, None) == 1     # ffn needed


def test_attention_validation_before_launch(lib):
    A = 1 << 40
    need = vgv.vg_attn_workspace_bytes(4, 3, 512)
    assert need > 0 and vgv.vg_attn_workspace_bytes(4, 8, 512) == 0 and vgv.vg_attn_workspace_bytes(4, 3, 40000) == 0
    f = lib.vg_attn_verify
    args = lambda **kw: [kw.get(k, v) for k, v in dict(B=4, K=3, L=512, x=A, wq=A + (1 << 30), wo=A + (2 << 30),
                                                          c=A + (3 << 30), lens=A + (4 << 30), out=A + (5 << 30),
                                                          o=None, ws=A + (6 << 30), n=need, s=None).items()]
    assert f(*args(B=0)) == 0
    assert f(*args(K=8)) == 1                     # at most 8 new rows per sequence
    assert f(*args(L=0)) == 1
    assert f(*args(x=None)) == 1
    assert f(*args(out=A + 64)) == 1              # out overlaps x
    assert f(*args(wq=A + 8)) == 1                # misaligned weights
    assert f(*args(out=A + (3 << 30) + 4096)) == 1  # out inside the cache
    assert f(*args(o=A + 64)) == 1                # o_out overlaps x
    assert f(*args(o=A + (5 << 30))) == 1         # o_out overlaps out
    assert f(*args(o=A + (3 << 30))) == 1         # o_out inside the cache
    assert f(*args(o=A + (7 << 30) + 8)) == 1     # misaligned o_out
    assert f(*args(n=need - 1)) == 3
    assert f(*args(ws=A + (6 << 30) + 8)) == 3    # misaligned workspace
    assert f(*args(B=600_000)) == 2               # B (K+1) H items overflow int launch sizes


def test_attention_binding_checks_cache_shape():
    """The binding passes the cache's third dimension as L_max, so it refuses a
    cache that is not a dense [B, 2, L_max, H] tensor before any library call."""
    import torch

    good = torch.zeros(2, 2, 16, 1280, dtype=torch.bfloat16)
    for bad in (torch.zeros(3, 2, 16, 1280, dtype=torch.bfloat16),       # wrong B
                torch.zeros(2, 16, 1280, dtype=torch.bfloat16),          # not 4-d
                good.transpose(2, 3)):                                    # not dense
        with pytest.raises(ValueError):
            vgv.vg_attn_verify(2, 3, None, None, None, bad, None, None, None)


def test_debug_wait_validation_before_launch(lib):
    A = 1 << 40
    f = lib.vg_debug_wait_site
    assert f(0, A, 1000, None) == 1              # unknown wait kind
    assert f(3, A, 1000, None) == 1
    assert f(vgv.VG_WAIT_MBARRIER, A, 0, None) == 1           # zero limit
    assert f(vgv.VG_WAIT_MBARRIER, A, 61_000_000_000, None) == 1  # over a minute
    assert f(vgv.VG_WAIT_GRID_BARRIER, None, 1000, None) == 1     # the counter is needed
    assert f(vgv.VG_WAIT_GRID_BARRIER, A + 2, 1000, None) == 1    # misaligned counter


def test_small_step_validation_before_launch(lib):
    A = 1 << 40
    need = lib.vg_verify_step_small_workspace_bytes()
    assert need > 10 << 20
    L = 12
    arr = ctypes.c_void_p * L
    w = arr(*[A + (i << 30) for i in range(L)])
    d = ctypes.byref(vgv.MOE_DIMS)
    f = lib.vg_verify_step_small

    def call(n_layers=L, B=1, K=3, x=A, lm=A, V=129280, drafts=A, ws=A, n=need, rw=w, states=None, dims=d):
        return f(dims, n_layers, B, K, x, rw, None, w, w, lm, V, drafts, A, A, A, states, None, ws, n, None)

    assert call(B=0) == 0                       # no-op
    assert call(B=-1) == 1
    assert call(n_layers=0) == 1
    assert call(n_layers=13) == 2               # at most 12 layers
    assert call(B=5, K=3) == 2                  # 20 rows > 16
    assert call(x=None) == 1
    assert call(drafts=None) == 1               # drafts needed when K > 0
    assert call(x=A + 8) == 1                   # misaligned
    assert call(states=A + 8) == 1
    assert call(rw=None) == 1
    assert call(n=need - 1) == 3
    assert call(ws=A + 8) == 3
    assert call(dims=ctypes.byref(vgv.vg_moe_dims(1280, 896, 64, 2, 8))) == 2

