"""vg_verify_greedy_noalloc: the verify entry point for callers that cannot
allocate device memory (a plugin whose memory belongs to its host
application's pool, a loop that must not synchronise the device through
cudaMalloc). It keeps its scratch (the running argmax key of each verify row
and a counter of finished CTAs) in a fixed 2 MiB array inside the library
instead of a caller-provided workspace.

The GPU test calls it through the C ABI twice in a row, with different shapes,
and requires the same argmax, accepted lengths and committed tokens as the
workspace entry point on the same inputs (integer outputs: bit-exact). This
file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import greedy_speculative_verify_b200 as vgv
import synth_inputs as si
from gpu_common import D, assert_device_ok, dev, ensure_lib


def _noalloc(lib, B, K, V, h, lm, drafts, am, acc, tok):
    ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.vg_verify_greedy_noalloc(B, K, D.H, V, ptr(h), ptr(lm), ptr(drafts), ptr(am), ptr(acc), ptr(tok),
                                        stream)


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_two_calls():
    ensure_lib()
    lib = vgv.load()
    cuda = torch.device("cuda")
    lm = dev(si.lm_head(0, 30, D.V, D.H))
    for B, K, cfg in [(32, 3, 31), (64, 1, 32)]:
        R = B * (K + 1)
        h = dev(si.hidden_states(0, cfg, R, D.H, tensor_id=si.TID_HID))
        # reference: the workspace entry point; drafts agree with its argmax at p = 0.7
        am0 = torch.empty(R, dtype=torch.int32, device=cuda)
        acc0 = torch.empty(B, dtype=torch.int32, device=cuda)
        tok0 = torch.empty(B, K + 1, dtype=torch.int32, device=cuda)
        ws = torch.zeros(vgv.vg_verify_workspace_bytes(B, K, D.H, D.V), dtype=torch.uint8, device=cuda)
        zeros = torch.zeros(B, K, dtype=torch.int32, device=cuda)
        vgv.vg_verify_greedy(B, K, D.H, D.V, h, lm, zeros, am0, acc0, tok0, ws)
        torch.cuda.synchronize()
        drafts_np = si.drafts_from_argmax(am0.cpu().numpy(), B, K, 0.7, D.V, seed=0, cfg=cfg)
        drafts = torch.from_numpy(drafts_np).to(cuda)
        vgv.vg_verify_greedy(B, K, D.H, D.V, h, lm, drafts, am0, acc0, tok0, ws)
        # the allocation-free entry on the same inputs
        am1 = torch.full((R,), -5, dtype=torch.int32, device=cuda)
        acc1 = torch.full((B,), -5, dtype=torch.int32, device=cuda)
        tok1 = torch.full((B, K + 1), -5, dtype=torch.int32, device=cuda)
        assert _noalloc(lib, B, K, D.V, h, lm, drafts, am1, acc1, tok1) == 0
        torch.cuda.synchronize()
        assert_device_ok()
        assert torch.equal(am1, am0)
        assert torch.equal(acc1, acc0)
        assert torch.equal(tok1, tok0)
        assert int(acc1.sum()) > 0


def test_noalloc_rejects_calls_beyond_its_scratch():
    """One 8-byte key per verify row plus the counter slot must fit the 2 MiB
    array (at most 262,143 rows); a larger call returns VG_ERR_WORKSPACE before
    any CUDA call (so this runs without a GPU)."""
    lib = vgv.load()
    A = 1 << 40
    R_max = vgv.NOALLOC_SCRATCH_KEYS - 1
    B_bad = R_max // 4 + 1  # K = 3 -> 4 rows per sequence, just past the limit
    assert lib.vg_verify_greedy_noalloc(B_bad, 3, D.H, D.V, A, A, A, A, A, A, None) == 3
    assert lib.vg_verify_greedy_noalloc(0, 3, D.H, D.V, A, A, A, A, A, A, None) == 0
    assert lib.vg_verify_greedy_noalloc(4, 3, 1024, D.V, A, A, A, A, A, A, None) == 2
