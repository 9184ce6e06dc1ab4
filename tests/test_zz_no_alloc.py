"""The no-allocation forward (library-held static scratch) against the regular forward.

entmax_attn_fwd_noalloc serves callers that are given only their input and output
buffers and may not allocate device memory. It must give the same O and tau as
entmax_attn_fwd with a caller workspace, call after call. This file sorts last so
that a run stopping at the first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

from entmax_sm_attention_b200 import binding as eb
from entmax_sm_attention_b200.workloads import make_inputs, small_case

from parity import TOL_O, TOL_TAU

pytestmark = pytest.mark.gpu


def _regular(desc, d):
    ws = eb.alloc_workspace(desc, "cuda")
    O = torch.empty(d["Q"].shape, dtype=torch.float32, device="cuda")
    tau = torch.empty(d["Q"].shape[:3], dtype=torch.float32, device="cuda")
    eb.entmax_attn_fwd(desc, d["Q"], d["K"], d["V"], O, tau, ws)
    return O, tau


def _noalloc(desc, d):
    O = torch.empty(d["Q"].shape, dtype=torch.float32, device="cuda")
    tau = torch.empty(d["Q"].shape[:3], dtype=torch.float32, device="cuda")
    eb.entmax_attn_fwd_noalloc(desc, d["Q"], d["K"], d["V"], O, tau)
    return O, tau


def test_noalloc_matches_regular_forward_twice():
    # Calls in a row with different shapes; the third is smaller than the second, so
    # contents left in the shared scratch by an earlier call would show up in its result.
    cases = [(small_case("na1", B=2, H=3, L=700, causal=True), 1.5),
             (small_case("na2", B=1, H=2, L=1500, kv_len=1100), 2.0),
             (small_case("na3", B=1, H=1, L=300, causal=True, window=32), 1.5)]
    for w, alpha in cases:
        d = {k: v.cuda() for k, v in make_inputs(w, seed=3).items()}
        kv = None if w.kv_len is None else torch.tensor(w.kv_len_list(), dtype=torch.int32, device="cuda")
        desc = eb.make_desc(w.B, w.H, w.L, alpha=alpha, scale=w.scale, causal=w.causal, window=w.window,
                            kv_len=kv)
        assert eb.entmax_attn_workspace_bytes(desc) <= eb.ENTMAX_NOALLOC_SCRATCH_BYTES
        O1, t1 = _regular(desc, d)
        O2, t2 = _noalloc(desc, d)
        torch.cuda.synchronize()
        # The same kernel on the same inputs: bit-identical results.
        assert torch.equal(O1, O2), (w.name, (O1 - O2).abs().max().item())
        assert torch.equal(t1, t2), (w.name, (t1 - t2).abs().max().item())
        assert (O1 - O2).abs().max().item() <= TOL_O and (t1 - t2).abs().max().item() <= TOL_TAU
        assert np.isfinite(O2.cpu().numpy()).all()
        # The scratch's status word of that call (workspace = NULL reads it).
        code, word = eb.entmax_last_device_status(desc, None)
        assert code == eb.ENTMAX_OK and word == 0, (code, word)


def test_noalloc_status_word_reports_device_conditions():
    """A V value beyond fp16's range is reported through the scratch's status word, and
    the next clean call clears it."""
    w = small_case("na_range", B=1, H=1, L=256)
    d = {k: v.cuda() for k, v in make_inputs(w, seed=5).items()}
    desc = eb.make_desc(1, 1, w.L, alpha=1.5, scale=w.scale)
    d["V"][0, 0, 9, 4] = 1.0e5
    _noalloc(desc, d)
    code, word = eb.entmax_last_device_status(desc, None)
    assert code == eb.ENTMAX_ERANGE and word & 4
    d["V"][0, 0, 9, 4] = 0.25
    _noalloc(desc, d)
    assert eb.entmax_last_device_status(desc, None) == (eb.ENTMAX_OK, 0)


def test_noalloc_rejects_problems_beyond_the_scratch():
    desc = eb.make_desc(4, 16, 8192)            # ~200 MB of workspace: far over 16 MiB
    assert eb.entmax_attn_workspace_bytes(desc) > eb.ENTMAX_NOALLOC_SCRATCH_BYTES
    rc = eb.load_library().entmax_attn_fwd_noalloc(__import__("ctypes").byref(desc), 1 << 20, 1 << 20, 1 << 20,
                                                   1 << 20, 1 << 20, None)
    assert rc == eb.ENTMAX_EUNSUPPORTED
