"""GPU test of hstu_attn_bwd_noalloc, the backward that needs no workspace.

That entry point serves callers that cannot allocate device memory themselves
(another allocator already owns the free device memory, or a host framework
forbids direct CUDA allocation): its scratch is a fixed array in device memory
that the library itself reserves.  Here it is called through the C ABI, twice
in a row, and each result is checked against the regular hstu_attn_bwd (which
takes a caller-provided workspace) within the bf16 tolerance of the parity
tests.  The file name makes pytest collect it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import hstu_inputs as hi
import pointwise_attention_b200 as pa
from tests.gpu_util import assert_close, np64, run_bwd, run_fwd

pytestmark = pytest.mark.gpu

NAMES = ("dq", "dk", "dv", "du", "d_rab_pos", "d_rab_time", "d_ln_weight", "d_ln_bias")


def call_noalloc(inp, dev, saved):
    lib = pa.load_library()
    p = pa.make_problem(dev["q"], dev["v"], dev["offsets"], inp.max_seq_len, dev["timestamps"],
                        dev["rab_pos"], dev["rab_time"], inp.norm_len,
                        offsets_host=inp.offsets, ln_weight=dev["ln_weight"],
                        ln_bias=dev["ln_bias"])
    out = dict(dq=torch.empty_like(dev["q"]), dk=torch.empty_like(dev["k"]),
               dv=torch.empty_like(dev["v"]), du=torch.empty_like(dev["u"]),
               d_rab_pos=torch.empty_like(dev["rab_pos"]),
               d_rab_time=torch.empty_like(dev["rab_time"]),
               d_ln_weight=torch.empty_like(dev["ln_weight"]),
               d_ln_bias=torch.empty_like(dev["ln_bias"]))
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib.hstu_attn_bwd_noalloc(ctypes.byref(p), ptr(dev["dy"]), ptr(dev["q"]), ptr(dev["k"]),
                                   ptr(dev["v"]), ptr(dev["u"]), ptr(saved[0]), ptr(saved[1]),
                                   ptr(saved[2]), *(ptr(out[n]) for n in NAMES), stream)
    torch.cuda.synchronize()
    return rc, out


def test_noalloc_backward_matches_workspace_backward():
    spec = hi.Spec("noalloc", "bf16", batch=3, heads=2, d_qk=128, d_v=128,
                   lengths=(200, 77, 131), qk_std=1 / np.sqrt(128), rab_pos_len=200,
                   rab_time=True, norm="own", grad=True, ln_affine=True)
    inp = hi.make_inputs(spec, seed=21)
    y, saved, dev = run_fwd(inp)
    ref = run_bwd(inp, dev, saved)
    for call in range(2):                       # the shared scratch keeps old contents
        rc, got = call_noalloc(inp, dev, saved)
        assert rc == 0, pa.status_string(rc)
        for n in NAMES:
            assert_close(np64(got[n]), np64(ref[n]), "bf16", "%s (call %d)" % (n, call))


def test_noalloc_rejects_problems_beyond_its_scratch():
    lib = pa.load_library()
    p = pa.hstu_problem_t()
    p.dtype, p.batch, p.total_tokens, p.max_seq_len = 1, 1, 65536, 65536
    p.num_heads, p.d_qk, p.d_v, p.ln_eps = 4, 128, 128, 1e-5
    p.offsets = 0x7F0000000000          # placeholder, rejected before any use
    assert pa.hstu_attn_workspace_size(p, True) > 16 << 20
    fake = ctypes.c_void_p(0x7F0000000000)
    # valid arguments (no bias tables, so no bias gradients) except the size
    rc = lib.hstu_attn_bwd_noalloc(ctypes.byref(p), *([fake] * 12), None, None, None, None,
                                   None)
    assert rc == 5        # HSTU_ERR_WORKSPACE
