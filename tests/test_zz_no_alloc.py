"""dsa_decode_paged_noalloc: the paged decode for callers that cannot allocate
device memory (host callbacks, plugins living in another framework's memory
pool, tools without a device allocator). Its scratch is a fixed array inside
libdsa.so, so it takes no workspace.

Checked through the raw C ABI: two calls in a row, on different inputs,
each against dsa_decode_paged with a caller-owned workspace, within the
tolerances the parity tests use (identical index sets; attention output
max-abs <= 2e-2, mean-abs <= 2e-3). The second call also shows that what
the first call left in the shared scratch does not leak into its result.
This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu


def _inputs(lens, nq, seed):
    cfg = W.Config(92, "decode_noalloc", "decode", k=2048, Hi=64, H=128, seed=seed, nq=nq,
                   ctx_lo=1, ctx_hi=2)
    inp = W.make_decode(cfg, lens=torch.tensor(lens))
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _call_noalloc(lib, g, stream):
    B, nq = g["B"], g["nq"]
    out = torch.full((B, nq, g["H"], 512), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, nq, g["H"]), float("nan"), dtype=torch.float32, device="cuda")
    idx = torch.full((B, nq, g["k"]), -7, dtype=torch.int32, device="cuda")
    st = lib.dsa_decode_paged_noalloc(
        _p(g["q8"]), _p(g["q_scale"]), _p(g["w"]), _p(g["q"]), _p(g["k8_pool"]),
        _p(g["k_scale_pool"]), _p(g["kv_pool"]), _p(g["block_table"]), _p(g["seq_len"]), B, nq,
        g["max_blocks"], g["nblk"], g["Hi"], g["H"], g["k"], g["scale"], g["sm_scale"], _p(idx),
        _p(out), _p(lse), stream)
    return st, out, lse, idx


def _call_with_workspace(lib, g, stream):
    B, nq = g["B"], g["nq"]
    need = lib.dsa_decode_paged_workspace_size(B, nq, g["max_blocks"], g["Hi"], g["H"], g["k"])
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    out = torch.empty(B, nq, g["H"], 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, nq, g["H"], dtype=torch.float32, device="cuda")
    idx = torch.empty(B, nq, g["k"], dtype=torch.int32, device="cuda")
    st = lib.dsa_decode_paged(
        _p(g["q8"]), _p(g["q_scale"]), _p(g["w"]), _p(g["q"]), _p(g["k8_pool"]),
        _p(g["k_scale_pool"]), _p(g["kv_pool"]), _p(g["block_table"]), _p(g["seq_len"]), B, nq,
        g["max_blocks"], g["nblk"], g["Hi"], g["H"], g["k"], g["scale"], g["sm_scale"], _p(idx),
        _p(out), _p(lse), _p(ws), need, stream)
    return st, out, lse, idx


def test_noalloc_decode_matches_workspace_decode_twice():
    import sparse_attention_long_02_b200 as dsa
    lib = dsa.lib()
    torch.cuda.set_device(0)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    cases = [_inputs([3000, 100, 2049, 8000], nq=2, seed=11),
             _inputs([5000, 2048, 64, 1000, 7777, 300], nq=1, seed=12)]
    for g in cases:                       # two calls in a row through the C ABI
        st, out, lse, idx = _call_noalloc(lib, g, stream)
        assert st == 0, dsa.STATUS.get(st, st)
        assert lib.dsa_get_device_error(stream) == 0
        st, out_r, lse_r, idx_r = _call_with_workspace(lib, g, stream)
        assert st == 0, dsa.STATUS.get(st, st)
        assert lib.dsa_get_device_error(stream) == 0
        assert torch.equal(idx, idx_r)
        err = (out.float() - out_r.float()).abs()
        assert torch.isfinite(out.float()).all()
        assert err.max().item() <= 2e-2 and err.mean().item() <= 2e-3
        fin = torch.isfinite(lse_r)
        assert torch.equal(fin, torch.isfinite(lse))
        assert (lse[fin] - lse_r[fin]).abs().max().item() <= 2e-3


def test_noalloc_rejects_requests_beyond_its_scratch():
    import sparse_attention_long_02_b200 as dsa
    lib = dsa.lib()
    fake = ctypes.c_void_p(1 << 20)       # never dereferenced: rejected on the host
    # 128 rows x 131072 keys of fp32 scores is 64 MiB, above the 32 MiB scratch
    st = lib.dsa_decode_paged_noalloc(fake, None, fake, fake, fake, None, fake, fake, fake,
                                      128, 1, 2048, 1, 64, 128, 2048, 0.1, 0.1, None, fake, None,
                                      None)
    assert st == -3                       # DSA_ERR_WORKSPACE
    assert b"32 MiB" in lib.dsa_last_error_string()
