"""Python binding of libdsa.so: DeepSeek Sparse Attention on one B200.

Argument marshalling only: every step of the path runs in the library's
CUDA kernels (include/dsa.h documents each entry point). PyTorch provides
device memory and the current stream. Importing this package loads
libdsa.so and raises ImportError when it has not been built (build with
``python sparse_attention_long_02_b200/build.py``); there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdsa.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "dsa.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python sparse_attention_long_02_b200/build.py`")

_lib = ctypes.CDLL(LIB_PATH)

P, I32, I64, F32, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t


def _sig(name, res, *args):
    fn = getattr(_lib, name)
    fn.restype = res
    fn.argtypes = list(args)
    return fn


_sig("dsa_status_string", ctypes.c_char_p, I32)
_sig("dsa_version", I32)
_sig("dsa_last_error_string", ctypes.c_char_p)
_sig("dsa_get_device_error", I32, P)
_sig("dsa_debug_stall", I32, ctypes.c_uint)
_sig("dsa_indexer_scores", I32, P, P, P, P, P, I32, I32, I32, I32, F32, P, I64, P)
_sig("dsa_topk", I32, P, I32, I32, I64, I32, I32, P, P)
_sig("dsa_sparse_mla_fwd", I32, P, P, P, I32, I32, I32, I32, F32, P, P, P)
_sig("dsa_window_indices", I32, I32, I32, I32, I32, I32, P, P)
_sig("dsa_project_workspace_size", SZ, I32, I32)
_sig("dsa_attention_probs_workspace_size", SZ, I32, I32, I32)
_sig("dsa_attention_probs_mean", I32, P, P, P, I32, I32, I32, I32, F32, P, I64, P, SZ, P)
_sig("dsa_indexer_kl", I32, P, I64, P, I64, I32, I32, I32, P, P, I64, P)
_sig("dsa_indexer_backward_workspace_size", SZ, I32, I32, I32)
_sig("dsa_indexer_backward", I32, P, P, P, P, P, I32, I32, I32, I32, F32, P, I64, P, P, P, P, SZ,
     P)
_sig("dsa_project_indexer_inputs", I32, P, P, P, I32, I32, I32, P, P, P, P, P, P, SZ, P)
_sig("dsa_forward_workspace_size", SZ, I32, I32, I32, I32, I32, I32)
_sig("dsa_forward_fused_workspace_size", SZ, I32, I32, I32, I32, I32, I32)
_sig("dsa_forward_fused", I32, P, P, P, P, P, P, P, I32, I32, I32, I32, I32, I32, I32, F32, F32,
     P, P, P, P, SZ, P)
_sig("dsa_forward_fused_fallback_rows", I32, P, I32, I32, I32, I32, P)
_sig("dsa_forward", I32, P, P, P, P, P, P, P, I32, I32, I32, I32, I32, I32, I32, F32, F32,
     P, P, P, P, SZ, P)
_sig("dsa_decode_paged_workspace_size", SZ, I32, I32, I32, I32, I32, I32)
_sig("dsa_decode_paged", I32, P, P, P, P, P, P, P, P, P, I32, I32, I32, I32, I32, I32, I32,
     F32, F32, P, P, P, P, SZ, P)
_sig("dsa_decode_paged_noalloc", I32, P, P, P, P, P, P, P, P, P, I32, I32, I32, I32, I32, I32,
     I32, F32, F32, P, P, P, P)
_sig("dsa_plan_prefill_chunks", I32, I32, I32, I32, I32, I32, I32, I32, I32, I32, P, I32)
_sig("dsa_plan_decode_sequences", I32, P, I32, I32, I32, I32, I32, I32, I32, P, I32)
_sig("dsa_dense_causal_mla", I32, P, P, I32, I32, I32, I32, F32, P, P, P)
_sig("dsa_dense_causal_mla_decode_paged", I32, P, P, P, P, I32, I32, I32, I32, I32, F32, P, P, P)
_sig("dsa_sparse_mla_decode_paged", I32, P, P, P, P, P, I32, I32, I32, I32, I32, I32, F32, P,
     P, P)

DSA_OK = 0
STATUS = {0: "DSA_OK", -1: "DSA_ERR_INVALID_ARG", -2: "DSA_ERR_UNSUPPORTED",
          -3: "DSA_ERR_WORKSPACE", -4: "DSA_ERR_CUDA", -5: "DSA_ERR_TIMEOUT",
          -6: "DSA_ERR_DEVICE_BOUNDS", -7: "DSA_ERR_NOT_IMPLEMENTED"}


class DSAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.dsa_status_string(status).decode()
        if status == -4:
            msg += ": " + _lib.dsa_last_error_string().decode()
        super().__init__(f"{where}: {STATUS.get(status, status)} ({msg})")


def lib():
    """The loaded ctypes library (for callers that use the raw C ABI)."""
    return _lib


def declared_functions():
    """Names of the functions include/dsa.h declares."""
    text = open(HEADER_PATH).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]*?\b(dsa_\w+)\s*\(", text, re.M)))


def _check(status, where):
    if status != DSA_OK:
        raise DSAError(status, where)


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _u8(t):
    if t.dtype == torch.float8_e4m3fn:
        t = t.view(torch.uint8)
    if t.dtype != torch.uint8:
        raise TypeError("FP8 inputs must be uint8 codes or float8_e4m3fn")
    return _dev(t)


def _dev(t, dtype=None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must be on a CUDA device")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t


def _ld(S):
    return (S + 3) // 4 * 4


DEBUG_STALL_INDEXER = 1
DEBUG_STALL_MLA = 2


def debug_stall(mask: int) -> None:
    """Debug aid: later launches of the named kernels (DEBUG_STALL_INDEXER,
    DEBUG_STALL_MLA) on the current device wait on a barrier nothing arrives
    at until their bounded wait runs out; 0 restores normal operation."""
    _check(_lib.dsa_debug_stall(mask), "dsa_debug_stall")


def get_device_error(stream=None) -> int:
    """Synchronise and read-and-clear the device error word (a status code)."""
    return _lib.dsa_get_device_error(_stream(stream))


def check_device_error(stream=None):
    _check(get_device_error(stream), "device")


def indexer_scores(q8, q_scale, k8, k_scale, w, scale, q_pos0=0, scores=None, stream=None):
    """I[t, s] for every visible key -> float32 [T][ld] (ld = S rounded up to 4)."""
    q8, k8 = _u8(q8), _u8(k8)
    w = _dev(w, torch.float32)
    T, Hi = q8.shape[0], q8.shape[1]
    S = k8.shape[0]
    if scores is None:
        scores = torch.empty(T, _ld(S), dtype=torch.float32, device=q8.device)
    _check(_lib.dsa_indexer_scores(_p(q8), _p(_dev(q_scale, torch.float32)), _p(k8),
                                   _p(_dev(k_scale, torch.float32)), _p(w), T, S, Hi, q_pos0,
                                   float(scale), _p(_dev(scores, torch.float32)),
                                   scores.shape[1], _stream(stream)), "dsa_indexer_scores")
    return scores


def project_indexer_inputs(h, wt, rope, Hi, workspace=None, stream=None):
    """Hidden states -> FP8 indexer inputs: (q8 u8 [T][Hi][128], q_scale [T],
    k8 u8 [T][128], k_scale [T], a f32 [T][Hi]); ``wt`` holds the rows of W_Q,
    W_K and W_a ([Hi*128 + 128 + Hi][d] bf16), ``rope`` the (cos, sin) table
    [T][64][2]."""
    h = _dev(h, torch.bfloat16)
    wt = _dev(wt, torch.bfloat16)
    rope = _dev(rope, torch.float32)
    T, d = h.shape
    dev = h.device
    q8 = torch.empty(T, Hi, 128, dtype=torch.uint8, device=dev)
    k8 = torch.empty(T, 128, dtype=torch.uint8, device=dev)
    q_scale = torch.empty(T, dtype=torch.float32, device=dev)
    k_scale = torch.empty(T, dtype=torch.float32, device=dev)
    a = torch.empty(T, Hi, dtype=torch.float32, device=dev)
    need = _lib.dsa_project_workspace_size(T, Hi)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    _check(_lib.dsa_project_indexer_inputs(_p(h), _p(wt), _p(rope), T, d, Hi, _p(q8), _p(q_scale),
                                           _p(k8), _p(k_scale), _p(a), _p(workspace),
                                           workspace.numel(), _stream(stream)),
           "dsa_project_indexer_inputs")
    return q8, q_scale, k8, k_scale, a


def attention_probs_mean(q, kv, lse, sm_scale, q_pos0=0, workspace=None, stream=None):
    """Head-mean dense causal attention weights -> float32 [T][S] (the warm-up target)."""
    q, kv = _dev(q, torch.bfloat16), _dev(kv, torch.bfloat16)
    lse = _dev(lse, torch.float32)
    T, H = q.shape[0], q.shape[1]
    S = kv.shape[0]
    p = torch.empty(T, S, dtype=torch.float32, device=q.device)
    if workspace is None:
        need = _lib.dsa_attention_probs_workspace_size(T, S, H)
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _check(_lib.dsa_attention_probs_mean(_p(q), _p(kv), _p(lse), T, S, H, q_pos0,
                                         float(sm_scale), _p(p), S, _p(workspace),
                                         workspace.numel(), _stream(stream)),
           "dsa_attention_probs_mean")
    return p


def indexer_kl(I, p, S, q_pos0=0, stream=None):
    """KL(p || softmax(I)) per row -> (loss [T], grad [T][ld] = dloss/dI)."""
    I, p = _dev(I, torch.float32), _dev(p, torch.float32)
    T = I.shape[0]
    loss = torch.empty(T, dtype=torch.float32, device=I.device)
    grad = torch.empty(T, I.shape[1], dtype=torch.float32, device=I.device)
    _check(_lib.dsa_indexer_kl(_p(I), I.shape[1], _p(p), p.shape[1], T, S, q_pos0, _p(loss),
                               _p(grad), grad.shape[1], _stream(stream)), "dsa_indexer_kl")
    return loss, grad


def indexer_backward(q8, q_scale, k8, k_scale, w, scale, grad, q_pos0=0, workspace=None,
                     stream=None):
    """Gradients of the warm-up loss w.r.t. the dequantised indexer inputs ->
    (dq [T][Hi][128], dk [S][128], dw [T][Hi]) in float32."""
    q8, k8 = _u8(q8), _u8(k8)
    w, grad = _dev(w, torch.float32), _dev(grad, torch.float32)
    T, Hi = q8.shape[0], q8.shape[1]
    S = k8.shape[0]
    dev = q8.device
    dq = torch.empty(T, Hi, 128, dtype=torch.float32, device=dev)
    dk = torch.empty(S, 128, dtype=torch.float32, device=dev)
    dw = torch.empty(T, Hi, dtype=torch.float32, device=dev)
    if workspace is None:
        need = _lib.dsa_indexer_backward_workspace_size(T, S, Hi)
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    _check(_lib.dsa_indexer_backward(_p(q8), _p(_dev(q_scale, torch.float32)), _p(k8),
                                     _p(_dev(k_scale, torch.float32)), _p(w), T, S, Hi, q_pos0,
                                     float(scale), _p(grad), grad.shape[1], _p(dq), _p(dk),
                                     _p(dw), _p(workspace), workspace.numel(), _stream(stream)),
           "dsa_indexer_backward")
    return dq, dk, dw


def window_indices(T, S, window, k, q_pos0=0, idx=None, device="cuda", stream=None):
    """Sliding-window (or, with window >= the prefix, dense causal) index sets
    -> int32 [T][k]: row t takes keys max(0, p - window + 1) .. p, p = q_pos0 + t."""
    if idx is None:
        idx = torch.empty(T, k, dtype=torch.int32, device=device)
    _check(_lib.dsa_window_indices(T, S, q_pos0, window, k, _p(_dev(idx, torch.int32)),
                                   _stream(stream)), "dsa_window_indices")
    return idx


def topk(scores, S, k, q_pos0=0, idx=None, stream=None):
    """Selected keys per row -> int32 [T][k], sorted by key, -1 padded."""
    scores = _dev(scores, torch.float32)
    T = scores.shape[0]
    if idx is None:
        idx = torch.empty(T, k, dtype=torch.int32, device=scores.device)
    _check(_lib.dsa_topk(_p(scores), T, S, scores.shape[1], q_pos0, k, _p(_dev(idx, torch.int32)),
                         _stream(stream)), "dsa_topk")
    return idx


def sparse_mla(q, kv, idx, sm_scale, out=None, lse=None, with_lse=True, stream=None):
    """Sparse MLA over the selected rows -> (out bf16 [T][H][512], lse f32 [T][H])."""
    q = _dev(q, torch.bfloat16)
    kv = _dev(kv, torch.bfloat16)
    idx = _dev(idx, torch.int32)
    T, H = q.shape[0], q.shape[1]
    S, k = kv.shape[0], idx.shape[1]
    if out is None:
        out = torch.empty(T, H, 512, dtype=torch.bfloat16, device=q.device)
    if lse is None and with_lse:
        lse = torch.empty(T, H, dtype=torch.float32, device=q.device)
    _check(_lib.dsa_sparse_mla_fwd(_p(q), _p(kv), _p(idx), T, S, H, k, float(sm_scale), _p(out),
                                   _p(lse), _stream(stream)), "dsa_sparse_mla_fwd")
    return out, lse


def forward_workspace_size(T, S, Hi, H, k, chunk=0) -> int:
    return int(_lib.dsa_forward_workspace_size(T, S, Hi, H, k, chunk))


def forward(q8, q_scale, k8, k_scale, w, q, kv, k, scale, sm_scale, q_pos0=0, chunk=0,
            idx=None, out=None, lse=None, workspace=None, return_idx=True, stream=None):
    """Whole prefill path -> (out, lse, idx or None)."""
    q8, k8 = _u8(q8), _u8(k8)
    q, kv = _dev(q, torch.bfloat16), _dev(kv, torch.bfloat16)
    T, Hi = q8.shape[0], q8.shape[1]
    S, H = k8.shape[0], q.shape[1]
    dev = q.device
    if out is None:
        out = torch.empty(T, H, 512, dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty(T, H, dtype=torch.float32, device=dev)
    if idx is None and return_idx:
        idx = torch.empty(T, k, dtype=torch.int32, device=dev)
    need = forward_workspace_size(T, S, Hi, H, k, chunk)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    _check(_lib.dsa_forward(_p(q8), _p(_dev(q_scale, torch.float32)), _p(k8),
                            _p(_dev(k_scale, torch.float32)), _p(_dev(w, torch.float32)), _p(q),
                            _p(kv), T, S, Hi, H, q_pos0, k, chunk, float(scale), float(sm_scale),
                            _p(idx), _p(out), _p(lse), _p(workspace), workspace.numel(),
                            _stream(stream)), "dsa_forward")
    return out, lse, idx


def forward_fused_workspace_size(T, S, Hi, H, k, chunk=0) -> int:
    return int(_lib.dsa_forward_fused_workspace_size(T, S, Hi, H, k, chunk))


def forward_fused(q8, q_scale, k8, k_scale, w, q, kv, k, scale, sm_scale, q_pos0=0, chunk=0,
                  idx=None, out=None, lse=None, workspace=None, return_idx=True, stream=None):
    """Whole prefill path with the top-k fused into the indexer (no score rows in
    HBM) -> (out, lse, idx or None); the same results as forward()."""
    q8, k8 = _u8(q8), _u8(k8)
    q, kv = _dev(q, torch.bfloat16), _dev(kv, torch.bfloat16)
    T, Hi = q8.shape[0], q8.shape[1]
    S, H = k8.shape[0], q.shape[1]
    dev = q.device
    if out is None:
        out = torch.empty(T, H, 512, dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty(T, H, dtype=torch.float32, device=dev)
    if idx is None and return_idx:
        idx = torch.empty(T, k, dtype=torch.int32, device=dev)
    if workspace is None:
        need = forward_fused_workspace_size(T, S, Hi, H, k, chunk)
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    _check(_lib.dsa_forward_fused(_p(q8), _p(_dev(q_scale, torch.float32)), _p(k8),
                                  _p(_dev(k_scale, torch.float32)), _p(_dev(w, torch.float32)),
                                  _p(q), _p(kv), T, S, Hi, H, q_pos0, k, chunk, float(scale),
                                  float(sm_scale), _p(idx), _p(out), _p(lse), _p(workspace),
                                  workspace.numel(), _stream(stream)), "dsa_forward_fused")
    return out, lse, idx


def forward_fused_fallback_rows(workspace, T, S, k, chunk=0, stream=None) -> int:
    """Rows of the last forward_fused call on `workspace` that were recomputed on
    CUDA cores (their candidate count missed [k, 4096]); synchronises."""
    n = _lib.dsa_forward_fused_fallback_rows(_p(workspace), T, S, k, chunk, _stream(stream))
    if n < 0:
        _check(n, "dsa_forward_fused_fallback_rows")
    return n


def decode_workspace_size(B, nq, max_blocks, Hi, H, k) -> int:
    return int(_lib.dsa_decode_paged_workspace_size(B, nq, max_blocks, Hi, H, k))


def decode_paged(q8, q_scale, w, q, k8_pool, k_scale_pool, kv_pool, block_table, seq_len, k,
                 scale, sm_scale, idx=None, out=None, lse=None, workspace=None,
                 return_idx=True, stream=None):
    """Paged decode -> (out [B][nq][H][512], lse [B][nq][H], idx [B][nq][k] or None)."""
    q8, k8_pool = _u8(q8), _u8(k8_pool)
    q, kv_pool = _dev(q, torch.bfloat16), _dev(kv_pool, torch.bfloat16)
    block_table = _dev(block_table, torch.int32)
    seq_len = _dev(seq_len, torch.int32)
    B, nq, Hi = q8.shape[0], q8.shape[1], q8.shape[2]
    H = q.shape[2]
    nblk, max_blocks = k8_pool.shape[0], block_table.shape[1]
    dev = q.device
    if out is None:
        out = torch.empty(B, nq, H, 512, dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty(B, nq, H, dtype=torch.float32, device=dev)
    if idx is None and return_idx:
        idx = torch.empty(B, nq, k, dtype=torch.int32, device=dev)
    need = decode_workspace_size(B, nq, max_blocks, Hi, H, k)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    _check(_lib.dsa_decode_paged(_p(q8), _p(_dev(q_scale, torch.float32)),
                                 _p(_dev(w, torch.float32)), _p(q), _p(k8_pool),
                                 _p(_dev(k_scale_pool, torch.float32)), _p(kv_pool),
                                 _p(block_table), _p(seq_len), B, nq, max_blocks, nblk, Hi, H, k,
                                 float(scale), float(sm_scale), _p(idx), _p(out), _p(lse),
                                 _p(workspace), workspace.numel(), _stream(stream)),
           "dsa_decode_paged")
    return out, lse, idx


def sparse_mla_decode_paged(q, kv_pool, block_table, seq_len, idx, sm_scale, out=None, lse=None,
                            stream=None):
    """Sparse MLA of the paged decode for given logical selections."""
    q, kv_pool = _dev(q, torch.bfloat16), _dev(kv_pool, torch.bfloat16)
    block_table, seq_len = _dev(block_table, torch.int32), _dev(seq_len, torch.int32)
    idx = _dev(idx, torch.int32)
    B, nq, H = q.shape[0], q.shape[1], q.shape[2]
    k = idx.shape[-1]
    dev = q.device
    if out is None:
        out = torch.empty(B, nq, H, 512, dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty(B, nq, H, dtype=torch.float32, device=dev)
    _check(_lib.dsa_sparse_mla_decode_paged(_p(q), _p(kv_pool), _p(block_table), _p(seq_len),
                                            _p(idx), B, nq, block_table.shape[1],
                                            kv_pool.shape[0], H, k, float(sm_scale), _p(out),
                                            _p(lse), _stream(stream)),
           "dsa_sparse_mla_decode_paged")
    return out, lse


def dense_causal_mla(q, kv, sm_scale, q_pos0=0, out=None, lse=None, stream=None):
    """Dense causal MLA: row t attends to every key 0 .. min(q_pos0 + t, S - 1) -> (out, lse)."""
    q, kv = _dev(q, torch.bfloat16), _dev(kv, torch.bfloat16)
    T, H, S = q.shape[0], q.shape[1], kv.shape[0]
    if out is None:
        out = torch.empty(T, H, 512, dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty(T, H, dtype=torch.float32, device=q.device)
    _check(_lib.dsa_dense_causal_mla(_p(q), _p(kv), T, S, H, q_pos0, float(sm_scale), _p(out),
                                     _p(lse), _stream(stream)), "dsa_dense_causal_mla")
    return out, lse


def dense_causal_mla_decode_paged(q, kv_pool, block_table, seq_len, sm_scale, out=None, lse=None,
                                  stream=None):
    """Dense causal MLA of a paged decode: every key of each query's causal prefix."""
    q, kv_pool = _dev(q, torch.bfloat16), _dev(kv_pool, torch.bfloat16)
    block_table, seq_len = _dev(block_table, torch.int32), _dev(seq_len, torch.int32)
    B, nq, H = q.shape[0], q.shape[1], q.shape[2]
    if out is None:
        out = torch.empty(B, nq, H, 512, dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty(B, nq, H, dtype=torch.float32, device=q.device)
    _check(_lib.dsa_dense_causal_mla_decode_paged(_p(q), _p(kv_pool), _p(block_table),
                                                  _p(seq_len), B, nq, block_table.shape[1],
                                                  kv_pool.shape[0], H, float(sm_scale), _p(out),
                                                  _p(lse), _stream(stream)),
           "dsa_dense_causal_mla_decode_paged")
    return out, lse


def decode_paged_noalloc(q8, q_scale, w, q, k8_pool, k_scale_pool, kv_pool, block_table, seq_len,
                         k, scale, sm_scale, idx=None, out=None, lse=None, stream=None):
    """Paged decode whose scratch is the library's fixed device array (no workspace).

    For callers that cannot allocate device memory; see dsa_decode_paged_noalloc
    in include/dsa.h for the size limit and the sharing rules.
    """
    q8, k8_pool = _u8(q8), _u8(k8_pool)
    q, kv_pool = _dev(q, torch.bfloat16), _dev(kv_pool, torch.bfloat16)
    block_table = _dev(block_table, torch.int32)
    seq_len = _dev(seq_len, torch.int32)
    B, nq, Hi = q8.shape[0], q8.shape[1], q8.shape[2]
    H = q.shape[2]
    dev = q.device
    if out is None:
        out = torch.empty(B, nq, H, 512, dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty(B, nq, H, dtype=torch.float32, device=dev)
    _check(_lib.dsa_decode_paged_noalloc(_p(q8), _p(_dev(q_scale, torch.float32)),
                                         _p(_dev(w, torch.float32)), _p(q), _p(k8_pool),
                                         _p(_dev(k_scale_pool, torch.float32)), _p(kv_pool),
                                         _p(block_table), _p(seq_len), B, nq,
                                         block_table.shape[1], k8_pool.shape[0], Hi, H, k,
                                         float(scale), float(sm_scale), _p(idx), _p(out), _p(lse),
                                         _stream(stream)), "dsa_decode_paged_noalloc")
    return out, lse, idx


def plan_prefill_chunks(T, S, Hi, H, k, chunk, parts, part, q_pos0=0):
    """First rows of worker `part`'s chunks of a T-row prefill split over `parts`
    workers, balanced by causal cost (host only)."""
    nch = max(1, (T + chunk - 1) // chunk)
    out = (ctypes.c_int32 * nch)()
    n = _lib.dsa_plan_prefill_chunks(T, S, q_pos0, Hi, H, k, chunk, parts, part, out, nch)
    _check(min(n, 0), "dsa_plan_prefill_chunks")
    return list(out[:n])


def plan_decode_sequences(seq_len, nq, Hi, H, k, parts, part):
    """Sequence numbers of worker `part`'s share of a decode batch, balanced by
    context length (host only)."""
    lens = [int(x) for x in (seq_len.tolist() if hasattr(seq_len, "tolist") else seq_len)]
    B = len(lens)
    arr = (ctypes.c_int32 * max(1, B))(*lens)
    out = (ctypes.c_int32 * max(1, B))()
    n = _lib.dsa_plan_decode_sequences(arr, B, nq, Hi, H, k, parts, part, out, max(1, B))
    _check(min(n, 0), "dsa_plan_decode_sequences")
    return list(out[:n])
