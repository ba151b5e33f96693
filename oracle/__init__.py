"""CPU oracle for the DSA hot path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg import this package. The product library never imports it; it shares no
code with the CUDA path.

The arithmetic lives in ``dsa_oracle.c`` (plain C, double precision, one
thread per call). This module builds it with gcc, calls it through ctypes
(the call releases the GIL, so disjoint row sets can run on several threads
when the CPU baseline is timed) and adds the two pieces of glue the paged
decode needs: translating logical positions through the block table with a
numpy gather, and chaining indexer -> top-k -> sparse MLA.

Citations (page titles and sections):
  * indexer, top-k, sparse MLA: "DeepSeek-V3.2-Exp 模型优势与 DSA 工作原理",
    section 4 "DSA 的四步工作流程", steps 2-4;
  * FP8 + ReLU in the indexer: "DeepSeek V3.2 ... DSA" (m.gxzdkb.com),
    section "秘密武器";
  * the short-context fallback (context <= k selects every key): page 3,
    section 2 "风险边界明确" and step 3.

Parity status of each function is pinned by tests/test_oracle_pins.py.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dsa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

P = ctypes.c_void_p
I64 = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile dsa_oracle.c into liboracle.so (gcc -O2, no fast-math)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared",
                           "-fno-fast-math", "-o", tmp, _SRC, "-lm"])
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            L.dsa_oracle_e4m3.restype = ctypes.c_double
            L.dsa_oracle_e4m3.argtypes = [ctypes.c_uint8]
            L.dsa_oracle_bf16.restype = ctypes.c_double
            L.dsa_oracle_bf16.argtypes = [ctypes.c_uint16]
            L.dsa_oracle_indexer.restype = ctypes.c_int
            L.dsa_oracle_indexer.argtypes = [P, P, P, P, P, I64, I64, ctypes.c_int,
                                             I64, ctypes.c_double, P, I64, P, P]
            L.dsa_oracle_topk.restype = ctypes.c_int
            L.dsa_oracle_topk.argtypes = [P, I64, I64, P, ctypes.c_int, P]
            L.dsa_oracle_window.restype = ctypes.c_int
            L.dsa_oracle_project.restype = ctypes.c_int
            L.dsa_oracle_attn_probs.restype = ctypes.c_int
            L.dsa_oracle_attn_probs.argtypes = [P, P, I64, I64, ctypes.c_int, I64, ctypes.c_double,
                                                P, I64, P]
            L.dsa_oracle_indexer_kl.restype = ctypes.c_int
            L.dsa_oracle_indexer_kl.argtypes = [P, P, I64, I64, P, P, P]
            L.dsa_oracle_indexer_backward.restype = ctypes.c_int
            L.dsa_oracle_indexer_backward.argtypes = [P, P, P, P, P, I64, I64, ctypes.c_int, I64,
                                                      ctypes.c_double, P, P, P, P]
            L.dsa_oracle_project.argtypes = [P, P, P, I64, I64, ctypes.c_int, P, I64, P]
            L.dsa_oracle_window.argtypes = [I64, I64, I64, ctypes.c_int, ctypes.c_int, P]
            L.dsa_oracle_sparse_mla.restype = ctypes.c_int
            L.dsa_oracle_sparse_mla.argtypes = [P, P, P, I64, I64, ctypes.c_int,
                                                ctypes.c_int, ctypes.c_double, P, I64, P, P]
            _lib = L
    return _lib


def _np(x, dtype):
    """Contiguous host numpy array of ``x`` with the given dtype.

    Integer codes of equal width (bf16 bits, e4m3 bytes) are reinterpreted
    bit for bit; anything else is converted.
    """
    if x is None:
        return None
    if hasattr(x, "detach"):                      # torch tensor
        import torch
        x = x.detach().cpu().contiguous()
        if x.dtype == torch.bfloat16:
            x = x.view(torch.int16)
        x = x.numpy()
    x = np.ascontiguousarray(x)
    dt = np.dtype(dtype)
    if x.dtype != dt:
        if x.dtype.itemsize == dt.itemsize and x.dtype.kind in "iu" and dt.kind in "iu":
            x = x.view(dt)
        else:
            x = x.astype(dt)
    return x


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def e4m3(code: int) -> float:
    return lib().dsa_oracle_e4m3(code)


def bf16(bits: int) -> float:
    return lib().dsa_oracle_bf16(bits)


def _rows(rows, T):
    return np.arange(T, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, np.int64)


def indexer(q8, q_scale, k8, k_scale, w, scale, q_pos0=0, rows=None, with_mag=False):
    """I[t, s] for the given query rows -> float32 [nrows][S] (and |w|-magnitudes)."""
    q8 = _np(q8, np.uint8)
    k8 = _np(k8, np.uint8)
    w = _np(w, np.float32)
    T, Hi = q8.shape[0], q8.shape[1]
    S = k8.shape[0]
    qs = _np(q_scale, np.float32)
    ks = _np(k_scale, np.float32)
    r = _rows(rows, T)
    out = np.empty((len(r), S), np.float32)
    mag = np.empty((len(r), S), np.float32) if with_mag else None
    rc = lib().dsa_oracle_indexer(_ptr(q8), _ptr(qs), _ptr(k8), _ptr(ks), _ptr(w),
                                  T, S, Hi, int(q_pos0), float(scale), _ptr(r), len(r),
                                  _ptr(out), _ptr(mag))
    if rc != 0:
        raise ValueError(f"oracle indexer failed ({rc})")
    return (out, mag) if with_mag else out


def topk(I, row_len, k):
    """Selected key positions [nrows][k] (score desc, index asc; -1 padded)."""
    I = np.ascontiguousarray(I, np.float32)
    n = np.ascontiguousarray(row_len, np.int64)
    out = np.empty((I.shape[0], k), np.int32)
    rc = lib().dsa_oracle_topk(_ptr(I), I.shape[0], I.shape[1], _ptr(n), int(k), _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle topk failed ({rc})")
    return out


def project(h, wt, rope, Hi, rows=None):
    """Projection of hidden states h [T][d] (bf16) through wt [N][d] (bf16) with
    the rotation table rope [T][64][2] -> float64 [nrows][N]: rotated q heads,
    rotated k, then a_h (before any FP8 encoding)."""
    hb = _np(h, np.uint16)
    wb = _np(wt, np.uint16)
    rp = np.ascontiguousarray(_np(rope, np.float32))
    T, d = hb.shape
    r = _rows(rows, T)
    N = Hi * 128 + 128 + Hi
    out = np.empty((len(r), N), np.float64)
    rc = lib().dsa_oracle_project(_ptr(hb), _ptr(wb), _ptr(rp), T, d, int(Hi), _ptr(r), len(r),
                                  _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle project failed ({rc})")
    return out


def attention_probs(q, kv, sm_scale, q_pos0=0, rows=None):
    """Warm-up target: head-mean dense causal attention weights -> float64 [nrows][S]."""
    qb = _np(q, np.uint16)
    kvb = _np(kv, np.uint16)
    T, H = qb.shape[0], qb.shape[1]
    S = kvb.shape[0]
    r = _rows(rows, T)
    out = np.empty((len(r), S), np.float64)
    rc = lib().dsa_oracle_attn_probs(_ptr(qb), _ptr(kvb), T, S, H, int(q_pos0), float(sm_scale),
                                     _ptr(r), len(r), _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle attn_probs failed ({rc})")
    return out


def indexer_kl(I, p, row_len):
    """KL(p || softmax(I)) per row and its gradient r - p (float64)."""
    Id = np.ascontiguousarray(I, np.float64)
    pd = np.ascontiguousarray(p, np.float64)
    n = np.ascontiguousarray(row_len, np.int64)
    loss = np.empty(Id.shape[0], np.float64)
    grad = np.empty_like(Id)
    rc = lib().dsa_oracle_indexer_kl(_ptr(Id), _ptr(pd), Id.shape[0], Id.shape[1], _ptr(n),
                                     _ptr(loss), _ptr(grad))
    if rc != 0:
        raise ValueError(f"oracle indexer_kl failed ({rc})")
    return loss, grad


def indexer_backward(q8, q_scale, k8, k_scale, w, scale, grad, q_pos0=0):
    """(dq [T][Hi][128], dk [S][128], dw [T][Hi]) float64: gradients of the warm-up
    loss w.r.t. the dequantised indexer inputs, given grad = dloss/dI [T][S]."""
    q8 = _np(q8, np.uint8)
    k8 = _np(k8, np.uint8)
    qs = None if q_scale is None else np.ascontiguousarray(_np(q_scale, np.float32))
    ks = None if k_scale is None else np.ascontiguousarray(_np(k_scale, np.float32))
    w = np.ascontiguousarray(_np(w, np.float32))
    T, Hi = q8.shape[0], q8.shape[1]
    S = k8.shape[0]
    g = np.ascontiguousarray(grad, np.float64)[:, :S]
    g = np.ascontiguousarray(g)
    dq = np.empty((T, Hi, 128), np.float64)
    dk = np.empty((S, 128), np.float64)
    dw = np.empty((T, Hi), np.float64)
    rc = lib().dsa_oracle_indexer_backward(_ptr(q8), None if qs is None else _ptr(qs), _ptr(k8),
                                           None if ks is None else _ptr(ks), _ptr(w), T, S, Hi,
                                           int(q_pos0), float(scale), _ptr(g), _ptr(dq),
                                           _ptr(dk), _ptr(dw))
    if rc != 0:
        raise ValueError(f"oracle indexer_backward failed ({rc})")
    return dq, dk, dw


def window(nrows, S, window, k, q_pos0=0):
    """Sliding-window key positions [nrows][k] (increasing, -1 padded)."""
    out = np.empty((nrows, k), np.int32)
    rc = lib().dsa_oracle_window(int(nrows), int(S), int(q_pos0), int(window), int(k), _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle window failed ({rc})")
    return out


def sparse_mla(q, kv, idx, sm_scale, rows=None):
    """(out [nrows][H][512] float64, lse [nrows][H] float64) for the given rows.

    ``idx`` is indexed by the absolute query row t (shape [T][k]).
    """
    qb = _np(q, np.uint16)
    kvb = _np(kv, np.uint16)
    idx = np.ascontiguousarray(_np(idx, np.int32))
    T, H = qb.shape[0], qb.shape[1]
    S = kvb.shape[0]
    k = idx.shape[1]
    r = _rows(rows, T)
    out = np.empty((len(r), H, 512), np.float64)
    lse = np.empty((len(r), H), np.float64)
    rc = lib().dsa_oracle_sparse_mla(_ptr(qb), _ptr(kvb), _ptr(idx), T, S, H, k,
                                     float(sm_scale), _ptr(r), len(r), _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError(f"oracle sparse_mla failed ({rc})")
    return out, lse


def prefill_row_len(T, S, q_pos0=0, rows=None):
    """Keys visible to each query row: min(q_pos0 + t + 1, S)."""
    r = _rows(rows, T)
    return np.minimum(q_pos0 + r + 1, S)


def forward(inp, rows=None):
    """Whole prefill path (indexer -> top-k -> sparse MLA) for query rows.

    ``inp`` is a dict as made by ``workloads.make_prefill``. Returns dict with
    I [nrows][S], idx [nrows][k], out [nrows][H][512], lse [nrows][H].
    """
    T, S, k = inp["T"], inp["S"], inp["k"]
    r = _rows(rows, T)
    I = indexer(inp["q8"], inp["q_scale"], inp["k8"], inp["k_scale"], inp["w"],
                inp["scale"], inp.get("q_pos0", 0), rows=r)
    idx_r = topk(I, prefill_row_len(T, S, inp.get("q_pos0", 0), r), k)
    idx_full = np.full((T, k), -1, np.int32)
    idx_full[r] = idx_r
    out, lse = sparse_mla(inp["q"], inp["kv"], idx_full, inp["sm_scale"], rows=r)
    return dict(I=I, idx=idx_r, out=out, lse=lse, rows=r)


def gather_sequence(pool, block_table_row, n_tokens):
    """Logical rows 0..n_tokens-1 of one sequence from a paged pool [nblk][64][...]."""
    pool = np.asarray(pool)
    pos = np.arange(n_tokens)
    blk = np.asarray(block_table_row)[pos // 64]
    return pool[blk, pos % 64]


def decode(inp, seqs=None):
    """Paged decode for the given sequences (default: all).

    Each sequence's cache is first gathered into logical order through its
    block table; the new queries j = 0..nq-1 sit at positions
    seq_len - nq + j. Returns dict with per-(b, j) I rows (list), idx
    [ns][nq][k] (logical positions), out [ns][nq][H][512], lse [ns][nq][H].
    """
    B, nq, k = inp["B"], inp["nq"], inp["k"]
    seqs = list(range(B)) if seqs is None else list(seqs)
    q8 = _np(inp["q8"], np.uint8)
    qs = _np(inp["q_scale"], np.float32)
    w = _np(inp["w"], np.float32)
    q = _np(inp["q"], np.uint16)
    k8p = _np(inp["k8_pool"], np.uint8)
    ksp = _np(inp["k_scale_pool"], np.float32)
    kvp = _np(inp["kv_pool"], np.uint16)
    table = _np(inp["block_table"], np.int32)
    lens = _np(inp["seq_len"], np.int32)
    H = q.shape[2]
    idx = np.full((len(seqs), nq, k), -1, np.int32)
    out = np.empty((len(seqs), nq, H, 512), np.float64)
    lse = np.empty((len(seqs), nq, H), np.float64)
    Is = []
    for i, b in enumerate(seqs):
        n = int(lens[b])
        k8 = gather_sequence(k8p, table[b], n)
        ks = gather_sequence(ksp, table[b], n)
        kv = gather_sequence(kvp, table[b], n)
        pos0 = n - nq
        I = indexer(q8[b], qs[b], k8, ks, w[b], inp["scale"], q_pos0=pos0)
        sel = topk(I, prefill_row_len(nq, n, pos0), k)
        o, l = sparse_mla(q[b], kv, sel, inp["sm_scale"])
        idx[i], out[i], lse[i] = sel, o, l
        Is.append(I)
    return dict(I=Is, idx=idx, out=out, lse=lse, seqs=seqs)
