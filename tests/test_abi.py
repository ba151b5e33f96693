"""The C ABI without a GPU: the library loads, exports every declared entry
point, and rejects bad arguments on the host before touching the device."""
import ctypes
import importlib.util
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _build():
    spec = importlib.util.spec_from_file_location(
        "dsa_build", os.path.join(ROOT, "sparse_attention_long_02_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.build()


@pytest.fixture(scope="module")
def dsa():
    _build()
    import sparse_attention_long_02_b200 as d
    return d


def test_every_declared_function_is_exported(dsa):
    names = dsa.declared_functions()
    header = open(os.path.join(ROOT, "include", "dsa.h")).read()
    assert len(names) >= 11
    for n in names:
        assert hasattr(dsa.lib(), n), n
    # every entry point in the header is extern "C" (no mangling)
    assert 'extern "C"' in header


def test_status_strings(dsa):
    for s in range(-7, 1):
        assert dsa.lib().dsa_status_string(s)
    assert dsa.lib().dsa_status_string(42) == b"unknown status"
    assert dsa.lib().dsa_version() >= 100


def test_host_validation_rejects_before_launch(dsa):
    L = dsa.lib()
    # null pointers
    assert L.dsa_indexer_scores(None, None, None, None, None, 4, 4, 4, 0, 1.0, None, 4, None) == -1
    assert L.dsa_topk(None, 4, 4, 4, 0, 4, None, None) == -1
    assert L.dsa_sparse_mla_fwd(None, None, None, 1, 1, 8, 4, 0.1, None, None, None) == -1
    fake = ctypes.c_void_p(1 << 20)       # aligned, never dereferenced
    # unsupported indexer head count
    assert L.dsa_indexer_scores(fake, None, fake, None, fake, 4, 4, 3, 0, 1.0, fake, 4, None) == -2
    # k not a multiple of 4, ld not a multiple of 4, ld < S
    assert L.dsa_topk(fake, 4, 4, 4, 0, 6, fake, None) == -1
    assert L.dsa_topk(fake, 4, 6, 6, 0, 4, fake, None) == -1
    assert L.dsa_topk(fake, 4, 8, 4, 0, 4, fake, None) == -1
    # misaligned pointer
    assert L.dsa_topk(ctypes.c_void_p((1 << 20) + 4), 4, 4, 4, 0, 4, fake, None) == -1
    # MLA head count out of range
    assert L.dsa_sparse_mla_fwd(fake, fake, fake, 1, 1, 129, 4, 0.1, fake, None, None) == -2
    # non-positive scales
    assert L.dsa_indexer_scores(fake, None, fake, None, fake, 4, 4, 4, 0, 0.0, fake, 4, None) == -1
    # forward: workspace missing / too small
    assert L.dsa_forward(fake, None, fake, None, fake, fake, fake, 8, 8, 4, 8, 0, 4, 0, 1.0, 0.1,
                         None, fake, None, None, 0, None) == -3
    # window indices: window above k, non-positive window, k not a multiple of 4
    assert L.dsa_window_indices(4, 16, 0, 9, 8, fake, None) == -1
    assert L.dsa_window_indices(4, 16, 0, 0, 8, fake, None) == -1
    assert L.dsa_window_indices(4, 16, 0, 4, 6, fake, None) == -1
    assert L.dsa_window_indices(4, 16, 0, 4, 8, None, None) == -1
    # warm-up target: logits workspace missing / too small; ldp below S
    assert L.dsa_attention_probs_mean(fake, fake, fake, 4, 8, 2, 0, ctypes.c_float(0.1), fake, 8,
                                      None, 0, None) == -3
    assert L.dsa_attention_probs_mean(fake, fake, fake, 4, 8, 2, 0, ctypes.c_float(0.1), fake, 8,
                                      fake, 4 * 2 * 8 * 4 - 1, None) == -3
    assert L.dsa_attention_probs_mean(fake, fake, fake, 4, 8, 2, 0, ctypes.c_float(0.1), fake, 7,
                                      fake, 1 << 20, None) == -1
    # warm-up backward: workspace missing / too small; misaligned dq
    need = L.dsa_indexer_backward_workspace_size(4, 8, 2)
    assert L.dsa_indexer_backward(fake, None, fake, None, fake, 4, 8, 2, 0, ctypes.c_float(1.0),
                                  fake, 8, fake, fake, fake, None, 0, None) == -3
    assert L.dsa_indexer_backward(fake, None, fake, None, fake, 4, 8, 2, 0, ctypes.c_float(1.0),
                                  fake, 8, fake, fake, fake, fake, need - 1, None) == -3
    assert L.dsa_indexer_backward(fake, None, fake, None, fake, 4, 8, 2, 0, ctypes.c_float(1.0),
                                  fake, 8, ctypes.c_void_p((1 << 20) + 4), fake, fake, fake,
                                  need, None) == -1
    assert L.dsa_indexer_backward(fake, None, fake, None, fake, 4, 8, 3, 0, ctypes.c_float(1.0),
                                  fake, 8, fake, fake, fake, fake, need, None) == -2
    # GEMM row tiles: at most 65535 tiles of 128 rows
    big = 65535 * 128
    assert L.dsa_project_indexer_inputs(fake, fake, fake, big + 1, 64, 4, fake, fake, fake, fake,
                                        fake, fake, 1 << 40, None) == -1
    assert L.dsa_attention_probs_mean(fake, fake, fake, big // 2 + 1, 8, 2, 0,
                                      ctypes.c_float(0.1), fake, 8, fake, 1 << 40, None) == -1
    assert L.dsa_indexer_backward(fake, None, fake, None, fake, big // 4 + 1, 8, 4, 0,
                                  ctypes.c_float(1.0), fake, 8, fake, fake, fake, fake, 1 << 40,
                                  None) == -1
    assert L.dsa_indexer_backward(fake, None, fake, None, fake, 4, big + 1, 4, 0,
                                  ctypes.c_float(1.0), fake, big + 1, fake, fake, fake, fake,
                                  1 << 40, None) == -1
    # fused prefill: k above 2048 or rows above 131072 keys unsupported; workspace checked
    assert L.dsa_forward_fused(fake, None, fake, None, fake, fake, fake, 8, 8, 4, 8, 0, 4096, 0,
                               ctypes.c_float(1.0), ctypes.c_float(0.1), None, fake, None, fake,
                               1 << 40, None) == -2
    assert L.dsa_forward_fused(fake, None, fake, None, fake, fake, fake, 8, 131073, 4, 8, 0, 4, 0,
                               ctypes.c_float(1.0), ctypes.c_float(0.1), None, fake, None, fake,
                               1 << 40, None) == -2
    assert L.dsa_forward_fused(fake, None, fake, None, fake, fake, fake, 8, 8, 4, 8, 0, 4, 0,
                               ctypes.c_float(1.0), ctypes.c_float(0.1), None, fake, None, None, 0,
                               None) == -3
    assert L.dsa_forward_fused(None, None, fake, None, fake, fake, fake, 8, 8, 4, 8, 0, 4, 0,
                               ctypes.c_float(1.0), ctypes.c_float(0.1), None, fake, None, fake,
                               1 << 40, None) == -1
    # paged decode: more than 256 indexer columns (nq * Hi), too many MLA heads, no queries,
    # k not a multiple of 4, workspace missing or too small; an empty batch is a no-op
    def decode(nq=1, Hi=64, H=128, k=2048, B=2, ws=None, ws_bytes=0):
        return L.dsa_decode_paged(fake, None, fake, fake, fake, None, fake, fake, fake, B, nq, 4,
                                  8, Hi, H, k, ctypes.c_float(1.0), ctypes.c_float(0.1), None,
                                  fake, None, ws, ws_bytes, None)
    assert decode(nq=5) == -2
    assert decode(H=129) == -2
    assert decode(nq=0) == -1
    assert decode(k=2046) == -1
    assert decode() == -3
    assert decode(ws=fake, ws_bytes=L.dsa_decode_paged_workspace_size(2, 1, 4, 64, 128, 2048) - 1) == -3
    assert decode(B=0) == 0
    # empty problems are a no-op
    assert L.dsa_topk(fake, 0, 4, 4, 0, 4, fake, None) == 0


def test_workspace_sizes(dsa):
    L = dsa.lib()
    # one chunk of fp32 scores (pitch rounded to 4) + the index rows, each 256-B rounded
    assert L.dsa_forward_workspace_size(1024, 1024, 4, 8, 256, 0) == 1024 * 1024 * 4 + 1024 * 256 * 4
    # several chunks: two score chunks (the top-k of one overlaps the next indexer)
    assert L.dsa_forward_workspace_size(131072, 131072, 64, 128, 2048, 4096) == \
        2 * 4096 * 131072 * 4 + 131072 * 2048 * 4
    assert L.dsa_forward_workspace_size(10, 7, 4, 8, 4, 3) == 2 * 256 + 256
    assert L.dsa_decode_paged_workspace_size(64, 1, 512, 64, 128, 2048) == \
        64 * 512 * 64 * 4 + 64 * 2048 * 4
    assert L.dsa_forward_workspace_size(0, 8, 4, 8, 4, 0) == 0
    # fused prefill: the sampled keys (the first 256 of every 4096) and their
    # scales, per chunk row the sample scores and threshold, then twice (by
    # chunk parity) the count, 4096 candidates and the failure list; the call's
    # failure total, 148 scratch score rows, and idx
    r256 = lambda x: (x + 255) // 256 * 256
    T, S, k, rows = 131072, 131072, 2048, 4096
    M = 32 * 256
    per_parity = [rows * 4, rows * 4096 * 4, rows * 4096 * 4, 4 + rows * 4]
    parts = [M * 128, M * 4, rows * M * 4, rows * 4] + 2 * per_parity + \
        [4, 148 * S * 4, T * k * 4]
    assert L.dsa_forward_fused_workspace_size(T, S, 64, 128, k, rows) == sum(r256(x) for x in parts)
    # one chunk: a single set of candidate buffers
    parts1 = [M * 128, M * 4, T * M * 4, T * 4] + [T * 4, T * 4096 * 4, T * 4096 * 4,
                                                    4 + T * 4] + [4, 148 * S * 4, T * k * 4]
    assert L.dsa_forward_fused_workspace_size(T, S, 64, 128, k, 0) == sum(r256(x) for x in parts1)
    assert L.dsa_forward_fused_workspace_size(T, S, 64, 128, 4096, rows) == 0
    # warm-up target: T * H rows of fp32 logits, S rounded up to 4
    assert L.dsa_attention_probs_workspace_size(2048, 2048, 128) == 2048 * 128 * 2048 * 4
    assert L.dsa_attention_probs_workspace_size(3, 10, 2) == 3 * 2 * 12 * 4
    # warm-up backward: fp32 products, three bf16 pieces per coefficient, bf16
    # copies of q and k with their transposes, split-K partials of dk
    R, S = 2048 * 64, 2048
    parts = [4 * R * S, 2 * 3 * R * S, 2 * R * 128, 2 * R * 128, 2 * S * 128, 2 * S * 128,
             4 * 9 * S * 128]
    assert L.dsa_indexer_backward_workspace_size(2048, 2048, 64) == sum(parts)
    assert L.dsa_indexer_backward_workspace_size(4, 8, 3) == 0


def _row_cost(n, Hi, H, k):
    """Cost of one query row seeing n keys: FP8 indexer flops at half weight plus MLA flops."""
    return 128 * Hi * n + 2176 * H * min(n, k)


@pytest.mark.parametrize("T,S,q_pos0,chunk,parts", [(131072, 131072, 0, 4096, 2),
                                                    (131072, 131072, 0, 4096, 8),
                                                    (10000, 20000, 7000, 999, 3),
                                                    (5, 5, 0, 4096, 4)])
def test_prefill_plan_covers_every_chunk_once_and_balances(dsa, T, S, q_pos0, chunk, parts):
    Hi, H, k = 64, 128, 2048
    plans = [dsa.plan_prefill_chunks(T, S, Hi, H, k, chunk, parts, p, q_pos0=q_pos0)
             for p in range(parts)]
    got = sorted(c for plan in plans for c in plan)
    assert got == list(range(0, T, chunk))                 # disjoint and complete
    for plan in plans:
        assert plan == sorted(plan)

    def chunk_cost(c0):
        return sum(_row_cost(min(q_pos0 + t, S - 1) + 1, Hi, H, k)
                   for t in range(c0, min(c0 + chunk, T)))

    costs = {c0: chunk_cost(c0) for c0 in got}
    loads = [sum(costs[c] for c in plan) for plan in plans]
    # longest-first greedy: the heaviest worker exceeds the mean by at most one unit
    assert max(loads) <= sum(loads) / parts + max(costs.values()) + 1e-6
    # an idle worker only where there are fewer chunks than workers
    assert min(len(p) for p in plans) >= (1 if len(got) >= parts else 0)


def test_prefill_plan_is_the_longest_first_rule(dsa):
    # three chunks of one row each at positions 0, 1, 2 over two workers: the
    # costliest (row 2) goes to worker 0, then row 1 to worker 1, then row 0 to
    # worker 1 (the lighter one)
    assert dsa.plan_prefill_chunks(3, 3, 1, 1, 2048, 1, 2, 0) == [2]
    assert dsa.plan_prefill_chunks(3, 3, 1, 1, 2048, 1, 2, 1) == [0, 1]
    # one worker takes every chunk in order
    assert dsa.plan_prefill_chunks(9, 9, 1, 1, 4, 2, 1, 0) == [0, 2, 4, 6, 8]


def test_decode_plan_balances_by_context(dsa):
    rng = np.random.default_rng(5)
    lens = np.exp(rng.uniform(np.log(512), np.log(131072), 128)).astype(np.int32)
    Hi, H, k, nq, parts = 64, 128, 2048, 2, 4
    plans = [dsa.plan_decode_sequences(lens, nq, Hi, H, k, parts, p) for p in range(parts)]
    assert sorted(b for plan in plans for b in plan) == list(range(128))
    cost = [sum(_row_cost(int(n) - nq + j + 1, Hi, H, k) for j in range(nq)) for n in lens]
    loads = [sum(cost[b] for b in plan) for plan in plans]
    assert max(loads) <= sum(loads) / parts + max(cost) + 1e-6


def test_plan_rejects_bad_arguments(dsa):
    L = dsa.lib()
    out = (ctypes.c_int32 * 8)()
    assert L.dsa_plan_prefill_chunks(16, 16, 0, 4, 8, 4, 4, 0, 0, out, 8) == -1    # parts 0
    assert L.dsa_plan_prefill_chunks(16, 16, 0, 4, 8, 4, 4, 2, 2, out, 8) == -1    # part >= parts
    assert L.dsa_plan_prefill_chunks(16, 16, 0, 4, 8, 4, 0, 1, 0, out, 8) == -1    # chunk 0
    assert L.dsa_plan_prefill_chunks(16, 16, 0, 4, 8, 4, 4, 1, 0, out, 3) == -1    # out too short
    assert L.dsa_plan_prefill_chunks(16, 16, 0, 4, 8, 4, 4, 1, 0, None, 8) == -1
    assert L.dsa_plan_prefill_chunks(16, 16, 0, 4, 8, 4, 4, 1, 0, out, 8) == 4
    lens = (ctypes.c_int32 * 2)(1, 9)
    assert L.dsa_plan_decode_sequences(lens, 2, 2, 4, 8, 4, 1, 0, out, 8) == -1   # seq_len < nq
    assert L.dsa_plan_decode_sequences(None, 2, 1, 4, 8, 4, 1, 0, out, 8) == -1
    assert L.dsa_plan_decode_sequences(lens, 2, 1, 4, 8, 4, 1, 0, out, 8) == 2
