"""Parity at the benchmark sizes, in the launch configuration bench.py times.

The GPU runs the whole path at full size: the prefill configs through
dsa_forward_fused (the top-k fused into the indexer, the path bench.py times)
and through dsa_forward (scores in HBM), both with their chunking; the decode
configs through dsa_decode_paged.
The oracle then recomputes sampled rows one by one: the indexer scores of the
row, its selection (exact, or within the tie rule on random inputs) and the
attention on the GPU's own selection (bf16 tolerances).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from test_gpu_parity import (assert_mla_close, assert_sets_within_tolerance, kv_norm_max,
                             lse_atol, no_device_error)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import sparse_attention_long_02_b200 as d
    return d


def _host(t):
    return t.detach().cpu()


def _prefill_rows(dsa, cfg_id, rows, fused):
    """Every sampled row's selection against the oracle's (exact, or within the
    tie rule judged on the oracle's own scores; no row is exempt), and its
    attention on the GPU's selection against the oracle on that selection."""
    cfg = W.CONFIGS[cfg_id]
    inp = W.make_prefill(cfg, device="cuda")
    T, S, k = inp["T"], inp["S"], inp["k"]
    chunk = cfg.chunk or 4096
    run = dsa.forward_fused if fused else dsa.forward
    out, lse, idx = run(inp["q8"], inp["q_scale"], inp["k8"], inp["k_scale"], inp["w"],
                        inp["q"], inp["kv"], k, inp["scale"], inp["sm_scale"], chunk=chunk)
    no_device_error(dsa)
    k8, ks, kv = _host(inp["k8"]), _host(inp["k_scale"]), _host(inp["kv"])
    kn = kv_norm_max(kv)
    for r in rows:
        sub = dict(T=1, S=S, k=k, q_pos0=r, scale=inp["scale"], sm_scale=inp["sm_scale"],
                   q8=_host(inp["q8"][r:r + 1]), q_scale=_host(inp["q_scale"][r:r + 1]),
                   w=_host(inp["w"][r:r + 1]), q=_host(inp["q"][r:r + 1]), k8=k8, k_scale=ks,
                   kv=kv)
        ref = oracle.forward(sub)
        gidx = _host(idx[r:r + 1]).numpy()
        assert_sets_within_tolerance(gidx, ref["idx"], ref["I"], k)
        o, l = oracle.sparse_mla(sub["q"], kv, gidx, inp["sm_scale"])
        assert_mla_close(out[r:r + 1], o, lse[r:r + 1], l,
                         lse_atol(sub["q"], kn, inp["sm_scale"], l, k))
    del inp, out, lse, idx
    torch.cuda.empty_cache()


ROWS_128K = [0, 2046, 2047, 2048, 4095, 4096, 40961, 65537, 98303, 131071]
ROWS_16K = [0, 2047, 2048, 4095, 4096, 9000, 12287, 16383]


@pytest.mark.parametrize("fused", [True, False], ids=["fused", "scores_in_hbm"])
def test_prefill_128k_in_4096_row_chunks(dsa, fused):
    """Config 4 (L = 131072): rows at both ends, on chunk edges, at the k boundary."""
    _prefill_rows(dsa, 4, ROWS_128K, fused)


@pytest.mark.parametrize("fused", [True, False], ids=["fused", "scores_in_hbm"])
def test_prefill_16k(dsa, fused):
    """Config 2 (L = 16384, planted keys) in 4096-row chunks, as bench.py runs it."""
    _prefill_rows(dsa, 2, ROWS_16K, fused)


def _decode_seqs(dsa, inp, seqs):
    g = inp
    out, lse, idx = dsa.decode_paged(g["q8"], g["q_scale"], g["w"], g["q"], g["k8_pool"],
                                     g["k_scale_pool"], g["kv_pool"], g["block_table"],
                                     g["seq_len"], g["k"], g["scale"], g["sm_scale"])
    no_device_error(dsa)
    ref = oracle.decode(inp, seqs=seqs)
    kvp = _host(inp["kv_pool"])
    table = _host(inp["block_table"]).numpy()
    lens = _host(inp["seq_len"]).numpy()
    for i, b in enumerate(seqs):
        gidx = _host(idx[b]).numpy()
        assert_sets_within_tolerance(gidx, ref["idx"][i], ref["I"][i], g["k"])
        kv_seq = torch.from_numpy(
            oracle.gather_sequence(kvp.view(torch.int16).numpy(), table[b], int(lens[b]))
        ).view(torch.bfloat16)
        o, l = oracle.sparse_mla(_host(inp["q"][b]), kv_seq, gidx, g["sm_scale"])
        assert_mla_close(out[b], o, lse[b], l,
                         lse_atol(_host(inp["q"][b]), kv_seq, g["sm_scale"], l, g["k"]))


def test_decode_64_by_32k_paged(dsa):
    """Config 3 (B = 64 sequences of 32768 tokens, shuffled block table)."""
    inp = W.make_decode(W.CONFIGS[3], device="cuda")
    _decode_seqs(dsa, inp, [0, 31, 63])
    del inp
    torch.cuda.empty_cache()


def test_decode_variable_lengths_two_queries(dsa):
    """Config 5 (B = 128, log-uniform contexts, nq = 2): shortest, longest, a middle one."""
    inp = W.make_decode(W.CONFIGS[5], device="cuda")
    lens = _host(inp["seq_len"]).numpy()
    order = np.argsort(lens)
    seqs = sorted({int(order[0]), int(order[len(order) // 2]), int(order[-1])})
    _decode_seqs(dsa, inp, seqs)
    del inp
    torch.cuda.empty_cache()
