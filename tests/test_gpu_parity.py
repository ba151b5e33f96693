"""CUDA path vs the CPU oracle, element by element, through the C ABI.

Tolerances (from the path's definition):
  * indexer scores: |gpu - oracle| <= 1e-3 * max(|oracle|, A), A = sum_h |w| ReLU(.)
    (bit-exact on the integer FP8 grid, where every fp32 partial sum is exact);
  * top-k: identical sets on the grid; on random inputs a key may differ only
    if its oracle score is within 1e-3 * |tau| of the oracle's k-th score tau;
  * sparse MLA (bf16 in/out, fp32 accumulate): max-abs <= 2e-2 and
    mean-abs <= 2e-3 against the float64 oracle on identical selections;
  * lse: the bound lse_atol() derives from the kernel's fp32 arithmetic.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W

pytestmark = pytest.mark.gpu

MLA_MAX_ABS = 2e-2
MLA_MEAN_ABS = 2e-3
IDX_REL = 1e-3
U32 = 2.0 ** -24          # unit roundoff of fp32


def _gamma(n):
    """Worst-case relative error of an n-term fp32 sum in any order (Higham's gamma_n)."""
    return n * U32 / (1 - n * U32)


def _f64(x):
    return x.double().cpu().numpy() if isinstance(x, torch.Tensor) else np.asarray(x, np.float64)


def kv_norm_max(kv):
    """Largest Euclidean norm of a 576-wide cache row (bf16 tensor or array)."""
    if isinstance(kv, torch.Tensor):
        return float(kv.reshape(-1, 576).float().norm(dim=1).max())
    return float(np.linalg.norm(np.asarray(kv, np.float64).reshape(-1, 576), axis=-1).max())


def lse_atol(q, kv, sm_scale, ref_lse, k):
    """Largest |lse_gpu - lse_oracle| the kernel's arithmetic allows, per (row, head).

    The kernel forms each logit as two fp32 tensor-core sums over 288 dims
    (products of bf16 values are exact in fp32), adds the two halves in fp32
    and scales them into log2 units: |dz| <= sm_scale * gamma_580 * sum_d |q_d kv_d|
    <= sm_scale * gamma_580 * |q| * max_s |kv_s| (Cauchy-Schwarz; `kv` is the cache or
    that largest row norm, kv_norm_max), which moves lse
    by at most as much. The row sum l adds at most k exponentials in fp32
    (gamma_k relative), each exp2 and each re-base factor (at most one per
    64-key tile) adding at most 2^-20 relative. The result is formed and
    converted in fp32 (4 roundings of |lse|)."""
    qn = np.linalg.norm(_f64(q).reshape(*np.shape(ref_lse), 576), axis=-1)
    kn = kv if np.isscalar(kv) else kv_norm_max(kv)
    ntiles = -(-k // 64)
    return (sm_scale * _gamma(580) * qn * kn + _gamma(k) + (ntiles + 1) * 2.0 ** -20
            + 4 * U32 * np.abs(np.where(np.isfinite(ref_lse), ref_lse, 0.0)))


@pytest.fixture(scope="module")
def dsa():
    import sparse_attention_long_02_b200 as d
    return d


def cuda(inp):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}


def no_device_error(dsa):
    st = dsa.get_device_error()
    assert st == 0, dsa.STATUS.get(st, st)


def assert_mla_close(got, ref, lse=None, ref_lse=None, lse_tol=None):
    got = got.float().cpu().numpy().astype(np.float64)
    err = np.abs(got - ref)
    assert np.isfinite(got).all()
    assert err.max() <= MLA_MAX_ABS, err.max()
    assert err.mean() <= MLA_MEAN_ABS, err.mean()
    if lse is not None:
        assert lse_tol is not None, "an lse check needs its derived tolerance"
        l = lse.cpu().numpy().astype(np.float64)
        fin = np.isfinite(ref_lse)
        assert (np.isfinite(l) == fin).all()
        tol = np.broadcast_to(lse_tol, ref_lse.shape)
        bad = np.abs(l[fin] - ref_lse[fin]) > tol[fin]
        assert not bad.any(), (np.abs(l[fin] - ref_lse[fin])[bad][:5], tol[fin][bad][:5])


def assert_sets_within_tolerance(gpu_idx, ref_idx, ref_I, k):
    """Index sets agree except where the oracle score ties the k-th within 1e-3."""
    for r in range(ref_idx.shape[0]):
        g = set(int(x) for x in gpu_idx[r] if x >= 0)
        o = set(int(x) for x in ref_idx[r] if x >= 0)
        assert len(g) == len(o), r
        if g == o:
            continue
        row = ref_I[r]
        tau = min(row[i] for i in o)
        for i in g ^ o:
            assert abs(row[i] - tau) <= IDX_REL * abs(tau) + 1e-30, (r, i, row[i], tau)


# ------------------------------------------------------------ config 1 grid

@pytest.fixture(scope="module")
def cfg1():
    inp = W.make_prefill(W.CONFIGS[1])
    ref = oracle.forward(inp)
    return inp, ref


def test_indexer_bit_exact_on_grid(dsa, cfg1):
    inp, ref = cfg1
    g = cuda(inp)
    sc = dsa.indexer_scores(g["q8"], None, g["k8"], None, g["w"], inp["scale"])
    no_device_error(dsa)
    got = sc[:, : inp["S"]].cpu().numpy()
    vis = np.isfinite(ref["I"])
    assert np.array_equal(got[vis], ref["I"][vis])


def test_topk_bit_exact_on_grid(dsa, cfg1):
    inp, ref = cfg1
    scores = torch.from_numpy(ref["I"]).cuda()
    idx = dsa.topk(scores, inp["S"], inp["k"])
    no_device_error(dsa)
    exp = np.sort(np.where(ref["idx"] < 0, np.iinfo(np.int32).max, ref["idx"]), axis=1)
    exp = np.where(exp == np.iinfo(np.int32).max, -1, exp)
    assert np.array_equal(idx.cpu().numpy(), exp)


def test_sparse_mla_on_oracle_selection(dsa, cfg1):
    inp, ref = cfg1
    g = cuda(inp)
    out, lse = dsa.sparse_mla(g["q"], g["kv"], torch.from_numpy(ref["idx"]).cuda(), inp["sm_scale"])
    no_device_error(dsa)
    assert_mla_close(out, ref["out"], lse, ref["lse"],
                     lse_atol(inp["q"], inp["kv"], inp["sm_scale"], ref["lse"], inp["k"]))


def test_forward_end_to_end_on_grid(dsa, cfg1):
    inp, ref = cfg1
    g = cuda(inp)
    out, lse, idx = dsa.forward(g["q8"], None, g["k8"], None, g["w"], g["q"], g["kv"], inp["k"],
                                inp["scale"], inp["sm_scale"], chunk=300)
    no_device_error(dsa)
    got = idx.cpu().numpy()
    for r in range(inp["T"]):
        assert set(got[r][got[r] >= 0]) == set(ref["idx"][r][ref["idx"][r] >= 0]), r
    assert_mla_close(out, ref["out"], lse, ref["lse"],
                     lse_atol(inp["q"], inp["kv"], inp["sm_scale"], ref["lse"], inp["k"]))


@pytest.mark.parametrize("chunk", [300, 0])
def test_forward_fused_end_to_end_on_grid(dsa, cfg1, chunk):
    """The top-k fused into the indexer (no score rows in HBM): bit-exact
    selection on the exact grid, in chunks and in one piece."""
    inp, ref = cfg1
    g = cuda(inp)
    out, lse, idx = dsa.forward_fused(g["q8"], None, g["k8"], None, g["w"], g["q"], g["kv"],
                                      inp["k"], inp["scale"], inp["sm_scale"], chunk=chunk)
    no_device_error(dsa)
    got = idx.cpu().numpy()
    for r in range(inp["T"]):
        assert set(got[r][got[r] >= 0]) == set(ref["idx"][r][ref["idx"][r] >= 0]), r
    assert_mla_close(out, ref["out"], lse, ref["lse"],
                     lse_atol(inp["q"], inp["kv"], inp["sm_scale"], ref["lse"], inp["k"]))


@pytest.mark.parametrize("L,Hi,k,chunk", [(1500, 64, 256, 512), (6000, 64, 2048, 2048),
                                          (2000, 32, 512, 0)])
def test_forward_fused_on_grid_wide_heads(dsa, L, Hi, k, chunk):
    """The fused path with 32 and 64 indexer heads (the epilogue that gives
    each thread four key rows and each warp its own candidate lists) on the
    exact grid: every row's selection equals the chunked path's, and sampled
    rows equal the oracle's. At k = 2048 over 6000 keys the rows keep more
    candidates than a warp's shared-memory list holds, so appends also go
    straight to the global lists."""
    cfg = W.Config(92, "grid_wide", "prefill", k=k, Hi=Hi, H=8, seed=L + Hi, L=L, grid=True,
                   scale=1.0 / 16, sm_scale=1.0 / 24)
    inp = W.make_prefill(cfg)
    g = cuda(inp)
    out, lse, idx = dsa.forward_fused(g["q8"], None, g["k8"], None, g["w"], g["q"], g["kv"], k,
                                      inp["scale"], inp["sm_scale"], chunk=chunk)
    no_device_error(dsa)
    _, _, idx_ref = dsa.forward(g["q8"], None, g["k8"], None, g["w"], g["q"], g["kv"], k,
                                inp["scale"], inp["sm_scale"], chunk=chunk)
    no_device_error(dsa)
    got, exp = idx.cpu().numpy(), idx_ref.cpu().numpy()
    for r in range(L):
        assert set(got[r][got[r] >= 0]) == set(exp[r][exp[r] >= 0]), r
    rows = np.unique(np.clip(np.array([0, 1, k - 1, k, k + 1, L // 2, chunk - 1, chunk,
                                       L - 2, L - 1]), 0, L - 1))
    ref = oracle.forward(inp, rows=rows)
    for i, r in enumerate(rows):
        assert set(got[r][got[r] >= 0]) == set(ref["idx"][i][ref["idx"][i] >= 0]), r
    assert_mla_close(out[rows], ref["out"], lse[rows], ref["lse"],
                     lse_atol(inp["q"][rows], inp["kv"], inp["sm_scale"], ref["lse"], k))


def test_forward_fused_recomputes_rows_whose_threshold_misses(dsa):
    """Keys at the sampled positions (the first 256 of every 4096) hold each
    row's largest scores, all distinct from the rest, so the threshold taken
    from the sample lies above the k-th score, fewer than k candidates are
    kept, and the row's scores are recomputed on CUDA cores. Exact-grid
    integers keep every score exact: the selection must equal the oracle's."""
    rng = np.random.default_rng(61)
    L, Hi, H, k = 6000, 4, 8, 256
    pos = np.arange(L)
    sampled = (pos % 4096) < 256
    ones = np.where(sampled, rng.integers(32, 129, L), rng.integers(0, 17, L))
    kf = (np.arange(128)[None, :] < ones[:, None]).astype(np.float32)      # q.k = ones[s]
    k8 = torch.from_numpy(kf).to(torch.float8_e4m3fn).view(torch.uint8)
    q8 = torch.ones(L, Hi, 128).to(torch.float8_e4m3fn).view(torch.uint8)
    w = torch.full((L, Hi), 0.25)
    q = torch.from_numpy(rng.normal(size=(L, H, 576))).to(torch.bfloat16)
    kv = torch.from_numpy(rng.normal(size=(L, 576))).to(torch.bfloat16)
    inp = dict(q8=q8, q_scale=None, k8=k8, k_scale=None, w=w, q=q, kv=kv, scale=1 / 16,
               sm_scale=1 / 24, k=k, q_pos0=0, T=L, S=L, Hi=Hi, H=H)
    g = cuda(inp)
    out, lse, idx = dsa.forward_fused(g["q8"], None, g["k8"], None, g["w"], g["q"], g["kv"], k,
                                      inp["scale"], inp["sm_scale"], chunk=2048)
    no_device_error(dsa)
    _, _, idx_ref = dsa.forward(g["q8"], None, g["k8"], None, g["w"], g["q"], g["kv"], k,
                                inp["scale"], inp["sm_scale"], chunk=2048)
    got, exp = idx.cpu().numpy(), idx_ref.cpu().numpy()
    for r in range(L):                   # the chunked path, bit-exact on this grid
        assert set(got[r][got[r] >= 0]) == set(exp[r][exp[r] >= 0]), r
    rows = np.array([0, 255, 256, 1500, 2047, 4095, 4096, 4400, 5999])
    ref = oracle.forward(inp, rows=rows)
    for i, r in enumerate(rows):
        assert set(got[r][got[r] >= 0]) == set(ref["idx"][i][ref["idx"][i] >= 0]), r
    assert_mla_close(out[rows], ref["out"], lse[rows], ref["lse"],
                     lse_atol(q[rows], kv, inp["sm_scale"], ref["lse"], k))


@pytest.mark.parametrize("gain", [1.0, 40.0, 1e3, 4e3, 4e4])
def test_mla_large_and_peaked_logits(dsa, gain):
    """Logits far from the N(0,1) range, against the float64 oracle.

    q is scaled by `gain`, so raw q.kv products reach about 24 * gain (1e3 to
    1e6 over the gains); in the even rows every head of q is `gain` times one
    selected key's row, so that key's logit stands ~gain * 576 above the rest
    (a one-hot softmax whose raw logit passes 1e7). The two CTAs of a query
    each hold a partial logit over half the dims; these partials cover the
    range where a 16-bit float would lose all resolution (gain 1e3) and
    overflow (gain 4e3 and above, peaked rows). Odd rows keep fewer than k
    keys and a ragged last tile."""
    rng = np.random.default_rng(int(gain) + 11)
    T, S, H, k = 6, 3000, 128, 2048
    kv = torch.from_numpy(rng.normal(size=(S, 576))).to(torch.bfloat16)
    qf = rng.normal(size=(T, H, 576)) * gain
    idx = np.full((T, k), -1, np.int32)
    for t in range(T):
        n = k if t % 2 == 0 else 2048 - 37 * t
        idx[t, :n] = rng.choice(S, n, replace=False)
        if t % 2 == 0:
            star = idx[t, rng.integers(0, n)]
            qf[t] = gain * kv[star].double().numpy()[None, :] + rng.normal(size=(H, 576))
    q = torch.from_numpy(qf).to(torch.bfloat16)
    out, lse = dsa.sparse_mla(q.cuda(), kv.cuda(), torch.from_numpy(idx).cuda(), 1 / 24)
    no_device_error(dsa)
    ref, ref_lse = oracle.sparse_mla(q, kv, idx, 1 / 24)
    assert_mla_close(out, ref, lse, ref_lse, lse_atol(q, kv, 1 / 24, ref_lse, k))


# ------------------------------------------------------ random FP8 inputs

def _random_prefill(L, Hi, H, k, seed, plant=True):
    cfg = W.Config(90, "random", "prefill", k=k, Hi=Hi, H=H, seed=seed, L=L,
                   plant_block=256 if plant else 0, plant_n=16)
    return W.make_prefill(cfg)


@pytest.mark.parametrize("L,Hi,H,k,rows", [
    (2500, 64, 128, 2048, [0, 1, 777, 2046, 2047, 2048, 2049, 2300, 2499]),
    (1111, 4, 8, 256, [0, 255, 256, 600, 1110]),
    (700, 1, 1, 64, [0, 63, 64, 65, 699]),
    (300, 32, 16, 512, [0, 150, 299]),
])
def test_random_prefill_stages(dsa, L, Hi, H, k, rows):
    inp = _random_prefill(L, Hi, H, k, seed=L + Hi)
    g = cuda(inp)
    rows = np.array(rows)
    sc = dsa.indexer_scores(g["q8"], g["q_scale"], g["k8"], g["k_scale"], g["w"], inp["scale"])
    out, lse, idx = dsa.forward(g["q8"], g["q_scale"], g["k8"], g["k_scale"], g["w"], g["q"],
                                g["kv"], k, inp["scale"], inp["sm_scale"])
    no_device_error(dsa)
    I, A = oracle.indexer(inp["q8"], inp["q_scale"], inp["k8"], inp["k_scale"], inp["w"],
                          inp["scale"], rows=rows, with_mag=True)
    got = sc[rows, :L].cpu().numpy()
    vis = np.isfinite(I)
    tol = IDX_REL * np.maximum(np.abs(I), A)
    assert (np.abs(got[vis] - I[vis]) <= tol[vis] + 1e-30).all()
    ref_idx = oracle.topk(I, oracle.prefill_row_len(L, L, 0, rows), k)
    gidx = idx[rows].cpu().numpy()
    assert_sets_within_tolerance(gidx, ref_idx, I, k)
    # attention on the GPU's own selection, oracle fed the identical selection
    full_idx = np.full((L, k), -1, np.int32)
    full_idx[rows] = gidx
    ref_out, ref_lse = oracle.sparse_mla(inp["q"], inp["kv"], full_idx, inp["sm_scale"], rows=rows)
    assert_mla_close(out[rows], ref_out, lse[rows], ref_lse,
                     lse_atol(inp["q"][rows], inp["kv"], inp["sm_scale"], ref_lse, k))


def test_indexer_offset_chunk_and_ragged_edges(dsa):
    """Query rows at an offset into the cache; S not a multiple of 128."""
    inp = _random_prefill(777, 64, 8, 128, seed=5, plant=False)
    g = cuda(inp)
    T0, T = 300, 213                       # rows 300..512 as a chunk
    sc = dsa.indexer_scores(g["q8"][T0:T0 + T].contiguous(), g["q_scale"][T0:T0 + T].contiguous(),
                            g["k8"], g["k_scale"], g["w"][T0:T0 + T].contiguous(), inp["scale"],
                            q_pos0=T0)
    no_device_error(dsa)
    rows = np.array([0, 1, 100, 212])
    I, A = oracle.indexer(inp["q8"][T0:T0 + T], inp["q_scale"][T0:T0 + T], inp["k8"],
                          inp["k_scale"], inp["w"][T0:T0 + T], inp["scale"], q_pos0=T0,
                          rows=rows, with_mag=True)
    got = sc[rows, :777].cpu().numpy()
    vis = np.isfinite(I)
    assert (np.abs(got[vis] - I[vis]) <= IDX_REL * np.maximum(np.abs(I), A)[vis] + 1e-30).all()


def test_mla_short_rows_single_key_and_all_padding(dsa):
    rng = np.random.default_rng(3)
    T, S, H, k = 5, 97, 8, 16
    q = torch.from_numpy(rng.normal(size=(T, H, 576))).to(torch.bfloat16)
    kv = torch.from_numpy(rng.normal(size=(S, 576))).to(torch.bfloat16)
    idx = np.full((T, k), -1, np.int32)
    idx[0, 0] = 96                         # one key: output is that row exactly
    idx[1, :16] = rng.choice(S, 16, replace=False)
    idx[2, :3] = [5, 6, 7]
    # row 3: no key at all -> zeros, lse = -inf
    idx[4, :7] = rng.choice(S, 7, replace=False)
    out, lse = dsa.sparse_mla(q.cuda(), kv.cuda(), torch.from_numpy(idx).cuda(), 1 / 24)
    no_device_error(dsa)
    ref, ref_lse = oracle.sparse_mla(q, kv, idx, 1 / 24)
    assert torch.equal(out[0].cpu(), kv[96, :512].expand(H, 512))
    assert (out[3].float().cpu() == 0).all() and torch.isneginf(lse[3].cpu()).all()
    assert_mla_close(out, ref, lse, ref_lse, lse_atol(q, kv, 1 / 24, ref_lse, k))


def test_unselected_nan_rows_never_read(dsa):
    """Poisoning every key outside the selection leaves the output bit-identical."""
    rng = np.random.default_rng(4)
    T, S, H, k = 9, 400, 128, 128
    q = torch.from_numpy(rng.normal(size=(T, H, 576))).to(torch.bfloat16).cuda()
    kv = torch.from_numpy(rng.normal(size=(S, 576))).to(torch.bfloat16).cuda()
    idx = torch.from_numpy(np.stack([rng.choice(S, k, replace=False) for _ in range(T)])
                           .astype(np.int32)).cuda()
    out, lse = dsa.sparse_mla(q, kv, idx, 1 / 24)
    poisoned = kv.clone()
    keep = torch.zeros(S, dtype=torch.bool, device="cuda")
    keep[idx.flatten().long()] = True
    poisoned[~keep] = float("nan")
    out2, lse2 = dsa.sparse_mla(q, poisoned, idx, 1 / 24)
    no_device_error(dsa)
    assert torch.equal(out, out2) and torch.equal(lse, lse2)


def test_out_of_range_index_is_reported_and_skipped(dsa):
    rng = np.random.default_rng(5)
    T, S, H, k = 2, 64, 8, 8
    q = torch.from_numpy(rng.normal(size=(T, H, 576))).to(torch.bfloat16).cuda()
    kv = torch.from_numpy(rng.normal(size=(S, 576))).to(torch.bfloat16).cuda()
    idx = torch.tensor([[1, 2, 3, 999, -1, -1, -1, -1], [4, 5, -7, 6, -1, -1, -1, -1]],
                       dtype=torch.int32).cuda()
    out, _ = dsa.sparse_mla(q, kv, idx, 1 / 24)
    st = dsa.get_device_error()
    assert st == -6, st                              # DSA_ERR_DEVICE_BOUNDS
    assert torch.isfinite(out.float()).all()
    clean = torch.tensor([[1, 2, 3, -1, -1, -1, -1, -1], [4, 5, 6, -1, -1, -1, -1, -1]],
                         dtype=torch.int32).cuda()
    out2, _ = dsa.sparse_mla(q, kv, clean, 1 / 24)
    no_device_error(dsa)
    # the -7 entry is simply skipped (slot order does not matter up to rounding)
    assert (out[0] == out2[0]).all()
    assert (out[1].float() - out2[1].float()).abs().max() < 1e-2


# ------------------------------------------------------------ paged decode

def _small_decode(lens, nq, seed, Hi=64, H=128, k=2048):
    cfg = W.Config(91, "decode_test", "decode", k=k, Hi=Hi, H=H, seed=seed, nq=nq,
                   ctx_lo=1, ctx_hi=2)
    return W.make_decode(cfg, lens=torch.tensor(lens))


@pytest.mark.parametrize("lens,nq,Hi", [([100, 2048, 2049, 2050, 5000, 9000], 2, 64),
                                        ([64, 65, 4097, 3000], 1, 64),
                                        ([300, 2100, 4500], 2, 32),
                                        ([700, 2200, 2051], 3, 64),
                                        ([2300, 5000], 4, 64)])
def test_decode_paged_vs_oracle(dsa, lens, nq, Hi):
    inp = _small_decode(lens, nq, seed=len(lens) + nq, Hi=Hi)
    g = cuda(inp)
    out, lse, idx = dsa.decode_paged(g["q8"], g["q_scale"], g["w"], g["q"], g["k8_pool"],
                                     g["k_scale_pool"], g["kv_pool"], g["block_table"],
                                     g["seq_len"], inp["k"], inp["scale"], inp["sm_scale"])
    no_device_error(dsa)
    ref = oracle.decode(inp)
    gidx = idx.cpu().numpy()
    for b in range(inp["B"]):
        assert_sets_within_tolerance(gidx[b], ref["idx"][b], ref["I"][b], inp["k"])
    # MLA on the oracle's selection through the paged stage entry point
    o2, l2 = dsa.sparse_mla_decode_paged(g["q"], g["kv_pool"], g["block_table"], g["seq_len"],
                                         torch.from_numpy(ref["idx"]).cuda(), inp["sm_scale"])
    no_device_error(dsa)
    tol = lse_atol(inp["q"], inp["kv_pool"], inp["sm_scale"], ref["lse"], inp["k"])
    assert_mla_close(o2, ref["out"], l2, ref["lse"], tol)
    same = [b for b in range(inp["B"])
            if all(set(gidx[b, j]) == set(ref["idx"][b, j]) for j in range(nq))]
    assert same
    assert_mla_close(out[same], ref["out"][same], lse[same], ref["lse"][same], tol[same])


@pytest.mark.parametrize("kind,n,k", [("random", 20000, 2048), ("ties", 20000, 2048),
                                      ("constant", 9000, 1024), ("random", 12000, 5000),
                                      ("ties", 3000, 256), ("sample_high", 20000, 2048),
                                      ("random", 131072, 2048), ("random", 70001, 2048),
                                      ("random", 8192, 2048), ("planted", 65536, 2048)])
def test_topk_fast_and_general_paths(dsa, kind, n, k):
    """Every selection path against the oracle's full sort:
    - random, planted, periodically boosted, full-length (131072) and
      ragged rows take the in-shared-memory path (their k-th bucket is small);
    - rows whose k-th bucket is crowded (heavy ties, constant rows) and
      k > 4096 take the general path."""
    rng = np.random.default_rng(n + k)
    R = 6
    if kind in ("random", "sample_high", "planted"):
        I = rng.normal(size=(R, n)).astype(np.float32)
        if kind == "sample_high":
            I[:, (np.arange(n) % 4096) < 256] += 10.0
        if kind == "planted":
            for r in range(R):
                I[r, rng.choice(n, 300, replace=False)] += 8.0
    elif kind == "ties":
        I = (rng.integers(-3, 4, size=(R, n)) / 8.0).astype(np.float32)
    else:
        I = np.full((R, n), 0.5, np.float32)
    q_pos0 = n - R                       # rows see n-R+1 .. n keys
    ld = (n + 3) // 4 * 4                # row stride: a multiple of 4 (ragged n pads it)
    Ig = np.zeros((R, ld), np.float32)
    Ig[:, :n] = I
    idx = dsa.topk(torch.from_numpy(Ig).cuda(), n, k, q_pos0=q_pos0)
    no_device_error(dsa)
    ref = oracle.topk(I, oracle.prefill_row_len(R, n, q_pos0), k)
    exp = np.sort(np.where(ref < 0, np.iinfo(np.int32).max, ref), axis=1)
    exp = np.where(exp == np.iinfo(np.int32).max, -1, exp)
    assert np.array_equal(idx.cpu().numpy(), exp)


# ------------------------------------------- sliding window / dense causal

@pytest.mark.parametrize("T,S,q_pos0,window,k", [(37, 37, 0, 1, 4), (300, 300, 0, 64, 64),
                                                 (50, 400, 333, 128, 132), (20, 100, 90, 16, 16),
                                                 (129, 129, 0, 129, 132)])
def test_window_indices_bit_exact(dsa, T, S, q_pos0, window, k):
    got = dsa.window_indices(T, S, window, k, q_pos0=q_pos0)
    no_device_error(dsa)
    ref = oracle.window(T, S, window, k, q_pos0=q_pos0)
    assert torch.equal(got.cpu(), torch.from_numpy(ref))


@pytest.mark.parametrize("window,k", [(96, 96), (300, 300)])
def test_sliding_window_and_dense_causal_mla(dsa, window, k):
    """The sparse MLA over window index sets: sliding-window attention (a
    window shorter than the rows) and dense causal attention (a window
    covering every prefix), against the oracle on sampled rows."""
    rng = np.random.default_rng(7)
    T, H = 300, 128
    q = torch.from_numpy(rng.normal(size=(T, H, 576))).to(torch.bfloat16)
    kv = torch.from_numpy(rng.normal(size=(T, 576))).to(torch.bfloat16)
    idx = dsa.window_indices(T, T, window, k)
    out, lse = dsa.sparse_mla(q.cuda(), kv.cuda(), idx, 1 / 24)
    no_device_error(dsa)
    rows = [0, 1, 63, 64, 95, 96, 97, 150, 255, 299]
    ref, ref_lse = oracle.sparse_mla(q, kv, oracle.window(T, T, window, k), 1 / 24, rows=rows)
    assert_mla_close(out[rows], ref, lse[rows], ref_lse, lse_atol(q[rows], kv, 1 / 24, ref_lse, k))


@pytest.mark.parametrize("T,S,q_pos0,H", [(300, 300, 0, 128), (100, 400, 300, 8), (70, 650, 580, 16)])
def test_dense_causal_mla_range_mode(dsa, T, S, q_pos0, H):
    """Dense causal attention with the slots generated in the kernel (no index
    sets): against the oracle's sparse MLA over every key of each row's causal
    prefix, on rows spanning several tiles, a ragged last tile and an offset."""
    rng = np.random.default_rng(T + S + H)
    q = torch.from_numpy(rng.normal(size=(T, H, 576))).to(torch.bfloat16)
    kv = torch.from_numpy(rng.normal(size=(S, 576))).to(torch.bfloat16)
    out, lse = dsa.dense_causal_mla(q.cuda(), kv.cuda(), 1 / 24, q_pos0=q_pos0)
    no_device_error(dsa)
    k = (S + 3) // 4 * 4
    rows = sorted({0, 1, 63, 64, T // 2, T - 1})
    ref, ref_lse = oracle.sparse_mla(q, kv, oracle.window(T, S, S, k, q_pos0=q_pos0), 1 / 24,
                                     rows=rows)
    assert_mla_close(out[rows], ref, lse[rows], ref_lse, lse_atol(q[rows], kv, 1 / 24, ref_lse, k))


def test_dense_causal_mla_decode_paged_range_mode(dsa):
    """The paged decode's dense attention: every key of each query's causal
    prefix through the block table, against the oracle on the gathered sequence."""
    inp = _small_decode([100, 2049, 5000, 64], 2, seed=12, H=128)
    g = cuda(inp)
    out, lse = dsa.dense_causal_mla_decode_paged(g["q"], g["kv_pool"], g["block_table"],
                                                 g["seq_len"], inp["sm_scale"])
    no_device_error(dsa)
    kvp, table, lens = inp["kv_pool"], inp["block_table"].numpy(), inp["seq_len"].numpy()
    for b in range(inp["B"]):
        n = int(lens[b])
        kv_seq = torch.from_numpy(
            oracle.gather_sequence(kvp.view(torch.int16).numpy(), table[b], n)).view(torch.bfloat16)
        k = (n + 3) // 4 * 4
        idx = oracle.window(2, n, n, k, q_pos0=n - 2)
        ref, ref_lse = oracle.sparse_mla(inp["q"][b], kv_seq, idx, inp["sm_scale"])
        assert_mla_close(out[b], ref, lse[b], ref_lse,
                         lse_atol(inp["q"][b], kv_seq, inp["sm_scale"], ref_lse, k))


# ------------------------------------------------ projection (workflow step 1)

@pytest.mark.parametrize("T,d,Hi", [(300, 200, 64), (129, 64, 4), (5, 8, 1)])
def test_projection_vs_oracle(dsa, T, d, Hi):
    """The GEMM + rotation against the float64 oracle; the FP8 encoding of the
    kernel's own fp32 values against torch's e4m3 cast (same precision, so the
    codes and scales must be identical)."""
    inp = W.make_projection(T, d, Hi, seed=T + d + Hi)
    need = dsa.lib().dsa_project_workspace_size(T, Hi)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    q8, q_scale, k8, k_scale, a = dsa.project_indexer_inputs(
        inp["h"].cuda(), inp["wt"].cuda(), inp["rope"].cuda(), Hi, workspace=ws)
    no_device_error(dsa)
    nq, nqk = Hi * 128, Hi * 128 + 128
    y = ws[: T * nqk * 4].view(torch.float32).view(T, nqk).cpu()      # rotated q | k, fp32
    ref = oracle.project(inp["h"], inp["wt"], inp["rope"], Hi)
    np.testing.assert_allclose(y.double().numpy(), ref[:, :nqk], rtol=1e-4, atol=1e-4)
    np.testing.assert_allclose(a.cpu().double().numpy(), ref[:, nqk:], rtol=1e-4, atol=1e-4)
    for part, codes, scale in ((y[:, :nq], q8.view(T, nq), q_scale), (y[:, nq:], k8, k_scale)):
        amax = part.abs().amax(dim=1)
        s = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
        assert torch.equal(scale.cpu(), s)
        want = (part / s.unsqueeze(1)).clamp(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8)
        assert torch.equal(codes.cpu(), want)


# ------------------------------------------------- indexer warm-up objective

def test_warmup_target_kl_and_backward(dsa):
    """The warm-up objective end to end on one small prefill:
    - target: per-head lse from the sparse MLA over dense window indices, then
      the head-mean attention weights;
    - KL and its gradient on the indexer scores;
    - backward to the dequantised indexer inputs.
    Each is checked against the oracle on the GPU's own inputs."""
    rng = np.random.default_rng(51)
    T, H, Hi, scale = 150, 8, 4, 1 / 16
    q = torch.from_numpy(rng.normal(size=(T, H, 576))).to(torch.bfloat16)
    kv = torch.from_numpy(rng.normal(size=(T, 576))).to(torch.bfloat16)
    k = (T + 3) // 4 * 4
    idx = dsa.window_indices(T, T, T, k)
    _, lse = dsa.sparse_mla(q.cuda(), kv.cuda(), idx, 1 / 24)
    p = dsa.attention_probs_mean(q.cuda(), kv.cuda(), lse, 1 / 24)
    no_device_error(dsa)
    p_ref = oracle.attention_probs(q, kv, 1 / 24)
    # each term exp(sm_scale z - lse) carries the logit's and the lse's fp32 error, each
    # within the bound lse_atol derives, as a relative error of the probability
    l_h = lse.cpu().double().numpy()
    rtol = 2 * lse_atol(q, kv, 1 / 24, l_h, k).max() + 1e-5
    np.testing.assert_allclose(p.cpu().numpy(), p_ref, rtol=rtol, atol=1e-7)
    # KL on indexer scores from FP8 inputs
    q8 = torch.from_numpy(rng.integers(-8, 9, size=(T, Hi, 128))).float().to(
        torch.float8_e4m3fn).view(torch.uint8)
    k8 = torch.from_numpy(rng.integers(-8, 9, size=(T, 128))).float().to(
        torch.float8_e4m3fn).view(torch.uint8)
    q_scale = torch.from_numpy(rng.uniform(0.01, 0.02, T)).float()
    k_scale = torch.from_numpy(rng.uniform(0.01, 0.02, T)).float()
    w = torch.from_numpy(rng.normal(size=(T, Hi)) / 8).float()
    I = dsa.indexer_scores(q8.cuda(), q_scale.cuda(), k8.cuda(), k_scale.cuda(), w.cuda(), scale)
    p_used = p.cpu().double().numpy()
    loss, grad = dsa.indexer_kl(I, p, T)
    no_device_error(dsa)
    n = np.arange(1, T + 1)
    I_h = I.cpu().double().numpy()[:, :T]
    I_h = np.where(np.isfinite(I_h), I_h, 0.0)
    l_ref, g_ref = oracle.indexer_kl(I_h, p_used, n)
    np.testing.assert_allclose(loss.cpu().numpy(), l_ref, rtol=1e-4, atol=1e-6)
    np.testing.assert_allclose(grad.cpu().numpy()[:, :T], g_ref, rtol=1e-4, atol=1e-6)
    # backward on the GPU's own gradient
    dq, dk, dw = dsa.indexer_backward(q8.cuda(), q_scale.cuda(), k8.cuda(), k_scale.cuda(),
                                      w.cuda(), scale, grad)
    no_device_error(dsa)
    dq_r, dk_r, dw_r = oracle.indexer_backward(q8, q_scale, k8, k_scale, w, scale,
                                               grad.cpu().double().numpy())
    for got, ref in ((dq, dq_r), (dk, dk_r), (dw, dw_r)):
        mag = np.abs(ref).max()
        np.testing.assert_allclose(got.cpu().double().numpy(), ref, rtol=0, atol=1e-4 * mag)


@pytest.mark.parametrize("T,S,q_pos0,Hi", [(37, 300, 263, 64), (64, 64, 0, 1), (40, 300, 0, 8),
                                           (150, 1000, 850, 16)])
def test_warmup_backward_offset_rows(dsa, T, S, q_pos0, Hi):
    """Backward for a chunk of rows at an offset (keys 0 .. q_pos0 + t), for one head, and
    for keys no row sees (S past the last row's position): several GEMM tiles, split-K
    steps and a ragged tail in each product."""
    rng = np.random.default_rng(T + S + Hi)
    q8 = torch.from_numpy(rng.integers(-8, 9, size=(T, Hi, 128))).float().to(
        torch.float8_e4m3fn).view(torch.uint8)
    k8 = torch.from_numpy(rng.integers(-8, 9, size=(S, 128))).float().to(
        torch.float8_e4m3fn).view(torch.uint8)
    w = torch.from_numpy(rng.normal(size=(T, Hi))).float()
    ld = (S + 3) // 4 * 4
    g = torch.from_numpy(rng.normal(size=(T, ld))).float()
    dq, dk, dw = dsa.indexer_backward(q8.cuda(), None, k8.cuda(), None, w.cuda(), 0.5, g.cuda(),
                                      q_pos0=q_pos0)
    no_device_error(dsa)
    dq_r, dk_r, dw_r = oracle.indexer_backward(q8, None, k8, None, w, 0.5, g.double().numpy(),
                                               q_pos0=q_pos0)
    for got, ref in ((dq, dq_r), (dk, dk_r), (dw, dw_r)):
        mag = np.abs(ref).max()
        np.testing.assert_allclose(got.cpu().double().numpy(), ref, rtol=0, atol=1e-5 * mag)
