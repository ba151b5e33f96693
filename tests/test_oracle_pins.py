"""Pins for the CPU oracle: each check ties it to something other than itself.

What pins what:
  * e4m3 / bf16 decoding: every code against torch's own dtype conversion.
  * indexer: with one head, w = 1 it must equal ReLU(scale * q.k^T) computed
    by a library matmul (the reduction stated in the path's definition);
    one-hot and negated head weights, positive homogeneity in the scales and
    head permutation then fix how heads, weights and scales enter; the
    causal boundary is checked at an offset.
  * top-k: equals a brute-force full sort (numpy lexsort) on tiny rows with
    many ties; the short-context fallback selects every key.
  * sparse MLA: when every causal key is selected it must equal dense causal
    softmax attention from torch's scaled_dot_product_attention in float64;
    a single selected row returns that row's latent exactly; the selection
    order does not matter and unselected rows (even NaN) have no effect.
  * paged decode: equals the contiguous path on the same logical sequence,
    and a permutation of the physical blocks changes nothing.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W


def e4m3_codes(rng, shape, lo=-8, hi=8):
    v = torch.from_numpy(rng.integers(lo, hi + 1, size=shape)).float()
    return v.to(torch.float8_e4m3fn).view(torch.uint8)


def e4m3_random(rng, shape):
    """Arbitrary finite e4m3 codes (not only integers)."""
    codes = rng.integers(0, 256, size=shape).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x3C      # replace NaN codes by 1.5
    return torch.from_numpy(codes)


def lib_float(codes_u8):
    return codes_u8.view(torch.float8_e4m3fn).double()


# ----------------------------------------------------------------- decoding

def test_e4m3_every_code_matches_torch():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double()
    for c in range(256):
        got = oracle.e4m3(c)
        if np.isnan(ref[c].item()):
            assert np.isnan(got), c
        else:
            assert got == ref[c].item(), (c, got, ref[c].item())


def test_bf16_decode_matches_torch():
    rng = np.random.default_rng(7)
    bits = rng.integers(0, 1 << 16, size=4096).astype(np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    got = np.array([oracle.bf16(int(b)) for b in bits])
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all()


# ------------------------------------------------------------------ indexer

def _single_head_library(q_f, k_f, scale, q_pos0):
    """ReLU(scale * q.k^T) with the causal mask, via a library matmul."""
    x = scale * (q_f @ k_f.T)
    T, S = x.shape
    pos = q_pos0 + torch.arange(T).unsqueeze(1)
    x = torch.clamp(x, min=0.0)
    return torch.where(torch.arange(S).unsqueeze(0) <= pos, x, torch.tensor(-np.inf, dtype=x.dtype))


@pytest.mark.parametrize("grid", [True, False])
def test_indexer_one_head_unit_weight_is_relu_qk(grid):
    rng = np.random.default_rng(1)
    T, S = 37, 53
    mk = e4m3_codes if grid else e4m3_random
    q8 = mk(rng, (T, 1, 128))
    k8 = mk(rng, (S, 128))
    w = torch.ones(T, 1)
    scale, q_pos0 = 0.3125, 11
    got = oracle.indexer(q8, None, k8, None, w, scale, q_pos0)
    ref = _single_head_library(lib_float(q8[:, 0]), lib_float(k8), scale, q_pos0)
    ref32 = ref.float().numpy()
    fin = np.isfinite(ref32)
    assert (np.isfinite(got) == fin).all()
    if grid:
        assert (got[fin] == ref32[fin]).all()
    else:
        np.testing.assert_allclose(got[fin], ref32[fin], rtol=2e-7, atol=0)


def test_indexer_head_weights_and_sign():
    """One-hot (+1 and -1) weights pick one head's ReLU score, with its sign."""
    rng = np.random.default_rng(2)
    T, S, Hi = 19, 40, 4
    q8 = e4m3_codes(rng, (T, Hi, 128))
    k8 = e4m3_codes(rng, (S, 128))
    scale = 1.0 / 16
    for h in range(Hi):
        for sign in (1.0, -1.0):
            w = torch.zeros(T, Hi)
            w[:, h] = sign
            got = oracle.indexer(q8, None, k8, None, w, scale)
            ref = sign * _single_head_library(lib_float(q8[:, h]), lib_float(k8), scale, 0)
            ref = torch.where(torch.isfinite(ref), ref, torch.tensor(-np.inf, dtype=ref.dtype))
            ref32 = ref.float().numpy()
            fin = np.isfinite(ref32)
            assert (np.isfinite(got) == fin).all()
            assert (got[fin] == ref32[fin]).all(), (h, sign)


def test_indexer_linear_in_weights_and_head_permutation():
    rng = np.random.default_rng(3)
    T, S, Hi = 23, 31, 4
    q8 = e4m3_codes(rng, (T, Hi, 128))
    k8 = e4m3_codes(rng, (S, 128))
    w1 = torch.from_numpy(rng.integers(-4, 5, size=(T, Hi)) / 4.0).float()
    w2 = torch.from_numpy(rng.integers(-4, 5, size=(T, Hi)) / 4.0).float()
    I1 = oracle.indexer(q8, None, k8, None, w1, 1 / 16)
    I2 = oracle.indexer(q8, None, k8, None, w2, 1 / 16)
    I12 = oracle.indexer(q8, None, k8, None, w1 + w2, 1 / 16)
    fin = np.isfinite(I12)
    assert (I1[fin] + I2[fin] == I12[fin]).all()       # exact on the grid
    perm = torch.from_numpy(rng.permutation(Hi))
    Ip = oracle.indexer(q8[:, perm].contiguous(), None, k8, None, w1[:, perm].contiguous(), 1 / 16)
    assert np.array_equal(Ip, I1)


def test_indexer_positive_homogeneity_in_scales():
    """I scales by q_scale[t] * k_scale[s] * scale (all > 0): ReLU commutes with them."""
    rng = np.random.default_rng(4)
    T, S, Hi = 17, 29, 3
    q8 = e4m3_random(rng, (T, Hi, 128))
    k8 = e4m3_random(rng, (S, 128))
    w = torch.from_numpy(rng.normal(size=(T, Hi))).float()
    qs = torch.from_numpy(rng.uniform(0.01, 3.0, size=T)).float()
    ks = torch.from_numpy(rng.uniform(0.01, 3.0, size=S)).float()
    base = oracle.indexer(q8, None, k8, None, w, 1.0)
    got = oracle.indexer(q8, qs, k8, ks, w, 0.125)
    ref = base.astype(np.float64) * qs.double().numpy()[:, None] * ks.double().numpy()[None, :] * 0.125
    fin = np.isfinite(base)
    assert (np.isfinite(got) == fin).all()
    np.testing.assert_allclose(got[fin], ref[fin], rtol=1e-6, atol=1e-30)


def test_indexer_causal_boundary_and_row_subset():
    rng = np.random.default_rng(5)
    T, S, Hi = 8, 20, 2
    q8 = e4m3_codes(rng, (T, Hi, 128))
    k8 = e4m3_codes(rng, (S, 128))
    w = torch.ones(T, Hi)
    q_pos0 = 9
    I = oracle.indexer(q8, None, k8, None, w, 1 / 16, q_pos0)
    for t in range(T):
        p = q_pos0 + t
        assert np.isfinite(I[t, : min(p + 1, S)]).all()
        assert np.isneginf(I[t, p + 1:]).all()
    rows = np.array([6, 1, 3])
    Ir = oracle.indexer(q8, None, k8, None, w, 1 / 16, q_pos0, rows=rows)
    assert np.array_equal(Ir, I[rows])


# -------------------------------------------------------------------- top-k

def brute_topk(row, n, k):
    if n <= k:
        return np.concatenate([np.arange(n), -np.ones(k - n, np.int64)])
    s = np.arange(n)
    order = np.lexsort((s, -row[:n].astype(np.float64)))
    return order[:k]


def test_topk_equals_full_sort_with_ties():
    rng = np.random.default_rng(6)
    R, ld, k = 40, 300, 17
    I = rng.integers(-6, 7, size=(R, ld)).astype(np.float32)   # many ties
    I[:5] = rng.normal(size=(5, ld)).astype(np.float32)
    n = rng.integers(1, ld + 1, size=R)
    n[:3] = [1, k, k + 1]
    got = oracle.topk(I, n, k)
    for r in range(R):
        assert np.array_equal(got[r], brute_topk(I[r], n[r], k)), r


def test_topk_short_context_takes_every_key_and_scale_invariance():
    rng = np.random.default_rng(8)
    I = rng.normal(size=(6, 64)).astype(np.float32)
    n = np.array([1, 5, 32, 33, 64, 2])
    got = oracle.topk(I, n, 32)
    for r in range(6):
        if n[r] <= 32:
            assert list(got[r, : n[r]]) == list(range(n[r]))
            assert (got[r, n[r]:] == -1).all()
    scaled = oracle.topk(I * np.float32(4.0), n, 32)     # power of two: exact
    assert np.array_equal(scaled, got)


# --------------------------------------------------------------- sparse MLA

def _bf16(rng, shape):
    return torch.from_numpy(rng.normal(size=shape)).to(torch.bfloat16)


def dense_causal_sdpa(q, kv, sm_scale):
    """Library dense causal attention in float64: K = kv (576), V = kv[:, :512]."""
    T, H, _ = q.shape
    qd = q.double().permute(1, 0, 2)                         # [H][T][576]
    kd = kv.double().unsqueeze(0).expand(H, -1, -1)
    vd = kv[:, :512].double().unsqueeze(0).expand(H, -1, -1)
    o = torch.nn.functional.scaled_dot_product_attention(qd, kd, vd, is_causal=True, scale=sm_scale)
    logits = (qd @ kd.transpose(1, 2)) * sm_scale
    mask = torch.ones(T, T, dtype=torch.bool).tril()
    lse = torch.logsumexp(logits.masked_fill(~mask, -np.inf), dim=-1)
    return o.permute(1, 0, 2).numpy(), lse.T.numpy()


def test_mla_all_keys_selected_is_dense_causal_attention():
    rng = np.random.default_rng(9)
    T, H, k = 24, 3, 32
    q, kv = _bf16(rng, (T, H, 576)), _bf16(rng, (T, 576))
    idx = np.full((T, k), -1, np.int32)
    for t in range(T):
        idx[t, : t + 1] = rng.permutation(t + 1)
    out, lse = oracle.sparse_mla(q, kv, idx, 1 / 24)
    ref, ref_lse = dense_causal_sdpa(q, kv, 1 / 24)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)


def test_mla_single_selected_row_is_that_row():
    rng = np.random.default_rng(10)
    T, H, k = 5, 4, 8
    q, kv = _bf16(rng, (T, H, 576)), _bf16(rng, (11, 576))
    idx = np.full((T, k), -1, np.int32)
    for t in range(T):
        idx[t, rng.integers(0, k)] = t + 3
    out, lse = oracle.sparse_mla(q, kv, idx, 0.1)
    for t in range(T):
        row = kv[t + 3, :512].double().numpy()
        assert (out[t] == row[None, :]).all()
        z = 0.1 * (q[t].double() @ kv[t + 3].double()).numpy()
        np.testing.assert_allclose(lse[t], z, rtol=1e-13)


def test_mla_order_free_and_unselected_rows_have_no_effect():
    rng = np.random.default_rng(11)
    T, S, H, k = 6, 50, 2, 12
    q, kv = _bf16(rng, (T, H, 576)), _bf16(rng, (S, 576))
    idx = np.stack([rng.choice(S, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    idx[2, 5:] = -1
    out, lse = oracle.sparse_mla(q, kv, idx, 1 / 24)
    perm = np.stack([rng.permutation(k) for _ in range(T)])
    out_p, lse_p = oracle.sparse_mla(q, kv, np.take_along_axis(idx, perm, 1), 1 / 24)
    np.testing.assert_allclose(out_p, out, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse_p, lse, rtol=1e-13)
    poisoned = kv.clone()
    sel = set(idx[idx >= 0].tolist())
    for s in range(S):
        if s not in sel:
            poisoned[s] = float("nan")
    out_n, lse_n = oracle.sparse_mla(q, poisoned, idx, 1 / 24)
    assert np.array_equal(out_n, out) and np.array_equal(lse_n, lse)


# ---------------------------------------------------------------- full path

def test_short_context_dsa_is_dense_causal_attention():
    """Context <= k: the whole DSA path reproduces dense causal attention."""
    cfg = W.CONFIGS[1]
    inp = W.make_prefill(cfg, L=160)            # every row has <= 256 keys
    r = oracle.forward(inp)
    ref, ref_lse = dense_causal_sdpa(inp["q"], inp["kv"], inp["sm_scale"])
    np.testing.assert_allclose(r["out"], ref, rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(r["lse"], ref_lse, rtol=1e-12, atol=1e-12)


def test_long_context_selection_is_the_indexer_top_k():
    """Past k keys, the output only depends on the selected rows."""
    cfg = W.CONFIGS[1]
    inp = W.make_prefill(cfg, L=400)
    rows = np.array([399, 300, 257, 256, 255, 10])
    r = oracle.forward(inp, rows=rows)
    kv = inp["kv"].clone()
    for i, t in enumerate(rows):
        sel = set(r["idx"][i][r["idx"][i] >= 0].tolist())
        assert len(sel) == min(t + 1, 256)
    # shifting every unselected causal key of row 399 leaves its output alone
    sel = set(r["idx"][0].tolist())
    for s in range(400):
        if s not in sel:
            kv[s] = kv[s] + 3.0
    out2, _ = oracle.sparse_mla(inp["q"], kv, np.tile(r["idx"][:1], (400, 1)), inp["sm_scale"], rows=[399])
    assert np.array_equal(out2[0], r["out"][0])


# ------------------------------------------------------------- paged decode

def _small_decode(lens, seed=3, nq=2):
    cfg = W.Config(99, "tiny_decode", "decode", k=48, Hi=4, H=3, seed=seed, nq=nq,
                   ctx_lo=1, ctx_hi=2)
    return W.make_decode(cfg, lens=torch.tensor(lens))


def test_decode_equals_contiguous_prefill_rows():
    inp = _small_decode([130, 40, 200], nq=2)
    d = oracle.decode(inp)
    for i, b in enumerate(range(inp["B"])):
        n = int(inp["seq_len"][b])
        k8 = oracle.gather_sequence(inp["k8_pool"].numpy(), inp["block_table"][b].numpy(), n)
        ks = oracle.gather_sequence(inp["k_scale_pool"].numpy(), inp["block_table"][b].numpy(), n)
        kv = oracle.gather_sequence(inp["kv_pool"].view(torch.int16).numpy(),
                                    inp["block_table"][b].numpy(), n)
        # contiguous prefill of n tokens whose last nq rows are the decode queries
        T = n
        q8 = torch.zeros(T, 4, 128, dtype=torch.uint8)
        q8[n - 2:] = inp["q8"][b]
        qs = torch.ones(T)
        qs[n - 2:] = inp["q_scale"][b]
        w = torch.zeros(T, 4)
        w[n - 2:] = inp["w"][b]
        q = torch.zeros(T, 3, 576, dtype=torch.bfloat16)
        q[n - 2:] = inp["q"][b]
        pre = dict(q8=q8, q_scale=qs, k8=torch.from_numpy(k8), k_scale=torch.from_numpy(ks),
                   w=w, q=q, kv=torch.from_numpy(kv).view(torch.bfloat16), scale=inp["scale"],
                   sm_scale=inp["sm_scale"], k=inp["k"], q_pos0=0, T=T, S=n)
        r = oracle.forward(pre, rows=[n - 2, n - 1])
        assert np.array_equal(np.sort(r["idx"], 1), np.sort(d["idx"][i], 1))
        np.testing.assert_array_equal(r["out"], d["out"][i])


def test_decode_invariant_under_physical_block_permutation():
    inp = _small_decode([100, 64, 65], nq=1)
    d = oracle.decode(inp)
    rng = np.random.default_rng(12)
    nblk = inp["nblk"]
    perm = torch.from_numpy(rng.permutation(nblk))       # new physical slot of each block
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(nblk)
    inp2 = dict(inp)
    for key in ("k8_pool", "k_scale_pool", "kv_pool"):
        inp2[key] = inp[key][inv].contiguous()
    tab = inp["block_table"].clone()
    tab[tab >= 0] = perm[tab[tab >= 0].long()].int()
    inp2["block_table"] = tab
    d2 = oracle.decode(inp2)
    assert np.array_equal(d2["idx"], d["idx"])
    assert np.array_equal(d2["out"], d["out"])


# ------------------------------------------- sliding window / dense causal

def band_mask(T, window):
    """Library band: key s visible from row t iff t - window < s <= t."""
    return torch.ones(T, T, dtype=torch.bool).tril().triu(-(window - 1))


@pytest.mark.parametrize("window,q_pos0,S", [(1, 0, 40), (7, 0, 40), (16, 5, 40), (40, 0, 40),
                                             (9, 30, 34)])
def test_window_is_the_band_of_a_library_mask(window, q_pos0, S):
    nrows, k = 12, 40
    sel = oracle.window(nrows, S, window, k, q_pos0=q_pos0)
    band = band_mask(S, window)
    for r in range(nrows):
        p = min(q_pos0 + r, S - 1)                # rows past the cache clamp to its end
        want = torch.nonzero(band[p]).flatten().numpy()
        got = sel[r][sel[r] >= 0]
        np.testing.assert_array_equal(got, want)
        assert (sel[r][len(got):] == -1).all()


def test_sliding_window_attention_is_banded_sdpa():
    rng = np.random.default_rng(21)
    T, H, window, k = 30, 3, 6, 8
    q, kv = _bf16(rng, (T, H, 576)), _bf16(rng, (T, 576))
    out, lse = oracle.sparse_mla(q, kv, oracle.window(T, T, window, k), 1 / 24)
    qd = q.double().permute(1, 0, 2)
    kd = kv.double().unsqueeze(0).expand(H, -1, -1)
    vd = kv[:, :512].double().unsqueeze(0).expand(H, -1, -1)
    mask = band_mask(T, window)
    ref = torch.nn.functional.scaled_dot_product_attention(qd, kd, vd, attn_mask=mask,
                                                           scale=1 / 24)
    ref_lse = torch.logsumexp(((qd @ kd.transpose(1, 2)) / 24).masked_fill(~mask, -np.inf), -1)
    np.testing.assert_allclose(out, ref.permute(1, 0, 2).numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse.T.numpy(), rtol=1e-12, atol=1e-12)


def test_window_covering_the_prefix_is_dense_causal_attention():
    rng = np.random.default_rng(22)
    T, H = 20, 2
    q, kv = _bf16(rng, (T, H, 576)), _bf16(rng, (T, 576))
    out, lse = oracle.sparse_mla(q, kv, oracle.window(T, T, T, 20), 1 / 24)
    ref, ref_lse = dense_causal_sdpa(q, kv, 1 / 24)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)


# ------------------------------------------------ projection (workflow step 1)

def test_projection_with_identity_rotation_is_a_matmul():
    inp = W.make_projection(20, 48, 2, seed=31)
    ident = torch.zeros(20, 64, 2)
    ident[..., 0] = 1.0
    y = oracle.project(inp["h"], inp["wt"], ident, 2)
    ref = (inp["h"].double() @ inp["wt"].double().T).numpy()
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_projection_rotation_is_complex_multiplication():
    """Pair (2i, 2i+1) of every q head and of k is multiplied, as a complex
    number, by cos + i sin of the table entry i; a_h is not rotated."""
    Hi, T = 3, 9
    inp = W.make_projection(T, 40, Hi, seed=32)
    rng = np.random.default_rng(33)
    ang = rng.uniform(-np.pi, np.pi, size=(T, 64))
    table = torch.from_numpy(np.stack([np.cos(ang), np.sin(ang)], -1)).float()
    rows = [8, 0, 5]
    y = oracle.project(inp["h"], inp["wt"], table, Hi, rows=rows)
    plain = (inp["h"].double() @ inp["wt"].double().T).numpy()[rows]
    nqk = Hi * 128 + 128
    z = plain[:, :nqk:2] + 1j * plain[:, 1:nqk:2]                # [rows][pairs]
    tab = table.double().numpy()[rows]
    rot = np.tile(tab[..., 0] + 1j * tab[..., 1], (1, nqk // 128))
    zr = z * rot
    np.testing.assert_allclose(y[:, :nqk:2], zr.real, rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(y[:, 1:nqk:2], zr.imag, rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(y[:, nqk:], plain[:, nqk:], rtol=1e-12, atol=1e-12)


# ------------------------------------------------- indexer warm-up objective

def test_warmup_target_rows_sum_to_one_and_match_softmax_and_attention():
    rng = np.random.default_rng(41)
    T, H = 12, 3
    q, kv = _bf16(rng, (T, H, 576)), _bf16(rng, (T, 576))
    p = oracle.attention_probs(q, kv, 1 / 24)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=1e-12)
    assert (p[np.triu_indices(T, 1)] == 0).all()                 # causal
    # one head: the library softmax of the masked logits
    p1 = oracle.attention_probs(q[:, :1], kv, 1 / 24)
    z = (q[:, 0].double() @ kv.double().T) / 24
    ref = torch.softmax(z.masked_fill(~torch.ones(T, T, dtype=torch.bool).tril(), -np.inf), -1)
    np.testing.assert_allclose(p1, ref.numpy(), rtol=1e-10, atol=1e-14)
    # the same weights give the pinned sparse-MLA oracle's dense output
    idx = np.full((T, T), -1, np.int32)
    for t in range(T):
        idx[t, : t + 1] = np.arange(t + 1)
    out, _ = oracle.sparse_mla(q[:, :1], kv, idx, 1 / 24)
    np.testing.assert_allclose(out[:, 0], p1 @ kv[:, :512].double().numpy(), rtol=1e-9, atol=1e-12)


def test_warmup_target_is_the_mean_of_the_per_head_softmax_rows():
    """The H-head target is the plain mean over heads of each head's own
    library softmax of its masked logits, with heads of very different
    sharpness so that any other weighting of the heads (a sum, one head, a
    softmax of averaged logits, weights by head index) moves the result."""
    rng = np.random.default_rng(43)
    T, H = 10, 4
    gains = torch.tensor([0.2, 1.0, 3.0, 8.0], dtype=torch.float64)
    qf = torch.from_numpy(rng.normal(size=(T, H, 576))) * gains[None, :, None]
    q, kv = qf.to(torch.bfloat16), _bf16(rng, (T, 576))
    p = oracle.attention_probs(q, kv, 1 / 24)
    mask = torch.ones(T, T, dtype=torch.bool).tril()
    z = torch.einsum("thd,sd->ths", q.double(), kv.double()) / 24
    per_head = torch.softmax(z.masked_fill(~mask[:, None, :], -np.inf), dim=-1)
    np.testing.assert_allclose(p, per_head.mean(dim=1).numpy(), rtol=1e-10, atol=1e-14)
    # the alternatives a mistake would produce differ from it
    pooled = torch.softmax(z.mean(dim=1).masked_fill(~mask, -np.inf), dim=-1)
    assert np.abs(p - pooled.numpy()).max() > 1e-3
    assert np.abs(p - per_head[:, -1].numpy()).max() > 1e-3


def test_warmup_kl_zero_at_the_target_and_gradient_by_finite_differences():
    rng = np.random.default_rng(42)
    R, n = 4, 17
    p = rng.dirichlet(np.ones(n), size=R)
    I = np.log(p) + rng.normal(size=(R, 1))                      # softmax(I) == p
    loss, grad = oracle.indexer_kl(I, p, np.full(R, n))
    np.testing.assert_allclose(loss, 0.0, atol=1e-12)
    np.testing.assert_allclose(grad, 0.0, atol=1e-12)
    I = rng.normal(size=(R, n)) * 2.0
    loss, grad = oracle.indexer_kl(I, p, np.full(R, n))
    assert (loss > 0).all()
    eps = 1e-6
    for s in (0, 5, 16):
        e = np.zeros_like(I)
        e[:, s] = eps
        lp, _ = oracle.indexer_kl(I + e, p, np.full(R, n))
        lm, _ = oracle.indexer_kl(I - e, p, np.full(R, n))
        np.testing.assert_allclose((lp - lm) / (2 * eps), grad[:, s], rtol=1e-6, atol=1e-9)


def _float_indexer(qf, kf, w, scale, q_pos0=0):
    """I[t, s] from dequantised inputs, float64, causal (-inf past the row's keys)."""
    x = np.einsum("thd,sd->ths", qf, kf)
    I = np.einsum("th,ths->ts", w, np.maximum(scale * x, 0.0))
    T, S = I.shape
    mask = np.arange(S)[None, :] <= (q_pos0 + np.arange(T))[:, None]
    return np.where(mask, I, -np.inf)


def test_warmup_backward_matches_finite_differences():
    rng = np.random.default_rng(43)
    T, Hi, scale = 6, 2, 0.25
    q8 = e4m3_codes(rng, (T, Hi, 128), -4, 4)
    k8 = e4m3_codes(rng, (T, 128), -4, 4)
    q_scale = torch.from_numpy(rng.uniform(0.5, 1.5, T)).float()
    k_scale = torch.from_numpy(rng.uniform(0.5, 1.5, T)).float()
    w = torch.from_numpy(rng.normal(size=(T, Hi)) / 8).float()
    qf = lib_float(q8).numpy() * q_scale.double().numpy()[:, None, None]
    kf = lib_float(k8).numpy() * k_scale.double().numpy()[:, None]
    wd = w.double().numpy()
    p = np.tril(rng.uniform(0.1, 1.0, (T, T)))
    p /= p.sum(axis=1, keepdims=True)
    n = np.arange(1, T + 1)

    def loss_of(qf_, kf_, w_):
        I = _float_indexer(qf_, kf_, w_, scale)
        I = np.where(np.isfinite(I), I, 0.0)
        return oracle.indexer_kl(I, p, n)[0].sum()

    I0 = np.where(np.isfinite(_float_indexer(qf, kf, wd, scale)),
                  _float_indexer(qf, kf, wd, scale), 0.0)
    _, g = oracle.indexer_kl(I0, p, n)
    dq, dk, dw = oracle.indexer_backward(q8, q_scale, k8, k_scale, w, scale, g)
    eps = 1e-5
    for (t, h, d) in [(5, 1, 3), (2, 0, 100), (4, 1, 64)]:
        e = np.zeros_like(qf)
        e[t, h, d] = eps
        num = (loss_of(qf + e, kf, wd) - loss_of(qf - e, kf, wd)) / (2 * eps)
        np.testing.assert_allclose(dq[t, h, d], num, rtol=1e-5, atol=1e-9)
    for (s, d) in [(0, 7), (3, 127), (5, 50)]:
        e = np.zeros_like(kf)
        e[s, d] = eps
        num = (loss_of(qf, kf + e, wd) - loss_of(qf, kf - e, wd)) / (2 * eps)
        np.testing.assert_allclose(dk[s, d], num, rtol=1e-5, atol=1e-9)
    for (t, h) in [(5, 0), (3, 1)]:
        e = np.zeros_like(wd)
        e[t, h] = eps
        num = (loss_of(qf, kf, wd + e) - loss_of(qf, kf, wd - e)) / (2 * eps)
        np.testing.assert_allclose(dw[t, h], num, rtol=1e-5, atol=1e-9)
