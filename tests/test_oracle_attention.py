"""Pins of the oracle's append / decode against an independent dense brute force,
closed forms and invariants.

The brute force never looks at pages: it quantizes the logical K/V sequence
with torch.float8_e4m3fn (clamped: saturating reading), dequantizes with
torch, and runs dense fp64 attention with numpy/scipy.  The oracle instead
scatters tokens into pages through a slot mapping and gathers them back
through the block table.  A dropped term, a wrong sign, a transposed operand,
a wrong GQA head map or a wrong page/offset split fails here.
"""
import math

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

import oracle
from fp8_kv_paged_kvq_b200 import workloads as W

MODE = {W.SCALE_TENSOR: oracle.SCALE_TENSOR, W.SCALE_HEAD: oracle.SCALE_HEAD,
        W.SCALE_TOKEN: oracle.SCALE_TOKEN}


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def bf16_f64(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.float64).numpy()


def new_cache(wl):
    s = wl.spec
    P, ps, H = wl.num_pages, s.page_size, s.num_kv_heads
    if s.kv_dtype == W.FP8:
        kp = np.full((P, H, ps, s.head_dim_k), 0xCD, np.uint8)
        vp = None if s.v_alias else np.full((P, H, ps, s.head_dim_v), 0xCD, np.uint8)
    else:
        kp = np.zeros((P, H, ps, s.head_dim_k), np.uint16)
        vp = None if s.v_alias else np.zeros((P, H, ps, s.head_dim_v), np.uint16)
    if s.scale_mode == W.SCALE_TOKEN:
        ks = np.zeros((P, H, ps), np.float32)
        vs = None if s.v_alias else np.zeros((P, H, ps), np.float32)
    else:
        n = 1 if s.scale_mode == W.SCALE_TENSOR else H
        ks, vs = np.ones(n, np.float32), (None if s.v_alias else np.ones(n, np.float32))
    return oracle.Cache(oracle.FP8 if s.kv_dtype == W.FP8 else oracle.BF16, MODE[s.scale_mode],
                        P, ps, H, s.head_dim_k, s.head_dim_v, kp, vp, ks, vs,
                        wl.page_tags.copy())


def fill(wl, cache):
    """Pre-fill with the history, then append the step's token.  Returns logical bf16 K, V."""
    s = wl.spec
    ks, vs = [], []
    hist = list(wl.hist_chunks())
    hk = torch.cat([h[0] for h in hist]) if hist else None
    hv = None if s.v_alias or not hist else torch.cat([h[1] for h in hist])
    if s.kv_dtype == W.FP8 and s.scale_mode != W.SCALE_TOKEN:
        per_head = s.scale_mode == W.SCALE_HEAD
        cache.k_scale[:] = oracle.scales(bf16_bits(hk), per_head)
        if not s.v_alias:
            cache.v_scale[:] = oracle.scales(bf16_bits(hv), per_head)
    if hist:
        oracle.append(cache, bf16_bits(hk), None if hv is None else bf16_bits(hv),
                      wl.hist_slots)
    kn, vn, slots = wl.new_tokens()
    oracle.append(cache, bf16_bits(kn), None if vn is None else bf16_bits(vn), slots)
    return hk, hv, kn, vn


def logical_sequences(wl, hk, hv, kn, vn):
    """Dense per-sequence bf16 K/V in logical order (history then new token)."""
    out, pos = [], 0
    for b, L in enumerate(wl.seq_lens.tolist()):
        if L == 0:
            out.append((None, None))
            continue
        k = torch.cat([hk[pos:pos + L - 1], kn[b:b + 1]])
        v = None if vn is None else torch.cat([hv[pos:pos + L - 1], vn[b:b + 1]])
        pos += L - 1
        out.append((k, v))
    return out


def torch_q8(x32: torch.Tensor) -> torch.Tensor:
    return torch.clamp(x32, -448, 448).to(torch.float8_e4m3fn)


def brute_force(wl, cache, seqs, abort=None):
    """Dense fp64 attention from logical tensors; quantization by torch."""
    s = wl.spec
    q = bf16_f64(wl.q())
    G = s.group
    res_o = np.zeros((s.B, s.num_q_heads, s.head_dim_v))
    res_l = np.full((s.B, s.num_q_heads), -np.inf)
    for b, (k, v) in enumerate(seqs):
        if k is None or (abort is not None and abort[b]):
            continue
        for hk in range(s.num_kv_heads):
            kk = k[:, hk].to(torch.float32)
            if s.kv_dtype == W.FP8:
                if s.scale_mode == W.SCALE_TOKEN:
                    amax = kk.abs().amax(dim=1, keepdim=True)
                    sc = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
                else:
                    sc = torch.tensor(cache.k_scale[0 if s.scale_mode == W.SCALE_TENSOR else hk])
                khat = (torch_q8(kk / sc).to(torch.float32) * sc).to(torch.float64).numpy()
                if s.v_alias:
                    vhat = khat[:, : s.head_dim_v]
                else:
                    vv = v[:, hk].to(torch.float32)
                    if s.scale_mode == W.SCALE_TOKEN:
                        am = vv.abs().amax(dim=1, keepdim=True)
                        vsc = torch.where(am > 0, am / 448.0, torch.ones_like(am))
                    else:
                        vsc = torch.tensor(cache.v_scale[0 if s.scale_mode == W.SCALE_TENSOR else hk])
                    vhat = (torch_q8(vv / vsc).to(torch.float32) * vsc).to(torch.float64).numpy()
            else:
                khat = kk.to(torch.float64).numpy()
                vhat = khat[:, : s.head_dim_v] if s.v_alias else v[:, hk].to(torch.float64).numpy()
            for g in range(G):
                h = hk * G + g
                sc_ = (khat @ q[b, h]) * np.float64(np.float32(wl.sm_scale))
                lse = logsumexp(sc_)
                res_o[b, h] = np.exp(sc_ - lse) @ vhat
                res_l[b, h] = lse
    return res_o, res_l


def run_oracle(wl, cache, abort=None):
    o, l = oracle.decode(cache, bf16_bits(wl.q()), wl.block_table, wl.seq_lens, abort, wl.sm_scale)
    s = wl.spec
    return o.reshape(s.B, s.num_q_heads, s.head_dim_v), l.reshape(s.B, s.num_q_heads)


SMALL = [
    W.Spec("s_tensor", [37, 100], 16, 4, 1, 64, 64, scale_mode=W.SCALE_TENSOR, pool_pages=16),
    W.Spec("s_head", [1, 15, 16, 17, 50], 16, 8, 2, 32, 32, outlier_p=0.05),
    W.Spec("s_bf16", [5, 33, 70], 16, 6, 3, 16, 16, kv_dtype=W.BF16),
    W.Spec("s_token_alias", [3, 64, 65, 130], 64, 8, 1, 40, 32, v_alias=True,
           scale_mode=W.SCALE_TOKEN),
    W.Spec("s_token_sep", [7, 40], 8, 4, 2, 24, 16, scale_mode=W.SCALE_TOKEN),
    W.Spec("s_empty", [0, 9, 0], 4, 2, 1, 8, 8, scale_mode=W.SCALE_HEAD),
]


@pytest.mark.parametrize("spec", SMALL, ids=lambda s: s.name)
def test_oracle_matches_dense_brute_force(spec):
    wl = W.make_workload(spec, seed=11)
    cache = new_cache(wl)
    seqs = logical_sequences(wl, *fill(wl, cache))
    o, l = run_oracle(wl, cache)
    bo, bl = brute_force(wl, cache, seqs)
    assert np.array_equal(np.isinf(l), np.isinf(bl))
    fin = np.isfinite(bl)
    np.testing.assert_allclose(l[fin], bl[fin], rtol=0, atol=1e-11)
    np.testing.assert_allclose(o, bo, rtol=0, atol=1e-11)


@pytest.mark.parametrize("spec", SMALL[:2] + SMALL[3:4], ids=lambda s: s.name)
def test_append_codes_match_torch_quantization(spec):
    """Every written code equals torch's e4m3 cast of x/s; untouched bytes keep the canary."""
    wl = W.make_workload(spec, seed=5)
    cache = new_cache(wl)
    seqs = logical_sequences(wl, *fill(wl, cache))
    s = wl.spec
    touched = np.zeros(cache.k_pages.shape[:3], bool)
    for b, (k, v) in enumerate(seqs):
        if k is None:
            continue
        for j in range(k.shape[0]):
            p, o = wl.block_table[b, j // s.page_size], j % s.page_size
            for hk in range(s.num_kv_heads):
                x = k[j, hk].to(torch.float32)
                if s.scale_mode == W.SCALE_TOKEN:
                    am = x.abs().max()
                    sc = am / 448.0 if am > 0 else torch.tensor(1.0)
                    assert np.float32(sc) == cache.k_scale[p, hk, o]
                else:
                    sc = torch.tensor(cache.k_scale[0 if s.scale_mode == W.SCALE_TENSOR else hk])
                want = torch_q8(x / sc).view(torch.uint8).numpy()
                assert np.array_equal(cache.k_pages[p, hk, o], want)
                touched[p, hk, o] = True
    assert np.all(cache.k_pages[~touched] == 0xCD)


def _single_page_cache(D, ps=16, P=4, Hkv=1):
    kp = np.zeros((P, Hkv, ps, D), np.uint8)
    vp = np.zeros((P, Hkv, ps, D), np.uint8)
    return oracle.Cache(oracle.FP8, oracle.SCALE_HEAD, P, ps, Hkv, D, D, kp, vp,
                        np.full(Hkv, 0.5, np.float32), np.full(Hkv, 0.25, np.float32),
                        np.zeros(P, np.uint32))


def test_single_token_returns_its_value_exactly():
    r = np.random.default_rng(3)
    c = _single_page_cache(32)
    c.k_pages[2, 0, 0] = r.integers(0, 0x7E, 32)
    c.v_pages[2, 0, 0] = r.integers(0, 0x7E, 32)
    q = bf16_bits(torch.randn(1, 1, 32, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16))
    o, l = oracle.decode(c, q, np.array([[2]], np.int32), np.array([1], np.int32), None, 0.3)
    vhat = (torch.from_numpy(c.v_pages[2, 0, 0]).view(torch.float8_e4m3fn).float() * 0.25)
    assert np.array_equal(o[0].astype(np.float32), vhat.numpy())
    khat = torch.from_numpy(c.k_pages[2, 0, 0]).view(torch.float8_e4m3fn).double() * 0.5
    s = float(np.float32(0.3)) * float(khat @ torch.from_numpy(q.view(np.int16)).view(torch.bfloat16).double()[0, 0])
    assert abs(l[0] - s) <= 1e-14 * max(1.0, abs(s))


def test_two_tokens_closed_form():
    r = np.random.default_rng(4)
    c = _single_page_cache(16)
    c.k_pages[1, 0, :2] = r.integers(0, 0x7E, (2, 16))
    c.v_pages[1, 0, :2] = r.integers(0, 0x7E, (2, 16))
    qt = torch.randn(1, 1, 16, generator=torch.Generator().manual_seed(4)).to(torch.bfloat16)
    o, l = oracle.decode(c, bf16_bits(qt), np.array([[1]], np.int32), np.array([2], np.int32),
                         None, 1.0)
    kh = torch.from_numpy(c.k_pages[1, 0, :2]).view(torch.float8_e4m3fn).double() * 0.5
    vh = torch.from_numpy(c.v_pages[1, 0, :2]).view(torch.float8_e4m3fn).double() * 0.25
    s = (kh @ qt.double()[0, 0]).numpy()
    d = s[1] - s[0]                                    # weight of token 0: sigma(s0 - s1)
    w1 = 1.0 / (1.0 + math.exp(d)) if d <= 0 else math.exp(-d) / (1.0 + math.exp(-d))
    want = w1 * vh[0].numpy() + (1 - w1) * vh[1].numpy()
    scale = float(np.abs(vh.numpy()).max())
    np.testing.assert_allclose(o[0], want, rtol=0, atol=1e-14 * max(1.0, scale))
    np.testing.assert_allclose(l[0], max(s) + math.log1p(math.exp(-abs(d))),
                               rtol=0, atol=1e-14 * max(1.0, float(np.abs(s).max())))


def test_zero_query_gives_mean_of_values():
    wl = W.make_workload(SMALL[1], seed=2)
    cache = new_cache(wl)
    fill(wl, cache)
    q0 = np.zeros_like(bf16_bits(wl.q()))
    o, l = oracle.decode(cache, q0, wl.block_table, wl.seq_lens, None, wl.sm_scale)
    s = wl.spec
    o = o.reshape(s.B, s.num_q_heads, -1)
    for b, L in enumerate(wl.seq_lens):
        for h in range(s.num_q_heads):
            hk = h // s.group
            idx = [(wl.block_table[b, j // s.page_size], j % s.page_size) for j in range(L)]
            v = np.stack([cache.v_pages[p, hk, off] for p, off in idx])
            vhat = torch.from_numpy(v).view(torch.float8_e4m3fn).double().numpy() * np.float64(cache.v_scale[hk])
            np.testing.assert_allclose(o[b, h], vhat.astype(np.float32).astype(np.float64).mean(0), atol=1e-12)
            assert abs(l.reshape(s.B, -1)[b, h] - math.log(L)) < 1e-12


def test_page_permutation_leaves_output_unchanged():
    wl = W.make_workload(SMALL[1], seed=9)
    cache = new_cache(wl)
    fill(wl, cache)
    o1, l1 = run_oracle(wl, cache)
    perm = np.random.default_rng(1).permutation(wl.num_pages).astype(np.int32)  # new id of page p
    c2 = new_cache(wl)
    c2.k_pages[perm] = cache.k_pages
    c2.v_pages[perm] = cache.v_pages
    c2.k_scale[:] = cache.k_scale
    c2.v_scale[:] = cache.v_scale
    bt2 = np.where(wl.block_table >= 0, perm[np.maximum(wl.block_table, 0)], -1).astype(np.int32)
    o2, l2 = oracle.decode(c2, bf16_bits(wl.q()), bt2, wl.seq_lens, None, wl.sm_scale)
    assert np.array_equal(o1.ravel(), o2.ravel()) and np.array_equal(l1.ravel(), l2.ravel())


def test_aborted_and_empty_rows():
    wl = W.make_workload(SMALL[5], seed=1)
    cache = new_cache(wl)
    fill(wl, cache)
    o, l = run_oracle(wl, cache, abort=np.array([0, 1, 0], np.uint8))
    assert np.all(o == 0) and np.all(np.isneginf(l))
    o, l = run_oracle(wl, cache)
    assert np.all(np.isneginf(l[[0, 2]])) and np.all(np.isfinite(l[1]))


def test_rows_subset_equals_full():
    wl = W.make_workload(SMALL[1], seed=3)
    cache = new_cache(wl)
    fill(wl, cache)
    o, l = oracle.decode(cache, bf16_bits(wl.q()), wl.block_table, wl.seq_lens, None, wl.sm_scale)
    rows = np.array([5, 0, 17, 39], np.int32)
    o2, l2 = oracle.decode(cache, bf16_bits(wl.q()), wl.block_table, wl.seq_lens, None,
                           wl.sm_scale, rows=rows)
    assert np.array_equal(o2, o[rows]) and np.array_equal(l2, l[rows])


def test_fp8_cache_is_half_the_bf16_bytes():
    """The FP8 cache holds the same tokens in half the bytes (codes only)."""
    f = W.make_workload(W.spec_by_name("ragged"), 0)
    b = W.make_workload(W.spec_by_name("ragged_bf16"), 0)
    assert 2 * f.kv_bytes_read() == b.kv_bytes_read()
    wl = W.make_workload(SMALL[1], seed=1)
    c8 = new_cache(wl)
    spec16 = W.Spec(**{**SMALL[1].__dict__, "kv_dtype": W.BF16})
    c16 = new_cache(W.make_workload(spec16, seed=1))
    assert 2 * (c8.k_pages.nbytes + c8.v_pages.nbytes) == c16.k_pages.nbytes + c16.v_pages.nbytes


@pytest.mark.parametrize("spec", [SMALL[0], SMALL[1]], ids=lambda s: s.name)
def test_scales_independent_of_oracle(spec):
    """Per-tensor / per-head scale = fl32(amax / 448) over the pre-filled tokens (torch)."""
    wl = W.make_workload(spec, seed=4)
    cache = new_cache(wl)
    hk, hv, _, _ = fill(wl, cache)
    for x, sc in ((hk, cache.k_scale), (hv, cache.v_scale)):
        a = x.float().abs()
        am = a.amax() if spec.scale_mode == W.SCALE_TENSOR else a.amax(dim=(0, 2))
        want = (am / torch.tensor(448.0)).numpy().astype(np.float32).reshape(-1)
        assert np.array_equal(sc, want)


def test_amax_ignores_nan_and_folds_into_the_running_value():
    """Reading R18 (NaN elements do not take part in the amax) against
    numpy's nanmax, per head and over the whole tensor, with infinities, a head
    that is all NaN (its amax stays at the running value) and a running value
    larger than the data (kept)."""
    r = np.random.default_rng(21)
    x = (r.standard_normal((50, 4, 24)) * 3).astype(np.float32)
    x[r.random(x.shape) < 0.05] = np.nan
    x[7, 1, 3] = -np.inf
    x[:, 2, :] = np.nan
    bits = torch.from_numpy(x).to(torch.bfloat16)
    xb = bits.float().numpy()                       # the bf16 values both sides see
    with np.errstate(all="ignore"), __import__("warnings").catch_warnings():
        __import__("warnings").simplefilter("ignore")
        want = np.nanmax(np.abs(xb), axis=(0, 2))
    want = np.where(np.isnan(want), 0.0, want).astype(np.float32)
    got = oracle.amax(bf16_bits(bits), True, np.zeros(4, np.float32))
    assert np.array_equal(got, want) and got[1] == np.inf and got[2] == 0.0
    run = np.array([0.0, 0.0, 5.0, 1e9], np.float32)
    got = oracle.amax(bf16_bits(bits), True, run.copy())
    assert np.array_equal(got, np.maximum(run, want))
    flat = np.float32(np.nanmax(np.abs(xb)))
    assert oracle.amax(bf16_bits(bits), False, np.zeros(1, np.float32))[0] == flat
    # all-NaN data leaves the scale at 1 (amax 0)
    s = oracle.scales(bf16_bits(bits[:, 2:3]), per_head=False)
    assert s[0] == 1.0


def test_out_of_range_page_ids_read_as_zero_rows():
    """Reading R16: a block-table entry outside [0, P) contributes tokens whose
    K and V are zero.  Brute force: the sequence gathered by hand from the
    pages with torch's E4M3 decoding, explicit zero rows for the bad entries,
    dense fp64 softmax.  Every page (page 0 included) holds nonzero codes, so
    reading any real page in place of the zeros would fail."""
    r = np.random.default_rng(31)
    P, ps, H, D = 6, 4, 2, 16
    codes = lambda: r.integers(0, 0x7E, (P, H, ps, D)).astype(np.uint8) | \
        (r.integers(0, 2, (P, H, ps, D)).astype(np.uint8) << 7)
    kp, vp = codes(), codes()
    ks, vs = np.array([0.5, 0.125], np.float32), np.array([0.25, 2.0], np.float32)
    c = oracle.Cache(oracle.FP8, oracle.SCALE_HEAD, P, ps, H, D, D, kp, vp, ks, vs,
                     np.zeros(P, np.uint32))
    bt = np.array([[2, P + 3, 0, -1, 5], [-4, 1, 3, 0, 0]], np.int32)
    lens = np.array([18, 9], np.int32)
    G = 3
    qt = torch.randn(2, G * H, D, generator=torch.Generator().manual_seed(31)).to(torch.bfloat16)
    sm = 0.37
    o, l = oracle.decode(c, bf16_bits(qt), bt, lens, None, sm)
    q = qt.double().numpy()
    for b in range(2):
        for h in range(G * H):
            hk = h // G
            kh, vh = [], []
            for j in range(lens[b]):
                p, off = bt[b, j // ps], j % ps
                if 0 <= p < P:
                    k8 = torch.from_numpy(kp[p, hk, off].copy()).view(torch.float8_e4m3fn)
                    v8 = torch.from_numpy(vp[p, hk, off].copy()).view(torch.float8_e4m3fn)
                    kh.append((k8.float() * float(ks[hk])).double().numpy())
                    vh.append((v8.float() * float(vs[hk])).double().numpy())
                else:
                    kh.append(np.zeros(D))
                    vh.append(np.zeros(D))
            kh, vh = np.stack(kh), np.stack(vh)
            s = (kh @ q[b, h]) * np.float64(np.float32(sm))
            lse = logsumexp(s)
            i = b * G * H + h
            np.testing.assert_allclose(o[i], np.exp(s - lse) @ vh, rtol=0, atol=1e-11)
            assert abs(l[i] - lse) <= 1e-11
