"""GPU parity: libkvq (through its C ABI) against the CPU oracle on the same
seeded inputs.

Bar: E4M3 codes, page writes, scales, tags and abort masks bit-exact; decode
outputs within max-abs 2e-3 and max-rel 1e-2 (relative error taken over
elements with |ref| >= 0.2, where it is meaningful), lse within 2e-3,
aborted/empty rows exactly 0 / -inf.  Both sides start from the same
dequantised values; the GPU's error comes from f16 probabilities and FP32
accumulation order.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import fp8_kv_paged_kvq_b200 as kvq
from fp8_kv_paged_kvq_b200 import workloads as W
from fp8_kv_paged_kvq_b200.pipeline import DecodeBatch
from tests import oracle_side as OS

pytestmark = pytest.mark.gpu

ATOL, RTOL, REL_FLOOR = 2e-3, 1e-2, 0.2


def assert_decode_close(out, lse, ref_out, ref_lse, what=""):
    out = out.detach().cpu().double().numpy().reshape(ref_out.shape)
    lse = lse.detach().cpu().double().numpy().reshape(ref_lse.shape)
    inf_ref = np.isneginf(ref_lse)
    assert np.array_equal(np.isneginf(lse), inf_ref), what
    assert np.all(out[inf_ref] == 0.0), what
    fin = ~inf_ref
    d = np.abs(out - ref_out)
    assert d.max(initial=0.0) <= ATOL, (what, d.max())
    big = np.abs(ref_out) >= REL_FLOOR
    if big.any():
        rel = (d[big] / np.abs(ref_out[big])).max()
        assert rel <= RTOL, (what, rel)
    if fin.any():
        assert np.abs(lse[fin] - ref_lse[fin]).max() <= ATOL, what


SPECS = {
    "tiny": W.spec_by_name("tiny"),
    "g8_d128_head": W.Spec("g8_d128_head", [1, 15, 16, 17, 300, 1000], 16, 16, 2, 128, 128,
                           outlier_p=0.01, n_stale=2),
    "g16_d128": W.Spec("g16_d128", [50, 129, 700], 16, 32, 2, 128, 128),
    "g3_d64_ps48": W.Spec("g3_d64_ps48", [5, 48, 49, 500], 48, 6, 2, 64, 64,
                          scale_mode=W.SCALE_TENSOR),
    "g8_token_ps32": W.Spec("g8_token_ps32", [31, 32, 33, 400], 32, 8, 1, 128, 128,
                            scale_mode=W.SCALE_TOKEN),
    "bf16_g8_d128": W.Spec("bf16_g8_d128", [1, 15, 16, 17, 300, 1000], 16, 16, 2, 128, 128,
                           kv_dtype=W.BF16),
    "bf16_g12_d64": W.Spec("bf16_g12_d64", [7, 64, 333], 32, 24, 2, 64, 64, kv_dtype=W.BF16),
    "bf16_g16_d128": W.Spec("bf16_g16_d128", [100, 257], 16, 16, 1, 128, 128, kv_dtype=W.BF16),
    # 128 query heads on one KV head, K 576 / V = first 512 dims, per-token scales
    "wide_ps64": W.Spec("wide_ps64", [1, 63, 64, 65, 200, 700], 64, 128, 1, 576, 512,
                        v_alias=True, scale_mode=W.SCALE_TOKEN, n_stale=1),
    "wide_ps128": W.Spec("wide_ps128", [129, 500, 1000], 128, 128, 1, 576, 512, v_alias=True,
                         scale_mode=W.SCALE_TOKEN),
}


def build_both(spec, seed=0, num_ctas=0, canary=True):
    wl = W.make_workload(spec, seed=seed, device="cuda")
    db = DecodeBatch(wl, num_ctas=num_ctas)
    if canary and db.cache.fp8:
        db.cache.k_pages.fill_(0xCD)
        if db.cache.v_pages is not None:
            db.cache.v_pages.fill_(0xCD)
    db.prefill()
    db.append_new()          # the oracle side's fill() also appends the step's token
    oc = OS.new_cache(wl)
    OS.fill(wl, oc)
    return wl, db, oc


@pytest.mark.parametrize("name", list(SPECS))
def test_append_and_scales_bit_exact(name):
    wl, db, oc = build_both(SPECS[name], seed=1)
    db.append_new()
    torch.cuda.synchronize()
    c = db.cache
    if c.fp8:
        assert np.array_equal(c.k_pages.cpu().numpy(), oc.k_pages)
        if oc.v_pages is not None:
            assert np.array_equal(c.v_pages.cpu().numpy(), oc.v_pages)
        assert np.array_equal(c.k_scale.cpu().numpy(), oc.k_scale)
        if oc.v_scale is not None:
            assert np.array_equal(c.v_scale.cpu().numpy(), oc.v_scale)
    else:
        assert np.array_equal(c.k_pages.cpu().view(torch.int16).numpy().view(np.uint16), oc.k_pages)
        assert np.array_equal(c.v_pages.cpu().view(torch.int16).numpy().view(np.uint16), oc.v_pages)
    assert np.array_equal(c.page_tags.cpu().numpy().view(np.uint32), oc.page_tags)


@pytest.mark.parametrize("name", list(SPECS))
def test_decode_matches_oracle(name):
    wl, db, oc = build_both(SPECS[name], seed=2)
    out, lse = db.step(check_tags=True)
    torch.cuda.synchronize()
    mask = db.abort.cpu().numpy()
    ref_mask = oracle.validate(oc.page_tags, wl.block_table, wl.expected_tags, wl.seq_lens,
                               wl.spec.page_size)
    assert np.array_equal(mask, ref_mask)
    want = np.zeros(wl.B, np.uint8)
    for b, _ in wl.stale:
        want[b] = 1
    assert np.array_equal(mask, want)
    ro, rl = OS.decode(wl, oc, abort=ref_mask)
    assert_decode_close(out, lse, ro.reshape(out.shape), rl.reshape(lse.shape), name)
    # with the check disabled every row is decoded
    out2, lse2 = db.decode(use_abort=False)
    ro2, rl2 = OS.decode(wl, oc, abort=None)
    assert_decode_close(out2, lse2, ro2.reshape(out.shape), rl2.reshape(lse.shape), name)
    assert kvq.device_error() == 0


@pytest.mark.parametrize("num_ctas", [1, 2, 3, 7, 64, 148, 296, 1000, 5000])
def test_split_count_sweep(num_ctas):
    spec = SPECS["g8_d128_head"]
    wl, db, oc = build_both(spec, seed=3, num_ctas=num_ctas)
    out, lse = db.step(check_tags=False)
    torch.cuda.synchronize()
    ro, rl = OS.decode(wl, oc)
    assert_decode_close(out, lse, ro.reshape(out.shape), rl.reshape(lse.shape), str(num_ctas))
    assert kvq.device_error() == 0


@pytest.mark.parametrize("num_pairs", [1, 2, 3, 7, 74, 200])
def test_wide_split_count_sweep(num_pairs):
    wl, db, oc = build_both(SPECS["wide_ps64"], seed=13, num_ctas=num_pairs)
    out, lse = db.step(check_tags=False)
    torch.cuda.synchronize()
    ro, rl = OS.decode(wl, oc)
    assert_decode_close(out, lse, ro.reshape(out.shape), rl.reshape(lse.shape), str(num_pairs))
    assert kvq.device_error() == 0


def test_wide_outlier_query_and_peaky_scores():
    """Queries with a wide magnitude range (the two-term E4M3 split) and a few
    very large scores (the reference max has to move)."""
    spec = W.Spec("wide_peaky", [300, 77], 64, 128, 1, 576, 512, v_alias=True,
                  scale_mode=W.SCALE_TOKEN)
    wl = W.make_workload(spec, seed=14, device="cuda")
    q = wl.q().float()
    q[:, :, :8] *= 40.0                       # a few large dims: peaky softmax
    q[:, 5, :] *= 1e-3                        # a tiny-magnitude head
    wl._q = q.to(torch.bfloat16)
    db = DecodeBatch(wl)
    db.prefill()
    db.append_new()
    oc = OS.new_cache(wl)
    OS.fill(wl, oc)
    out, lse = db.decode(use_abort=False)
    torch.cuda.synchronize()
    ro, rl = OS.decode(wl, oc)
    assert_decode_close(out, lse, ro.reshape(out.shape), rl.reshape(lse.shape), "peaky")
    assert kvq.device_error() == 0


def test_wide_out_of_range_pages_empty_and_aborted_rows():
    """The tensor-core path: an out-of-range and a negative page inside a
    sequence read as zero codes with zero scale, an empty sequence and an
    aborted one give 0 / -inf, the rest match the oracle."""
    spec = W.Spec("wide_edges", [0, 130, 64, 300, 129], 64, 128, 1, 576, 512, v_alias=True,
                  scale_mode=W.SCALE_TOKEN)
    wl, db, oc = build_both(spec, seed=15)
    bt = wl.block_table.copy()
    bt[1, 1] = wl.num_pages + 3
    bt[3, 2] = -1
    wl.block_table = bt
    db.block_table = torch.from_numpy(bt).cuda()
    abort = np.array([0, 0, 1, 0, 0], np.uint8)
    db.abort.copy_(torch.from_numpy(abort))
    out, lse = db.decode(use_abort=True)
    torch.cuda.synchronize()
    ro, rl = OS.decode(wl, oc, abort=abort)
    assert_decode_close(out, lse, ro.reshape(out.shape), rl.reshape(lse.shape), "wide edges")
    assert torch.all(out[[0, 2]] == 0) and torch.all(torch.isneginf(lse[[0, 2]]))
    assert kvq.device_error() == 0


def test_page_permutation_is_bit_exact():
    spec = SPECS["g8_d128_head"]
    wl, db, _ = build_both(spec, seed=4, canary=False)
    out1, lse1 = [t.clone() for t in db.step(check_tags=False)]
    perm = torch.randperm(wl.num_pages, generator=torch.Generator().manual_seed(9)).cuda()
    c = db.cache
    k2 = torch.empty_like(c.k_pages)
    v2 = torch.empty_like(c.v_pages)
    k2[perm] = c.k_pages
    v2[perm] = c.v_pages
    c.k_pages.copy_(k2)
    c.v_pages.copy_(v2)
    bt = db.block_table
    db.block_table = torch.where(bt >= 0, perm[bt.clamp(min=0).long()].int(), bt).contiguous()
    out2, lse2 = db.decode(use_abort=False)
    torch.cuda.synchronize()
    assert torch.equal(out1, out2) and torch.equal(lse1, lse2)


def test_single_token_returns_value_bit_exact():
    spec = W.Spec("one", [1, 1, 1], 16, 8, 1, 128, 128)
    wl, db, oc = build_both(spec, seed=5)
    out, lse = db.step(check_tags=False)
    torch.cuda.synchronize()
    ro, _ = OS.decode(wl, oc)
    # p = 1: out is exactly fl32(decode(code) * s_v)
    assert np.array_equal(out.cpu().numpy().reshape(ro.shape), ro.astype(np.float32))


def test_aborted_rows_read_nothing():
    spec = SPECS["g8_d128_head"]
    wl, db, oc = build_both(spec, seed=6)
    db.abort.copy_(torch.tensor([1, 0, 1, 0, 0, 1], dtype=torch.uint8))
    out, lse = db.decode(use_abort=True)
    torch.cuda.synchronize()
    ro, rl = OS.decode(wl, oc, abort=np.array([1, 0, 1, 0, 0, 1], np.uint8))
    assert_decode_close(out, lse, ro.reshape(out.shape), rl.reshape(lse.shape))
    assert torch.all(out[[0, 2, 5]] == 0) and torch.all(torch.isneginf(lse[[0, 2, 5]]))


def test_all_rows_aborted_or_empty():
    spec = W.Spec("empty", [0, 20, 0], 16, 8, 1, 128, 128)
    wl, db, oc = build_both(spec, seed=7)
    db.abort.copy_(torch.tensor([0, 1, 0], dtype=torch.uint8))
    out, lse = db.decode(use_abort=True)
    torch.cuda.synchronize()
    assert torch.all(out == 0) and torch.all(torch.isneginf(lse))


def test_out_of_range_pages_read_zero_and_validate_aborts():
    spec = SPECS["g8_d128_head"]
    wl, db, oc = build_both(spec, seed=8)
    bt = wl.block_table.copy()
    bt[4, 3] = wl.num_pages + 5
    bt[5, 0] = -7
    wl.block_table = bt
    db.block_table = torch.from_numpy(bt).cuda()
    m = db.validate()
    ref = oracle.validate(oc.page_tags, bt, wl.expected_tags, wl.seq_lens, spec.page_size)
    torch.cuda.synchronize()
    assert np.array_equal(m.cpu().numpy(), ref) and ref[4] == 1 and ref[5] == 1
    out, lse = db.decode(use_abort=False)
    torch.cuda.synchronize()
    ro, rl = OS.decode(wl, oc)
    assert_decode_close(out, lse, ro.reshape(out.shape), rl.reshape(lse.shape))


def test_validate_random_bit_exact():
    r = np.random.default_rng(0)
    for trial in range(30):
        P, B, maxp, ps = int(r.integers(1, 3000)), int(r.integers(1, 40)), int(r.integers(1, 5000)), int(r.integers(1, 33))
        tags = r.integers(0, 3, P).astype(np.uint32)
        bt = r.integers(-2, P + 2, (B, maxp)).astype(np.int32)
        bt[r.random((B, maxp)) < 0.999] = r.integers(0, P, 1)[0]
        exp = tags[np.clip(bt, 0, P - 1)].copy()
        flip = r.random((B, maxp)) < 2e-4
        exp[flip] ^= 1
        lens = r.integers(-3, maxp * ps + 5, B).astype(np.int32)
        n_ab = torch.full((1,), 12345, dtype=torch.int32, device="cuda")   # zeroed by the call
        first = torch.empty(B, dtype=torch.int32, device="cuda")
        got = kvq.validate(torch.from_numpy(tags.view(np.int32)).cuda(), torch.from_numpy(bt).cuda(),
                           torch.from_numpy(exp.view(np.int32)).cuda(), torch.from_numpy(lens).cuda(), ps,
                           n_aborted=n_ab, first_bad=first)
        ref, ref_first = oracle.validate(tags, bt, exp, lens, ps, first_bad=True)
        assert np.array_equal(got.cpu().numpy(), ref), trial
        assert np.array_equal(first.cpu().numpy(), ref_first), trial
        assert int(n_ab.item()) == int(ref.sum()), trial


@pytest.mark.parametrize("B", [1, 4095, 4096, 4097, 6000])
def test_validate_batch_sizes_and_reset(B):
    """Batches on both sides of the flat / per-request-cluster switch, each
    checked after a failing call so that state carried between calls would
    show: failing, then clean, then failing again."""
    r = np.random.default_rng(B)
    P, maxp, ps = 5000, 6, 16
    tags = r.integers(0, 1 << 32, P, dtype=np.uint64).astype(np.uint32)
    bt = r.integers(0, P, (B, maxp)).astype(np.int32)
    lens = r.integers(0, maxp * ps + 1, B).astype(np.int32)
    clean = tags[bt].copy()
    stale = clean.copy()
    hit = r.integers(0, B, max(1, B // 50))
    stale[hit, r.integers(0, maxp, hit.size)] ^= 1
    dev = lambda a: torch.from_numpy(a).cuda()
    for exp in (stale, clean, stale):
        n_ab = torch.full((1,), -7, dtype=torch.int32, device="cuda")
        first = torch.full((B,), -9, dtype=torch.int32, device="cuda")
        got = kvq.validate(dev(tags.view(np.int32)), dev(bt), dev(exp.view(np.int32)), dev(lens), ps,
                           n_aborted=n_ab, first_bad=first)
        ref, ref_first = oracle.validate(tags, bt, exp, lens, ps, first_bad=True)
        assert np.array_equal(got.cpu().numpy(), ref)
        assert np.array_equal(first.cpu().numpy(), ref_first)
        assert int(n_ab.item()) == int(ref.sum())


@pytest.mark.parametrize("with_first_bad", [False, True])
def test_validate_graph_replays_with_changing_tags(with_first_bad):
    """One kvq_validate call captured in a CUDA graph and replayed with the
    expected tags changed between replays (stale entries in different
    requests, then none, then again): each replay's mask, abort count and
    first failing index equal the oracle's, so nothing of one replay's
    outcome leaks into the next."""
    r = np.random.default_rng(40)
    P, B, maxp, ps = 3000, 64, 40, 16
    tags = r.integers(0, 1 << 32, P, dtype=np.uint64).astype(np.uint32)
    bt = r.integers(0, P, (B, maxp)).astype(np.int32)
    lens = r.integers(0, maxp * ps + 1, B).astype(np.int32)
    clean = tags[bt].copy()
    dev = lambda a: torch.from_numpy(a).cuda()
    d_tags, d_bt, d_lens = dev(tags.view(np.int32)), dev(bt), dev(lens)
    d_exp = dev(clean.view(np.int32))
    mask = torch.empty(B, dtype=torch.uint8, device="cuda")
    n_ab = torch.full((1,), 77, dtype=torch.int32, device="cuda")
    first = torch.full((B,), 5, dtype=torch.int32, device="cuda") if with_first_bad else None
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        kvq.validate(d_tags, d_bt, d_exp, d_lens, ps, mask, stream, n_aborted=n_ab, first_bad=first)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            kvq.validate(d_tags, d_bt, d_exp, d_lens, ps, mask, stream, n_aborted=n_ab,
                         first_bad=first)
    for trial in range(12):
        exp = clean.copy()
        if trial % 3 != 1:
            hit = r.integers(0, B, int(r.integers(1, 6)))
            exp[hit, r.integers(0, maxp, hit.size)] ^= 1
        d_exp.copy_(torch.from_numpy(exp.view(np.int32)))
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        ref, ref_first = oracle.validate(tags, bt, exp, lens, ps, first_bad=True)
        assert np.array_equal(mask.cpu().numpy(), ref), trial
        assert int(n_ab.item()) == int(ref.sum()), trial
        if with_first_bad:
            assert np.array_equal(first.cpu().numpy(), ref_first), trial
    assert kvq.device_error() == 0


def test_validate_abort_count_without_first_bad():
    """The abort count alone (no per-request index requested), over calls in
    a row where the same requests fail again: each call counts each aborted
    request once."""
    r = np.random.default_rng(41)
    for trial in range(10):
        P, B, maxp, ps = 2000, int(r.integers(1, 300)), int(r.integers(1, 200)), 16
        tags = r.integers(0, 1 << 32, P, dtype=np.uint64).astype(np.uint32)
        bt = r.integers(-1, P + 1, (B, maxp)).astype(np.int32)
        lens = r.integers(0, maxp * ps + 1, B).astype(np.int32)
        exp = tags[np.clip(bt, 0, P - 1)].copy()
        exp[r.random((B, maxp)) < 0.01] ^= 1
        dev = lambda a: torch.from_numpy(a).cuda()
        for _ in range(2):
            n_ab = torch.full((1,), -3, dtype=torch.int32, device="cuda")
            got = kvq.validate(dev(tags.view(np.int32)), dev(bt), dev(exp.view(np.int32)),
                               dev(lens), ps, n_aborted=n_ab)
            ref = oracle.validate(tags, bt, exp, lens, ps)
            assert np.array_equal(got.cpu().numpy(), ref), trial
            assert int(n_ab.item()) == int(ref.sum()), trial
    assert kvq.device_error() == 0


def test_tag_bump_matches_oracle():
    P = 50
    tags = np.random.default_rng(1).integers(0, 2**32, P, dtype=np.uint64).astype(np.uint32)
    tags[3] = 0xFFFFFFFF
    realloc = np.array([3, 3, 7, -1, 50, 49, 0, 7, 7], np.int32)
    c = kvq.PagedCache(kvq.FP8_E4M3, kvq.SCALE_HEAD, P, 16, 1, 16, 16,
                       tags=torch.from_numpy(tags.view(np.int32)))
    kvq.append(c, torch.zeros((0, 1, 16), dtype=torch.bfloat16, device="cuda"),
               torch.zeros((0, 1, 16), dtype=torch.bfloat16, device="cuda"),
               torch.zeros(0, dtype=torch.int32, device="cuda"),
               realloc_pages=torch.from_numpy(realloc).cuda())
    oc = oracle.Cache(oracle.FP8, oracle.SCALE_HEAD, P, 16, 1, 16, 16,
                      np.zeros((P, 1, 16, 16), np.uint8), np.zeros((P, 1, 16, 16), np.uint8),
                      np.ones(1, np.float32), np.ones(1, np.float32), tags.copy())
    oracle.append(oc, np.zeros((0, 1, 16), np.uint16), np.zeros((0, 1, 16), np.uint16),
                  np.zeros(0, np.int32), realloc_pages=realloc)
    assert np.array_equal(c.page_tags.cpu().numpy().view(np.uint32), oc.page_tags)


def test_amax_chunked_and_nan():
    x = torch.randn(1000, 3, 64, device="cuda").to(torch.bfloat16)
    x[5, 1, 7] = float("nan")
    a = torch.zeros(3, device="cuda")
    for lo in range(0, 1000, 300):
        kvq.amax(x[lo:lo + 300].contiguous(), True, a)
    s = kvq.scale_from_amax(a)
    torch.cuda.synchronize()
    want = oracle.scales(OS.bf16_bits(x), per_head=True)
    assert np.array_equal(s.cpu().numpy(), want)
    s1 = kvq.scale_from_amax(kvq.amax(x, False))
    assert np.array_equal(s1.cpu().numpy(), oracle.scales(OS.bf16_bits(x), per_head=False))


def test_e4m3_encode_all_2_32_patterns():
    """Device conversion vs the oracle's integer-arithmetic encoder, every float bit pattern."""
    chunk = 1 << 28
    dev = torch.empty(chunk, dtype=torch.uint8, device="cuda")
    for i in range((1 << 32) // chunk):
        start = i * chunk
        kvq.e4m3_encode_bits(start, chunk, dev)
        ref = oracle.e4m3_encode_bits_range(start, chunk)
        got = dev.cpu().numpy()
        if not np.array_equal(got, ref):
            bad = np.nonzero(got != ref)[0][:5]
            raise AssertionError([(hex(start + int(j)), hex(got[j]), hex(ref[j])) for j in bad])


@pytest.mark.parametrize("scale", [3.7 / 448, 0.0123, 2.0 ** -6, 3.0e-11, 7.5e8, 2.0 ** -50])
def test_e4m3_quantize_division_all_2_32_patterns(scale):
    """The append's quantize step (device quotient and conversion) against the
    oracle's IEEE quotient and integer-arithmetic encoder, every float bit
    pattern: scales with inexact quotients, a power of two (exact ones), the
    edges of the division-free range and one outside it."""
    scale = float(np.float32(scale))
    chunk = 1 << 28
    dev = torch.empty(chunk, dtype=torch.uint8, device="cuda")
    for i in range((1 << 32) // chunk):
        start = i * chunk
        kvq.e4m3_quantize_bits(start, chunk, scale, dev)
        ref = oracle.e4m3_quantize_bits_range(start, chunk, scale)
        got = dev.cpu().numpy()
        if not np.array_equal(got, ref):
            bad = np.nonzero(got != ref)[0][:5]
            raise AssertionError([(hex(start + int(j)), hex(got[j]), hex(ref[j])) for j in bad])


def test_host_argument_errors():
    c = kvq.PagedCache(kvq.FP8_E4M3, kvq.SCALE_HEAD, 4, 16, 1, 128, 128)
    q = torch.zeros((1, 8, 128), dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros((1, 1), dtype=torch.int32, device="cuda")
    sl = torch.ones(1, dtype=torch.int32, device="cuda")
    with pytest.raises(kvq.KvqError) as e:
        kvq.decode(c, q, bt, sl, None, 1.0, workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))
    assert e.value.status == kvq.KVQ_ERR_WORKSPACE
    q7 = torch.zeros((1, 7, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(kvq.KvqError):
        kvq.decode(c, q7, bt, sl, None, 1.0, workspace=torch.empty(1 << 20, dtype=torch.uint8, device="cuda"))
    cb = kvq.PagedCache(kvq.BF16, kvq.SCALE_HEAD, 4, 16, 1, 128, 128)
    ws = kvq.alloc_workspace(cb, 1, 8)
    with pytest.raises(kvq.KvqError) as e:   # fp8 entry point on a bf16 cache
        kvq.lib().kvq_decode  # noqa: B018
        import ctypes
        st = kvq.lib().kvq_decode(ctypes.byref(cb.desc), ctypes.c_void_p(q.data_ptr()), 8,
                                  ctypes.c_void_p(bt.data_ptr()), 1, ctypes.c_void_p(sl.data_ptr()),
                                  1, None, ctypes.c_float(1.0), ctypes.c_void_p(q.data_ptr()), None,
                                  ctypes.c_void_p(ws.data_ptr()), ws.numel(), 0, None)
        kvq._check("kvq_decode", st)
    assert e.value.status == kvq.KVQ_ERR_INVALID_ARG


@pytest.mark.parametrize("mode", [kvq.SCALE_TENSOR, kvq.SCALE_HEAD, kvq.SCALE_TOKEN])
def test_append_every_bf16_pattern(mode):
    """Every bf16 bit pattern (zeros, subnormals, infinities, NaNs) through
    kvq_append, with scales inside and outside the range the division-free
    quotient covers, against the oracle's append: codes and scales bit-exact."""
    P, ps, H, D = 40, 16, 2, 128
    T = (1 << 16) // (H * D)                          # 256 tokens: each pattern once in K
    rng = np.random.default_rng(5)
    kb = np.arange(1 << 16, dtype=np.uint16).reshape(T, H, D)
    vb = rng.permutation(np.arange(1 << 16, dtype=np.uint16)).reshape(T, H, D)
    slots = rng.permutation(P * ps)[:T].astype(np.int32)
    slots[::37] = -1                                   # some tokens not stored
    if mode == kvq.SCALE_TENSOR:
        ks, vs = np.array([0.0123], np.float32), np.array([2.0 ** -50], np.float32)
    elif mode == kvq.SCALE_HEAD:
        ks = np.array([3.7 / 448, 1.0e13], np.float32)
        vs = np.array([2.0 ** -6, 1.0e-40], np.float32)   # the last one subnormal
    else:
        ks = vs = None
    c = kvq.PagedCache(kvq.FP8_E4M3, mode, P, ps, H, D, D)
    c.k_pages.fill_(0xCD)
    c.v_pages.fill_(0xCD)
    if ks is not None:
        c.k_scale.copy_(torch.from_numpy(ks))
        c.v_scale.copy_(torch.from_numpy(vs))
    kt = torch.from_numpy(kb.view(np.int16)).view(torch.bfloat16).cuda()
    vt = torch.from_numpy(vb.view(np.int16)).view(torch.bfloat16).cuda()
    kvq.append(c, kt, vt, torch.from_numpy(slots).cuda())
    torch.cuda.synchronize()
    sshape = (P, H, ps) if mode == kvq.SCALE_TOKEN else ks.shape
    oc = oracle.Cache(oracle.FP8, mode, P, ps, H, D, D,
                      np.full((P, H, ps, D), 0xCD, np.uint8), np.full((P, H, ps, D), 0xCD, np.uint8),
                      np.ones(sshape, np.float32) if ks is None else ks.copy(),
                      np.ones(sshape, np.float32) if vs is None else vs.copy(),
                      np.zeros(P, np.uint32))
    oracle.append(oc, kb, vb, slots)
    assert np.array_equal(c.k_pages.cpu().numpy(), oc.k_pages)
    assert np.array_equal(c.v_pages.cpu().numpy(), oc.v_pages)
    assert np.array_equal(c.k_scale.cpu().numpy().view(np.uint32), oc.k_scale.view(np.uint32))
    assert np.array_equal(c.v_scale.cpu().numpy().view(np.uint32), oc.v_scale.view(np.uint32))


@pytest.mark.parametrize("num_ctas", [0, 1000])
def test_single_long_sequence_split_into_many_pieces(num_ctas):
    """One 40,000-token sequence on one KV head: its 2,500 tiles go to 78
    CTAs of at least 32 tiles, so the one segment has 78 pieces and the
    combine merges them in two chunks, far more than one warp's worth of
    partials per head."""
    spec = W.Spec("one_long", [40000], 16, 8, 1, 128, 128, outlier_p=0.01)
    wl, db, oc = build_both(spec, seed=16, num_ctas=num_ctas)
    out, lse = db.step(check_tags=False)
    torch.cuda.synchronize()
    ro, rl = OS.decode(wl, oc)
    assert_decode_close(out, lse, ro.reshape(out.shape), rl.reshape(lse.shape), "one long")
    assert kvq.device_error() == 0


@pytest.mark.parametrize("num_ctas", [0, 5, 12, 20])
def test_equal_tile_counts_split_on_segment_edges(num_ctas):
    """Sequences of one tile count (126 tiles of 16 tokens each, ragged last
    tiles), 8 segments: with at least two CTAs per segment each segment gets
    its own CTAs (3 each by default, 2 at 20 CTAs); with 5 or 12 CTAs the
    split falls back to the stream-K ranges.  With a stale tag one row aborts
    and the plan redone after the wait is the stream-K one."""
    spec = W.Spec("even_tiles", [2001, 2002, 2016, 2010], 16, 16, 2, 128, 128,
                  outlier_p=0.01, n_stale=1)
    wl, db, oc = build_both(spec, seed=18, num_ctas=num_ctas)
    out, lse = db.step(check_tags=True)
    torch.cuda.synchronize()
    mask = db.abort.cpu().numpy()
    ref_mask = oracle.validate(oc.page_tags, wl.block_table, wl.expected_tags, wl.seq_lens,
                               wl.spec.page_size)
    assert np.array_equal(mask, ref_mask) and mask.sum() == 1
    ro, rl = OS.decode(wl, oc, abort=ref_mask)
    assert_decode_close(out, lse, ro.reshape(out.shape), rl.reshape(lse.shape), "aborted")
    out2, lse2 = db.decode(use_abort=False)
    ro2, rl2 = OS.decode(wl, oc, abort=None)
    assert_decode_close(out2, lse2, ro2.reshape(out.shape), rl2.reshape(lse.shape), "even")
    assert kvq.device_error() == 0


@pytest.mark.parametrize("num_ctas", [0, 1000])
def test_weighted_split_with_ctas_inside_a_segments_start(num_ctas):
    """A ragged batch (2,048 tiles and 1 tile on one KV head) with many CTAs:
    the weighted split charges each segment 48 extra units at its start, so
    with 1,000 CTAs the first CTAs' shares lie inside that charge and own no
    tile; the combine must skip them when it looks up a segment's pieces."""
    spec = W.Spec("weighted_empty", [32768, 16], 16, 8, 1, 128, 128, outlier_p=0.01)
    wl, db, oc = build_both(spec, seed=22, num_ctas=num_ctas)
    out, lse = db.step(check_tags=False)
    torch.cuda.synchronize()
    ro, rl = OS.decode(wl, oc)
    assert_decode_close(out, lse, ro.reshape(out.shape), rl.reshape(lse.shape), "weighted")
    assert kvq.device_error() == 0


def test_weighted_split_beyond_the_staged_starts():
    """More than 2,047 working CTAs over a ragged batch (two long sequences on
    two KV heads, 70,000 tiles, 2,100 CTAs): the combine searches the CTAs'
    starts in global memory instead of staging them."""
    spec = W.Spec("weighted_many_ctas", [300000, 260000], 16, 4, 2, 128, 128)
    wl, db, oc = build_both(spec, seed=23, num_ctas=2100, canary=False)
    out, lse = db.step(check_tags=False)
    torch.cuda.synchronize()
    ro, rl = OS.decode(wl, oc)
    assert_decode_close(out, lse, ro.reshape(out.shape), rl.reshape(lse.shape), "many ctas")
    assert kvq.device_error() == 0


def test_many_short_segments_group_1():
    """32 KV heads with one query head each and 520 short ragged rows (1..60
    tokens, head dim 64): 16,640 segments, each CTA's range crossing about
    fifty of them; two stale tags."""
    B = 520
    r = np.random.default_rng(20)
    lens = [int(x) for x in r.integers(1, 61, B)]
    spec = W.Spec(f"segs_{B}", lens, 16, 32, 32, 64, 64, n_stale=2)
    wl, db, oc = build_both(spec, seed=20)
    out, lse = db.step(check_tags=True)
    torch.cuda.synchronize()
    mask = db.abort.cpu().numpy()
    ref_mask = oracle.validate(oc.page_tags, wl.block_table, wl.expected_tags, wl.seq_lens,
                               wl.spec.page_size)
    assert np.array_equal(mask, ref_mask)
    ro, rl = OS.decode(wl, oc, abort=ref_mask)
    assert_decode_close(out, lse, ro.reshape(out.shape), rl.reshape(lse.shape), spec.name)
    assert kvq.device_error() == 0


def test_few_kv_heads_long_context_bf16_and_group_16():
    """B = 1 with four KV heads (about 74 pieces per segment at the default
    CTA count) on the BF16 cache, and a 16-head group on the FP8 cache."""
    for spec in (W.Spec("b1_bf16", [4096], 16, 32, 4, 128, 128, kv_dtype=W.BF16),
                 W.Spec("b1_g16", [3000], 16, 16, 1, 64, 64)):
        wl, db, oc = build_both(spec, seed=17)
        out, lse = db.step(check_tags=False)
        torch.cuda.synchronize()
        ro, rl = OS.decode(wl, oc)
        assert_decode_close(out, lse, ro.reshape(out.shape), rl.reshape(lse.shape), spec.name)
    assert kvq.device_error() == 0


def test_wide_single_long_sequence_many_pieces():
    """The tensor-core path with one 8,192-token sequence: 128 blocks of 64
    tokens over the default CTA pairs, one piece per pair."""
    spec = W.Spec("wide_one_long", [8192], 64, 128, 1, 576, 512, v_alias=True,
                  scale_mode=W.SCALE_TOKEN)
    wl, db, oc = build_both(spec, seed=18)
    out, lse = db.step(check_tags=False)
    torch.cuda.synchronize()
    ro, rl = OS.decode(wl, oc)
    assert_decode_close(out, lse, ro.reshape(out.shape), rl.reshape(lse.shape), "wide one long")
    assert kvq.device_error() == 0
