"""GPU parity of ksa_interleave_rope and ksa_prefill_fwd against the fp64
oracle, through the C ABI (Kwai Summary Attention Technical Report, Eqs.
(1)-(3) and (10))."""
import math

import numpy as np
import pytest
import torch

import oracle
from kv_cache_compression_ksa_b200 import _lib as L
from kv_cache_compression_ksa_b200 import api
from kv_cache_compression_ksa_b200.inputs import prefill_inputs
from ksa_testutil import (LSE_ABS, assert_close, sample_rows, summary_rows, text_rows, to_f64)

pytestmark = pytest.mark.gpu

THETA = 1e6

# name, seqlens, k, w, Hq, Hkv, d, scale, seed
CASES = [
    ("small_d64_2q1kv", [256], 8, 2, 2, 1, 64, 1.0, 0),        # the small prefill case
    ("varlen_partial_chunks", [100, 37, 256, 3, 8], 8, 2, 8, 2, 128, 1.0, 11),
    ("k4_gqa4_w3", [300], 4, 3, 16, 4, 128, 0.5, 12),
    ("k1_w0", [150, 41], 1, 0, 4, 4, 64, 1.0, 13),
    ("k3_w1_ragged_tiles", [97, 64, 5], 3, 1, 4, 2, 128, 1.0, 14),
    ("two_summary_tiles", [2000], 8, 8, 32, 8, 128, 0.5, 15),
    ("window_covers_all", [200], 8, 100, 4, 1, 128, 1.0, 16),
    ("gqa8_k16", [700], 16, 2, 16, 2, 64, 1.0, 17),
    ("k16_gqa4_w8", [4096], 16, 8, 32, 8, 128, 1.0, 22),       # k ablation shapes of the report's Table 7
    ("k32_gqa4_w4", [1500, 333], 32, 4, 32, 8, 128, 1.0, 18),
    ("k64_gqa4_head_split", [2000, 130], 64, 2, 32, 8, 128, 1.0, 19),   # 4 heads x 64 slots > 128 rows
    ("k128_gqa8_head_split", [1300], 128, 1, 16, 2, 64, 1.0, 20),
    ("w128_k8", [3000], 8, 128, 8, 2, 128, 0.5, 21),           # the report's sliding chunk number
]


def run_gpu(seqlens, k, w, Hq, Hkv, d, scale, seed, want_lse=True):
    x = prefill_inputs(seqlens, k, Hq, Hkv, d, seed=seed, scale=scale, device="cpu")
    p = L.make_params(k, w, Hq, Hkv, d, 0.0, THETA)
    dev = torch.device("cuda")
    out = api.prefill(p, seqlens, x.cu_seqlens.to(dev), x.q_text.to(dev), x.k_text.to(dev), x.v_text.to(dev),
                      x.q_sum.to(dev), x.k_sum.to(dev), x.v_sum.to(dev), want_lse=want_lse)
    torch.cuda.synchronize()
    return x, out


def check_against_oracle(x, out, k, w, text_sel=None, sum_sel=None, tag=""):
    seqlens = x.seqlens
    ref = oracle.ksa_prefill(seqlens, k, w, to_f64(x.q_text), to_f64(x.k_text), to_f64(x.v_text),
                             to_f64(x.q_sum), to_f64(x.k_sum), to_f64(x.v_sum), THETA,
                             text_rows=text_sel, sum_rows=sum_sel)
    o = to_f64(out.o_aug)
    lse = to_f64(out.lse)
    got_t, want_t, got_s, want_s, lt_g, lt_w, ls_g, ls_w = [], [], [], [], [], [], [], []
    for b, r in enumerate(ref):
        rows = text_rows(seqlens, k, b, r.text_rows)
        got_t.append(o[rows]); want_t.append(r.text_o)
        lt_g.append(lse[rows]); lt_w.append(r.text_lse)
        if len(r.sum_rows):
            srows = summary_rows(seqlens, k, b, r.sum_rows)
            got_s.append(o[srows]); want_s.append(r.sum_o)
            ls_g.append(lse[srows]); ls_w.append(r.sum_lse)
    assert_close(np.concatenate(got_t), np.concatenate(want_t), f"{tag} text O")
    assert_close(np.concatenate(lt_g), np.concatenate(lt_w), f"{tag} text LSE", max_abs=LSE_ABS, rel_frob=None)
    if got_s:
        assert_close(np.concatenate(got_s), np.concatenate(want_s), f"{tag} summary O")
        assert_close(np.concatenate(ls_g), np.concatenate(ls_w), f"{tag} summary LSE", max_abs=LSE_ABS,
                     rel_frob=None)


@pytest.mark.parametrize("name,seqlens,k,w,Hq,Hkv,d,scale,seed", CASES, ids=[c[0] for c in CASES])
def test_prefill_matches_oracle(name, seqlens, k, w, Hq, Hkv, d, scale, seed):
    x, out = run_gpu(seqlens, k, w, Hq, Hkv, d, scale, seed)
    check_against_oracle(x, out, k, w, tag=name)


@pytest.mark.parametrize("name,seqlens,k,w,Hq,Hkv,d,scale,seed", CASES[:5], ids=[c[0] for c in CASES[:5]])
def test_interleave_rope_matches_oracle(name, seqlens, k, w, Hq, Hkv, d, scale, seed):
    """Eq. (1) layout with RoPE at text position i / summary position jk+k-1;
    V is a bit-exact copy, Q and K within one bf16 rounding of the fp64
    rotation; padding rows are zero."""
    x, out = run_gpu(seqlens, k, w, Hq, Hkv, d, scale, seed, want_lse=False)
    qa, ka, va = to_f64(out.q_aug), to_f64(out.k_aug), to_f64(out.v_aug)
    live = np.zeros(qa.shape[0], bool)
    t0 = s0 = 0
    for b, n in enumerate(seqlens):
        m = n // k
        tr = text_rows(seqlens, k, b, np.arange(n))
        sr = summary_rows(seqlens, k, b, np.arange(m))
        live[tr] = True
        live[sr] = True
        pt, ps = oracle.text_positions(n), oracle.summary_positions(n, k)
        for got, raw, pos, rows in ((qa, x.q_text[t0:t0 + n], pt, tr), (ka, x.k_text[t0:t0 + n], pt, tr),
                                    (qa, x.q_sum[s0:s0 + m], ps, sr), (ka, x.k_sum[s0:s0 + m], ps, sr)):
            if len(rows) == 0:
                continue
            want = oracle.rope(to_f64(raw), pos, THETA)
            err = np.abs(got[rows] - want)
            assert np.all(err <= 2.0 ** -8 * np.abs(want) + 1e-5), f"{name}: rope err {err.max()}"
        np.testing.assert_array_equal(va[tr], to_f64(x.v_text[t0:t0 + n]))
        if m:
            np.testing.assert_array_equal(va[sr], to_f64(x.v_sum[s0:s0 + m]))
        t0 += n
        s0 += m
    for t in (qa, ka, va):
        assert np.all(t[~live] == 0)


@pytest.mark.parametrize("seqlens,k,w,Hq,Hkv", [([100], 8, 2, 4, 1), ([37, 5, 50], 4, 1, 2, 2),
                                                ([40, 50], 3, 0, 8, 1), ([64], 64, 0, 8, 2)])
def test_visible_set_bit_exact_one_hot(seqlens, k, w, Hq, Hkv):
    """Q = K = 0 makes the softmax uniform over the visible keys; V of the key
    at augmented row a is e_a.  The output row is then nonzero exactly on the
    keys the rule makes visible: compared bit for bit with the oracle's
    dense mask of every sequence."""
    d = 128
    p = L.make_params(k, w, Hq, Hkv, d, 0.0, THETA)
    rows_total = L.ksa_aug_rows(p, seqlens)
    assert rows_total <= d
    x = prefill_inputs(seqlens, k, Hq, Hkv, d, seed=3)
    for t in (x.q_text, x.k_text, x.q_sum, x.k_sum, x.v_text, x.v_sum):
        t.zero_()
    t0 = s0 = 0
    for b, n in enumerate(seqlens):
        m = n // k
        tr = text_rows(seqlens, k, b, np.arange(n))
        sr = summary_rows(seqlens, k, b, np.arange(m))
        for i in range(n):
            x.v_text[t0 + i, :, tr[i]] = 1
        for j in range(m):
            x.v_sum[s0 + j, :, sr[j]] = 1
        t0 += n
        s0 += m
    dev = torch.device("cuda")
    out = api.prefill(p, seqlens, x.cu_seqlens.to(dev), x.q_text.to(dev), x.k_text.to(dev), x.v_text.to(dev),
                      x.q_sum.to(dev), x.k_sum.to(dev), x.v_sum.to(dev))
    o = to_f64(out.o_aug)
    for b, n in enumerate(seqlens):
        mask = oracle.dense_mask(n, k, w)          # [L_b, L_b] in the sequence's own order
        m = n // k
        # the sequence's augmented rows in the library layout, in Eq. (1) order
        aug_of_local = []
        for a in range(n + m):
            j, r = divmod(a, k + 1)
            if r < k:
                aug_of_local.append(text_rows(seqlens, k, b, [j * k + r])[0])
            else:
                aug_of_local.append(summary_rows(seqlens, k, b, [j])[0])
        aug_of_local = np.array(aug_of_local)
        for a in range(n + m):
            R = aug_of_local[a]
            want = np.zeros(d)
            want[aug_of_local[mask[a] == 1]] = 1
            for h in range(Hq):
                got_nz = (o[R, h] != 0).astype(int)
                np.testing.assert_array_equal(got_nz, want.astype(int))
                cnt = int(mask[a].sum())
                expect = float(torch.tensor(1.0 / cnt).to(torch.bfloat16).double())
                np.testing.assert_array_equal(o[R, h][want == 1], expect)


def closed_form_counts(n, k, w):
    i = np.arange(n)
    c = i // k
    lo = np.maximum(c - w, 0) * k
    m = n // k
    text = (i - lo + 1) + np.clip(c - w, 0, m)
    return text, np.full(m, k + 1)


@pytest.mark.parametrize("seqlens,k,w,Hq,Hkv,d", [
    ([32768], 8, 8, 32, 8, 128),                          # Qwen3-4B-shaped prefill
    ([131072, 65536, 16384, 4000], 8, 16, 32, 8, 128),    # long varlen batch
    ([131072, 65536, 16384, 4003], 8, 16, 32, 8, 128),    # with a trailing partial chunk
])
def test_visible_counts_full_size(seqlens, k, w, Hq, Hkv, d):
    """At full size: with Q = K = 0 every visible key scores 0, so
    LSE = ln(#visible keys).  The count recovered from every row's LSE equals
    the closed form of Eqs. (2)-(3) exactly."""
    p = L.make_params(k, w, Hq, Hkv, d, 0.0, THETA)
    dev = torch.device("cuda")
    nt = sum(seqlens)
    ns = sum(n // k for n in seqlens)
    z = lambda r, h: torch.zeros(r, h, d, dtype=torch.bfloat16, device=dev)
    v1 = lambda r, h: torch.ones(r, h, d, dtype=torch.bfloat16, device=dev)
    cu = torch.tensor([0] + list(np.cumsum(seqlens)), dtype=torch.int32, device=dev)
    out = api.prefill(p, seqlens, cu, z(nt, Hq), z(nt, Hkv), v1(nt, Hkv), z(ns, Hq), z(ns, Hkv), v1(ns, Hkv))
    lse = out.lse.double().cpu().numpy()
    o = out.o_aug.double().cpu().numpy()
    for b, n in enumerate(seqlens):
        tc, sc = closed_form_counts(n, k, w)
        tr = text_rows(seqlens, k, b, np.arange(n))
        got = np.rint(np.exp(lse[tr]))
        np.testing.assert_array_equal(got, np.repeat(tc[:, None], Hq, 1))
        if len(sc):
            sr = summary_rows(seqlens, k, b, np.arange(len(sc)))
            np.testing.assert_array_equal(np.rint(np.exp(lse[sr])), np.repeat(sc[:, None], Hq, 1))
        assert np.all(o[tr] == 1.0)


@pytest.mark.parametrize("seqlens,w,scale,seed,nsample", [
    ([32768], 8, 0.5, 1, 160),
    ([131072, 65536, 16384, 4000], 16, 1.0, 2, 48),     # the long varlen batch as written
    ([131072, 65536, 16384, 4003], 16, 1.0, 2, 48),     # with a trailing partial chunk
])
def test_prefill_full_size_sampled(seqlens, w, scale, seed, nsample):
    """Full-size workloads in the benchmark's launch configuration, checked on
    sampled rows the oracle computes one by one (spread over every sequence,
    including its first and last rows)."""
    k, Hq, Hkv, d = 8, 32, 8, 128
    dev = torch.device("cuda")
    x = prefill_inputs(seqlens, k, Hq, Hkv, d, seed=seed, scale=scale, device="cuda")
    p = L.make_params(k, w, Hq, Hkv, d, 0.0, THETA)
    out = api.prefill(p, seqlens, x.cu_seqlens, x.q_text, x.k_text, x.v_text, x.q_sum, x.k_sum, x.v_sum)
    torch.cuda.synchronize()
    tsel = [sample_rows(n, nsample, seed + b) for b, n in enumerate(seqlens)]
    ssel = [sample_rows(n // k, max(8, nsample // 4), seed + 7 * b) for b, n in enumerate(seqlens)]
    check_against_oracle(x, out, k, w, tsel, ssel, tag=f"full {seqlens}")


def test_device_error_on_inconsistent_cu_seqlens():
    """cu_seqlens that disagree with the host totals: the plan kernel records
    KSA_ERR_INVALID in the caller's error word and nothing is computed."""
    k, w, Hq, Hkv, d = 8, 2, 4, 1, 64
    p = L.make_params(k, w, Hq, Hkv, d, 0.0, THETA)
    dev = torch.device("cuda")
    seqlens = [64]
    x = prefill_inputs(seqlens, k, Hq, Hkv, d, seed=5, device="cuda")
    rows = L.ksa_aug_rows(p, seqlens)
    bad_cu = torch.tensor([0, 72], dtype=torch.int32, device=dev)  # says 72, host says 64
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    ws = torch.empty(L.ksa_prefill_workspace_size(p, 1, 64), dtype=torch.uint8, device=dev)
    o = torch.full((rows, Hq, d), 7.0, dtype=torch.bfloat16, device=dev)
    qa = torch.zeros(rows, Hq, d, dtype=torch.bfloat16, device=dev)
    ka = torch.zeros(rows, Hkv, d, dtype=torch.bfloat16, device=dev)
    L.ksa_prefill_fwd(p, bad_cu, 64, rows, qa, ka, ka, o, None, ws, dev_err=err)
    assert L.ksa_get_device_error(err) == L.KSA_ERR_INVALID
    assert L.ksa_get_device_error(err) == L.KSA_OK  # read-and-clear
    assert torch.all(o == 7.0)
