"""GPU parity of ksa_prefill_bwd (gradients of Eq. (10) of the Kwai Summary
Attention Technical Report under the KSA mask, sections 2.2.1-2.2.2) against
the oracle's fp64 backward, over varlen batches with partial chunks, GQA,
w = 0, k = 1, a k that does not divide the 128-row tiles of the tensor-core
kernels (warp-level path), k = 128 (dk/dv steps of 128 queries instead of
64), k = 64 (a dk/dv step is one chunk) and a sequence long enough that the
summary key tiles' text queries are split over several CTAs; and
inconsistent cu_seqlens on both paths (error recorded, nothing written).

Tolerance: the kernels feed P and dS to the tensor cores in bf16 (relative
rounding 2^-9 each) and write bf16 gradients, accumulating in fp32, so the
gradients carry a few bf16 ulps of relative error: relative Frobenius error
<= 1e-2 per tensor and max-abs error <= 3e-2 of the tensor's largest entry."""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_compression_ksa_b200 import _lib as L
from kv_cache_compression_ksa_b200.inputs import prefill_inputs
from ksa_testutil import to_f64

pytestmark = pytest.mark.gpu
THETA = 1e6
REL_FROB = 1e-2
MAX_REL = 3e-2

CASES = [
    ("varlen_partial_chunks", [100, 37, 8, 3], 8, 2, 8, 2, 128, 11),
    ("k1_w0", [150, 41], 1, 0, 4, 4, 64, 13),
    ("k4_gqa4_w3", [300], 4, 3, 16, 4, 128, 12),
    ("long_summaries", [1500], 8, 4, 8, 2, 128, 15),
    ("k16_d64", [700, 333], 16, 2, 8, 4, 64, 17),
    ("k6_warp_path", [200, 50], 6, 2, 8, 2, 128, 19),          # k does not divide 128: warp-level dk/dv
    ("summary_shares", [2600, 300], 8, 1, 16, 2, 128, 23),     # 8 heads x 41 steps: summary tile 0 over two CTAs
    ("k128_steps_of_128", [700, 300], 128, 1, 4, 2, 128, 29),  # k does not divide 64: 128-query dk/dv steps
    ("k64_one_chunk_steps", [1300, 260], 64, 2, 8, 2, 128, 31),  # a dk/dv step is one chunk of 64 slots
]


def _check(name, got, want, live):
    g, w = got[live], want[live]
    err = np.linalg.norm(g - w) / max(np.linalg.norm(w), 1e-30)
    mx = np.abs(g - w).max() / max(np.abs(w).max(), 1e-30)
    assert err <= REL_FROB and mx <= MAX_REL, f"{name}: rel-Frob {err:.3e}, max-abs/max {mx:.3e}"


@pytest.mark.parametrize("name,seqlens,k,w,Hq,Hkv,d,seed", CASES, ids=[c[0] for c in CASES])
def test_prefill_bwd_matches_oracle(name, seqlens, k, w, Hq, Hkv, d, seed):
    dev = torch.device("cuda")
    x = prefill_inputs(seqlens, k, Hq, Hkv, d, seed=seed, device=dev)
    p = L.make_params(k, w, Hq, Hkv, d, 0.0, THETA)
    nt, ns = sum(seqlens), sum(n // k for n in seqlens)
    rows = L.ksa_aug_rows(p, seqlens)
    qa = torch.empty(rows, Hq, d, dtype=torch.bfloat16, device=dev)
    ka = torch.empty(rows, Hkv, d, dtype=torch.bfloat16, device=dev)
    va = torch.empty_like(ka)
    oa = torch.empty_like(qa)
    lse = torch.empty(rows, Hq, dtype=torch.float32, device=dev)
    ws = torch.empty(L.ksa_prefill_workspace_size(p, len(seqlens), nt), dtype=torch.uint8, device=dev)
    L.ksa_interleave_rope(p, x.cu_seqlens, nt, ns, rows, x.q_text, x.k_text, x.v_text, x.q_sum, x.k_sum, x.v_sum,
                          qa, ka, va, ws)
    L.ksa_prefill_fwd(p, x.cu_seqlens, nt, rows, qa, ka, va, oa, lse, ws)
    gen = torch.Generator(device=dev).manual_seed(seed + 100)
    do = torch.randn(rows, Hq, d, generator=gen, device=dev).to(torch.bfloat16)
    dq = torch.zeros_like(qa)
    dk = torch.zeros_like(ka)
    dv = torch.zeros_like(va)
    wsb = torch.empty(L.ksa_prefill_bwd_workspace_size(p, len(seqlens), rows), dtype=torch.uint8, device=dev)
    L.ksa_prefill_bwd(p, x.cu_seqlens, nt, rows, qa, ka, va, oa, lse, do, dq, dk, dv, wsb)
    torch.cuda.synchronize()
    assert L.ksa_get_device_error(wsb) == 0
    want = oracle.ksa_prefill_bwd_aug(seqlens, k, w, to_f64(qa), to_f64(ka), to_f64(va), to_f64(do))
    live = np.zeros(rows, bool)
    base = 0
    for n in seqlens:
        live[base + oracle.aug_index(n, k)] = True
        base += ((n + k - 1) // k) * (k + 1)
    _check(name + " dq", to_f64(dq), want[0], live)
    _check(name + " dk", to_f64(dk), want[1], live)
    _check(name + " dv", to_f64(dv), want[2], live)


@pytest.fixture(scope="module")
def full_size():
    """The 32768-token Qwen3-4B-layer prefill (32 q / 8 kv heads, d 128, k 8,
    w 8) and its backward through the library, with fp64 host copies of the
    tensors the oracle needs (n % k == 0: the padded layout has no padding
    rows and equals Eq. (1) order)."""
    dev = torch.device("cuda")
    seqlens, k, w, Hq, Hkv, d = [32768], 8, 8, 32, 8, 128
    x = prefill_inputs(seqlens, k, Hq, Hkv, d, seed=1, scale=0.5, device=dev)
    p = L.make_params(k, w, Hq, Hkv, d, 0.0, THETA)
    nt, ns = sum(seqlens), sum(n // k for n in seqlens)
    rows = L.ksa_aug_rows(p, seqlens)
    qa = torch.empty(rows, Hq, d, dtype=torch.bfloat16, device=dev)
    ka = torch.empty(rows, Hkv, d, dtype=torch.bfloat16, device=dev)
    va = torch.empty_like(ka)
    oa = torch.empty_like(qa)
    lse = torch.empty(rows, Hq, dtype=torch.float32, device=dev)
    ws = torch.empty(L.ksa_prefill_workspace_size(p, 1, nt), dtype=torch.uint8, device=dev)
    L.ksa_interleave_rope(p, x.cu_seqlens, nt, ns, rows, x.q_text, x.k_text, x.v_text, x.q_sum, x.k_sum, x.v_sum,
                          qa, ka, va, ws)
    L.ksa_prefill_fwd(p, x.cu_seqlens, nt, rows, qa, ka, va, oa, lse, ws)
    gen = torch.Generator(device=dev).manual_seed(7)
    do = torch.randn(rows, Hq, d, generator=gen, device=dev).to(torch.bfloat16)
    dq, dk, dv = torch.empty_like(qa), torch.empty_like(ka), torch.empty_like(va)
    wsb = torch.empty(L.ksa_prefill_bwd_workspace_size(p, 1, rows), dtype=torch.uint8, device=dev)
    L.ksa_prefill_bwd(p, x.cu_seqlens, nt, rows, qa, ka, va, oa, lse, do, dq, dk, dv, wsb)
    torch.cuda.synchronize()
    assert L.ksa_get_device_error(wsb) == 0
    return dict(n=seqlens[0], k=k, w=w, Hq=Hq, Hkv=Hkv, d=d, rows=rows, do_dev=do, dk_dev=dk, dv_dev=dv,
                q=to_f64(qa), kk=to_f64(ka), v=to_f64(va), do=to_f64(do), dq=to_f64(dq), dk=to_f64(dk),
                dv=to_f64(dv))


def test_prefill_bwd_full_size_identities_and_sampled_rows(full_size):
    """Per kv head the key gradients sum to zero and the value gradients sum
    to the output gradients of its q heads (exact for softmax attention;
    checked to 1e-2 of the summed magnitudes); sampled dq rows against the
    oracle's per-row backward."""
    F = full_size
    rows, Hq, Hkv, d = F["rows"], F["Hq"], F["Hkv"], F["d"]
    dkf, dvf, dof = F["dk_dev"].double(), F["dv_dev"].double(), F["do_dev"].double()
    sk = dkf.sum(0)
    assert (sk.abs().sum(-1) <= 1e-2 * dkf.abs().sum(0).sum(-1)).all()
    want_v = dof.view(rows, Hkv, Hq // Hkv, d).sum((0, 2))
    assert ((dvf.sum(0) - want_v).abs().sum(-1) <= 1e-2 * dvf.abs().sum(0).sum(-1)).all()
    # sampled dq rows (Eq. (1) order = the layout here): text rows early, mid
    # and late, and summary rows
    sample = np.array([0, 5, 80, 9 * 1000 + 3, 9 * 2047 + 8, 9 * 3000 + 4, rows - 2, rows - 1])
    want = oracle.ksa_attention_bwd_dq_rows(F["n"], F["k"], F["w"], F["q"], F["kk"], F["v"], F["do"], sample)
    got = F["dq"][sample]
    err = np.linalg.norm(got - want) / np.linalg.norm(want)
    assert err <= REL_FROB, f"sampled dq rel-Frob {err:.3e}"


# Per kv head, the first key of one summary tile (128 summaries s_j0 ..) and
# one text tile (128 text positions p0 ..) of the dk/dv kernel.  The summary
# tile j0 = 3456 is seen by 5048 text queries x 4 q heads, more than one CTA
# share of 256 steps of 64 queries, so its dk/dv is summed over two CTAs;
# the others fit one share.  Text tiles: the sequence start (window clipped),
# middle ones, and the end.
KEY_TILES = [(3968, 0), (3456, 128), (3968, 12800), (3840, 20480), (3968, 8192), (3968, 24576), (3840, 29952),
             (3968, 32640)]


def test_prefill_bwd_full_size_sampled_key_tiles(full_size):
    """dk and dv element by element on whole key tiles of the full-size
    backward, one summary tile and one text tile per kv head, against the
    oracle's per-key backward of the same kv head."""
    F = full_size
    k, G = F["k"], F["Hq"] // F["Hkv"]
    for g, (j0, p0) in enumerate(KEY_TILES):
        hs = slice(g * G, (g + 1) * G)
        kv = slice(g, g + 1)
        for name, keys in (("summary", np.arange(j0, j0 + 128) * (k + 1) + k),
                           ("text", np.arange(p0, p0 + 128) + np.arange(p0, p0 + 128) // k)):
            wk, wv = oracle.ksa_attention_bwd_dkv_keys(F["n"], k, F["w"], F["q"][:, hs], F["kk"][:, kv],
                                                       F["v"][:, kv], F["do"][:, hs], keys)
            live = np.ones(len(keys), bool)
            _check(f"kv head {g} {name} tile {keys[0]} dk", F["dk"][keys, g], wk[:, 0], live)
            _check(f"kv head {g} {name} tile {keys[0]} dv", F["dv"][keys, g], wv[:, 0], live)


@pytest.mark.parametrize("seqlens,k,w,Hq,Hkv,d", [([100, 37, 8, 3], 8, 2, 8, 2, 128), ([150, 41], 4, 1, 4, 4, 64)])
def test_training_chain_gradients_of_the_projections(seqlens, k, w, Hq, Hkv, d):
    """The whole prefill training step: text/summary projections -> RoPE +
    interleave -> attention -> loss sum(dO * O) and back through
    ksa_prefill_bwd and ksa_interleave_rope_bwd, against the oracle's chain
    (its own fp64 rotation of the same inputs, its backward, the transpose of
    the rotation)."""
    dev = torch.device("cuda")
    x = prefill_inputs(seqlens, k, Hq, Hkv, d, seed=21, device=dev)
    p = L.make_params(k, w, Hq, Hkv, d, 0.0, THETA)
    nt, ns = sum(seqlens), sum(n // k for n in seqlens)
    rows = L.ksa_aug_rows(p, seqlens)
    qa = torch.empty(rows, Hq, d, dtype=torch.bfloat16, device=dev)
    ka = torch.empty(rows, Hkv, d, dtype=torch.bfloat16, device=dev)
    va = torch.empty_like(ka)
    oa = torch.empty_like(qa)
    lse = torch.empty(rows, Hq, dtype=torch.float32, device=dev)
    ws = torch.empty(L.ksa_prefill_workspace_size(p, len(seqlens), nt), dtype=torch.uint8, device=dev)
    L.ksa_interleave_rope(p, x.cu_seqlens, nt, ns, rows, x.q_text, x.k_text, x.v_text, x.q_sum, x.k_sum, x.v_sum,
                          qa, ka, va, ws)
    L.ksa_prefill_fwd(p, x.cu_seqlens, nt, rows, qa, ka, va, oa, lse, ws)
    gen = torch.Generator(device=dev).manual_seed(22)
    do = torch.randn(rows, Hq, d, generator=gen, device=dev).to(torch.bfloat16)
    dqa, dka, dva = torch.zeros_like(qa), torch.zeros_like(ka), torch.zeros_like(va)
    wsb = torch.empty(L.ksa_prefill_bwd_workspace_size(p, len(seqlens), rows), dtype=torch.uint8, device=dev)
    L.ksa_prefill_bwd(p, x.cu_seqlens, nt, rows, qa, ka, va, oa, lse, do, dqa, dka, dva, wsb)
    outs = [torch.empty_like(t) for t in (x.q_text, x.k_text, x.v_text, x.q_sum, x.k_sum, x.v_sum)]
    L.ksa_interleave_rope_bwd(p, x.cu_seqlens, nt, ns, rows, dqa, dka, dva, *outs, ws)
    torch.cuda.synchronize()
    # the oracle's chain from the same bf16 inputs
    f64 = lambda t: to_f64(t)
    base = 0
    qa64, ka64, va64 = (np.zeros((rows, H, d)) for H in (Hq, Hkv, Hkv))
    t0 = s0 = 0
    for n in seqlens:
        m = n // k
        i = np.arange(n)
        tr = base + (i // k) * (k + 1) + i % k
        sr = base + np.arange(m) * (k + 1) + k
        pt, ps = oracle.text_positions(n), oracle.summary_positions(n, k)
        qa64[tr] = oracle.rope(f64(x.q_text[t0:t0 + n]), pt, THETA)
        ka64[tr] = oracle.rope(f64(x.k_text[t0:t0 + n]), pt, THETA)
        va64[tr] = f64(x.v_text[t0:t0 + n])
        if m:
            qa64[sr] = oracle.rope(f64(x.q_sum[s0:s0 + m]), ps, THETA)
            ka64[sr] = oracle.rope(f64(x.k_sum[s0:s0 + m]), ps, THETA)
            va64[sr] = f64(x.v_sum[s0:s0 + m])
        base += ((n + k - 1) // k) * (k + 1)
        t0 += n
        s0 += m
    g = oracle.ksa_prefill_bwd_aug(seqlens, k, w, qa64, ka64, va64, f64(do))
    want = oracle.interleave_rope_bwd(seqlens, k, THETA, *g)
    names = ["dq_text", "dk_text", "dv_text", "dq_sum", "dk_sum", "dv_sum"]
    for nm, got, wt in zip(names, outs, want):
        allrows = np.ones(wt.shape[0], bool)
        if wt.shape[0]:
            _check(nm, f64(got), wt, allrows)


def test_autograd_function_matches_the_library_chain():
    """KSAAttention (torch.autograd over the library) gives, bit for bit, the
    gradients of the explicit chain interleave -> prefill -> prefill_bwd ->
    interleave_bwd that test_training_chain_gradients_of_the_projections
    checks against the oracle; padding rows' incoming gradient is ignored."""
    from kv_cache_compression_ksa_b200.api import KSAAttention
    seqlens, k, w, Hq, Hkv, d = [37, 64, 5], 4, 2, 4, 2, 64
    dev = torch.device("cuda")
    x = prefill_inputs(seqlens, k, Hq, Hkv, d, seed=31, device=dev)
    p = L.make_params(k, w, Hq, Hkv, d, 0.0, THETA)
    ins = [t.clone().requires_grad_(True) for t in (x.q_text, x.k_text, x.v_text, x.q_sum, x.k_sum, x.v_sum)]
    o = KSAAttention.apply(p, seqlens, x.cu_seqlens, *ins)
    gen = torch.Generator(device=dev).manual_seed(32)
    G = torch.randn(o.shape, generator=gen, device=dev).to(torch.bfloat16)
    grads = torch.autograd.grad((o.float() * G.float()).sum(), ins)
    # the same chain through the C ABI
    nt, ns = sum(seqlens), sum(n // k for n in seqlens)
    rows = L.ksa_aug_rows(p, seqlens)
    qa = torch.empty(rows, Hq, d, dtype=torch.bfloat16, device=dev)
    ka = torch.empty(rows, Hkv, d, dtype=torch.bfloat16, device=dev)
    va, oa = torch.empty_like(ka), torch.empty_like(qa)
    lse = torch.empty(rows, Hq, dtype=torch.float32, device=dev)
    ws = torch.empty(L.ksa_prefill_workspace_size(p, len(seqlens), nt), dtype=torch.uint8, device=dev)
    L.ksa_interleave_rope(p, x.cu_seqlens, nt, ns, rows, x.q_text, x.k_text, x.v_text, x.q_sum, x.k_sum, x.v_sum,
                          qa, ka, va, ws)
    L.ksa_prefill_fwd(p, x.cu_seqlens, nt, rows, qa, ka, va, oa, lse, ws)
    dqa, dka, dva = torch.empty_like(qa), torch.empty_like(ka), torch.empty_like(va)
    wsb = torch.empty(L.ksa_prefill_bwd_workspace_size(p, len(seqlens), rows), dtype=torch.uint8, device=dev)
    L.ksa_prefill_bwd(p, x.cu_seqlens, nt, rows, qa, ka, va, oa, lse, G, dqa, dka, dva, wsb)
    want = [torch.empty_like(t) for t in ins]
    L.ksa_interleave_rope_bwd(p, x.cu_seqlens, nt, ns, rows, dqa, dka, dva, *want, ws)
    torch.cuda.synchronize()
    for g_, w_ in zip(grads, want):
        assert g_.dtype == torch.bfloat16 and g_.shape == w_.shape
        assert torch.equal(g_, w_)


@pytest.mark.parametrize("k", [8, 6])   # tensor-core path; warp-level path (6 does not divide 128)
def test_prefill_bwd_inconsistent_cu_seqlens_writes_nothing(k):
    """cu_seqlens that disagree with the host totals: the plan kernel records
    KSA_ERR_INVALID in the caller's error word and every kernel of the call
    returns before writing a gradient (the offsets it would use are wrong)."""
    w, Hq, Hkv, d = 2, 4, 2, 64
    p = L.make_params(k, w, Hq, Hkv, d, 0.0, THETA)
    dev = torch.device("cuda")
    n = 10 * k
    rows = L.ksa_aug_rows(p, [n])
    bad_cu = torch.tensor([0, n + k], dtype=torch.int32, device=dev)   # says n + k, the host says n
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    gen = torch.Generator(device=dev).manual_seed(7)
    qa = torch.randn(rows, Hq, d, generator=gen, device=dev).to(torch.bfloat16)
    ka = torch.randn(rows, Hkv, d, generator=gen, device=dev).to(torch.bfloat16)
    oa = torch.randn(rows, Hq, d, generator=gen, device=dev).to(torch.bfloat16)
    lse = torch.zeros(rows, Hq, dtype=torch.float32, device=dev)
    dq = torch.full((rows, Hq, d), 5.0, dtype=torch.bfloat16, device=dev)
    dk = torch.full((rows, Hkv, d), 5.0, dtype=torch.bfloat16, device=dev)
    dv = torch.full((rows, Hkv, d), 5.0, dtype=torch.bfloat16, device=dev)
    wsb = torch.empty(L.ksa_prefill_bwd_workspace_size(p, 1, rows), dtype=torch.uint8, device=dev)
    L.ksa_prefill_bwd(p, bad_cu, n, rows, qa, ka, ka, oa, lse, oa, dq, dk, dv, wsb, dev_err=err)
    assert L.ksa_get_device_error(err) == L.KSA_ERR_INVALID
    for t in (dq, dk, dv):
        assert torch.all(t == 5.0)
