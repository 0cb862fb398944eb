"""fp64 CPU oracle for Kwai Summary Attention (KSA) -- test infrastructure.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it and
shares no code with it.  The arithmetic lives in ``ksa_oracle.c`` (plain C,
fp64); this module only compiles that file, marshals numpy arrays and strings
together the per-sequence calls of a packed (varlen) batch.

Citations are to "Kwai Summary Attention Technical Report": the augmented
sequence is section 2.2.1 Eq. (1); visibility is section 2.2.1 (summary rule)
and section 2.2.2 Eqs. (2)-(3); the attention is Eq. (10); the decode cache is
section 2.3.1 with Figure 4; a chunked prefill (ksa_prefill_chunk) is, by
definition, a range of rows of the prefill; KSA over an MLA latent cache
(section 3.2, Eq. (6)) is absorbed MLA written as multi-query attention over
the same slot map (mla_decode_image).  The prefill backward
(ksa_attention_bwd) is the textbook gradient of Eq. (10) under the same mask,
written in numpy.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ksa_oracle.c")
_SO = os.path.join(_HERE, "libksa_oracle.so")

_lib = None

_d = ctypes.POINTER(ctypes.c_double)
_i64 = ctypes.POINTER(ctypes.c_int64)
_u8 = ctypes.POINTER(ctypes.c_uint8)
_I64 = ctypes.c_int64
_I = ctypes.c_int


def build(force: bool = False) -> str:
    """Compile ksa_oracle.c into libksa_oracle.so (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", _SO + ".tmp", _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(_SO + ".tmp", _SO)
    return _SO


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        L.oracle_rope.argtypes = [_I64, _I, _I, _d, _i64, ctypes.c_double, _d]
        L.oracle_visible.argtypes = [_I64, _I, _I, _I, _I64, _I, _I64]
        L.oracle_visible.restype = _I
        L.oracle_aug_len.argtypes = [_I64, _I]
        L.oracle_aug_len.restype = _I64
        L.oracle_dense_mask.argtypes = [_I64, _I, _I, _u8]
        L.oracle_count_pairs.argtypes = [_I64, _I, _I]
        L.oracle_count_pairs.restype = _I64
        L.oracle_ksa_attention.argtypes = [_I64, _I, _I, _I, _I, _I, ctypes.c_double,
                                           _d, _d, _d, _d, _d, _d,
                                           _I64, _i64, _I64, _i64, _d, _d, _d, _d]
        L.oracle_cache_slots.argtypes = [_I, _I, _I64]
        L.oracle_cache_slots.restype = _I64
        L.oracle_cache_new.argtypes = [_I, _I, _I, _I, _I64]
        L.oracle_cache_new.restype = ctypes.c_void_p
        L.oracle_cache_free.argtypes = [ctypes.c_void_p]
        for nm in ("oracle_cache_k", "oracle_cache_v"):
            getattr(L, nm).argtypes = [ctypes.c_void_p]
            getattr(L, nm).restype = _d
        for nm in ("oracle_cache_n_text", "oracle_cache_m"):
            getattr(L, nm).argtypes = [ctypes.c_void_p]
            getattr(L, nm).restype = _I64
        L.oracle_cache_append_text.argtypes = [ctypes.c_void_p, _d, _d]
        L.oracle_cache_append_text.restype = _I
        L.oracle_cache_append_summary.argtypes = [ctypes.c_void_p, _d, _d]
        L.oracle_cache_append_summary.restype = _I
        L.oracle_cache_slice.argtypes = [ctypes.c_void_p, _I, _i64, _i64]
        L.oracle_cache_decode.argtypes = [ctypes.c_void_p, _I, _I, ctypes.c_double, _d, _d, _d]
        L.oracle_decode_image.argtypes = [_I, _I, _I, _I, _I64, _I64, _I64, _I, _d, _d,
                                          _I, ctypes.c_double, _d, _d, _d]
        _lib = L
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a: np.ndarray):
    if a is None:
        return None
    if a.dtype == np.float64:
        return a.ctypes.data_as(_d)
    if a.dtype == np.int64:
        return a.ctypes.data_as(_i64)
    if a.dtype == np.uint8:
        return a.ctypes.data_as(_u8)
    raise TypeError(a.dtype)


# --------------------------------------------------------------------------
# RoPE and positions
# --------------------------------------------------------------------------
def rope(x: np.ndarray, pos: np.ndarray, theta: float) -> np.ndarray:
    """Rotate-half RoPE in fp64.  x: [rows, heads, d]; pos: [rows]."""
    x = _f64(x)
    pos = np.ascontiguousarray(pos, dtype=np.int64)
    out = np.empty_like(x)
    lib().oracle_rope(x.shape[0], x.shape[1], x.shape[2], _p(x), _p(pos), float(theta), _p(out))
    return out


def text_positions(n: int) -> np.ndarray:
    """Text token t_i of a sequence has position id i (its local index)."""
    return np.arange(n, dtype=np.int64)


def summary_positions(n: int, k: int) -> np.ndarray:
    """Summary s_j takes the position id of its chunk's last text token, jk+k-1
    (section 2.2.1, second bullet after Eq. (1))."""
    m = n // k
    return np.arange(m, dtype=np.int64) * k + (k - 1)


# --------------------------------------------------------------------------
# Visibility
# --------------------------------------------------------------------------
def visible(n: int, k: int, C: int, q_kind: int, q_idx: int, key_kind: int, key_idx: int) -> bool:
    return bool(lib().oracle_visible(n, k, C, q_kind, q_idx, key_kind, key_idx))


def dense_mask(n: int, k: int, C: int) -> np.ndarray:
    """[L, L] uint8 mask over the augmented sequence of Eq. (1)."""
    L = int(lib().oracle_aug_len(n, k))
    out = np.zeros((L, L), dtype=np.uint8)
    lib().oracle_dense_mask(n, k, C, _p(out))
    return out


# --------------------------------------------------------------------------
# Prefill attention
# --------------------------------------------------------------------------
def ksa_attention(n, k, C, qt, kt, vt, qs, ks, vs, scale=None, tq_idx=None, sq_idx=None):
    """KSA attention of one sequence on already-RoPE'd fp64 inputs.

    qt [n, Hq, d], kt/vt [n, Hkv, d], qs [m, Hq, d], ks/vs [m, Hkv, d].
    Returns (ot, lse_t, os, lse_s) for the requested text / summary rows.
    """
    qt, kt, vt, qs, ks, vs = (_f64(a) for a in (qt, kt, vt, qs, ks, vs))
    Hq, d = qt.shape[1], qt.shape[2]
    Hkv = kt.shape[1]
    m = n // k
    assert qs.shape[0] == m and ks.shape[0] == m
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    tq = None if tq_idx is None else np.ascontiguousarray(tq_idx, dtype=np.int64)
    sq = None if sq_idx is None else np.ascontiguousarray(sq_idx, dtype=np.int64)
    ntq = n if tq is None else len(tq)
    nsq = m if sq is None else len(sq)
    ot = np.zeros((ntq, Hq, d))
    lt = np.zeros((ntq, Hq))
    os_ = np.zeros((nsq, Hq, d))
    ls = np.zeros((nsq, Hq))
    # empty arrays still need a valid pointer
    qs_ = qs if m > 0 else np.zeros((1, Hq, d))
    ks_ = ks if m > 0 else np.zeros((1, Hkv, d))
    vs_ = vs if m > 0 else np.zeros((1, Hkv, d))
    lib().oracle_ksa_attention(n, k, C, Hq, Hkv, d, float(scale),
                               _p(qt), _p(kt), _p(vt), _p(qs_), _p(ks_), _p(vs_),
                               ntq, _p(tq), nsq, _p(sq),
                               _p(ot) if ntq else None, _p(lt) if ntq else None,
                               _p(os_) if nsq else None, _p(ls) if nsq else None)
    return ot, lt, os_, ls


@dataclass
class SeqResult:
    text_o: np.ndarray      # [n_rows, Hq, d]
    text_lse: np.ndarray    # [n_rows, Hq]
    sum_o: np.ndarray       # [m_rows, Hq, d]
    sum_lse: np.ndarray     # [m_rows, Hq]
    text_rows: np.ndarray   # which text indices were computed
    sum_rows: np.ndarray    # which summary indices were computed


def ksa_prefill(seqlens, k, C, qt, kt, vt, qs, ks, vs, theta, scale=None,
                text_rows=None, sum_rows=None):
    """The whole prefill path for a packed batch, from un-rotated inputs.

    qt/kt/vt: [sum(n_b), H, d] text tensors packed by sequence;
    qs/ks/vs: [sum(floor(n_b/k)), H, d] summary tensors packed the same way.
    RoPE (theta; 0 disables it) is applied per sequence with text position i
    and summary position jk+k-1, then Eq. (10) under the KSA mask.
    text_rows / sum_rows: optional per-sequence index arrays to compute.
    Returns one SeqResult per sequence.
    """
    out = []
    t0 = s0 = 0
    for b, n in enumerate(seqlens):
        m = n // k
        sl_t = slice(t0, t0 + n)
        sl_s = slice(s0, s0 + m)
        q1, k1, v1 = _f64(qt[sl_t]), _f64(kt[sl_t]), _f64(vt[sl_t])
        q2, k2, v2 = _f64(qs[sl_s]), _f64(ks[sl_s]), _f64(vs[sl_s])
        if theta and theta > 0:
            pt, ps = text_positions(n), summary_positions(n, k)
            q1, k1 = rope(q1, pt, theta), rope(k1, pt, theta)
            if m:
                q2, k2 = rope(q2, ps, theta), rope(k2, ps, theta)
        tr = None if text_rows is None else text_rows[b]
        sr = None if sum_rows is None else sum_rows[b]
        ot, lt, os_, ls = ksa_attention(n, k, C, q1, k1, v1, q2, k2, v2, scale, tr, sr)
        out.append(SeqResult(ot, lt, os_, ls,
                             np.arange(n) if tr is None else np.asarray(tr),
                             np.arange(m) if sr is None else np.asarray(sr)))
        t0 += n
        s0 += m
    return out


# --------------------------------------------------------------------------
# Decode cache model
# --------------------------------------------------------------------------
TEXT, SUMMARY = 0, 1


def cache_slots(k: int, C: int, cap: int) -> int:
    return int(lib().oracle_cache_slots(k, C, cap))


class Cache:
    """One sequence's decode cache under the documented slot map."""

    def __init__(self, k: int, C: int, Hkv: int, d: int, cap: int):
        self.k, self.C, self.Hkv, self.d, self.cap = k, C, Hkv, d, cap
        self.S = cache_slots(k, C, cap)
        self._h = lib().oracle_cache_new(k, C, Hkv, d, cap)

    def __del__(self):
        if getattr(self, "_h", None):
            lib().oracle_cache_free(self._h)
            self._h = None

    @property
    def n_text(self) -> int:
        return int(lib().oracle_cache_n_text(self._h))

    @property
    def m(self) -> int:
        return int(lib().oracle_cache_m(self._h))

    def K(self) -> np.ndarray:
        p = lib().oracle_cache_k(self._h)
        return np.ctypeslib.as_array(p, shape=(self.S, self.Hkv, self.d)).copy()

    def V(self) -> np.ndarray:
        p = lib().oracle_cache_v(self._h)
        return np.ctypeslib.as_array(p, shape=(self.S, self.Hkv, self.d)).copy()

    def append_text(self, k_row, v_row) -> int:
        k_row, v_row = _f64(k_row), _f64(v_row)
        return int(lib().oracle_cache_append_text(self._h, _p(k_row), _p(v_row)))

    def append_summary(self, k_row, v_row) -> int:
        k_row, v_row = _f64(k_row), _f64(v_row)
        return int(lib().oracle_cache_append_summary(self._h, _p(k_row), _p(v_row)))

    def slice(self, kind: int):
        lo = ctypes.c_int64(0)
        hi = ctypes.c_int64(0)
        lib().oracle_cache_slice(self._h, kind, ctypes.byref(lo), ctypes.byref(hi))
        return int(lo.value), int(hi.value)

    def decode(self, kind: int, q, scale=None):
        q = _f64(q)
        Hq = q.shape[0]
        if scale is None:
            scale = 1.0 / np.sqrt(self.d)
        o = np.zeros((Hq, self.d))
        lse = np.zeros(Hq)
        lib().oracle_cache_decode(self._h, kind, Hq, float(scale), _p(q), _p(o), _p(lse))
        return o, lse


def decode_image(k, C, cap, n_text, m, kind, K, V, q, scale=None):
    """Decode against a cache image K/V [S, Hkv, d] (fp64) in the slot map."""
    K, V, q = _f64(K), _f64(V), _f64(q)
    S, Hkv, d = K.shape
    assert S == cache_slots(k, C, cap)
    Hq = q.shape[0]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    o = np.zeros((Hq, d))
    lse = np.zeros(Hq)
    lib().oracle_decode_image(k, C, Hkv, d, cap, n_text, m, kind, _p(K), _p(V),
                              Hq, float(scale), _p(q), _p(o), _p(lse))
    return o, lse


# --------------------------------------------------------------------------
# Prefill backward (gradients of Eq. (10) under the KSA mask)
# --------------------------------------------------------------------------
def aug_index(n: int, k: int) -> np.ndarray:
    """Rows of the padded augmented layout (chunk * (k+1) + slot, the layout
    of the CUDA library) that hold the n + floor(n/k) rows of Eq. (1), in
    Eq. (1) order (dense_mask's order)."""
    m = n // k
    idx = [c * (k + 1) + s for c in range(m) for s in range(k + 1)]
    idx += [m * (k + 1) + r for r in range(n - m * k)]
    return np.asarray(idx, dtype=np.int64)


def ksa_attention_bwd(n, k, C, q, kk, v, do, scale=None):
    """Gradients of the loss sum(do * o), o = softmax(scale q k^T + M_KSA) v
    (Eq. (10)), for one sequence.

    q, do [L, Hq, d] and kk, v [L, Hkv, d]: the L = n + floor(n/k) augmented
    rows of Eq. (1), already rotated (the tensors attention sees).  Query
    head h uses kv head h // (Hq / Hkv).  Returns (dq, dk, dv, o, lse) in
    fp64, written out from the definition: with P the masked softmax,
    dP = do v^T, D = rowsum(do * o), dS = P * (dP - D), dq = scale dS k,
    dk = scale dS^T q and dv = P^T do, the last two summed over the q heads
    that share a kv head.
    """
    q, kk, v, do = (_f64(a) for a in (q, kk, v, do))
    L, Hq, d = q.shape
    Hkv = kk.shape[1]
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    M = dense_mask(n, k, C).astype(bool)
    dq = np.zeros_like(q)
    dk = np.zeros_like(kk)
    dv = np.zeros_like(v)
    o = np.zeros_like(q)
    lse = np.zeros((L, Hq))
    for h in range(Hq):
        g = h // G
        S = scale * (q[:, h] @ kk[:, g].T)
        S = np.where(M, S, -np.inf)
        mx = S.max(axis=1, keepdims=True)
        E = np.exp(S - mx)
        den = E.sum(axis=1, keepdims=True)
        P = E / den
        o[:, h] = P @ v[:, g]
        lse[:, h] = (mx + np.log(den))[:, 0]
        dP = do[:, h] @ v[:, g].T
        D = (do[:, h] * o[:, h]).sum(axis=1)
        dS = P * (dP - D[:, None])
        dq[:, h] = scale * (dS @ kk[:, g])
        dk[:, g] += scale * (dS.T @ q[:, h])
        dv[:, g] += P.T @ do[:, h]
    return dq, dk, dv, o, lse


def ksa_prefill_bwd_aug(seqlens, k, C, q_aug, k_aug, v_aug, do_aug, scale=None):
    """ksa_attention_bwd over a packed batch in the padded augmented layout
    ([rows, H, d] with chunk * (k+1) + slot rows per sequence).  Returns
    (dq, dk, dv) in that layout; padding rows are zero."""
    q_aug, k_aug, v_aug, do_aug = (_f64(a) for a in (q_aug, k_aug, v_aug, do_aug))
    dq, dk, dv = np.zeros_like(q_aug), np.zeros_like(k_aug), np.zeros_like(v_aug)
    base = 0
    for n in seqlens:
        rows = base + aug_index(n, k)
        g = ksa_attention_bwd(n, k, C, q_aug[rows], k_aug[rows], v_aug[rows], do_aug[rows], scale)
        dq[rows], dk[rows], dv[rows] = g[0], g[1], g[2]
        base += ((n + k - 1) // k) * (k + 1)
    return dq, dk, dv


def visible_keys(n: int, k: int, C: int, a: int) -> np.ndarray:
    """Eq. (1) indices of the keys the query at Eq. (1) index a sees
    (section 2.2.1: a summary sees its chunk's text and itself; Eqs. (2)-(3):
    text t_i sees text t_{max(0, c-C)k} .. t_i and summaries s_j, j < c - C)."""
    m = n // k
    txt = lambda i: i + i // k                       # Eq. (1) index of text i
    if a < m * (k + 1) and a % (k + 1) == k:         # summary j
        j = a // (k + 1)
        return np.concatenate([txt(np.arange(j * k, j * k + k)), [a]]).astype(np.int64)
    i = a - min(a // (k + 1), m)                      # text token index
    c = i // k
    lo = max(0, c - C) * k
    summ = np.arange(0, max(0, min(c - C, m))) * (k + 1) + k
    return np.concatenate([summ, txt(np.arange(lo, i + 1))]).astype(np.int64)


def ksa_attention_bwd_dq_rows(n, k, C, q, kk, v, do, rows, scale=None):
    """dq of the given Eq. (1) query rows only (each row's gradient needs just
    its own visible keys): the same formulas as ksa_attention_bwd."""
    q, kk, v, do = (_f64(a) for a in (q, kk, v, do))
    Hq, d = q.shape[1], q.shape[2]
    G = Hq // kk.shape[1]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    out = np.zeros((len(rows), Hq, d))
    for r, a in enumerate(rows):
        keys = visible_keys(n, k, C, int(a))
        for h in range(Hq):
            g = h // G
            s = scale * (kk[keys, g] @ q[a, h])
            p = np.exp(s - s.max())
            p /= p.sum()
            o = p @ v[keys, g]
            dp = v[keys, g] @ do[a, h]
            ds = p * (dp - float(do[a, h] @ o))
            out[r, h] = scale * (ds @ kk[keys, g])
    return out


def seeing_queries(n: int, k: int, C: int, a: int) -> np.ndarray:
    """Eq. (1) indices of the queries that see the key at Eq. (1) index a:
    the visibility rules read from the key's side.  Summary s_j is seen by
    itself (section 2.2.1) and by every text t_i with j < c_i - C, that is
    i >= (j + C + 1) k (Eq. (3)).  Text t_p of chunk c_p is seen by the text
    t_i with p <= i and c_i - C <= c_p, that is p <= i < (c_p + C + 1) k
    (Eqs. (2)-(3)), and by its chunk's summary s_{c_p} when that chunk is
    complete (section 2.2.1)."""
    m = n // k
    txt = lambda i: i + i // k                       # Eq. (1) index of text i
    if a < m * (k + 1) and a % (k + 1) == k:         # summary j
        j = a // (k + 1)
        return np.concatenate([[a], txt(np.arange((j + C + 1) * k, n))]).astype(np.int64)
    p = a - min(a // (k + 1), m)                      # text token index
    c = p // k
    out = txt(np.arange(p, min(n, (c + C + 1) * k)))
    if c < m:
        out = np.concatenate([out, [c * (k + 1) + k]])
    return out.astype(np.int64)


def ksa_attention_bwd_dkv_keys(n, k, C, q, kk, v, do, keys, scale=None):
    """dk and dv of the given Eq. (1) key rows only: the same formulas as
    ksa_attention_bwd, summed over the query rows that see those keys.  Each
    such row needs its whole softmax row (its own visible keys) for P and
    D = rowsum(do * o); dk_a = scale sum_b dS_ba q_b and dv_a = sum_b P_ba
    do_b, over those rows b and the q heads of a's kv head.  Returns
    ([len(keys), Hkv, d], [len(keys), Hkv, d])."""
    q, kk, v, do = (_f64(a) for a in (q, kk, v, do))
    Hq, d = q.shape[1], q.shape[2]
    Hkv = kk.shape[1]
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    keys = np.asarray(keys, dtype=np.int64)
    out_of = np.full(q.shape[0], -1, dtype=np.int64)    # Eq. (1) index -> output row, -1 if not requested
    out_of[keys] = np.arange(len(keys))
    assert len(np.unique(keys)) == len(keys), "keys must be distinct"
    dk = np.zeros((len(keys), Hkv, d))
    dv = np.zeros((len(keys), Hkv, d))
    rows = np.unique(np.concatenate([seeing_queries(n, k, C, int(a)) for a in keys]))
    for b in rows:
        vis = visible_keys(n, k, C, int(b))
        at = np.flatnonzero(out_of[vis] >= 0)         # positions in vis of requested keys
        to = out_of[vis[at]]
        for g in range(Hkv):
            hs = slice(g * G, (g + 1) * G)
            Kb, Vb = kk[vis, g], v[vis, g]            # [nvis, d]
            S = scale * (Kb @ q[b, hs].T)             # [nvis, G]
            P = np.exp(S - S.max(axis=0))
            P /= P.sum(axis=0)
            O = P.T @ Vb                              # [G, d]
            dP = Vb @ do[b, hs].T                     # [nvis, G]
            D = (do[b, hs] * O).sum(axis=1)           # [G]
            dS = P * (dP - D)
            dk[to, g] += scale * (dS[at] @ q[b, hs])
            dv[to, g] += P[at] @ do[b, hs]
    return dk, dv


def interleave_rope_bwd(seqlens, k, theta, dq_aug, dk_aug, dv_aug):
    """Gradients of the text and summary projections from those of the
    augmented rows: the transpose of Eq. (1)'s interleave and of RoPE (an
    orthogonal rotation, so its transpose rotates by the opposite angle).
    Returns (dq_text, dk_text, dv_text, dq_sum, dk_sum, dv_sum), packed by
    sequence like the forward's inputs."""
    dq_aug, dk_aug, dv_aug = (_f64(a) for a in (dq_aug, dk_aug, dv_aug))
    out = [[], [], [], [], [], []]
    base = 0
    for n in seqlens:
        m = n // k
        i = np.arange(n)
        tr = base + (i // k) * (k + 1) + i % k
        sr = base + np.arange(m) * (k + 1) + k
        pt, ps = text_positions(n), summary_positions(n, k)
        neg = lambda x, pos: rope(x, -pos, theta) if theta and theta > 0 else x
        out[0].append(neg(dq_aug[tr], pt))
        out[1].append(neg(dk_aug[tr], pt))
        out[2].append(dv_aug[tr])
        out[3].append(neg(dq_aug[sr], ps) if m else dq_aug[sr])
        out[4].append(neg(dk_aug[sr], ps) if m else dk_aug[sr])
        out[5].append(dv_aug[sr])
        base += ((n + k - 1) // k) * (k + 1)
    return tuple(np.concatenate(x) for x in out)


# --------------------------------------------------------------------------
# Chunked prefill
# --------------------------------------------------------------------------
def ksa_prefill_chunk(n0, m0, T, k, C, qt, kt, vt, qs, ks, vs, theta, scale=None):
    """Rows of a block of T new text tokens appended to a sequence that holds
    n0 text tokens and m0 summaries (0 <= n0 - m0 k <= k): by definition the
    prefill rows (Eq. (10) under the KSA mask) of text positions n0 .. n0+T-1
    and of the summaries m0 .. m1-1, m1 = floor((n0+T)/k), of the sequence's
    first n0 + T tokens.  qt/kt/vt hold at least n0 + T text rows and qs/ks/vs
    at least m1 summary rows (not rotated).  Returns one SeqResult."""
    n1 = n0 + T
    m1 = n1 // k
    assert 0 <= n0 - m0 * k <= k and m0 <= m1
    return ksa_prefill([n1], k, C, qt[:n1], kt[:n1], vt[:n1], qs[:m1], ks[:m1], vs[:m1], theta, scale,
                       text_rows=[np.arange(n0, n1)], sum_rows=[np.arange(m0, m1)])[0]


# --------------------------------------------------------------------------
# KSA over an MLA latent cache (section 3.2, Eq. (6); MLA per section 3.1)
# --------------------------------------------------------------------------
def mla_kv_rows(lat, pos, theta, d_c):
    """K and V rows of absorbed MLA written as multi-query attention: a
    latent row [c (d_c), r (d_r)] gives K = [c, RoPE(r, pos)] and
    V = [c, 0] (the value is the latent; the zero tail keeps one row width).
    lat: [n, d_c + d_r] not rotated; pos: [n]."""
    lat = _f64(lat)
    K = lat.copy()
    if theta and theta > 0:
        K[:, d_c:] = rope(lat[:, None, d_c:], np.asarray(pos), theta)[:, 0]
    V = lat.copy()
    V[:, d_c:] = 0.0
    return K, V


def mla_query(q, pos, theta, d_c):
    """[q_c, RoPE(q_r, pos)] for q [H, d_c + d_r] of one query."""
    q = _f64(q).copy()
    if theta and theta > 0:
        q[:, d_c:] = rope(q[None, :, d_c:], np.asarray([pos]), theta)[0]
    return q


def mla_decode_image(k, C, cap, n_text, m, kind, lat_img, q, scale, theta, d_c=512):
    """Absorbed-MLA decode of one sequence against a latent cache image
    lat_img [S, d_c + d_r] (rope part already rotated) in the slot map:
    scores scale (q_c . c_j + RoPE(q_r) . r_j) over the slice the map makes
    visible, output sum_j p_j c_j.  q: [H, d_c + d_r], q_r not rotated
    (rotated at position n_text - 1).  Returns (o [H, d_c], lse [H])."""
    lat_img = _f64(lat_img)
    K = lat_img[:, None, :]
    V = lat_img.copy()
    V[:, d_c:] = 0.0
    qq = mla_query(q, n_text - 1, theta, d_c)
    o, lse = decode_image(k, C, cap, n_text, m, kind, K, V[:, None, :], qq, scale)
    return o[:, :d_c], lse
