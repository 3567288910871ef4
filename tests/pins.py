"""Pins of the CPU oracle: checks against facts that do not come from the oracle itself.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises ``AssertionError`` when
the oracle disagrees with what the pages and the mathematics fix:

* identities (the XOR/popcount form of the +-1 dot product, Hamming-distance
  similarity: every page's technical summary, section "theoretical motivation");
* library routines on special cases (``numpy.packbits``, ``numpy.mean``, float64 matmul);
* brute force over every sign pattern of a tiny head dimension;
* statistical laws (E|x| of a standard normal, Sheppard's arcsine law for sign
  correlations, which is the covariance content of the pages' Theorem 1);
* hand-derived closed forms of the quantised forward pass (``tests/golden/closed_forms.json``);
* a deterministic error bound against float64 softmax attention on the scaled binary logits.

The same functions are run against deliberately broken copies of the oracle in
``test_oracle_mutants.py``: every plausible mistake must fail at least one of them.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

import oracle as oracle_mod

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_forms.json")


def _rng(seed):
    return np.random.default_rng(seed)


def _signs(x):
    return np.where(x < 0, -1.0, 1.0)


def _ref_bits(x):
    """Independent packing: numpy.packbits of (x < 0), little bit order, 16 bytes per row."""
    d = x.shape[-1]
    flat = (x.reshape(-1, d) < 0)
    by = np.packbits(flat, axis=1, bitorder="little")
    pad = np.zeros((by.shape[0], 16 - by.shape[1]), np.uint8)
    return np.concatenate([by, pad], 1).view("<u4").reshape(x.shape[:-1] + (4,))


# --------------------------------------------------------------------------- signs
def pin_pack_signs_special_values(o: oracle_mod.Oracle):
    """Bit = (x < 0): -0.0, +0.0 and NaN give 0; subnormals and infinities keep their sign."""
    special = np.array([0.0, -0.0, np.nan, -np.nan, np.inf, -np.inf, 1e-45, -1e-45, 1e-38, -1e-38,
                        65504.0, -65504.0, 1.0, -1.0, 0.5, -0.5], np.float32)
    rng = _rng(0)
    for d in (1, 16, 31, 32, 33, 64, 72, 127, 128):
        x = rng.choice(special, size=(3, 7, d)).astype(np.float32)
        got = o.pack_signs(x)
        want = _ref_bits(x)
        assert np.array_equal(got, want), f"pack_signs differs from packbits at d={d}"


def pin_pack_signs_random(o: oracle_mod.Oracle):
    rng = _rng(1)
    for d in (5, 64, 72, 100, 128):
        x = rng.standard_normal((2, 3, 11, d)).astype(np.float32)
        assert np.array_equal(o.pack_signs(x), _ref_bits(x)), d
        neg = -np.abs(x) - 1e-3
        bits = o.pack_signs(neg).reshape(-1, 4)
        full = np.zeros(4, np.uint64)
        for c in range(d):
            full[c // 32] |= np.uint64(1) << np.uint64(c % 32)
        assert np.array_equal(bits, np.broadcast_to(full.astype(np.uint32), bits.shape)), "all-negative row"


# --------------------------------------------------------------------------- mu
def pin_mu_closed_forms(o: oracle_mod.Oracle):
    rng = _rng(2)
    x = np.where(rng.random((2, 3, 17, 40)) < 0.5, -1.0, 1.0).astype(np.float32)
    assert np.array_equal(o.mu(x), np.ones((2, 3), np.float32)), "|x| = 1 gives mu = 1"
    c = np.full((1, 2, 9, 8), -0.375, np.float32)
    assert np.array_equal(o.mu(c), np.full((1, 2), 0.375, np.float32)), "constant input"
    y = rng.standard_normal((2, 2, 33, 72)).astype(np.float32) * 3.0
    want = np.mean(np.abs(y.astype(np.float64)), axis=(2, 3)).astype(np.float32)
    assert np.array_equal(o.mu(y), want), "mean |x| over tokens and channels per (b,h)"
    # statistical: E|z| = sqrt(2/pi) for z ~ N(0,1)
    z = rng.standard_normal((1, 1, 4096, 64)).astype(np.float32)
    assert abs(float(o.mu(z)[0, 0]) - math.sqrt(2 / math.pi)) < 4 * 0.6 / math.sqrt(z.size)


# --------------------------------------------------------------------------- logits
def pin_logits_identity(o: oracle_mod.Oracle):
    """x_ij = d - 2 popc(s_i xor t_j) equals the float64 dot product of the +-1 vectors."""
    rng = _rng(3)
    for d in (1, 7, 31, 32, 33, 64, 72, 128):
        q = rng.standard_normal((2, 2, 13, d)).astype(np.float32)
        k = rng.standard_normal((2, 2, 11 + 2, d)).astype(np.float32)
        k = k[:, :, :13]
        x = o.logits(o.pack_signs(q), o.pack_signs(k), d)
        want = np.einsum("bhic,bhjc->bhij", _signs(q), _signs(k))
        assert np.array_equal(x, want.astype(np.int32)), f"identity fails at d={d}"


def pin_logits_bruteforce(o: oracle_mod.Oracle):
    """Every pair of sign patterns at d = 6: the similarity is sum_c s_c t_c."""
    d = 6
    pats = np.array([[(-1.0 if (p >> c) & 1 else 1.0) for c in range(d)] for p in range(2 ** d)],
                    np.float32)
    q = pats.reshape(1, 1, -1, d)
    x = o.logits(o.pack_signs(q), o.pack_signs(q), d)[0, 0]
    for a in range(2 ** d):
        for b in range(2 ** d):
            dot = sum(int(pats[a, c]) * int(pats[b, c]) for c in range(d))
            if x[a, b] != dot:
                raise AssertionError(f"pattern pair ({a},{b}): {x[a, b]} != {dot}")


def pin_logits_arcsine(o: oracle_mod.Oracle):
    """Sheppard's law: for unit Gaussians with correlation rho, E[sign(q) sign(k)] = (2/pi) asin(rho)."""
    rng = _rng(4)
    d, n = 64, 2048
    for rho in (-0.8, -0.3, 0.0, 0.5, 0.9):
        a = rng.standard_normal((n, d))
        b = rho * a + math.sqrt(1 - rho * rho) * rng.standard_normal((n, d))
        q = a.astype(np.float32).reshape(1, n, 1, d)
        k = b.astype(np.float32).reshape(1, n, 1, d)
        x = o.logits(o.pack_signs(q), o.pack_signs(k), d).reshape(n)
        est = x.mean() / d
        want = 2 / math.pi * math.asin(rho)
        assert abs(est - want) < 5 / math.sqrt(n * d), f"rho={rho}: {est} vs {want}"


# --------------------------------------------------------------------------- V quantiser
def pin_quant_v_closed_forms(o: oracle_mod.Oracle):
    B, H, N, d = 1, 2, 9, 6
    v = np.zeros((B, H, N, d), np.float32)
    v[0, 0, :, 0] = 0.75                      # constant positive channel
    v[0, 0, :, 1] = -2.0                      # constant negative channel
    v[0, 0, :, 2] = 0.0                       # zero channel
    v[0, 1, :, 3] = np.arange(N) - 4.0        # amax 4 at both ends
    v[0, 1, :, 4] = [127.0, 2.5, 3.5, -2.5, -3.5, 0.5, 1.5, -0.5, 0.0]   # inv = 1: ties
    vq, sv = o.quant_v(v)
    assert np.all(vq[0, 0, :, 0] == 127) and sv[0, 0, 0] == np.float32(0.75) / np.float32(127)
    assert np.all(vq[0, 0, :, 1] == -127) and sv[0, 0, 1] == np.float32(2.0) / np.float32(127)
    assert np.all(vq[0, 0, :, 2] == 0) and sv[0, 0, 2] == 0.0, "zero channel"
    assert vq[0, 1, 0, 3] == -127 and vq[0, 1, N - 1, 3] == 127, "amax entries map to +-127"
    assert list(vq[0, 1, :, 4]) == [127, 2, 4, -2, -4, 0, 2, 0, 0], "round half to even"
    assert sv[0, 1, 4] == np.float32(1.0)
    # A channel whose 127 / amax overflows fp32 (amax < 127 / FLT_MAX) is a zero channel; one
    # just above that bound still maps its amax entries to +-127.
    w = np.zeros((1, 1, 4, 2), np.float32)
    w[0, 0, :, 0] = [1e-38, 0.0, -5e-39, 2e-39]
    w[0, 0, :, 1] = [4e-37, 0.0, -4e-37, 2e-37]
    wq, ws = o.quant_v(w)
    assert np.all(wq[0, 0, :, 0] == 0) and ws[0, 0, 0] == 0.0, "overflowing 127/amax: zero channel"
    assert list(wq[0, 0, :, 1]) == [127, 0, -127, 64] and ws[0, 0, 1] == np.float32(4e-37) / np.float32(127)


def pin_quant_v_invariants(o: oracle_mod.Oracle):
    rng = _rng(5)
    v = (rng.standard_normal((2, 3, 37, 72)) * rng.uniform(0.01, 10, (1, 1, 1, 72))).astype(np.float32)
    vq, sv = o.quant_v(v)
    vh = vq.astype(np.float64) * sv[:, :, None, :].astype(np.float64)
    err = np.abs(vh - v.astype(np.float64))
    assert np.all(err <= sv[:, :, None, :] * 0.5 * (1 + 1e-5) + 1e-30), "|v^ - v| <= sv/2"
    assert np.all(np.abs(vq.astype(np.int32)).max(axis=2) == 127), "each channel reaches +-127"
    amax = np.abs(v).max(axis=2)
    assert np.array_equal(sv, (amax / np.float32(127)).astype(np.float32)), "scale = amax / 127"
    vq2, sv2 = o.quant_v(v * np.float32(4.0))
    assert np.array_equal(vq2, vq) and np.array_equal(sv2, sv * np.float32(4.0)), "power-of-two scaling"


# --------------------------------------------------------------------------- bias
def pin_relpos_bias(o: oracle_mod.Oracle):
    """A one-hot table at (dy, dx) yields 1 exactly where (y_i - y_j, x_i - x_j) = (dy, dx);
    prefix rows and columns are 0; the diagonal reads the table centre."""
    gh, gw, th, tw, npre = 3, 5, 4, 6, 1
    N = npre + gh * gw
    T = (2 * th - 1) * (2 * tw - 1)
    pos = [(t // gw, t % gw) for t in range(gh * gw)]
    for (dy, dx) in ((1, 0), (0, -2), (-2, 3), (0, 0)):
        table = np.zeros((2, T), np.float32)
        table[1, (dy + th - 1) * (2 * tw - 1) + (dx + tw - 1)] = 1.0
        dense = o.bias_materialize(oracle_mod.Bias(oracle_mod.BIAS_RELPOS2D, table, 0, gh, gw, th, tw, npre),
                                   2, N)
        assert np.all(dense[0] == 0) and np.all(dense[1, :npre, :] == 0) and np.all(dense[1, :, :npre] == 0)
        for i in range(gh * gw):
            for j in range(gh * gw):
                hit = (pos[i][0] - pos[j][0], pos[i][1] - pos[j][1]) == (dy, dx)
                assert dense[1, npre + i, npre + j] == (1.0 if hit else 0.0), (dy, dx, i, j)


# --------------------------------------------------------------------------- forward
def _equal_sign_case(N, d, B=1, H=1, seed=0, q_signs=None, k_signs=None):
    """q, k with prescribed sign patterns (magnitudes random), v random."""
    rng = _rng(seed)
    mag_q = rng.uniform(0.5, 2.0, (B, H, N, d)).astype(np.float32)
    mag_k = rng.uniform(0.5, 2.0, (B, H, N, d)).astype(np.float32)
    qs = np.ones(d, np.float32) if q_signs is None else np.asarray(q_signs, np.float32)
    ks = np.ones(d, np.float32) if k_signs is None else np.asarray(k_signs, np.float32)
    v = rng.standard_normal((B, H, N, d)).astype(np.float32)
    return mag_q * qs, mag_k * ks, v


def _vhat(o, v):
    vq, sv = o.quant_v(v)
    return vq.astype(np.float64) * sv[:, :, None, :].astype(np.float64), vq, sv


def pin_forward_uniform(o: oracle_mod.Oracle):
    """All-equal signs and zero bias: every logit equal, every code 255, O = mean_j v^_j."""
    for N, Bc in ((1, 128), (7, 3), (130, 128), (64, 64)):
        q, k, v = _equal_sign_case(N, 24, B=2, H=2, seed=N)
        vh, _, _ = _vhat(o, v)
        out = o.attention_fwd(q, k, v, block_c=Bc)
        want = vh.mean(axis=2, keepdims=True)
        assert np.allclose(out, np.broadcast_to(want, out.shape), rtol=2e-6, atol=1e-7), (N, Bc)
    q, k, v = _equal_sign_case(1, 9, seed=3)
    vh, _, _ = _vhat(o, v)
    assert np.allclose(o.attention_fwd(q, k, v), vh, rtol=1e-6, atol=0), "N = 1 gives v^_0"


def pin_forward_dense_spike(o: oracle_mod.Oracle):
    """Equal signs + a dense bias of +40 at key j*(i) = (3i+1) mod N: O_i = v^_{j*(i)}.
    The map i -> j* is not symmetric, so a transposed bias index fails."""
    N, d, H = 23, 16, 2
    q, k, v = _equal_sign_case(N, d, H=H, seed=7)
    bias = np.zeros((H, N, N), np.float32)
    js = [(3 * i + 1) % N for i in range(N)]
    for h in range(H):
        for i in range(N):
            bias[h, i, js[i]] = 40.0
    vh, _, _ = _vhat(o, v)
    for Bc in (4, 128):
        out = o.attention_fwd(q, k, v, oracle_mod.Bias(oracle_mod.BIAS_DENSE, bias), block_c=Bc)
        want = vh[:, :, js, :]
        assert np.allclose(out, want, rtol=1e-6, atol=1e-9), Bc


def pin_forward_relpos_spike(o: oracle_mod.Oracle):
    """Equal signs + a rel-pos table that is +40 at offset (dy, dx) = (+1, 0): each query
    attends to the key one grid row above it; first-row queries and the class token see
    no spike and average uniformly."""
    gh, gw, npre, d = 4, 5, 1, 8
    N = npre + gh * gw
    th, tw = gh, gw
    table = np.zeros((1, (2 * th - 1) * (2 * tw - 1)), np.float32)
    table[0, (1 + th - 1) * (2 * tw - 1) + (0 + tw - 1)] = 40.0
    q, k, v = _equal_sign_case(N, d, seed=8)
    vh, _, _ = _vhat(o, v)
    out = o.attention_fwd(q, k, v, oracle_mod.Bias(oracle_mod.BIAS_RELPOS2D, table, 0, gh, gw, th, tw, npre),
                          block_c=6)
    for i in range(N):
        if i < npre or (i - npre) // gw == 0:
            want = vh[0, 0].mean(axis=0)
        else:
            want = vh[0, 0, i - gw]
        assert np.allclose(out[0, 0, i], want, rtol=1e-6, atol=1e-9), i


def _zero_logit_case(N, seed):
    """d = 2, q signs (+,+), k signs (+,-): every x_ij = 0, so s_ij = b_ij exactly."""
    return _equal_sign_case(N, 2, seed=seed, q_signs=[1, 1], k_signs=[1, -1])


def pin_forward_golden(o: oracle_mod.Oracle):
    """Hand-derived closed forms (tests/golden/closed_forms.json)."""
    with open(GOLDEN) as f:
        cases = json.load(f)["cases"]
    for case in cases:
        b = np.asarray(case["bias_row"], np.float32)
        N = len(b)
        q, k, v = _zero_logit_case(N, seed=case["seed"])
        bias = np.broadcast_to(b, (1, N, N)).copy()
        out, dbg = o.attention_fwd(q, k, v, oracle_mod.Bias(oracle_mod.BIAS_DENSE, bias),
                                   block_c=case["block_c"], debug=True)
        vh, _, _ = _vhat(o, v)
        codes = [int(c) for c in dbg["pu8"][0]]
        assert codes == case["codes"], (case["name"], codes)
        # O_c = sum_j w_j code_j v^_jc / (255 l), with w_j the rescale each key's block received
        w = np.array([eval(str(e), {"exp": math.exp}) for e in case["weights"]], np.float64)
        l_want = eval(case["l"], {"exp": math.exp})
        want = (w[:, None] * np.array(case["codes"], np.float64)[:, None] * vh[0, 0]).sum(0) / (255.0 * l_want)
        assert np.allclose(out[0, 0, 0], want, rtol=1e-6, atol=1e-9), case["name"]
        assert abs(dbg["l"][0] - l_want) <= 1e-6 * l_want, case["name"]


def pin_forward_block_invariance(o: oracle_mod.Oracle):
    """With block_c >= N the blockwise pass equals the separately written one-pass
    definition exactly; the final normaliser equals sum_j exp(s_ij - m_i)."""
    rng = _rng(9)
    B, H, N, d = 2, 2, 37, 40
    q, k, v = (rng.standard_normal((B, H, N, d)).astype(np.float32) for _ in range(3))
    bias = (rng.standard_normal((H, N, N)) * 0.3).astype(np.float32)
    bz = oracle_mod.Bias(oracle_mod.BIAS_DENSE, bias)
    a = o.attention_fwd(q, k, v, bz, block_c=64)
    b = o.attention_twopass(q, k, v, bz)
    assert np.array_equal(a, b), "single block == one-pass definition"
    for Bc in (5, 16, 37):
        out, dbg = o.attention_fwd(q, k, v, bz, block_c=Bc, debug=True)
        s = dbg["s"].astype(np.float64)
        m = s.max(axis=1)
        assert np.array_equal(dbg["m"].astype(np.float64), m), "running max ends at the row max"
        lsum = np.exp(s - m[:, None]).sum(1)
        assert np.allclose(dbg["l"], lsum, rtol=3e-7), "rows of P~ / l sum to 1 before quantisation"
        assert np.all(dbg["pu8"][np.arange(s.shape[0]), s.argmax(1)] == 255), "row max maps to 255"


def pin_forward_logit_definition(o: oracle_mod.Oracle):
    """s_ij = alpha x_ij + b_ij with alpha = scale * mu_q * mu_k (fp32), bias not scaled."""
    rng = _rng(10)
    B, H, N, d = 1, 2, 19, 33
    q, k, v = (rng.standard_normal((B, H, N, d)).astype(np.float32) for _ in range(3))
    table = (rng.standard_normal((H, 9 * 7)) * 0.5).astype(np.float32)
    bz = oracle_mod.Bias(oracle_mod.BIAS_RELPOS2D, table, 0, 3, 6, 5, 4, 1)
    for scale in (0.0, 0.37):
        _, dbg = o.attention_fwd(q, k, v, bz, softmax_scale=scale, block_c=8, debug=True)
        x = np.einsum("bhic,bhjc->bhij", _signs(q), _signs(k))
        mu_q = np.mean(np.abs(q.astype(np.float64)), axis=(2, 3))
        mu_k = np.mean(np.abs(k.astype(np.float64)), axis=(2, 3))
        sc = np.float32(scale) if scale > 0 else np.float32(1.0) / np.sqrt(np.float32(d))
        alpha = (sc * mu_q.astype(np.float32)) * mu_k.astype(np.float32)
        dense = o.bias_materialize(bz, H, N)
        want = alpha[:, :, None, None].astype(np.float64) * x + dense[None].astype(np.float64)
        got = dbg["s"].reshape(B, H, N, N).astype(np.float64)
        assert np.allclose(got, want, rtol=1e-6, atol=1e-6), scale


def pin_forward_error_bound(o: oracle_mod.Oracle):
    """Against float64 softmax attention on the scaled binary logits with unquantised P
    and V: |O - R| <= (0.5/255) sum_j |v^_jc| / l + sv_c / 2 (+ fp rounding)."""
    rng = _rng(11)
    B, H, N, d = 1, 3, 150, 72
    q, k, v = (rng.standard_normal((B, H, N, d)).astype(np.float32) for _ in range(3))
    bias = (rng.standard_normal((H, N, N)) * 0.5).astype(np.float32)
    bz = oracle_mod.Bias(oracle_mod.BIAS_DENSE, bias)
    vh, _, sv = _vhat(o, v)
    for Bc in (16, 64, 150):
        out, dbg = o.attention_fwd(q, k, v, bz, block_c=Bc, debug=True)
        s = dbg["s"].reshape(B, H, N, N).astype(np.float64)
        p = np.exp(s - s.max(-1, keepdims=True))
        lsum = p.sum(-1, keepdims=True)
        ref = (p / lsum) @ v.astype(np.float64)
        bound = (0.5 / 255) * (np.abs(vh).sum(2, keepdims=True) / lsum) + 0.5 * sv[:, :, None, :] + 1e-5
        assert np.all(np.abs(out - ref) <= bound), Bc
        assert np.abs(out - ref).mean() < 0.02, "quantisation error is small on average"


def pin_forward_multiblock_bruteforce(o: oracle_mod.Oracle):
    """Ragged tails: an independent pure-Python transcription of the blockwise steps on
    tiny inputs, for several block sizes and N not a multiple of the block."""
    rng = _rng(12)
    for (N, d, Bc) in ((1, 3, 2), (5, 4, 2), (13, 10, 4), (33, 7, 8), (65, 5, 16)):
        q, k, v = (rng.standard_normal((1, 1, N, d)).astype(np.float32) for _ in range(3))
        bias = (rng.standard_normal((1, N, N)) * 0.7).astype(np.float32)
        out = o.attention_fwd(q, k, v, oracle_mod.Bias(oracle_mod.BIAS_DENSE, bias), block_c=Bc)
        sq, sk = _signs(q[0, 0]), _signs(k[0, 0])
        vq, sv = o.quant_v(v)
        mq = np.float32(np.mean(np.abs(q.astype(np.float64))))
        mk = np.float32(np.mean(np.abs(k.astype(np.float64))))
        alpha = float((np.float32(1.0) / np.sqrt(np.float32(d)) * mq) * mk)
        for i in range(N):
            m, l, acc = -math.inf, 0.0, [0.0] * d
            for t0 in range(0, N, Bc):
                blk = range(t0, min(N, t0 + Bc))
                s = {j: float(np.float32(alpha * float(sq[i] @ sk[j]) + float(bias[0, i, j]))) for j in blk}
                mt = max([m] + list(s.values()))
                c = 0.0 if m == -math.inf else math.exp(m - mt)
                p = {j: float(np.float32(math.exp(s[j] - mt))) for j in blk}
                code = {j: int(np.rint(np.float32(255.0) * np.float32(p[j]))) for j in blk}
                l = l * c + sum(p.values())
                for cc in range(d):
                    acc[cc] = acc[cc] * c + sum(code[j] * int(vq[0, 0, j, cc]) for j in blk)
                m = mt
            want = [acc[cc] * (float(sv[0, 0, cc]) / 255.0) / l for cc in range(d)]
            assert np.allclose(out[0, 0, i], want, rtol=2e-6, atol=1e-7), (N, Bc, i)


def pin_forward_fullprec_sanity(o: oracle_mod.Oracle):
    """Full-precision attention is only a loose reference: outputs are finite and, for
    keys that are sign-aligned with the queries, strongly correlated."""
    rng = _rng(13)
    B, H, N, d = 1, 2, 64, 64
    base = rng.standard_normal((B, H, 8, d))
    q = (base[:, :, rng.integers(0, 8, N)] + 0.3 * rng.standard_normal((B, H, N, d))).astype(np.float32)
    k = (base[:, :, rng.integers(0, 8, N)] + 0.3 * rng.standard_normal((B, H, N, d))).astype(np.float32)
    v = rng.standard_normal((B, H, N, d)).astype(np.float32)
    a = o.attention_fwd(q, k, v, softmax_scale=0.5)
    f = o.attention_fullprec(q, k, v, softmax_scale=0.5)
    assert np.all(np.isfinite(a))
    cos = (a * f).sum() / (np.linalg.norm(a) * np.linalg.norm(f))
    assert cos > 0.5, cos


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
