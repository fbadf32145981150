"""Pins for the CPU oracle: facts the pages and mathematics fix, checked without the oracle's own code path.

Every pin is written as a `check_*` function that takes the oracle function
under test, so the mutation tests at the bottom can plant plausible mistakes in
copies of the oracle (on the CPU) and show that some pin fails for each.
"""
import math

import numpy as np
import pytest
import scipy.special
import scipy.stats
import torch

import oracle
from oracle import fastmka as O
from fastmka_inputs import CONFIGS, FastMKAConfig, make_inputs, to_f64

RNG = np.random.default_rng(1234)


def tiny_cfg(**kw) -> FastMKAConfig:
    base = FastMKAConfig("pin", 2, 40, 12, 4, 2, 3, 5, 0.7, 4, 3, 4, "f32", 99)
    return base.replace(**kw)


def tiny_weights(cfg, rng):
    d, dq, dkv, rh, nb = cfg.d_model, cfg.dq, cfg.dkv, cfg.router_hidden, cfg.hash_bits
    return O.weights_f64(rng.standard_normal((d, dq)) / math.sqrt(d), rng.standard_normal((d, dkv)) / math.sqrt(d),
                         rng.standard_normal((d, dkv)) / math.sqrt(d), rng.standard_normal((dq, rh)) / math.sqrt(dq),
                         rng.standard_normal((rh, 3)) / math.sqrt(rh), rng.standard_normal((d, nb)))


# ============================================================================ router (notes §2)
def check_router_rows(router_fn):
    q = RNG.standard_normal((50, 8))
    lam = router_fn(q, RNG.standard_normal((8, 6)), RNG.standard_normal((6, 3)))
    assert lam.shape == (50, 3)
    assert np.all(lam > 0)
    np.testing.assert_allclose(lam.sum(-1), 1.0, rtol=0, atol=1e-15)


def check_router_closed_form(router_fn):
    # W_r1 = W_r2 = I and h = 10 + [0, ln 2, ln 4]: GELU(h) = h exactly in float64
    # (1 - Phi(10) ~ 7.6e-24), so lambda = softmax(h) = (1, 2, 4) / 7.
    h = 10.0 + np.log(np.array([1.0, 2.0, 4.0]))
    lam = router_fn(h[None], np.eye(3), np.eye(3))[0]
    np.testing.assert_allclose(lam, np.array([1.0, 2.0, 4.0]) / 7.0, rtol=1e-14)
    # A zero first layer gives GELU(0) = 0, hence equal gates.
    lam0 = router_fn(RNG.standard_normal((4, 5)), np.zeros((5, 7)), RNG.standard_normal((7, 3)))
    np.testing.assert_allclose(lam0, 1.0 / 3.0, rtol=1e-15)
    # Only the second column of W_r2 sees positive inputs -> lambda_2 dominates.
    lam1 = router_fn(np.full((1, 2), 20.0), np.eye(2), np.array([[0.0, 5.0, -5.0], [0.0, 5.0, -5.0]]))[0]
    # GELU(20) = 20, z = (0, 200, -200): lambda = (e^-200, 1, e^-400) / (1 + e^-200 + e^-400).
    np.testing.assert_allclose(lam1, [math.exp(-200), 1.0, math.exp(-400)], rtol=1e-13)
    # h = (-1, 0, 1): GELU(h) = (-Phi(-1), 0, Phi(1)) with the textbook normal-table values.
    lam2 = router_fn(np.array([[-1.0, 0.0, 1.0]]), np.eye(3), np.eye(3))[0]
    e = [math.exp(-0.15865525393145707), 1.0, math.exp(0.8413447460685429)]
    np.testing.assert_allclose(lam2, np.array(e) / sum(e), rtol=1e-14)


def test_router_rows_sum_to_one():
    check_router_rows(O.router)


def test_router_closed_form():
    check_router_closed_form(O.router)


def test_gelu_is_x_times_normal_cdf():
    x = np.linspace(-6, 6, 101)
    np.testing.assert_allclose(O.gelu_erf(x), x * scipy.stats.norm.cdf(x), rtol=1e-13, atol=1e-300)
    # Textbook: Phi(1) = 0.8413447460685429, Phi(-1) = 0.15865525393145707.
    np.testing.assert_allclose(O.gelu_erf(np.array([1.0, -1.0])), [0.8413447460685429, -0.15865525393145707],
                               rtol=1e-15)


# ============================================================================ L2 session EMA
def check_ema_closed_form(ema_fn):
    for alpha in (0.0, 0.5, 0.9, 0.999):
        X = RNG.standard_normal((2, 17, 3))
        M2, m_next = ema_fn(X, alpha)
        ref = np.zeros_like(X)
        for t in range(X.shape[1]):
            for k in range(t):
                ref[:, t] += alpha ** k * (1 - alpha) * X[:, t - 1 - k]
        np.testing.assert_allclose(M2, ref, rtol=1e-12, atol=1e-14)
        nxt = sum(alpha ** k * (1 - alpha) * X[:, X.shape[1] - 1 - k] for k in range(X.shape[1]))
        np.testing.assert_allclose(m_next, nxt, rtol=1e-12, atol=1e-14)
    # alpha = 0: a pure one-step shift; M2[0] = 0.
    X = RNG.standard_normal((1, 9, 4))
    M2, _ = ema_fn(X, 0.0)
    np.testing.assert_array_equal(M2[:, 1:], X[:, :-1])
    np.testing.assert_array_equal(M2[:, 0], 0.0)


def check_ema_carry(ema_fn):
    # Splitting a sequence and carrying the state gives the unsplit result.
    X = RNG.standard_normal((2, 30, 5))
    full, m_full = ema_fn(X, 0.8)
    a, m_a = ema_fn(X[:, :11], 0.8)
    b, m_b = ema_fn(X[:, 11:], 0.8, m_a)
    np.testing.assert_allclose(np.concatenate([a, b], 1), full, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(m_b, m_full, rtol=1e-14)


def test_ema_closed_form():
    check_ema_closed_form(O.session_ema)


def test_ema_carry():
    check_ema_carry(O.session_ema)


# ============================================================================ L3 recall
def brute_summaries(X1, b):
    S, d = X1.shape
    out = []
    for j in range(S // b):
        acc = np.zeros(d)
        for r in range(j * b, (j + 1) * b):
            acc += X1[r]
        out.append(acc / b)
    return np.array(out).reshape(-1, d)


def brute_code(v, P):
    code = 0
    for k in range(P.shape[1]):
        if float(sum(v[i] * P[i, k] for i in range(len(v)))) > 0:
            code |= 1 << k
    return code


def check_recall_brute_force(recall_fn, b=4, R=3, nb=4, S=60, d=5, seed=7):
    rng = np.random.default_rng(seed)
    X1 = rng.standard_normal((S, d))
    P = rng.standard_normal((d, nb))
    summ = brute_summaries(X1, b)
    idx, count, M3, xcodes, _ = recall_fn(X1, np.arange(S), summ, P, b, R)
    scodes = [brute_code(s, P) for s in summ]
    for t in range(S):
        xc = brute_code(X1[t], P)
        assert int(xcodes[t]) == xc
        eligible = [j for j in range(len(summ)) if (j + 1) * b <= t]   # strictly past, full blocks
        assert count[t] == min(R, len(eligible))
        sel = [int(j) for j in idx[t, : count[t]]]
        assert all(j == -1 for j in idx[t, count[t]:])
        key = {j: (bin(xc ^ scodes[j]).count("1"), j) for j in eligible}
        assert set(sel) <= set(eligible) and len(set(sel)) == len(sel)
        # Every recalled block beats every block left out, in (distance, index) order.
        for js in sel:
            for ju in set(eligible) - set(sel):
                assert key[js] < key[ju]
        assert [key[j] for j in sel] == sorted(key[j] for j in sel)
        ref = np.mean([summ[j] for j in sel], axis=0) if sel else np.zeros(d)
        np.testing.assert_allclose(M3[t], ref, rtol=1e-14, atol=1e-15)


def test_recall_brute_force_heavy_ties():
    check_recall_brute_force(O.longterm_recall)                      # 4-bit codes: ties everywhere
    check_recall_brute_force(O.longterm_recall, b=3, R=5, nb=7, S=50, seed=3)


def test_recall_special_cases():
    rng = np.random.default_rng(11)
    X1 = rng.standard_normal((40, 6))
    P = rng.standard_normal((6, 8))
    b = 8
    summ = O.block_summaries(X1[None], b)[0]
    # M3 == 0 and no index for t < b.
    idx, count, M3, *_ = O.longterm_recall(X1, np.arange(40), summ, P, b, 2)
    assert np.all(count[:b] == 0) and np.all(M3[:b] == 0) and np.all(idx[:b] == -1)
    # R >= number of eligible blocks: M3 is the mean of all eligible summaries, whatever the codes.
    idx, count, M3, *_ = O.longterm_recall(X1, np.arange(40), summ, P, b, 100)
    for t in range(40):
        n = t // b
        ref = summ[:n].mean(0) if n else np.zeros(6)
        np.testing.assert_allclose(M3[t], ref, rtol=1e-14, atol=1e-15)
    # b >= S: nothing is ever eligible.
    summ_big = O.block_summaries(X1[None], 64)[0]
    _, count, M3, *_ = O.longterm_recall(X1, np.arange(40), summ_big, P, 64, 2)
    assert np.all(count == 0) and np.all(M3 == 0)


def brute_reachable_recalls(x_proj_t, s_proj, n_elig, R, eps):
    """Every recalled list (as a tuple) that some flip of the hash bits with |p| < eps produces,
    found by enumerating all subsets of those bits (token's and blocks') and sorting by hand."""
    nb = len(x_proj_t)
    free = [("t", None, k) for k in range(nb) if abs(x_proj_t[k]) < eps]
    free += [("s", j, k) for j in range(n_elig) for k in range(nb) if abs(s_proj[j, k]) < eps]
    out = set()
    for m in range(1 << len(free)):
        tb = [x_proj_t[k] > 0 for k in range(nb)]
        sb = [[s_proj[j, k] > 0 for k in range(nb)] for j in range(n_elig)]
        for i, (who, j, k) in enumerate(free):
            if (m >> i) & 1:
                if who == "t":
                    tb[k] = not tb[k]
                else:
                    sb[j][k] = not sb[j][k]
        keys = sorted((sum(tb[k] != sb[j][k] for k in range(nb)), j) for j in range(n_elig))
        out.add(tuple(j for _, j in keys[:R]))
    return out


def check_recall_excuse_exact(excused_fn, seed, nb=4, nblk=7, R=3, n_free=3):
    """The excuse accepts exactly the lists that a flip of near-zero bits reaches (brute force),
    for a token with near-zero bits planted at random among its own and the blocks' projections."""
    rng = np.random.default_rng(seed)
    eps = 1e-4
    x = rng.standard_normal(nb)
    sp = rng.standard_normal((nblk, nb))
    for _ in range(n_free):                      # plant near-zero components
        if rng.random() < 0.3:
            x[rng.integers(nb)] = rng.uniform(-0.9, 0.9) * eps
        else:
            sp[rng.integers(nblk), rng.integers(nb)] = rng.uniform(-0.9, 0.9) * eps
    for n_elig in range(nblk + 1):
        reach = brute_reachable_recalls(x, sp, n_elig, R, eps)
        for lst in reach:
            assert excused_fn(list(lst), x, sp, n_elig, R, eps)
        cands = set()
        for _ in range(40):                       # wrong lists: random picks, orders and counts
            k = min(R, n_elig) if rng.random() < 0.8 else int(rng.integers(0, R + 1))
            cands.add(tuple(int(j) for j in rng.permutation(max(n_elig, 1))[:k] if j < n_elig))
        for lst in cands - reach:
            assert not excused_fn(list(lst), x, sp, n_elig, R, eps), (lst, reach)


def test_recall_excuse_matches_brute_force():
    for seed in range(30):
        check_recall_excuse_exact(O.recall_mismatch_excused, seed)
    check_recall_excuse_exact(O.recall_mismatch_excused, 99, nb=6, nblk=9, R=4, n_free=5)


def test_recall_excuse_needs_a_deciding_bit():
    """A near-zero component excuses a mismatch only where it can move the selection."""
    eps = 1e-4
    # token code 0000; blocks at distances 0, 1, 2, 4 (block 3's bit 0 projection is near zero)
    x = np.array([-1.0, -1.0, -1.0, -1.0])
    sp = np.array([[-1.0, -1.0, -1.0, -1.0],     # d 0
                   [1.0, -1.0, -1.0, -1.0],      # d 1
                   [1.0, 1.0, -1.0, -1.0],       # d 2
                   [0.5 * eps, 1.0, 1.0, 1.0]])  # d 4, bit 0 undecided -> d in {3, 4}
    assert O.recall_mismatch_excused([0, 1], x, sp, 4, 2)
    # block 3 is far from the R = 2 cutoff whatever its bit 0: it excuses no other list
    for wrong in ([0, 2], [1, 0], [0, 3], [1, 2], [0]):
        assert not O.recall_mismatch_excused(wrong, x, sp, 4, 2)
    # with R = 3 the cutoff sits at distance 2 vs 3-or-4: still fixed, (2 beats 3)
    assert not O.recall_mismatch_excused([0, 1, 3], x, sp, 4, 3)
    # make block 3's distance reach 2 (two undecided bits): now it can tie block 2 at d 2, and wins
    # only on (distance, index) order if its distance drops below 2 -- it cannot, so [0, 1, 3] stays out
    sp2 = sp.copy()
    sp2[3, 1] = -0.5 * eps
    assert O.recall_mismatch_excused([0, 1, 2], x, sp2, 4, 3)
    assert not O.recall_mismatch_excused([0, 1, 3], x, sp2, 4, 3)
    # three undecided bits: block 3 reaches distance 1 and ties block 1, which it loses on the index,
    # but it beats block 2 (distance 2): [0, 1, 3] becomes reachable, and so does [0, 3, 1]? no: index order
    sp3 = sp2.copy()
    sp3[3, 2] = 0.25 * eps
    assert O.recall_mismatch_excused([0, 1, 3], x, sp3, 4, 3)
    assert not O.recall_mismatch_excused([0, 3, 1], x, sp3, 4, 3)
    # a token's own undecided bit moves every block: flipping bit 3 of the token makes block 3 nearer
    xt = x.copy()
    xt[3] = 0.1 * eps
    assert O.recall_mismatch_excused([0, 1], xt, sp, 4, 2)
    assert not O.recall_mismatch_excused([2, 3], xt, sp, 4, 2)


def test_recall_excuse_planted_broad_rule_is_caught():
    """The broad rule -- excuse a token whenever any eligible block has a near-zero component --
    would excuse a recall that no flip reaches; the exact rule and brute force both reject it."""
    eps = 1e-4
    x = np.array([-1.0, -1.0, -1.0, -1.0])
    sp = np.array([[-1.0, -1.0, -1.0, -1.0], [1.0, -1.0, -1.0, -1.0], [1.0, 1.0, -1.0, -1.0],
                   [0.5 * eps, 1.0, 1.0, 1.0]])

    def broad(got, x_proj_t, s_proj, n_elig, R, eps=eps):
        return bool((np.abs(x_proj_t) < eps).any() or (np.abs(s_proj[:n_elig]) < eps).any())

    assert (1, 0) not in brute_reachable_recalls(x, sp, 4, 2, eps)
    assert broad([1, 0], x, sp, 4, 2) and not O.recall_mismatch_excused([1, 0], x, sp, 4, 2)
    with pytest.raises(AssertionError):
        check_recall_excuse_exact(broad, 0)


def test_recall_mismatches_counts():
    """recall_mismatches counts a mismatch the flip excuses and one it does not."""
    rng = np.random.default_rng(5)
    cfg = tiny_cfg(seq=24, block=4, recall_r=2, hash_bits=4)
    X = rng.standard_normal((1, cfg.seq, cfg.d_model))
    ref = O.fastmka_prefill(X, tiny_weights(cfg, rng), cfg, rows=np.array([23]))
    got = ref["idx"].copy()
    assert O.recall_mismatches(got, ref) == (0, 0, [])
    t = 20                                       # 5 eligible blocks
    got[0, t] = got[0, t][::-1]                  # reversed order: no flip reaches it (no bit is near zero)
    assert O.recall_mismatches(got, ref)[:2] == (1, 0)
    ref["x_proj"][0, t] = 0.0                    # every token bit undecided: brute force decides
    reach = brute_reachable_recalls(ref["x_proj"][0, t], ref["summary_proj"][0], 5, 2, O.EXCUSE_EPS)
    want = (0, 1) if tuple(got[0, t]) in reach else (1, 0)
    assert O.recall_mismatches(got, ref)[:2] == want


def test_hash_bit_order_and_zero():
    P = np.eye(5)
    v = np.array([[1.0, -1.0, 0.0, 2.0, -0.5]])
    codes, p = O.hash_codes(v, P)
    assert int(codes[0]) == (1 << 0) | (1 << 3)        # p = 0 gives bit 0
    assert O.hamming(0b1011, 0b0110) == 3


# ============================================================================ attention
def brute_causal_gqa(q, K, V, Hkv, scale):
    """Explicit S x S masked score matrix per head."""
    S, Hq, dh = q.shape
    G = Hq // Hkv
    out = np.zeros_like(q)
    for h in range(Hq):
        g = h // G
        sc = np.full((S, S), -np.inf)
        for t in range(S):
            for j in range(t + 1):
                sc[t, j] = scale * float(np.dot(q[t, h], K[j, g]))
        w = np.exp(sc - sc.max(1, keepdims=True))
        w /= w.sum(1, keepdims=True)
        out[:, h] = w @ V[:, g]
    return out


def check_attention_brute(attn_fn, S=23, Hq=6, Hkv=2, dh=4):
    rng = np.random.default_rng(5)
    q = rng.standard_normal((S, Hq, dh)) * 2
    K = rng.standard_normal((S, Hkv, dh))
    V = rng.standard_normal((S, Hkv, dh))
    got = attn_fn(q, np.arange(S), K, V, Hkv, 0.37, row_chunk=5)
    np.testing.assert_allclose(got, brute_causal_gqa(q, K, V, Hkv, 0.37), rtol=1e-12, atol=1e-13)


def test_attention_brute_force():
    check_attention_brute(O.causal_gqa_attention)
    check_attention_brute(O.causal_gqa_attention, S=9, Hq=3, Hkv=3, dh=5)    # Hq = Hkv: plain MHA


def test_attention_matches_torch_sdpa():
    rng = np.random.default_rng(8)
    S, Hq, Hkv, dh = 31, 8, 2, 16
    q, K, V = rng.standard_normal((S, Hq, dh)), rng.standard_normal((S, Hkv, dh)), rng.standard_normal((S, Hkv, dh))
    got = O.causal_gqa_attention(q, np.arange(S), K, V, Hkv, 1 / 4)
    tq = torch.from_numpy(q).permute(1, 0, 2)[None]
    tk = torch.from_numpy(K).permute(1, 0, 2).repeat_interleave(Hq // Hkv, 0)[None]
    tv = torch.from_numpy(V).permute(1, 0, 2).repeat_interleave(Hq // Hkv, 0)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True, scale=0.25)
    np.testing.assert_allclose(got, ref[0].permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("tile", [1, 7, 64])
def test_online_max_shift_equals_two_pass(tile):
    rng = np.random.default_rng(tile)
    for scale in (1.0, 30.0):                      # large scores force many max updates
        s = rng.standard_normal(150) * scale + np.linspace(-20, 20, 150)
        Vt = rng.standard_normal((150, 6))
        w = np.exp(s - s.max())
        np.testing.assert_allclose(O.online_softmax_attend(s, Vt, tile), (w / w.sum()) @ Vt, rtol=1e-12, atol=1e-14)


# ============================================================================ whole layer
def _run(cfg, X, w, **kw):
    return O.fastmka_prefill(X, w, cfg, **kw)


def test_layer_lambda_one_is_standard_causal_attention():
    """lambda = (1,0,0) ("L1 only (=MHA)" in the abstract page's Table 9) is textbook causal GQA."""
    cfg = tiny_cfg()
    w = tiny_weights(cfg, np.random.default_rng(2))
    X = np.random.default_rng(3).standard_normal((cfg.batch, cfg.seq, cfg.d_model))
    out = _run(cfg, X, w, lam_override=[1.0, 0.0, 0.0])
    for bi in range(cfg.batch):
        q = (X[bi] @ w.w_q).reshape(cfg.seq, cfg.n_q_heads, cfg.d_head)
        K = (X[bi] @ w.w_k).reshape(cfg.seq, cfg.n_kv_heads, cfg.d_head)
        V = (X[bi] @ w.w_v).reshape(cfg.seq, cfg.n_kv_heads, cfg.d_head)
        ref = brute_causal_gqa(q, K, V, cfg.n_kv_heads, cfg.scale)
        np.testing.assert_allclose(out["O"][bi].reshape(ref.shape), ref, rtol=1e-11, atol=1e-12)


def test_layer_sources_enter_as_defined():
    """lambda = e_2 or e_3 routes the EMA or the recalled mean alone into K/V."""
    cfg = tiny_cfg()
    w = tiny_weights(cfg, np.random.default_rng(4))
    X = np.random.default_rng(5).standard_normal((cfg.batch, cfg.seq, cfg.d_model))
    o2 = _run(cfg, X, w, lam_override=[0.0, 1.0, 0.0], keep_d_space=True)
    M2, _ = O.session_ema(X, cfg.alpha)
    np.testing.assert_allclose(o2["K"].reshape(cfg.batch, cfg.seq, -1), M2 @ w.w_k, rtol=1e-12, atol=1e-13)
    o3 = _run(cfg, X, w, lam_override=[0.0, 0.0, 1.0], keep_d_space=True)
    np.testing.assert_allclose(o3["V"].reshape(cfg.batch, cfg.seq, -1), o3["M3"] @ w.w_v, rtol=1e-12, atol=1e-13)


def test_layer_first_row_and_lambda_sum():
    cfg = tiny_cfg()
    w = tiny_weights(cfg, np.random.default_rng(6))
    X = np.random.default_rng(7).standard_normal((cfg.batch, cfg.seq, cfg.d_model))
    out = _run(cfg, X, w)
    np.testing.assert_allclose(out["lam"].sum(-1), 1.0, atol=1e-15)
    G = cfg.n_q_heads // cfg.n_kv_heads
    for bi in range(cfg.batch):
        V0 = out["lam"][bi, 0, 0] * (X[bi, 0] @ w.w_v)       # M2[0] = M3[0] = 0
        O0 = out["O"][bi, 0].reshape(cfg.n_q_heads, cfg.d_head)
        for h in range(cfg.n_q_heads):
            np.testing.assert_allclose(O0[h], V0.reshape(cfg.n_kv_heads, cfg.d_head)[h // G], rtol=1e-13)


def test_layer_causality_under_future_perturbation():
    cfg = tiny_cfg(seq=48)
    w = tiny_weights(cfg, np.random.default_rng(8))
    X = np.random.default_rng(9).standard_normal((cfg.batch, cfg.seq, cfg.d_model))
    base = _run(cfg, X, w)
    for t0 in (0, 5, 17, 31, 46):
        Xp = X.copy()
        Xp[:, t0 + 1:] = np.random.default_rng(t0).standard_normal(Xp[:, t0 + 1:].shape) * 3
        pert = _run(cfg, Xp, w)
        np.testing.assert_allclose(pert["O"][:, : t0 + 1], base["O"][:, : t0 + 1], rtol=1e-12, atol=1e-13)
        np.testing.assert_array_equal(pert["idx"][:, : t0 + 1], base["idx"][:, : t0 + 1])


def test_decode_equals_prefill_rows():
    cfg = tiny_cfg(seq=37)
    w = tiny_weights(cfg, np.random.default_rng(10))
    X = np.random.default_rng(11).standard_normal((cfg.batch, cfg.seq, cfg.d_model))
    pre = _run(cfg, X, w)
    dec = O.fastmka_decode(X, w, cfg)
    np.testing.assert_allclose(dec, pre["O"], rtol=1e-11, atol=1e-12)


def test_chunked_rows_equal_unchunked():
    cfg = tiny_cfg(seq=40)
    w = tiny_weights(cfg, np.random.default_rng(12))
    X = np.random.default_rng(13).standard_normal((cfg.batch, cfg.seq, cfg.d_model))
    a = _run(cfg, X, w)
    b = _run(cfg, X, w, row_chunk=7, rows=np.array([0, 3, 8, 9, 39]))
    np.testing.assert_allclose(b["O"], a["O"][:, [0, 3, 8, 9, 39]], rtol=1e-12, atol=1e-13)
    np.testing.assert_array_equal(b["idx"], a["idx"])
    np.testing.assert_allclose(b["K"], a["K"], rtol=1e-12, atol=1e-13)


def test_tiny_workload_runs():
    cfg = CONFIGS["tiny_f32"]
    inp = make_inputs(cfg)
    w = O.weights_f64(*(to_f64(t) for t in (inp.w_q, inp.w_k, inp.w_v, inp.w_r1, inp.w_r2, inp.hash_proj)))
    out = _run(cfg, to_f64(inp.x), w)
    assert np.isfinite(out["O"]).all()
    np.testing.assert_allclose(out["lam"].sum(-1), 1.0, atol=1e-15)
    assert out["count"][0, cfg.block] == 1 and out["count"][0, -1] == cfg.recall_r


# ============================================================================ planted mistakes
def _mut_ema_reads_current(X, alpha, m_init=None):
    B, S, d = X.shape
    M2 = np.zeros((B, S, d))
    m = np.zeros((B, d)) if m_init is None else m_init.copy()
    for t in range(S):
        m = alpha * m + (1 - alpha) * X[:, t]       # leaks token t into its own summary
        M2[:, t] = m
    return M2, m


def _mut_ema_swapped_weights(X, alpha, m_init=None):
    return O.session_ema(X, 1.0 - alpha, m_init)


def _mut_router_no_gelu(q, w_r1, w_r2):
    return O.softmax_rows((q @ w_r1) @ w_r2)


def _mut_router_softmax_axis(q, w_r1, w_r2):
    z = O.gelu_erf(q @ w_r1) @ w_r2
    e = np.exp(z - z.max(0, keepdims=True))
    return e / e.sum(0, keepdims=True)


def _mut_recall_factory(kind):
    def select(code_t, summary_codes, n_eligible, R):
        if kind == "eligible_off_by_one":
            n_eligible = min(n_eligible + 1, len(summary_codes))
        if n_eligible <= 0:
            return np.zeros(0, np.int64)
        dist = O.hamming(code_t, summary_codes[:n_eligible])
        if kind == "tie_high_index":
            order = np.lexsort((-np.arange(n_eligible), dist))
        elif kind == "farthest":
            order = np.lexsort((np.arange(n_eligible), -dist))
        else:
            order = np.lexsort((np.arange(n_eligible), dist))
        return order[:R]
    return select


def _mut_attention_factory(kind):
    def attn(q_rows, positions, K, V, n_kv_heads, scale, row_chunk=64):
        n, Hq, dh = q_rows.shape
        G = Hq // n_kv_heads
        out = np.zeros((n, Hq, dh))
        for i, t in enumerate(positions):
            for h in range(Hq):
                g = h % n_kv_heads if kind == "gqa_interleaved" else h // G
                hi = t if kind == "exclusive_mask" and t > 0 else t + 1
                s = K[:hi, g] @ q_rows[i, h] * scale
                p = np.exp(s - s.max())
                out[i, h] = p @ V[:hi, g] / p.sum()
        return out
    return attn


def test_planted_mistakes_are_caught(monkeypatch):
    for bad in (_mut_ema_reads_current, _mut_ema_swapped_weights):
        with pytest.raises(AssertionError):
            check_ema_closed_form(bad)
    for bad in (_mut_router_no_gelu, _mut_router_softmax_axis):
        with pytest.raises(AssertionError):
            check_router_rows(bad)
            check_router_closed_form(bad)
    for kind in ("eligible_off_by_one", "tie_high_index", "farthest"):
        with monkeypatch.context() as m:
            m.setattr(O, "recall_select", _mut_recall_factory(kind))
            with pytest.raises(AssertionError):
                check_recall_brute_force(O.longterm_recall)
    for kind in ("exclusive_mask", "gqa_interleaved"):
        with pytest.raises(AssertionError):
            check_attention_brute(_mut_attention_factory(kind))
    # The unplanted copy of the attention mutant passes, so the failures above are the mistakes'.
    check_attention_brute(_mut_attention_factory("none"))


# ============================================================================ routing and tier variants
# abstract page, Tables 9 (tiers) and 10 (routing); gates read as in oracle.route_gate.
_ZL = np.log(np.array([[1.0, 2.0, 4.0]]))  # softmax gives (1, 2, 4) / 7
ROUTE_CLOSED_FORMS = [
    ("soft", 7, [1 / 7, 2 / 7, 4 / 7]), ("fixed", 7, [1 / 3] * 3), ("top1", 7, [0, 0, 1]), ("top2", 7, [0, 1 / 3, 2 / 3]),
    ("soft", 3, [1 / 3, 2 / 3, 0]), ("fixed", 3, [0.5, 0.5, 0]), ("top1", 3, [0, 1, 0]), ("top2", 3, [1 / 3, 2 / 3, 0]),
    ("soft", 5, [1 / 5, 0, 4 / 5]), ("fixed", 5, [0.5, 0, 0.5]), ("top1", 5, [0, 0, 1]), ("top2", 5, [1 / 5, 0, 4 / 5]),
    ("soft", 1, [1, 0, 0]), ("fixed", 1, [1, 0, 0]), ("top1", 1, [1, 0, 0]), ("top2", 1, [1, 0, 0]),
]


def check_route_closed_forms(gate):
    for mode, tiers, want in ROUTE_CLOSED_FORMS:
        np.testing.assert_allclose(gate(_ZL, mode, tiers)[0], want, rtol=1e-14, atol=1e-15, err_msg=f"{mode} {tiers}")
    # ties go to the lower tier index
    np.testing.assert_array_equal(gate(np.array([[1.0, 1.0, 0.0]]), "top1", 7)[0], [1, 0, 0])
    np.testing.assert_array_equal(gate(np.array([[0.0, 2.0, 2.0]]), "top1", 7)[0], [0, 1, 0])
    np.testing.assert_allclose(gate(np.array([[0.0, 3.0, 3.0]]), "top2", 7)[0], [0, 0.5, 0.5], rtol=1e-15)
    e = math.exp(-3.0)
    np.testing.assert_allclose(gate(np.array([[3.0, 0.0, 0.0]]), "top2", 7)[0], [1 / (1 + e), e / (1 + e), 0],
                               rtol=1e-15)


def test_route_gate_closed_forms():
    check_route_closed_forms(O.route_gate)


def test_route_gate_soft_is_softmax_and_rows_sum_to_one():
    z = RNG.standard_normal((200, 3)) * 4
    np.testing.assert_allclose(O.route_gate(z), scipy.special.softmax(z, axis=1), rtol=1e-13)
    for mode in O.ROUTE_MODES:
        for tiers in range(1, 8):
            lam = O.route_gate(z, mode, tiers)
            np.testing.assert_allclose(lam.sum(-1), 1.0, atol=1e-15)
            for i in range(3):
                if not (tiers >> i) & 1:
                    assert (lam[:, i] == 0).all()
            if mode in ("top1", "top2"):
                k = 1 if mode == "top1" else min(2, bin(tiers).count("1"))
                assert ((lam > 0).sum(-1) <= k).all()


def test_route_margin():
    np.testing.assert_allclose(O.route_margin(_ZL, "top1"), [math.log(2.0)], rtol=1e-15)
    np.testing.assert_allclose(O.route_margin(_ZL, "top2"), [math.log(2.0)], rtol=1e-15)
    np.testing.assert_allclose(O.route_margin(_ZL, "top1", 5), [math.log(4.0)], rtol=1e-15)
    assert np.isinf(O.route_margin(_ZL, "soft")).all() and np.isinf(O.route_margin(_ZL, "top2", 3)).all()


def test_layer_l1_only_tier_is_standard_causal_attention():
    """tiers = L1 only ("L1 only (=MHA)", Table 9) through the configuration is textbook causal GQA."""
    cfg = tiny_cfg(tiers=1)
    w = tiny_weights(cfg, np.random.default_rng(21))
    X = np.random.default_rng(22).standard_normal((cfg.batch, cfg.seq, cfg.d_model))
    out = _run(cfg, X, w)
    assert (out["lam"] == np.array([1.0, 0.0, 0.0])).all()
    for bi in range(cfg.batch):
        q = (X[bi] @ w.w_q).reshape(cfg.seq, cfg.n_q_heads, cfg.d_head)
        K = (X[bi] @ w.w_k).reshape(cfg.seq, cfg.n_kv_heads, cfg.d_head)
        V = (X[bi] @ w.w_v).reshape(cfg.seq, cfg.n_kv_heads, cfg.d_head)
        ref = brute_causal_gqa(q, K, V, cfg.n_kv_heads, cfg.scale)
        np.testing.assert_allclose(out["O"][bi].reshape(ref.shape), ref, rtol=1e-11, atol=1e-12)


def test_layer_fixed_and_hard_routing():
    """Fixed routing equals lambda = 1/3 everywhere; hard top-1 picks each token's largest logit."""
    cfg = tiny_cfg()
    w = tiny_weights(cfg, np.random.default_rng(23))
    X = np.random.default_rng(24).standard_normal((cfg.batch, cfg.seq, cfg.d_model))
    fixed = _run(cfg.replace(route_mode="fixed"), X, w)
    ref = _run(cfg, X, w, lam_override=[1 / 3, 1 / 3, 1 / 3])
    np.testing.assert_allclose(fixed["O"], ref["O"], rtol=1e-13, atol=1e-14)
    top1 = _run(cfg.replace(route_mode="top1"), X, w)
    soft = _run(cfg, X, w)
    np.testing.assert_array_equal(top1["lam"].argmax(-1), soft["lam"].argmax(-1))
    assert ((top1["lam"] == 0) | (top1["lam"] == 1)).all()
    # the published layer is the soft gate
    np.testing.assert_allclose(soft["lam"], O.softmax_rows(O.router_logits(
        (X.reshape(-1, cfg.d_model) @ w.w_q), w.w_r1, w.w_r2)).reshape(soft["lam"].shape), rtol=1e-13)


def test_decode_equals_prefill_rows_for_variants():
    for kw in (dict(route_mode="top2"), dict(tiers=5), dict(route_mode="fixed", tiers=3)):
        cfg = tiny_cfg(seq=29, **kw)
        w = tiny_weights(cfg, np.random.default_rng(25))
        X = np.random.default_rng(26).standard_normal((cfg.batch, cfg.seq, cfg.d_model))
        np.testing.assert_allclose(O.fastmka_decode(X, w, cfg), _run(cfg, X, w)["O"], rtol=1e-11, atol=1e-12)


def _mut_route_top2_unnormalised(z, mode="soft", tiers=7):
    lam = O.route_gate(z, "soft", tiers)
    if mode == "top2":
        lam = np.where(lam == lam.min(-1, keepdims=True), 0.0, lam)
    return lam if mode in ("soft", "top2") else O.route_gate(z, mode, tiers)


def _mut_route_tie_high_index(z, mode="soft", tiers=7):
    if mode != "top1":
        return O.route_gate(z, mode, tiers)
    zz = np.where(np.array([(tiers >> i) & 1 for i in range(3)], bool), z, -np.inf)
    lam = np.zeros(np.shape(z))
    np.put_along_axis(lam, (2 - np.argmax(zz[..., ::-1], axis=-1))[..., None], 1.0, axis=-1)
    return lam


def test_planted_routing_mistakes_are_caught():
    for bad in (_mut_route_top2_unnormalised, _mut_route_tie_high_index):
        with pytest.raises(AssertionError):
            check_route_closed_forms(bad)


# ============================================================================ full MKA (three paths)
def brute_masked_gqa(q, K, V, Hkv, scale, allowed):
    """Softmax attention with an explicit boolean key mask allowed[t, j]; rows with no key give 0."""
    S, Hq, dh = q.shape
    G = Hq // Hkv
    out = np.zeros_like(q)
    for h in range(Hq):
        g = h // G
        for t in range(S):
            keys = [j for j in range(K.shape[0]) if allowed[t, j]]
            if not keys:
                continue
            sc = np.array([scale * float(np.dot(q[t, h], K[j, g])) for j in keys])
            wts = np.exp(sc - sc.max())
            out[t, h] = (wts / wts.sum()) @ V[keys, g]
    return out


def _mka_setup(seed, **kw):
    cfg = tiny_cfg(**kw)
    w = tiny_weights(cfg, np.random.default_rng(seed))
    X = np.random.default_rng(seed + 1).standard_normal((cfg.batch, cfg.seq, cfg.d_model))
    return cfg, w, X


def _heads(cfg, X, w, bi):
    q = (X[bi] @ w.w_q).reshape(cfg.seq, cfg.n_q_heads, cfg.d_head)
    K = (X[bi] @ w.w_k).reshape(cfg.seq, cfg.n_kv_heads, cfg.d_head)
    V = (X[bi] @ w.w_v).reshape(cfg.seq, cfg.n_kv_heads, cfg.d_head)
    return q, K, V


def check_mka_l1_path(fn):
    cfg, w, X = _mka_setup(30)
    out = fn(X, w, cfg, lam_override=[1.0, 0.0, 0.0])
    for bi in range(cfg.batch):
        q, K, V = _heads(cfg, X, w, bi)
        ref = brute_causal_gqa(q, K, V, cfg.n_kv_heads, cfg.scale)
        np.testing.assert_allclose(out["O"][bi].reshape(ref.shape), ref, rtol=1e-11, atol=1e-12)


def check_mka_l2_path(fn):
    """lambda = e_2: O[t, h] = (M2[t] W_v)[g(h)], M2 from the closed form sum_k a^k (1-a) X[t-1-k]."""
    cfg, w, X = _mka_setup(32)
    out = fn(X, w, cfg, lam_override=[0.0, 1.0, 0.0])
    a, G = cfg.alpha, cfg.n_q_heads // cfg.n_kv_heads
    for bi in range(cfg.batch):
        for t in range(cfg.seq):
            m2 = sum(a ** k * (1 - a) * X[bi, t - 1 - k] for k in range(t)) if t else np.zeros(cfg.d_model)
            v2 = (m2 @ w.w_v).reshape(cfg.n_kv_heads, cfg.d_head)
            want = v2[np.arange(cfg.n_q_heads) // G].reshape(-1)
            np.testing.assert_allclose(out["O"][bi, t], want, rtol=1e-11, atol=1e-12)


def check_mka_l3_path_recall_all(fn):
    """R >= every eligible block: a_3 attends to the whole prefix of full blocks [0, floor(t/b)*b)."""
    cfg, w, X = _mka_setup(34, recall_r=20)
    out = fn(X, w, cfg, lam_override=[0.0, 0.0, 1.0])
    S, b = cfg.seq, cfg.block
    allowed = np.arange(S)[None, :] < (np.arange(S) // b * b)[:, None]
    for bi in range(cfg.batch):
        q, K, V = _heads(cfg, X, w, bi)
        ref = brute_masked_gqa(q, K, V, cfg.n_kv_heads, cfg.scale, allowed)
        np.testing.assert_allclose(out["O"][bi].reshape(ref.shape), ref, rtol=1e-11, atol=1e-12)


def test_mka_l1_path_is_textbook_causal_attention():
    check_mka_l1_path(O.mka_full_prefill)


def test_mka_l2_path_is_the_ema_value():
    check_mka_l2_path(O.mka_full_prefill)


def test_mka_l3_path_with_every_block_recalled():
    check_mka_l3_path_recall_all(O.mka_full_prefill)


def test_mka_l3_path_matches_a_dense_block_mask():
    """Small R: the recalled blocks (pinned by the brute-force recall tests) as a dense key mask."""
    cfg, w, X = _mka_setup(36, recall_r=2)
    out = O.mka_full_prefill(X, w, cfg, lam_override=[0.0, 0.0, 1.0])
    S, b = cfg.seq, cfg.block
    for bi in range(cfg.batch):
        allowed = np.zeros((S, S), bool)
        for t in range(S):
            for j in out["idx"][bi, t, :out["count"][bi, t]]:
                allowed[t, j * b:(j + 1) * b] = True
        assert (allowed.sum(1) == out["count"][bi] * b).all()
        q, K, V = _heads(cfg, X, w, bi)
        ref = brute_masked_gqa(q, K, V, cfg.n_kv_heads, cfg.scale, allowed)
        np.testing.assert_allclose(out["O"][bi].reshape(ref.shape), ref, rtol=1e-11, atol=1e-12)


def test_mka_mixes_paths_linearly():
    cfg, w, X = _mka_setup(38)
    lam = np.array([0.2, 0.5, 0.3])
    mixed = O.mka_full_prefill(X, w, cfg, lam_override=lam)["O"]
    parts = [O.mka_full_prefill(X, w, cfg, lam_override=np.eye(3)[i])["O"] for i in range(3)]
    np.testing.assert_allclose(mixed, sum(l * p for l, p in zip(lam, parts)), rtol=1e-12, atol=1e-13)


def _mut_mka_a3_current_block(X, w, cfg, rows=None, lam_override=None):
    """Planted mistake: the L3 path also sees the current, unfinished block."""
    cfg2 = cfg.replace(block=cfg.block)
    out = O.mka_full_prefill(X, w, cfg2, rows, lam_override)
    S, b = cfg.seq, cfg.block
    for bi in range(cfg.batch):
        q, K, V = _heads(cfg, X, w, bi)
        allowed = np.arange(S)[None, :] < np.minimum(S, (np.arange(S) // b + 1) * b)[:, None]
        allowed &= np.arange(S)[None, :] <= np.arange(S)[:, None]
        extra = brute_masked_gqa(q, K, V, cfg.n_kv_heads, cfg.scale, allowed)
        lam = np.asarray(lam_override if lam_override is not None else [0, 0, 1], float)
        out["O"][bi] = out["O"][bi] * (1 - lam[2]) + lam[2] * extra.reshape(S, -1)
    return out


def _mut_mka_a2_leaks_current(X, w, cfg, rows=None, lam_override=None):
    """Planted mistake: the L2 summary at t already contains x_t."""
    Xs = np.concatenate([X[:, 1:], X[:, -1:]], axis=1)
    return O.mka_full_prefill(Xs, w, cfg, rows, lam_override) if lam_override is not None and \
        lam_override[1] == 1.0 else O.mka_full_prefill(X, w, cfg, rows, lam_override)


def test_planted_mka_mistakes_are_caught():
    with pytest.raises(AssertionError):
        check_mka_l3_path_recall_all(_mut_mka_a3_current_block)
    with pytest.raises(AssertionError):
        check_mka_l2_path(_mut_mka_a2_leaks_current)


# ============================================================================ Block-MKA block-sparse attention
def check_block_sparse_recall_all(fn):
    """R covering every eligible block: the block-sparse attention is the full causal one."""
    cfg = tiny_cfg(recall_r=20, seq=41)
    w = tiny_weights(cfg, np.random.default_rng(40))
    X = np.random.default_rng(41).standard_normal((cfg.batch, cfg.seq, cfg.d_model))
    causal = O.fastmka_prefill(X, w, cfg)
    sparse = fn(X, w, cfg.replace(block_sparse=1))
    np.testing.assert_allclose(sparse["O"], causal["O"], rtol=1e-11, atol=1e-12)


def check_block_sparse_dense_mask(fn):
    """Small R: own block up to t plus the recalled blocks, as an explicit key mask."""
    cfg = tiny_cfg(recall_r=2, seq=43, block_sparse=1)
    w = tiny_weights(cfg, np.random.default_rng(42))
    X = np.random.default_rng(43).standard_normal((cfg.batch, cfg.seq, cfg.d_model))
    out = fn(X, w, cfg)
    S, b = cfg.seq, cfg.block
    for bi in range(cfg.batch):
        allowed = np.zeros((S, S), bool)
        for t in range(S):
            allowed[t, (t // b) * b:t + 1] = True
            for j in out["idx"][bi, t, :out["count"][bi, t]]:
                allowed[t, j * b:(j + 1) * b] = True
        q = out["q"][bi]
        ref = brute_masked_gqa(q, out["K"][bi], out["V"][bi], cfg.n_kv_heads, cfg.scale, allowed)
        np.testing.assert_allclose(out["O"][bi].reshape(ref.shape), ref, rtol=1e-11, atol=1e-12)


def test_block_sparse_with_every_block_recalled_is_causal_attention():
    check_block_sparse_recall_all(O.fastmka_prefill)


def test_block_sparse_matches_a_dense_mask():
    check_block_sparse_dense_mask(O.fastmka_prefill)


def _mut_block_sparse_own_block_unmasked(X, w, cfg, **kw):
    """Planted mistake: the own block is attended whole, future keys included."""
    out = O.fastmka_prefill(X, w, cfg.replace(block_sparse=0), **kw)
    if not getattr(cfg, "block_sparse", 0):
        return out
    S, b = cfg.seq, cfg.block
    for bi in range(cfg.batch):
        allowed = np.zeros((S, S), bool)
        for t in range(S):
            allowed[t, (t // b) * b:min(S, (t // b + 1) * b)] = True
            for j in out["idx"][bi, t, :out["count"][bi, t]]:
                allowed[t, j * b:(j + 1) * b] = True
        ref = brute_masked_gqa(out["q"][bi], out["K"][bi], out["V"][bi], cfg.n_kv_heads, cfg.scale, allowed)
        out["O"][bi] = ref.reshape(S, -1)
    return out


def test_planted_block_sparse_mistake_is_caught():
    with pytest.raises(AssertionError):
        check_block_sparse_dense_mask(_mut_block_sparse_own_block_unmasked)


# ============================================================================ regression snapshot
def test_golden_snapshot_unchanged():
    """tests/golden/tiny_f32_oracle.json (written by tests/golden/make_golden.py from the oracle) still holds."""
    import importlib.util
    import json
    import os
    here = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
    spec = importlib.util.spec_from_file_location("make_golden", os.path.join(here, "make_golden.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    with open(os.path.join(here, "tiny_f32_oracle.json")) as f:
        stored = json.load(f)
    now = mod.compute()
    assert now["idx"] == stored["idx"] and now["x_codes"] == stored["x_codes"]
    assert now["summary_codes"] == stored["summary_codes"]
    for k in ("lam", "O_row_sums", "O_first8"):
        np.testing.assert_allclose(np.array(now[k]), np.array(stored[k]), rtol=1e-12, atol=1e-13)
