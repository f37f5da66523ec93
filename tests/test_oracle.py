"""Pins for the fp64 oracle: each test checks it against something other than
itself -- brute force over a different algorithm, closed forms, library
routines (torch fp64 softmax / SDPA), invariants, and hand-worked fixtures
under tests/golden/.  No GPU involved."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import steps as S

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(12345)


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ----------------------------------------------------------------- predict (a1)
def _predict_brute(conf, masked, k, w):
    """Rounds of argmax (ties -> lower index) then a distance test per position."""
    conf = [float(np.float32(c)) for c in conf]
    avail = [i for i in range(len(conf)) if masked[i]]
    chosen = []
    for _ in range(k):
        if not avail:
            break
        best = avail[0]
        for i in avail[1:]:
            if conf[i] > conf[best]:
                best = i
        chosen.append(best)
        avail.remove(best)
    return [i for i in range(len(conf)) if any(abs(i - p) <= w for p in chosen)]


def test_predict_hand_fixture():
    g = _golden("predict_hand.json")
    q = S.predict_queries(np.array(g["conf_prev"], dtype=np.float32), np.array(g["still_masked"]),
                          g["k"], g["w"])
    assert q.tolist() == g["q_idx"]


@pytest.mark.parametrize("trial", range(40))
def test_predict_brute_force(trial):
    L = int(rng.integers(1, 40))
    # coarse values so that ties occur
    conf = (rng.integers(0, 6, L) / 5.0).astype(np.float32)
    masked = rng.integers(0, 2, L)
    k = int(rng.integers(0, 6))
    w = int(rng.integers(0, 4))
    q = S.predict_queries(conf, masked, k, w)
    assert q.tolist() == _predict_brute(conf, masked, k, w)


def test_predict_special_cases():
    conf = rng.random(32).astype(np.float32)
    masked = np.ones(32, dtype=np.uint8)
    # w = 0: exactly the top-k positions
    q = S.predict_queries(conf, masked, 4, 0)
    assert sorted(np.argsort(-conf.astype(np.float64))[:4].tolist()) == q.tolist()
    # k >= #masked and w >= L_q: every position
    masked2 = np.zeros(32, dtype=np.uint8)
    masked2[[3, 17]] = 1
    assert S.predict_queries(conf, masked2, 5, 32).tolist() == list(range(32))
    # nothing masked: nothing predicted
    assert len(S.predict_queries(conf, np.zeros(32), 4, 2)) == 0
    # window clipped at both ends
    c = np.zeros(10, dtype=np.float32)
    c[0], c[9] = 1.0, 0.9
    assert S.predict_queries(c, np.ones(10), 2, 2).tolist() == [0, 1, 2, 7, 8, 9]


def test_predict_permutation_equivariance():
    # with w=0 and distinct confidences, permuting positions permutes the result
    conf = rng.permutation(32).astype(np.float32) / 32
    masked = rng.integers(0, 2, 32)
    perm = rng.permutation(32)
    q = set(S.predict_queries(conf, masked, 4, 0).tolist())
    qp = set(S.predict_queries(conf[perm], masked[perm], 4, 0).tolist())
    assert {int(perm[i]) for i in qp} == q


# ------------------------------------------------------------------- pool (a2)
def test_pool_closed_form_and_partial_block():
    d, L, B = 8, 70, 16
    K = rng.standard_normal((L, d))
    Kb = S.pooled_keys(K, L, B)
    cs = np.vstack([np.zeros(d), np.cumsum(K, axis=0)])   # prefix sums
    for j in range(Kb.shape[0]):
        lo, hi = j * B, min((j + 1) * B, L)
        ref = (cs[hi] - cs[lo]) / (hi - lo)
        assert np.allclose(Kb[j], ref.astype(np.float32), rtol=0, atol=1e-6)
    assert Kb.shape[0] == 5                                 # ceil(70/16)
    const = np.full((64, 4), 0.375)
    assert np.all(S.pooled_keys(const, 64, 64) == 0.375)


def test_pool_rounds_once_to_fp32():
    # Reading R6: the exact mean, rounded once to fp32
    x = np.array([[1.0], [2.0 ** -30], [0.0], [0.0]])
    out = S.pooled_keys(x, 4, 4)
    assert out[0, 0] == float(np.float32((1.0 + 2.0 ** -30) / 4))


# ----------------------------------------------------------------- scores (a3)
def test_scores_sum_to_row_count_and_uniform():
    Q = rng.standard_normal((7, 16))
    Kb = rng.standard_normal((11, 16))
    s = S.block_scores(Q, Kb, S.scale_for(16))
    assert abs(s.sum() - 7.0) < 1e-12
    same = np.tile(rng.standard_normal((1, 16)), (11, 1))
    assert np.allclose(S.block_scores(Q, same, 0.3), 7.0 / 11.0, atol=1e-14)
    assert np.all(S.block_scores(np.zeros((0, 16)), Kb, 0.3) == 0)


def test_scores_two_blocks_logistic():
    # with two blocks the softmax is the logistic function of the logit gap
    Q = rng.standard_normal((5, 8))
    Kb = rng.standard_normal((2, 8))
    sc = S.scale_for(8)
    s = S.block_scores(Q, Kb, sc)
    gap = sc * (Q @ (Kb[0] - Kb[1]))
    ref0 = sum(1.0 / (1.0 + math.exp(-x)) for x in gap)
    assert abs(s[0] - ref0) < 1e-12 and abs(s[1] - (5 - ref0)) < 1e-12


def test_scores_match_torch_softmax():
    Q = rng.standard_normal((9, 32))
    Kb = rng.standard_normal((40, 32))
    sc = S.scale_for(32)
    ref = torch.softmax(torch.from_numpy(Q) @ torch.from_numpy(Kb).T * sc, dim=1).sum(0)
    assert np.allclose(S.block_scores(Q, Kb, sc), ref.numpy(), rtol=1e-13, atol=0)


# ----------------------------------------------------------------- select (a5)
def test_select_hand_fixture():
    g = _golden("select_hand.json")
    out = S.select_blocks(np.array(g["score"]), g["sink_pos"], g["B"], g["topK"])
    assert out.tolist() == g["blk_idx"]


@pytest.mark.parametrize("trial", range(30))
def test_select_brute_force_subsets(trial):
    n = int(rng.integers(2, 13))
    B = 4
    score = rng.integers(0, 4, n).astype(np.float64)       # many ties
    n_s = int(rng.integers(0, 3))
    sinks = rng.integers(0, n * B, n_s)
    K = int(rng.integers(0, n + 1))
    out = S.select_blocks(score, sinks, B, K)
    sb = sorted({int(p) // B for p in sinks})
    cand = [j for j in range(n) if j not in sb]
    kk = min(K, len(cand))
    best = None
    for sub in itertools.combinations(cand, kk):          # lexicographic order
        tot = sum(score[j] for j in sub)
        if best is None or tot > best[0]:
            best = (tot, sub)
    ref = sorted(list(best[1]) + sb)
    assert out.tolist() == ref
    assert set(sb) <= set(out.tolist())
    assert len(out) == kk + len(sb)


def test_select_ignores_negative_sinks_and_dedups():
    score = np.arange(8, dtype=np.float64)
    out = S.select_blocks(score, [-1, 0, 3, 65], 64, 2)   # 0 and 3 share block 0
    assert out.tolist() == [0, 1, 6, 7]


# ------------------------------------------------------------------ sinks (a4)
def _sink_setup(H=4, H_kv=2, L_ctx=96, L_q=8, d=16, plant=(0, 37)):
    Q = rng.standard_normal((H, L_q, d))
    Kc = rng.standard_normal((H_kv, L_ctx, d))
    Kd = rng.standard_normal((H_kv, L_q, d))
    G = H // H_kv
    for g in range(H_kv):
        qbar = Q[g * G:(g + 1) * G].reshape(-1, d).mean(0)
        for p in plant:
            Kc[g, p] += 3 * qbar
    return Q, Kc, Kd


def test_sinks_match_torch_softmax_and_mass_total():
    Q, Kc, Kd = _sink_setup()
    rows = np.array([1, 2, 5])
    sc = S.scale_for(16)
    top, mass = S.find_sinks(Q, Kc, Kd, rows, 3, sc)
    ref = torch.zeros(Kc.shape[1] + Kd.shape[1], dtype=torch.float64)
    for h in range(4):
        keys = torch.from_numpy(np.concatenate([Kc[h // 2], Kd[h // 2]]))
        ref += torch.softmax(torch.from_numpy(Q[h, rows]) @ keys.T * sc, dim=1).sum(0)
    assert np.allclose(mass, ref[:96].numpy(), rtol=1e-13)
    assert abs(ref.sum().item() - 3 * 4) < 1e-12          # |P| * H
    assert set([0, 37]) <= set(top.tolist())


def test_sinks_tie_break_lower_index():
    # identical keys everywhere -> equal mass -> the lowest positions win
    Q = rng.standard_normal((2, 4, 8))
    Kc = np.tile(rng.standard_normal((1, 1, 8)), (2, 20, 1))
    Kd = rng.standard_normal((2, 4, 8))
    top, _ = S.find_sinks(Q, Kc, Kd, np.arange(4), 3, 0.5)
    assert top.tolist() == [0, 1, 2]


# -------------------------------------------------------------- attention (a6)
def _paged(K_log, B, perm=None):
    """Pack logical [H_kv][L][d] into a pool [n_pages][H_kv][B][d] (+table)."""
    H_kv, L, d = K_log.shape
    n_pages = -(-L // B)
    pad = np.zeros((H_kv, n_pages * B, d))
    pad[:, :L] = K_log
    pool_log = pad.reshape(H_kv, n_pages, B, d).transpose(1, 0, 2, 3)
    if perm is None:
        perm = np.arange(n_pages)
    pool = np.zeros_like(pool_log)
    pool[perm] = pool_log
    return pool, perm


def _sdpa(Q, K, V, mask=None):
    q = torch.from_numpy(Q)[None]
    k = torch.from_numpy(K)[None]
    v = torch.from_numpy(V)[None]
    m = None if mask is None else torch.from_numpy(mask)[None]
    return torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=m)[0].numpy()


def test_attention_all_blocks_equals_sdpa_gqa():
    H, H_kv, L_q, d, L, B = 6, 2, 5, 16, 100, 16
    Q = rng.standard_normal((H, L_q, d))
    Kc, Vc = rng.standard_normal((2, H_kv, L, d))
    Kd, Vd = rng.standard_normal((2, H_kv, L_q, d))
    Kp, pt = _paged(Kc, B)
    Vp, _ = _paged(Vc, B)
    O, lse = S.dense_attention(Q, Kp, Vp, pt, L, B, Kd, Vd, S.scale_for(d))
    G = H // H_kv
    for h in range(H):
        g = h // G
        K = np.concatenate([Kc[g], Kd[g]])
        V = np.concatenate([Vc[g], Vd[g]])
        ref = _sdpa(Q[h][None], K[None], V[None])[0]
        assert np.allclose(O[:, h], ref, rtol=1e-12, atol=1e-12)
        lref = torch.logsumexp(torch.from_numpy(Q[h] @ K.T / math.sqrt(d)), dim=1).numpy()
        assert np.allclose(lse[h], lref, rtol=1e-13)


def test_attention_subset_equals_masked_sdpa_and_page_permutation():
    H, L_q, d, L, B = 3, 4, 8, 90, 16         # 6 blocks, the last partial
    Q = rng.standard_normal((H, L_q, d))
    Kc, Vc = rng.standard_normal((2, H, L, d))
    Kd, Vd = rng.standard_normal((2, H, L_q, d))
    perm = rng.permutation(6)
    Kp, pt = _paged(Kc, B, perm)
    Vp, _ = _paged(Vc, B, perm)
    sel = [np.array([0, 5]), np.array([2, 3, 5]), np.array([], dtype=np.int64)]
    O, _ = S.sparse_attention(Q, Kp, Vp, pt, sel, L, B, Kd, Vd, S.scale_for(d))
    for h in range(H):
        allowed = np.zeros(L + L_q, dtype=bool)
        for j in sel[h]:
            allowed[j * B: min((j + 1) * B, L)] = True
        allowed[L:] = True
        K = np.concatenate([Kc[h], Kd[h]])
        V = np.concatenate([Vc[h], Vd[h]])
        mask = np.where(allowed, 0.0, -np.inf)[None, :].repeat(L_q, 0)
        ref = _sdpa(Q[h][None], K[None], V[None], mask[None])[0]
        assert np.allclose(O[:, h], ref, rtol=1e-12, atol=1e-12)
    # identity layout gives the same result
    Kp2, pt2 = _paged(Kc, B)
    Vp2, _ = _paged(Vc, B)
    O2, _ = S.sparse_attention(Q, Kp2, Vp2, pt2, sel, L, B, Kd, Vd, S.scale_for(d))
    assert np.array_equal(O, O2)


def test_attention_closed_forms():
    # two keys: weights are the logistic of the logit gap
    q = np.array([[1.0, 0.0]])
    k = np.array([[2.0, 0.0], [0.0, 2.0]])
    v = np.array([[1.0, 0.0], [0.0, 1.0]])
    o, l = S.attention_rows(q, k, v, S.scale_for(2))
    s1 = 2.0 / math.sqrt(2.0)
    p1 = 1.0 / (1.0 + math.exp(-s1))
    assert abs(o[0, 0] - p1) < 1e-15 and abs(o[0, 1] - (1 - p1)) < 1e-15
    assert abs(l[0] - math.log(math.exp(s1) + 1.0)) < 1e-14
    # single key: output is its value, lse is its logit
    o, l = S.attention_rows(q, k[:1], np.array([[3.0, -4.0]]), 0.5)
    assert np.array_equal(o[0], [3.0, -4.0]) and l[0] == 1.0
    # constant V gives V; one-hot V gives weights that sum to 1
    Q = rng.standard_normal((4, 8))
    K = rng.standard_normal((30, 8))
    o, _ = S.attention_rows(Q, K, np.tile([[0.25, -2.0]], (30, 1)), 0.3)
    assert np.allclose(o, [[0.25, -2.0]] * 4, atol=1e-15)
    w, _ = S.attention_rows(Q, K, np.eye(30), 0.3)
    assert np.allclose(w.sum(1), 1.0, atol=1e-14) and np.all(w > 0)


def test_gqa_group_of_one_equals_mha():
    H, L_q, d, L, B = 4, 3, 8, 64, 16
    Q = rng.standard_normal((H, L_q, d))
    Kc, Vc = rng.standard_normal((2, H, L, d))
    Kd, Vd = rng.standard_normal((2, H, L_q, d))
    Kp, pt = _paged(Kc, B)
    Vp, _ = _paged(Vc, B)
    sel = [np.array([1, 3])] * H
    O, _ = S.sparse_attention(Q, Kp, Vp, pt, sel, L, B, Kd, Vd, 0.35)
    for h in range(H):   # each head alone, as a one-head problem
        Kp1, pt1 = _paged(Kc[h:h + 1], B)
        Vp1, _ = _paged(Vc[h:h + 1], B)
        O1, _ = S.sparse_attention(Q[h:h + 1], Kp1, Vp1, pt1, [sel[h]], L, B, Kd[h:h + 1],
                                   Vd[h:h + 1], 0.35)
        assert np.array_equal(O[:, h], O1[:, 0])


# -------------------------------------------------------------- chunk path (a7)
def test_chunk_layout_fixture_matches_workload():
    import synth
    g = _golden("chunk_layout.json")
    wl = synth.workload("chunked32k")
    assert (wl.n_chunks, wl.chunk_content, wl.B) == (g["n_chunks"], g["chunk_content"], g["page"])
    assert (wl.chunk_tokens, wl.chunk_pages, wl.chunk_stride, wl.n_pages) == (
        g["chunk_tokens"], g["chunk_pages"], g["chunk_stride"], g["n_pages"])
    assert wl.chunk_tokens - (wl.chunk_pages - 1) * wl.B == g["last_page_valid_rows"]
    assert wl.topK_chunks * (wl.topT_tokens + 1) == g["attended_context_tokens_per_head"]


def test_token_select_brute_force_and_ties():
    Q = rng.standard_normal((6, 8))
    K = rng.standard_normal((20, 8))
    offs, tau = S.token_select(Q, K, 5, 0.4)
    ref = torch.softmax(torch.from_numpy(Q @ K.T * 0.4), dim=1).sum(0).numpy()
    assert np.allclose(tau, ref, rtol=1e-13)
    order = sorted(range(20), key=lambda t: (-ref[t], t))[:5]
    assert offs.tolist() == sorted(order)
    # equal keys -> equal tau -> lowest offsets
    offs, _ = S.token_select(Q, np.tile(K[:1], (20, 1)), 4, 0.4)
    assert offs.tolist() == [0, 1, 2, 3]


def test_chunked_step_bos_kept_and_excluded_from_pool():
    H, L_q, d, B = 2, 4, 8, 8
    n_chunks, content = 4, 10              # 11 tokens -> 2 pages, stride 16
    stride = 16
    Kc = rng.standard_normal((H, n_chunks * stride, d))
    Vc = rng.standard_normal((H, n_chunks * stride, d))
    Kc[:, ::stride] = 1e6                 # BOS keys huge: must not enter pooling
    Q = rng.standard_normal((1, H, L_q, d))
    Kd, Vd = rng.standard_normal((2, 1, H, L_q, d))
    perm = rng.permutation(n_chunks * 2)
    Kp, pt = _paged(Kc, B, perm)
    Vp, _ = _paged(Vc, B, perm)
    r = oracle.chunked_step(Q, Kp, Vp, pt[None], Kd, Vd, n_chunks=n_chunks, stride=stride,
                            content=content, B=B, topK_chunks=2, topT=3)
    for g in range(H):
        for c in range(n_chunks):
            ref = Kc[g, c * stride + 1: c * stride + 1 + content].mean(0)
            assert np.allclose(r.Kbar[0, g, c], ref.astype(np.float32), atol=1e-6)
        pos = r.tok_pos[0, g]
        for c in r.chunk_idx[0, g]:
            assert c * stride in pos                      # BOS anchor kept
        assert len(pos) == 2 * 4
    # attention over the chosen tokens equals masked SDPA over the logical stream
    for h in range(H):
        allowed = np.zeros(n_chunks * stride + L_q, dtype=bool)
        allowed[r.tok_pos[0, h]] = True
        allowed[n_chunks * stride:] = True
        K = np.concatenate([Kc[h], Kd[0, h]])
        V = np.concatenate([Vc[h], Vd[0, h]])
        mask = np.where(allowed, 0.0, -np.inf)[None, :].repeat(L_q, 0)
        ref = _sdpa(Q[0, h][None], K[None], V[None], mask[None])[0]
        assert np.allclose(r.O[0, :, h], ref, rtol=1e-11, atol=1e-11)


# ------------------------------------------------------------- layer step glue
def test_layer_step_tiny_invariants():
    import synth
    wl = synth.workload("tiny")
    inp = synth.make_step_inputs(wl)
    r = oracle.layer_step(inp.q_dec, inp.k_pool, inp.v_pool, inp.page_table, inp.k_dec,
                          inp.v_dec, wl.L_ctx, wl.B, wl.topK, conf_prev=inp.conf_prev,
                          still_masked=inp.still_masked, k=wl.k, w=wl.w,
                          sink_pos=inp.sinks_planted[:, :wl.sinks_given])
    assert r.q_cnt[0] <= (2 * wl.w + 1) * wl.k
    assert np.all(r.blk_cnt == wl.topK + 1)
    assert np.all(r.blk_idx[..., 0] == 0)                       # sink block 0
    assert np.allclose(r.score.sum(-1), r.q_cnt[0] * wl.G, atol=1e-12)
    # with K covering every block the layer equals dense attention
    rd = oracle.layer_step(inp.q_dec, inp.k_pool, inp.v_pool, inp.page_table, inp.k_dec,
                           inp.v_dec, wl.L_ctx, wl.B, wl.n_blk, q_idx=r.q_idx, q_cnt=r.q_cnt,
                           sink_pos=inp.sinks_planted[:, :1])
    rdense = oracle.layer_step(inp.q_dec, inp.k_pool, inp.v_pool, inp.page_table, inp.k_dec,
                               inp.v_dec, wl.L_ctx, wl.B, 0, q_idx=r.q_idx, q_cnt=r.q_cnt,
                               dense=True)
    assert np.allclose(rd.O, rdense.O, rtol=0, atol=1e-13)


# ------------------------------------------------------------ cache refresh
def _random_pool(n_pages, H_kv, B, d, seed):
    r = np.random.default_rng(seed)
    pool = r.standard_normal((n_pages, H_kv, B, d)).astype(np.float32).astype(np.float64)
    row = r.permutation(n_pages)
    return pool, row


def test_cache_write_of_cached_tokens_changes_nothing():
    B, d, H_kv, L_ctx = 8, 4, 2, 45
    Kp, row = _random_pool(6, H_kv, B, d, 1)
    Vp, _ = _random_pool(6, H_kv, B, d, 2)
    start, n = 13, 20
    pos = np.arange(start, start + n)
    Kn = np.stack([S.gather_context(Kp, row, g, pos, B) for g in range(H_kv)])
    Vn = np.stack([S.gather_context(Vp, row, g, pos, B) for g in range(H_kv)])
    K2, V2, kbar = oracle.cache_write(Kp, Vp, row, Kn, Vn, start, L_ctx, B)
    assert np.array_equal(K2, Kp) and np.array_equal(V2, Vp)
    assert sorted(kbar) == [1, 2, 3, 4]
    for g in range(H_kv):
        ref = S.pooled_keys(S.gather_context(Kp, row, g, np.arange(L_ctx), B), L_ctx, B)
        for j, v in kbar.items():
            assert np.array_equal(v[g], ref[j])


def test_cache_write_closed_forms_and_untouched_rows():
    B, d, H_kv, L_ctx = 8, 3, 1, 30   # blocks 0..3, the last holds 6 positions
    Kp = np.full((4, H_kv, B, d), 2.0)
    Vp = np.full((4, H_kv, B, d), -1.0)
    row = np.array([2, 0, 3, 1])
    start, n = 5, 20                  # positions 5..24: block 0 partly, 1 and 2 fully, 3 partly
    Kn = np.full((H_kv, n, d), 6.0)
    Vn = np.full((H_kv, n, d), 7.0)
    K2, V2, kbar = oracle.cache_write(Kp, Vp, row, Kn, Vn, start, L_ctx, B)
    assert sorted(kbar) == [0, 1, 2, 3]
    assert np.allclose(kbar[0], (5 * 2.0 + 3 * 6.0) / 8)   # 5 old rows, 3 new
    assert np.allclose(kbar[1], 6.0) and np.allclose(kbar[2], 6.0)
    assert np.allclose(kbar[3], (1 * 6.0 + 5 * 2.0) / 6)  # position 24: 1 new of 6 valid
    for t in range(32):
        k = K2[row[t // B], 0, t % B]
        v = V2[row[t // B], 0, t % B]
        new = start <= t < start + n
        assert np.all(k == (6.0 if new else 2.0)) and np.all(v == (7.0 if new else -1.0))


# ------------------------------------------------- sinks across a decode block
def _block_inputs(wl, n_layers, seeds):
    """Cached context of seed seeds[0] (unchanged over the block); the
    decode-block tensors and confidences of each step from its own seed."""
    import synth
    ctx = [synth.make_step_inputs(wl, layer=l) for l in range(n_layers)]
    steps = []
    for sd in seeds:
        xs = [synth.make_step_inputs(wl.replace(seed=sd), layer=l) for l in range(n_layers)]
        steps.append(dict(conf_prev=xs[0].conf_prev, still_masked=xs[0].still_masked,
                          q_dec=[x.q_dec for x in xs], k_dec=[x.k_dec for x in xs],
                          v_dec=[x.v_dec for x in xs]))
    return ctx, steps


def test_denoise_block_keeps_first_step_sinks():
    """R8: the later steps keep the first step's sinks, not sinks found anew
    from their own queries (which differ here), and every sparse layer of
    every step selects the sink blocks."""
    import synth
    wl = synth.workload("tiny", batch=2, H=4, H_kv=2, L_ctx=1024, n_layers=3, topK=3)
    ctx, steps = _block_inputs(wl, 3, [0, 7])
    res = oracle.denoise_block([x.k_pool for x in ctx], [x.v_pool for x in ctx],
                               ctx[0].page_table, steps, wl.L_ctx, wl.B, wl.topK,
                               first_sparse=1, n_sinks=4, k=wl.k, w=wl.w)
    s0 = res[0][1].sink_pos
    fresh = []
    for b in range(wl.batch):
        Kc = np.stack([S.gather_context(S.f64(ctx[1].k_pool), ctx[1].page_table[b].numpy(), g,
                                        np.arange(wl.L_ctx), wl.B) for g in range(wl.H_kv)])
        q_idx, q_cnt = res[1][1].q_idx[b], res[1][1].q_cnt[b]
        top, _ = S.find_sinks(steps[1]["q_dec"][1][b], Kc, steps[1]["k_dec"][1][b],
                              q_idx[:q_cnt], 4, S.scale_for(wl.d))
        fresh.append(top)
    assert not np.array_equal(np.stack(fresh), s0), "inputs do not tell the readings apart"
    for t, layers in enumerate(res):
        # the dense layer selects every block
        assert np.all(layers[0].blk_cnt == wl.n_blk)
        for r in layers[1:]:
            assert np.array_equal(r.sink_pos, s0)
            for b in range(wl.batch):
                sink_blocks = set((s0[b] // wl.B).tolist())
                for g in range(wl.H_kv):
                    sel = set(r.blk_idx[b, g, : r.blk_cnt[b, g]].tolist())
                    assert sink_blocks <= sel
                    # the rest are the topK highest-scoring non-sink blocks
                    rest = [j for j in np.argsort(-r.score[b, g], kind="stable")
                            if j not in sink_blocks][: wl.topK]
                    assert sel == sink_blocks | set(rest)
    # each step predicts its own queries
    assert not np.array_equal(res[0][1].q_idx, res[1][1].q_idx)


def test_head_shard_masses_sum_to_the_whole():
    """R9: the sink mass over all heads is the sum of the per-shard masses
    (any split of the KV heads), computed per head with torch's fp64
    softmax."""
    r = np.random.default_rng(5)
    H, H_kv, L_ctx, L_q, d = 6, 3, 40, 8, 16
    Q = r.standard_normal((H, L_q, d))
    Kc = r.standard_normal((H_kv, L_ctx, d))
    Kd = r.standard_normal((H_kv, L_q, d))
    rows = np.array([1, 2, 5])
    scale = S.scale_for(d)
    G = H // H_kv
    want = torch.zeros(L_ctx, dtype=torch.float64)
    for h in range(H):
        keys = torch.from_numpy(np.concatenate([Kc[h // G], Kd[h // G]]))
        p = torch.softmax(scale * torch.from_numpy(Q[h, rows]) @ keys.T, dim=-1)
        want += p[:, :L_ctx].sum(0)
    for split in ([0, 1, 3], [0, 2, 3], [0, 1, 2, 3]):
        parts = [S.find_sinks(Q[a * G:b * G], Kc[a:b], Kd[a:b], rows, 2, scale)[1]
                 for a, b in zip(split, split[1:])]
        assert np.allclose(sum(parts), want.numpy(), rtol=1e-13, atol=0)
