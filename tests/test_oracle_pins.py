"""Pins of the CPU oracle to facts other than itself (CPU only).

Each test checks an oracle routine against a closed form, a brute-force
computation in plain Python, an identity from another formulation, or an
invariant the mathematics fixes. A plausible slip in the oracle (a dropped
term, a wrong sign, swapped RoPE pairs, a wrong GQA head map, a missing
causal mask, a wrong softmax axis, a wrong tie rule) fails at least one test;
``test_planted_mistakes_are_caught`` checks a few of those explicitly.
"""
import dataclasses
import math

import numpy as np
import pytest

import oracle
from oracle import forward as F
from oracle.run import run_oracle
from synth.workloads import WORKLOADS, TEST_WORKLOADS, make_batch

RNG = np.random.default_rng(1234)


# --- bf16 rounding (the cache's element type) -----------------------------------------------------

def test_bf16_round_ties_and_exact_values():
    one = 1.0
    ulp = 2.0 ** -7                      # bf16 spacing in [1, 2)
    assert F.bf16_round(one) == one
    assert F.bf16_round(one + ulp / 2) == one            # tie -> even (1.0)
    assert F.bf16_round(one + 3 * ulp / 2) == one + 2 * ulp  # tie -> even (mantissa 2)
    assert F.bf16_round(one + ulp / 2 + 1e-12) == one + ulp
    assert F.bf16_round(-3.0) == -3.0
    assert F.bf16_round(0.0) == 0.0


def test_bf16_round_matches_fp32_bit_route():
    # independent route: fp32 values (exact in fp64) rounded by integer RNE on the fp32 bit pattern
    x32 = (RNG.standard_normal(100_000) * 10 ** RNG.uniform(-3, 3, 100_000)).astype(np.float32)
    u = x32.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    ref = (u.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.array_equal(F.bf16_round(x32.astype(np.float64)), ref)


# --- RMSNorm --------------------------------------------------------------------------------------

def test_rmsnorm_constant_rows_closed_form():
    c = np.array([[0.5] * 8, [-3.0] * 8, [1e-3] * 8])
    g = np.linspace(0.5, 2.0, 8)
    eps = 1e-5
    expect = g[None, :] * c / np.sqrt(c * c + eps)
    assert np.allclose(F.rmsnorm(c, g, eps), expect, rtol=1e-14, atol=0)


def test_rmsnorm_scale_invariance_and_unit_rms():
    x = RNG.standard_normal((4, 64))
    g = np.ones(64)
    y = F.rmsnorm(x, g, 0.0)
    assert np.allclose(np.sqrt(np.mean(y * y, axis=1)), 1.0, rtol=1e-13)
    assert np.allclose(F.rmsnorm(7.5 * x, g, 0.0), y, rtol=1e-13)


# --- RoPE -----------------------------------------------------------------------------------------

def test_rope_position_zero_is_identity_and_norm_preserving():
    x = RNG.standard_normal((5, 3, 16))
    pos = np.array([0, 1, 7, 100, 4095])
    c, s = F.rope_cos_sin(pos, 16, 10000.0)
    y = F.apply_rope(x, c, s)
    assert np.allclose(y[0], x[0], atol=0)
    assert np.allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)


def test_rope_equals_complex_rotation_of_half_pairs():
    # rotate-half RoPE == multiplying z_i = x_i + j x_{i+d/2} by exp(j * pos * theta^(-2i/d))
    d, theta = 8, 10000.0
    x = RNG.standard_normal((3, 2, d))
    pos = np.array([1, 13, 511])
    c, s = F.rope_cos_sin(pos, d, theta)
    y = F.apply_rope(x, c, s)
    z = x[..., : d // 2] + 1j * x[..., d // 2:]
    w = np.array([[complex(math.cos(p * theta ** (-2.0 * i / d)), math.sin(p * theta ** (-2.0 * i / d)))
                   for i in range(d // 2)] for p in pos])
    zr = z * w[:, None, :]
    assert np.allclose(y[..., : d // 2], zr.real, rtol=0, atol=1e-13)
    assert np.allclose(y[..., d // 2:], zr.imag, rtol=0, atol=1e-13)


def test_rope_relative_position_property():
    # <R_m q, R_n k> depends only on m - n
    d = 64
    q = RNG.standard_normal((1, 1, d))
    k = RNG.standard_normal((1, 1, d))
    vals = []
    for m, n in [(10, 3), (107, 100), (7, 0)]:
        cm, sm = F.rope_cos_sin(np.array([m]), d, 500000.0)
        cn, sn = F.rope_cos_sin(np.array([n]), d, 500000.0)
        vals.append(float(np.sum(F.apply_rope(q, cm, sm) * F.apply_rope(k, cn, sn))))
    assert np.allclose(vals, vals[0], rtol=1e-11)


# --- attention ------------------------------------------------------------------------------------

def _brute_attention(q, k, v, qpos, kpos):
    """Plain-Python loops with math.exp, no max subtraction, no numpy reductions."""
    Tq, nq, d = q.shape
    nkv = k.shape[1]
    G = nq // nkv
    out = np.zeros((Tq, nq, v.shape[2]))
    for i in range(Tq):
        for h in range(nq):
            g = h // G
            ws, acc = 0.0, [0.0] * v.shape[2]
            for j in range(k.shape[0]):
                if kpos[j] > qpos[i]:
                    continue
                s = sum(float(q[i, h, t]) * float(k[j, g, t]) for t in range(d)) / math.sqrt(d)
                e = math.exp(s)
                ws += e
                for t in range(v.shape[2]):
                    acc[t] += e * float(v[j, g, t])
            out[i, h] = [a / ws for a in acc]
    return out


def test_attention_matches_brute_force_gqa_causal():
    q = RNG.standard_normal((5, 4, 8))
    k = RNG.standard_normal((5, 2, 8))
    v = RNG.standard_normal((5, 2, 8))
    got = F.prefill_attention(q, k, v)
    ref = _brute_attention(q, k, v, np.arange(5), np.arange(5))
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-13)


def test_decode_attention_matches_brute_force():
    q = RNG.standard_normal((6, 16))
    k = RNG.standard_normal((9, 3, 16))
    v = RNG.standard_normal((9, 3, 16))
    got = F.decode_attention(q, k, v)
    ref = _brute_attention(q[None], k, v, np.array([8]), np.arange(9))[0]
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-13)


def test_attention_special_cases():
    v = RNG.standard_normal((1, 1, 8))
    q = RNG.standard_normal((2, 8))
    k = RNG.standard_normal((1, 1, 8))
    assert np.allclose(F.decode_attention(q, k, v), np.repeat(v[0], 2, axis=0), atol=1e-15)  # one key -> V
    kz = np.zeros((7, 1, 8))
    vv = RNG.standard_normal((7, 1, 8))
    assert np.allclose(F.decode_attention(q, kz, vv), np.repeat(vv.mean(axis=0), 2, axis=0), atol=1e-14)


def test_gqa_equals_mha_with_repeated_kv():
    q = RNG.standard_normal((4, 8, 16))
    k = RNG.standard_normal((4, 2, 16))
    v = RNG.standard_normal((4, 2, 16))
    gqa = F.prefill_attention(q, k, v)
    mha = F.prefill_attention(q, np.repeat(k, 4, axis=1), np.repeat(v, 4, axis=1))
    assert np.allclose(gqa, mha, rtol=1e-13, atol=1e-14)


def test_decode_row_equals_prefill_row_at_same_position():
    q = RNG.standard_normal((6, 4, 16))
    k = RNG.standard_normal((6, 2, 16))
    v = RNG.standard_normal((6, 2, 16))
    pre = F.prefill_attention(q, k, v)
    for p in range(6):
        dec = F.decode_attention(q[p], k[: p + 1], v[: p + 1])
        assert np.allclose(dec, pre[p], rtol=1e-13, atol=1e-14)


def test_paged_read_equals_contiguous():
    P, nkv, d = 4, 2, 8
    pool = RNG.standard_normal((6, 2, nkv, P, d))
    kv = F.PagedKV(lambda layer, pages: pool[pages], P)
    pages = np.array([4, 0, 5])
    K, V = kv.read(0, pages, 10)
    Kc = np.concatenate([pool[p, 0].transpose(1, 0, 2) for p in pages])[:10]
    Vc = np.concatenate([pool[p, 1].transpose(1, 0, 2) for p in pages])[:10]
    assert np.array_equal(K, Kc) and np.array_equal(V, Vc)
    kv.write(0, 0, 3, np.full((nkv, d), 1.0 + 2 ** -9), np.full((nkv, d), -2.0))
    K2, V2 = kv.read(0, pages, 10)
    assert np.all(K2[7] == 1.0) and np.all(V2[7] == -2.0)      # slot 3 of page 0 = position 4 + 3
    assert np.array_equal(np.delete(K2, 7, axis=0), np.delete(Kc, 7, axis=0))


# --- FFN, MoE, LM head ----------------------------------------------------------------------------

def test_silu_special_values():
    assert F.silu(np.array([0.0]))[0] == 0.0
    assert abs(F.silu(np.array([40.0]))[0] - 40.0) < 1e-12
    assert abs(F.silu(np.array([-40.0]))[0]) < 1e-15
    assert abs(F.silu(np.array([1.0]))[0] - 1.0 / (1.0 + math.exp(-1.0))) < 1e-16


def test_swiglu_brute_force():
    n = RNG.standard_normal((3, 5))
    wg, wu, wd = RNG.standard_normal((4, 5)), RNG.standard_normal((4, 5)), RNG.standard_normal((5, 4))
    ref = np.zeros((3, 5))
    for t in range(3):
        a = []
        for f in range(4):
            g = sum(n[t, i] * wg[f, i] for i in range(5))
            u = sum(n[t, i] * wu[f, i] for i in range(5))
            a.append(g / (1 + math.exp(-g)) * u)
        for o in range(5):
            ref[t, o] = sum(a[f] * wd[o, f] for f in range(4))
    assert np.allclose(F.swiglu_ffn(n, wg, wu, wd), ref, rtol=1e-12, atol=1e-14)


def test_moe_routing_brute_force_and_ties():
    z = np.array([[0.1, 2.0, 2.0, -1.0], [3.0, 1.0, 3.0, 3.0], [-1.0, -2.0, -0.5, -0.5]])
    idx, w = F.moe_route(z, 2)
    assert idx.tolist() == [[1, 2], [0, 2], [2, 3]]
    for t in range(3):
        a, b = z[t, idx[t, 0]], z[t, idx[t, 1]]
        assert np.allclose(w[t], [math.exp(a) / (math.exp(a) + math.exp(b)), math.exp(b) / (math.exp(a) + math.exp(b))])
    zr = RNG.standard_normal((50, 8))
    idx, _ = F.moe_route(zr, 2)
    for t in range(50):
        srt = sorted(range(8), key=lambda e: (-zr[t, e], e))
        assert idx[t].tolist() == srt[:2]


def test_moe_identical_experts_equal_dense_and_top1_single_expert():
    n = RNG.standard_normal((7, 6))
    wg, wu, wd = RNG.standard_normal((5, 6)), RNG.standard_normal((5, 6)), RNG.standard_normal((6, 5))
    dense = F.swiglu_ffn(n, wg, wu, wd)
    z = RNG.standard_normal((7, 3))
    idx, w = F.moe_route(z, 2)
    y = F.moe_ffn(n, [(wg, wu, wd)] * 3, idx, w)
    assert np.allclose(y, dense, rtol=1e-12, atol=1e-13)
    idx1, w1 = F.moe_route(RNG.standard_normal((7, 1)), 1)
    assert np.all(w1 == 1.0)
    assert np.allclose(F.moe_ffn(n, [(wg, wu, wd)], idx1, w1), dense, rtol=1e-13)


def test_lm_head_argmax_first_index_on_ties():
    x = np.ones((2, 4))
    head = np.array([[1.0, 0, 0, 0], [0, 0, 0, 1.0], [0.5, 0.5, 0, 0], [0, 0, 0, 1.0]])
    logits, nxt = F.lm_head_argmax(x, np.ones(4), head, 0.0)
    assert nxt.tolist() == [0, 0]                      # logits [1, 1, 1, 1]: first max wins
    head2 = head.copy()
    head2[0, 0] = 0.0
    _, nxt2 = F.lm_head_argmax(x, np.ones(4), head2, 0.0)
    assert nxt2.tolist() == [1, 1]


# --- whole iteration: invariants ------------------------------------------------------------------

@pytest.fixture(scope="module")
def tiny_full():
    return run_oracle(TEST_WORKLOADS["tiny_gamma"])


def test_iteration_sub_batch_rows_equal_full_batch(tiny_full):
    b, res, _ = tiny_full
    w = TEST_WORKLOADS["tiny_gamma"]
    sb, sres, _ = run_oracle(w, requests=[5, 1, 6], keep_prefill=False)
    assert np.allclose(sres["hidden"], res["hidden"][[5, 1, 6]], rtol=0, atol=1e-12)
    pb, pres, _ = run_oracle(w, requests=[], keep_prefill=True)
    assert np.allclose(pres["hidden"], res["hidden"][b.num_decode:], rtol=0, atol=1e-12)


def test_iteration_request_permutation_invariance(tiny_full):
    b, res, _ = tiny_full
    w = TEST_WORKLOADS["tiny_gamma"]
    perm = [3, 0, 7, 2, 6, 1, 5, 4]
    _, pres, _ = run_oracle(w, requests=perm, keep_prefill=True)
    assert np.allclose(pres["hidden"][: len(perm)], res["hidden"][perm], rtol=0, atol=1e-12)
    assert np.allclose(pres["hidden"][len(perm):], res["hidden"][b.num_decode:], rtol=0, atol=1e-12)


def test_iteration_is_idempotent(tiny_full):
    _, res, _ = tiny_full
    _, res2, _ = run_oracle(TEST_WORKLOADS["tiny_gamma"])
    assert np.array_equal(res["hidden"], res2["hidden"])


def test_iteration_moe_and_lm_head_run():
    _, res, _ = run_oracle(TEST_WORKLOADS["tiny_moe"])
    idx = res["layers"][0]["topk_idx"]
    assert idx.shape == (40, 2) and np.all(idx[:, 0] != idx[:, 1])
    _, r2, _ = run_oracle(TEST_WORKLOADS["tiny_lm"])
    assert r2["logits"].shape == (9, 1024) and r2["next_token"].shape == (9,)


def test_written_kv_slots_follow_page_table(tiny_full):
    b, res, kv = tiny_full
    R = b.num_decode
    w = res["layers"][0]["written"]
    for t in range(b.num_tokens):
        r = t if t < R else R
        pos = int(b.positions[t])
        assert w[t] == (int(b.page_indices[b.page_indptr[r] + pos // 16]), pos % 16)


def _lm_forward(s, batch, kv, bf16_act):
    from oracle.run import layer_weights_f64
    from synth import bf16_to_f64
    from synth import weights as SW
    g = SW.global_specs(s)
    return F.iteration_forward(s, batch, lambda l: layer_weights_f64(s, l), kv,
                               embed_rows=lambda t: bf16_to_f64(SW.host_rows(g["embed"], t)),
                               final_norm=bf16_to_f64(SW.host_tensor(g["final_norm"])),
                               lm_head=bf16_to_f64(SW.host_tensor(g["lm_head"])), bf16_act=bf16_act)


def test_cached_decode_step_equals_full_sequence_recompute():
    """Greedy decoding with a KV cache (prefill, then one decode row reading the cached pages)
    gives the same logits as running prompt + token as one fresh prompt with no cache: the
    identity that lets plain recomputation serve as the greedy-decoding reference."""
    from oracle.run import make_kv
    from synth.workloads import Batch
    s = TEST_WORKLOADS["tiny_lm"].shape
    prompt = RNG.integers(0, s.vocab, 21).tolist()
    L = len(prompt)
    npg = (L + 1 + 15) // 16
    pages = np.array([3, 0, 5][:npg], dtype=np.int32)  # scattered pages of a larger pool
    kv = make_kv(s)
    pre = Batch(num_decode=0, prefill_len=L, ctx_lens=np.zeros(0, np.int32), page_size=16, num_pages=6,
                page_indptr=np.array([0, npg], np.int32), page_indices=pages,
                positions=np.arange(L, dtype=np.int32), tokens=np.array(prompt, np.int32))
    r1 = _lm_forward(s, pre, kv, bf16_act=False)
    tok = int(r1["next_token"][0])
    dec = Batch(num_decode=1, prefill_len=0, ctx_lens=np.array([L], np.int32), page_size=16, num_pages=6,
                page_indptr=np.array([0, npg, npg], np.int32), page_indices=pages,
                positions=np.array([L], np.int32), tokens=np.array([tok], np.int32))
    r2 = _lm_forward(s, dec, kv, bf16_act=False)
    full = Batch(num_decode=0, prefill_len=L + 1, ctx_lens=np.zeros(0, np.int32), page_size=16, num_pages=npg,
                 page_indptr=np.array([0, npg], np.int32), page_indices=np.arange(npg, dtype=np.int32),
                 positions=np.arange(L + 1, dtype=np.int32), tokens=np.array(prompt + [tok], np.int32))
    r3 = _lm_forward(s, full, make_kv(s), bf16_act=False)
    assert np.allclose(r2["logits"][0], r3["logits"][0], rtol=0, atol=1e-9)
    assert int(r2["next_token"][0]) == int(r3["next_token"][0])
    # the first token agrees with the full recompute of the prompt alone, too
    full_p = dataclasses.replace(full, prefill_len=L, positions=np.arange(L, dtype=np.int32),
                                 tokens=np.array(prompt, np.int32))
    assert np.allclose(_lm_forward(s, full_p, make_kv(s), bf16_act=False)["logits"][0], r1["logits"][0],
                       rtol=0, atol=1e-9)


# --- planted mistakes must be caught by the pins above --------------------------------------------

def test_planted_mistakes_are_caught(monkeypatch):
    # swapped RoPE pairing (interleaved instead of rotate-half) breaks the complex-rotation pin
    def rope_interleaved(x, cos, sin):
        x1, x2 = x[..., 0::2], x[..., 1::2]
        c, s = cos[:, None, :], sin[:, None, :]
        y = np.empty_like(x)
        y[..., 0::2], y[..., 1::2] = x1 * c - x2 * s, x2 * c + x1 * s
        return y
    monkeypatch.setattr(F, "apply_rope", rope_interleaved)
    with pytest.raises(AssertionError):
        test_rope_equals_complex_rotation_of_half_pairs()
    monkeypatch.undo()

    # a wrong GQA head map (h % nkv) breaks the brute-force GQA pin
    orig = F.attention

    def attention_wrong_map(q, k, v, q_pos, k_pos, bf16_p=False):
        nq, nkv = q.shape[1], k.shape[1]
        kk = k[:, [h % nkv for h in range(nq)], :]
        vv = v[:, [h % nkv for h in range(nq)], :]
        return orig(q, kk, vv, q_pos, k_pos, bf16_p)
    monkeypatch.setattr(F, "attention", attention_wrong_map)
    with pytest.raises(AssertionError):
        test_attention_matches_brute_force_gqa_causal()
    monkeypatch.undo()

    # a dropped causal mask breaks the causal brute-force pin
    def attention_no_mask(q, k, v, q_pos, k_pos, bf16_p=False):
        return orig(q, k, v, np.full_like(np.asarray(q_pos), 10 ** 9), k_pos, bf16_p)
    monkeypatch.setattr(F, "attention", attention_no_mask)
    with pytest.raises(AssertionError):
        test_attention_matches_brute_force_gqa_causal()
    monkeypatch.undo()

    # RMSNorm without eps or with the wrong axis breaks the closed form
    monkeypatch.setattr(F, "rmsnorm", lambda x, g, eps: x / np.sqrt(np.mean(x * x, axis=0, keepdims=True) + eps) * g)
    with pytest.raises(AssertionError):
        test_rmsnorm_constant_rows_closed_form()
    monkeypatch.undo()

    # the prefill chunk's token taken from its first row instead of its last breaks the cached-decode
    # identity (the logits of a prompt's continuation)
    def lm_rows_first_chunk_row(batch):
        rows = list(range(batch.num_decode))
        if batch.prefill_len > 0:
            rows.append(batch.num_decode)
        return np.array(rows, dtype=np.int64)
    monkeypatch.setattr(F, "lm_rows", lm_rows_first_chunk_row)
    with pytest.raises(AssertionError):
        test_cached_decode_step_equals_full_sequence_recompute()


def test_bf16_p_attention_definition():
    """Attention of the bf16 model: P = bf16(2^(x - M)), M the integer ceiling of the row maximum, output
    (P V) / sum 2^(x - M). Any other integer M gives the same result (exact power-of-two scaling of
    bf16 values); it stays within bf16 resolution of exact attention; scores that make every weight a
    power of two (no rounding) reproduce exact attention to double precision."""
    import math
    from oracle import forward as F
    rng = np.random.default_rng(4)
    q = rng.standard_normal((3, 4, 16))
    k = rng.standard_normal((40, 2, 16))
    v = rng.standard_normal((40, 2, 16))
    qp, kp = np.array([39, 20, 5]), np.arange(40)
    got = F.attention(q, k, v, qp, kp, bf16_p=True)
    exact = F.attention(q, k, v, qp, kp)
    assert np.abs(got - exact).max() < 4e-3 * np.abs(v).max()
    # the same definition written with M + 7 instead of M
    man = np.zeros_like(got)
    for h in range(4):
        g = h // 2
        s = (q[:, h, :] @ k[:, g, :].T) / math.sqrt(16)
        x = np.where(kp[None, :] <= qp[:, None], s, -np.inf) * math.log2(math.e)
        p = np.exp2(x - (np.ceil(x.max(axis=1, keepdims=True)) + 7))
        man[:, h, :] = (F.bf16_round(p) @ v[:, g, :]) / p.sum(axis=1, keepdims=True)
    assert np.abs(got - man).max() < 1e-12   # (x - M - 7) and (x - M) round differently only in the last bit
    # integer log2 scores: every weight is an exact power of two, so bf16 P is exact
    d = 16
    qi = np.zeros((1, 1, d)); qi[0, 0, 0] = math.sqrt(d) / math.log2(math.e)
    ki = np.zeros((8, 1, d)); ki[:, 0, 0] = rng.integers(-6, 3, size=8)
    vi = rng.standard_normal((8, 1, d))
    a = F.attention(qi, ki, vi, np.array([7]), np.arange(8), bf16_p=True)
    b = F.attention(qi, ki, vi, np.array([7]), np.arange(8))
    assert np.abs(a - b).max() < 1e-12
