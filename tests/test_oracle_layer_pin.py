"""Pin of the oracle's layer composition by brute force (CPU only).

``oracle.forward.layer_forward`` composes pinned primitives (RMSNorm, RoPE, attention, SwiGLU,
routing) into one Llama / Mixtral layer. The composition itself -- which tensor each step reads,
where the residual adds happen, what the router sees, which K/V land in which page slot -- is
checked here against a second, independent statement of the same layer written with plain Python
loops, ``math.exp`` and scalar arithmetic only (no numpy contraction), on tiny shapes:

    n  = RMSNorm(x) * gamma_attn;  q, k, v = n Wq^T, n Wk^T, n Wv^T;  RoPE (rotate-half) on q, k
    K/V of token t -> slot pos % 16 of page table[request][pos // 16] (stored as bf16)
    o  = softmax(q K^T / sqrt(d)) V over the visible keys, query head h reads KV head h // G
    h  = x + o Wo^T;  n2 = RMSNorm(h) * gamma_ffn
    x' = h + SwiGLU(n2)  or  x' = h + sum_k w_k Expert_{i_k}(n2), router logits RMSNorm(h) Wr^T + b

(the standard Llama / Mixtral layer named by the workloads; the NanoFlow pages give no layer
equations). Both precision readings are covered: float64 activations, and the bf16 model in which
every tensor handed from one operation to the next is rounded to bf16 and the attention weights
are P = bf16(2^(x - M)) with M the integer ceiling of the row maximum.

``test_planted_composition_mistakes_are_caught`` edits the oracle's layer on the CPU (x' = x + y,
the FFN norm reading x instead of h, a dropped attention residual, the router reading x, K stored
without RoPE, the decode query at the wrong position) and checks that the brute-force pin fails
for each.
"""
import inspect
import math

import numpy as np
import pytest

from oracle import forward as F
from oracle.forward import PagedKV
from synth.workloads import Batch, ModelShape

P = 16


def _bf(x: float) -> float:
    """Round to the nearest bf16 value (8 significant bits), ties to even (Python's round)."""
    if x == 0.0 or not math.isfinite(x):
        return x
    m, e = math.frexp(x)
    return math.ldexp(round(m * 256.0), e - 8)


def _dot(a, b):
    s = 0.0
    for u, w in zip(a, b):
        s += u * w
    return s


def _matvec(W, v):
    return [_dot(row, v) for row in W]


def _brute_layer(s, lw, x, batch, init_pages, bf16_act):
    """The layer, token by token and element by element. Returns (x', cache dict, router info)."""
    H, nq, nkv, d = s.hidden, s.n_q_heads, s.n_kv_heads, s.head_dim
    G = nq // nkv
    R, C = batch.num_decode, batch.prefill_len
    T = R + C
    eps = s.rms_eps
    W = {k: np.asarray(v).tolist() for k, v in lw.items()}
    rnd = _bf if bf16_act else (lambda z: z)
    X = np.asarray(x).tolist()
    pos = [int(p) for p in batch.positions]
    indptr = [int(p) for p in batch.page_indptr]
    table = [int(p) for p in batch.page_indices]
    cache = {}  # (page, kind, kv head, slot) -> list of d values (bf16)
    for pg in range(init_pages.shape[0]):
        for kind in range(2):
            for g in range(nkv):
                for sl in range(P):
                    cache[(pg, kind, g, sl)] = init_pages[pg, kind, g, sl].tolist()

    def norm_op(row, gamma, rounded):
        rs = 1.0 / math.sqrt(sum(v * v for v in row) / len(row) + eps)
        src = [_bf(v) for v in row] if rounded else row
        return [src[i] * rs * gamma[i] for i in range(len(row))]

    def rope(vec, p):
        out = list(vec)
        for i in range(d // 2):
            ang = p * s.rope_theta ** (-2.0 * i / d)
            c, sn = math.cos(ang), math.sin(ang)
            a, b = vec[i], vec[i + d // 2]
            out[i] = a * c - b * sn
            out[i + d // 2] = b * c + a * sn
        return out

    def req_of(t):
        return t if t < R else R

    # projections, RoPE, K/V into the pages
    Q = []
    for t in range(T):
        n = norm_op(X[t], W["attn_norm"], bf16_act)
        qf, kf, vf = _matvec(W["wq"], n), _matvec(W["wk"], n), _matvec(W["wv"], n)
        qh = [rnd(z) for h in range(nq) for z in rope(qf[h * d:(h + 1) * d], pos[t])]
        Q.append(qh)
        r = req_of(t)
        page = table[indptr[r] + pos[t] // P]
        for g in range(nkv):
            kk = rope(kf[g * d:(g + 1) * d], pos[t])
            cache[(page, 0, g, pos[t] % P)] = [_bf(z) for z in kk]
            cache[(page, 1, g, pos[t] % P)] = [_bf(z) for z in vf[g * d:(g + 1) * d]]

    def key(r, p, kind, g):
        return cache[(table[indptr[r] + p // P], kind, g, p % P)]

    # attention: decode request r sees keys 0..pos[r]; chunk row i sees keys 0..i
    O = []
    for t in range(T):
        r = req_of(t)
        nvis = pos[t] + 1
        o = []
        for h in range(nq):
            g = h // G
            qv = Q[t][h * d:(h + 1) * d]
            sc = [_dot(qv, key(r, p, 0, g)) / math.sqrt(d) for p in range(nvis)]
            if bf16_act:
                xs = [z * math.log2(math.e) for z in sc]
                M = math.ceil(max(xs))
                pw = [2.0 ** (z - M) for z in xs]
                den = sum(pw)
                acc = [0.0] * d
                for p in range(nvis):
                    w = _bf(pw[p])
                    vv = key(r, p, 1, g)
                    for j in range(d):
                        acc[j] += w * vv[j]
                o.extend(rnd(a / den) for a in acc)
            else:
                mx = max(sc)
                ex = [math.exp(z - mx) for z in sc]
                den = sum(ex)
                acc = [0.0] * d
                for p in range(nvis):
                    vv = key(r, p, 1, g)
                    for j in range(d):
                        acc[j] += ex[p] / den * vv[j]
                o.extend(acc)
        O.append(o)

    def swiglu(n2, wg, wu, wd):
        gt, up = _matvec(wg, n2), _matvec(wu, n2)
        act = [rnd(gv / (1.0 + math.exp(-gv)) * uv) for gv, uv in zip(gt, up)]
        return _matvec(wd, act)

    out, router = [], []
    for t in range(T):
        proj = _matvec(W["wo"], O[t])
        h = [X[t][i] + proj[i] for i in range(H)]
        n2 = norm_op(h, W["ffn_norm"], bf16_act)
        if s.n_experts == 0:
            y = swiglu(n2, W["w_gate"], W["w_up"], W["w_down"])
        else:
            hn = norm_op(h, W["ffn_norm"], False)
            z = [_dot(W["router"][e], hn) + W["router_bias"][e] for e in range(s.n_experts)]
            chosen = []
            for _ in range(s.top_k):  # largest remaining logit, lowest index on ties
                best = None
                for e in range(s.n_experts):
                    if e not in chosen and (best is None or z[e] > z[best]):
                        best = e
                chosen.append(best)
            zm = max(z[e] for e in chosen)
            ew = [math.exp(z[e] - zm) for e in chosen]
            wts = [v / sum(ew) for v in ew]
            y = [0.0] * H
            for e, w in zip(chosen, wts):
                ye = swiglu(n2, W[f"e{e}_gate"], W[f"e{e}_up"], W[f"e{e}_down"])
                y = [a + w * b for a, b in zip(y, ye)]
            router.append((z, chosen, wts))
        out.append([h[i] + y[i] for i in range(H)])
    return np.array(out), cache, router


def _setup(n_experts):
    rng = np.random.default_rng(7 + n_experts)
    s = ModelShape(name="pin", n_layers=1, hidden=16, n_q_heads=4, n_kv_heads=2, head_dim=8, ffn=12,
                   n_experts=n_experts, top_k=2, rope_theta=10000.0)
    H, d, F_ = s.hidden, s.head_dim, s.ffn

    def w(*shape, sd=0.3):
        return F.bf16_round(rng.standard_normal(shape) * sd)

    lw = {"attn_norm": F.bf16_round(1 + 0.1 * rng.standard_normal(H)), "ffn_norm": F.bf16_round(1 + 0.1 * rng.standard_normal(H)),
          "wq": w(s.n_q_heads * d, H), "wk": w(s.n_kv_heads * d, H), "wv": w(s.n_kv_heads * d, H),
          "wo": w(H, s.n_q_heads * d)}
    if n_experts == 0:
        lw.update(w_gate=w(F_, H), w_up=w(F_, H), w_down=w(H, F_))
    else:
        lw.update(router=w(n_experts, H, sd=0.5), router_bias=w(n_experts, sd=0.5))
        for e in range(n_experts):
            lw.update({f"e{e}_gate": w(F_, H), f"e{e}_up": w(F_, H), f"e{e}_down": w(H, F_)})
    # decode contexts 5, 17 (the new key opens a second page) and 0 (only the new key); a 6-token chunk
    ctx = np.array([5, 17, 0], np.int32)
    npages = [(c + 1 + P - 1) // P for c in ctx] + [1]
    num_pages = sum(npages) + 2                      # two pages nobody owns
    table = rng.permutation(num_pages)[:sum(npages)].astype(np.int32)
    indptr = np.concatenate([[0], np.cumsum(npages)]).astype(np.int32)
    C = 6
    batch = Batch(num_decode=3, prefill_len=C, ctx_lens=ctx, page_size=P, num_pages=num_pages,
                  page_indptr=indptr, page_indices=table,
                  positions=np.concatenate([ctx, np.arange(C)]).astype(np.int32))
    init = F.bf16_round(rng.standard_normal((num_pages, 2, s.n_kv_heads, P, d)))
    x = F.bf16_round(rng.standard_normal((batch.num_tokens, H)))
    return s, lw, x, batch, init


def _check(n_experts, bf16_act):
    s, lw, x, batch, init = _setup(n_experts)
    kv = PagedKV(lambda layer, pages: init[pages], P)
    got, extras = F.layer_forward(s, lw, x, batch, kv, 0, bf16_act)
    ref, cache, router = _brute_layer(s, lw, x, batch, init, bf16_act)
    assert np.abs(got - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max()), np.abs(got - ref).max()
    # every slot the oracle's cache holds equals the brute-force cache (written and untouched)
    for (layer, page), buf in kv.pages.items():
        for kind in range(2):
            for g in range(s.n_kv_heads):
                for sl in range(P):
                    assert np.abs(buf[kind, g, sl] - np.array(cache[(page, kind, g, sl)])).max() <= 1e-12
    if n_experts:
        z = np.array([r[0] for r in router])
        assert np.abs(extras["router_logits"] - z).max() <= 1e-12
        assert extras["topk_idx"].tolist() == [r[1] for r in router]
        assert np.abs(extras["topk_w"] - np.array([r[2] for r in router])).max() <= 1e-12


@pytest.mark.parametrize("bf16_act", [False, True])
def test_dense_layer_equals_brute_force(bf16_act):
    _check(0, bf16_act)


@pytest.mark.parametrize("bf16_act", [False, True])
def test_moe_layer_equals_brute_force(bf16_act):
    _check(3, bf16_act)


def _mutant(old: str, new: str):
    src = inspect.getsource(F.layer_forward)
    assert old in src, old
    ns = dict(F.__dict__)
    exec(compile(src.replace(old, new), "<planted mistake>", "exec"), ns)
    return ns["layer_forward"]


MUTANTS = [
    ("return h + y, extras", "return x + y, extras"),                               # x' = x + y
    ('n2 = norm_operand(h, lw["ffn_norm"]', 'n2 = norm_operand(x, lw["ffn_norm"]'),  # FFN norm of x
    ("h = x + o.reshape(T, nq * d)", "h = 0 * x + o.reshape(T, nq * d)"),          # attention residual dropped
    ('z = rmsnorm(h, lw["ffn_norm"]', 'z = rmsnorm(x, lw["ffn_norm"]'),              # router reads x
    ("k = apply_rope(k, cos, sin)", "k = k"),                                        # K cached unrotated
    ("K, V = kv.read(layer, pages, int(pos[t]) + 1)",
     "K, V = kv.read(layer, pages, int(pos[t]))"),                                   # own new key left out
]


@pytest.mark.parametrize("old,new", MUTANTS)
def test_planted_composition_mistakes_are_caught(monkeypatch, old, new):
    monkeypatch.setattr(F, "layer_forward", _mutant(old, new))
    # caught = the pin's comparison fails (or the mutant cannot even run, e.g. a request left with no key)
    with pytest.raises((AssertionError, ValueError)):
        _check(3 if "router" in new or "rmsnorm" in new else 0, False)


@pytest.mark.parametrize("n_experts,bf16_act", [(0, False), (0, True), (3, True)])
def test_row_subset_equals_full_layer_rows(n_experts, bf16_act):
    """layer_forward on a row subset (decode and chunk rows, any order) returns exactly those rows of
    the full layer, and writes the same K/V."""
    s, lw, x, batch, init = _setup(n_experts)
    kv_a = PagedKV(lambda layer, pages: init[pages], P)
    full, _ = F.layer_forward(s, lw, x, batch, kv_a, 0, bf16_act)
    rows = [7, 0, 3, 2, 8]          # chunk rows 4, 0 (position 0: one key), 5; decode rows 0, 2
    kv_b = PagedKV(lambda layer, pages: init[pages], P)
    sub, _ = F.layer_forward(s, lw, x, batch, kv_b, 0, bf16_act, rows=rows)
    assert np.array_equal(sub, full[rows])
    for key, buf in kv_b.pages.items():      # every page the subset touched (all written pages among them)
        assert np.array_equal(buf, kv_a.pages[key])
