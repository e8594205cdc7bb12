"""Input generator: Philox known answers, distribution moments, batch structure (CPU)."""
import os

import numpy as np
import pytest

import synth
from synth import weights as W
from synth.workloads import WORKLOADS, TEST_WORKLOADS, make_batch, pages_needed

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "philox4x32_10_kat.txt")


def _kat_rows():
    rows = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        v = [int(x, 16) for x in line.split()]
        rows.append((v[0:4], v[4:6], v[6:10]))
    return rows


@pytest.mark.parametrize("ctr,key,expect", _kat_rows())
def test_philox_known_answers(ctr, key, expect):
    assert synth.philox(ctr, key).tolist() == expect


def test_counter_layout_matches_block_function():
    # element i of tensor (seed, tid) is the Philox block at counter (lo32(i), hi32(i), 0, 0), key (seed, tid)
    i = (5 << 32) + 77
    w = synth.raw_words(9, 1234, i, 1)[0]
    assert w.tolist() == synth.philox([77, 5, 0, 0], [9, 1234]).tolist()


def test_normal_moments_and_bounds():
    # Irwin-Hall of eight 16-bit uniforms: mean 0, variance 1 after scaling; |z| <= 262140 * scale
    z = synth.bf16_to_f64(synth.normal_bf16(7, 3, 4_000_000))
    assert abs(z.mean()) < 3e-3
    assert abs(z.var() - 1.0) < 5e-3
    # excess kurtosis of a sum of 8 uniforms is -6/(5*8) = -0.15
    k = np.mean(z ** 4) / z.var() ** 2 - 3.0
    assert abs(k + 0.15) < 0.02
    assert np.abs(z).max() <= 262140 * float(synth.normal_scale(1.0)) * (1 + 2 ** -8)


def test_normal_exact_formula_small():
    # recompute a few elements from the raw words with the spec's integer sum, in plain Python
    w = synth.raw_words(0, 42, 0, 16)
    scale = synth.normal_scale(0.02)
    got = synth.normal_bf16(0, 42, 16, sigma=0.02)
    for i in range(16):
        s = sum((int(x) & 0xFFFF) + (int(x) >> 16) for x in w[i]) - 262140
        f = np.float32(np.float32(s) * scale) + np.float32(0.0)
        u = int(np.float32(f).view(np.uint32))
        u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFFFFFF
        assert got[i] == (u >> 16)


def test_uniform_int_range_and_mean():
    v = synth.uniform_int(3, 0, 200_000, 1024, 1536)
    assert v.min() == 1024 and v.max() == 1536
    assert abs(v.mean() - 1280) < 2.0


def test_offsets_and_ranges_agree():
    a = synth.normal_bf16(1, 5, 1000)
    b = synth.normal_bf16(1, 5, 100, offset=300)
    assert np.array_equal(a[300:400], b)
    c = synth.ranges_normal_bf16(1, 5, np.array([10, 500]), 20)
    assert np.array_equal(c[0], a[10:30]) and np.array_equal(c[1], a[500:520])
    g = synth.gather_normal_bf16(1, 5, np.array([999, 0, 17]))
    assert g.tolist() == [a[999], a[0], a[17]]


@pytest.mark.parametrize("name", ["tiny_layer", "llama3_8b_layer", "mixtral_8x7b_slice"])
def test_batch_structure(name):
    w = WORKLOADS[name]
    b = make_batch(w)
    R, C = w.num_decode, w.prefill_len
    assert b.page_indptr.shape == (R + 2,)
    assert sorted(b.page_indices.tolist()) == list(range(b.num_pages))     # a permutation
    for r in range(R):
        assert b.page_indptr[r + 1] - b.page_indptr[r] == pages_needed(b.ctx_lens[r] + 1, 16)
    assert b.page_indptr[R + 1] - b.page_indptr[R] == pages_needed(C, 16)
    assert np.array_equal(b.positions[:R], b.ctx_lens)
    assert np.array_equal(b.positions[R:], np.arange(C))
    if w.ctx_lognormal_median > 0:
        assert b.ctx_lens.min() >= w.ctx_lo and b.ctx_lens.max() <= w.ctx_hi
        assert 700 < np.median(b.ctx_lens) < 840
    else:
        assert b.ctx_lens.min() >= w.ctx_lo and b.ctx_lens.max() <= w.ctx_hi


def test_kv_pages_match_pool():
    s = WORKLOADS["tiny_layer"].shape
    pool = W.host_kv_pool(s, 0, 12)
    sel = W.host_kv_pages(s, 0, np.array([11, 3]))
    assert np.array_equal(sel[0], pool[11]) and np.array_equal(sel[1], pool[3])


@pytest.mark.parametrize("d,nkv", [(64, 2), (128, 8)])
def test_kv_physical_layout_is_a_permutation_with_the_documented_formula(d, nkv):
    from synth.workloads import ModelShape
    s = ModelShape("t", 1, 256, nkv, nkv, d, 128)
    pe = W.kv_page_elems(s)
    phys = np.arange(2 * pe, dtype=np.int64).reshape(2, pe)
    logical = W.kv_phys_to_logical(phys, s)
    assert sorted(logical.ravel().tolist()) == list(range(2 * pe))
    rng = np.random.default_rng(0)
    for _ in range(200):
        n, kv, h, r, c = (rng.integers(2), rng.integers(2), rng.integers(nkv), rng.integers(16), rng.integers(d))
        off = (kv * (d // 64) * nkv * 16 * 64 + (c // 64) * nkv * 16 * 64 + (h * 16 + r) * 64
               + (((c % 64) // 8) ^ (r % 8)) * 8 + c % 8)
        assert logical[n, kv, h, r, c] == n * pe + off


def test_weight_rows_match_full_tensor():
    s = TEST_WORKLOADS["tiny_lm"].shape
    spec = W.global_specs(s)["embed"]
    full = W.host_tensor(spec)
    rows = W.host_rows(spec, np.array([5, 1023, 0]))
    assert np.array_equal(rows, full[[5, 1023, 0]])


def test_gamma_is_one_for_model_shapes():
    s = WORKLOADS["tiny_layer"].shape
    g = synth.bf16_to_f64(W.host_tensor(W.layer_specs(s, 0)["attn_norm"]))
    assert np.all(g == 1.0)
